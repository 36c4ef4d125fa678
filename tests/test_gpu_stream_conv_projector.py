"""GPU parity of the streaming conv-stem step (conv padding cache) and of the
audio projector against the float64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import compare_bf16, dev, host

pytestmark = pytest.mark.gpu


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def _conv_dev(vx, conv):
    return (vx.pack_conv_weight(dev(conv["w1"], torch.bfloat16)), dev(conv["b1"], torch.bfloat16),
            vx.pack_conv_weight(dev(conv["w2"], torch.bfloat16)), dev(conv["b2"], torch.bfloat16))


def _bf16_bits(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32) >> 16


def test_conv_stem_step_chain_matches_oracle_and_whole_clip():
    vx = _vx()
    S, C, d, chunk, n_chunks = 3, 128, 256, 8, 5
    conv = synth.conv_params(seed=21, n_mels=C, d=d)
    w = _conv_dev(vx, conv)
    mel = synth.mel(S, C, chunk * n_chunks, seed=22)
    cache = vx.ConvCache(S, C, d)
    cx, ch = np.zeros((S, C, 2)), np.zeros((S, d, 2))
    outs = []
    for s in range(n_chunks):
        part = mel[:, :, s * chunk:(s + 1) * chunk]
        got = host(vx.conv_stem_step(dev(np.ascontiguousarray(part)), *w, cache))
        want, cx, ch = oracle.conv_stem_step(part, conv["w1"], conv["b1"], conv["w2"], conv["b2"], cx, ch)
        compare_bf16(got, want, f"conv step chunk {s}")
        outs.append(got)
    # the cache holds the last two mel frames exactly as bf16, frame-major
    np.testing.assert_array_equal(host(cache.x.float()), synth.bf16_round(np.transpose(mel[:, :, -2:], (0, 2, 1))))
    compare_bf16(host(cache.h1.float()), np.transpose(ch, (0, 2, 1)), "conv step h1 cache")
    # chunked output == the GPU whole-clip stem on the same frames (same bf16 operands)
    whole = host(vx.conv_stem_fwd(dev(mel), *w))
    np.testing.assert_allclose(np.concatenate(outs, axis=1), whole, rtol=0, atol=1e-5)


def test_conv_stem_step_full_width_64_streams():
    # The 80 ms streaming shape: 64 streams x 8 mel frames -> 4 frames of 1280, warm caches.
    vx = _vx()
    S, C, d = 64, 128, 1280
    conv = synth.conv_params(seed=3, n_mels=C, d=d)
    w = _conv_dev(vx, conv)
    rng = np.random.default_rng(23)
    cx = synth.bf16_round(rng.standard_normal((S, C, 2)))
    ch = synth.bf16_round(rng.standard_normal((S, d, 2)) * 0.5)
    cache = vx.ConvCache(S, C, d)
    cache.x.copy_(dev(np.transpose(cx, (0, 2, 1)), torch.bfloat16))
    cache.h1.copy_(dev(np.transpose(ch, (0, 2, 1)), torch.bfloat16))
    mel = synth.mel(S, C, 8, seed=24)
    got = host(vx.conv_stem_step(dev(mel), *w, cache))
    want, _, _ = oracle.conv_stem_step(mel, conv["w1"], conv["b1"], conv["w2"], conv["b2"], cx, ch)
    assert got.shape == (S, 4, d)
    compare_bf16(got, want, "conv step 64x8")


def test_conv_stem_step_rejects_odd_chunks():
    vx = _vx()
    conv = synth.conv_params(seed=3, n_mels=128, d=256)
    cache = vx.ConvCache(2, 128, 256)
    with pytest.raises(vx.VxError, match="UNSUPPORTED"):
        vx.conv_stem_step(dev(synth.mel(2, 128, 7, seed=1)), *_conv_dev(vx, conv), cache)


@pytest.mark.parametrize("B,T", [(1, 4), (2, 13), (3, 40)])
def test_projector_small(B, T):
    vx = _vx()
    d, H = 256, 384
    pw = synth.projector_params(d=d, hidden=H, seed=31)
    x = synth.frames(B, T, d, seed=32)
    got = host(vx.projector_fwd(dev(x), dev(pw["w1"], torch.bfloat16), dev(pw["w2"], torch.bfloat16)))
    compare_bf16(got, oracle.projector(x, pw["w1"], pw["w2"]), f"projector B={B} T={T}")


def test_projector_fewer_than_four_frames_gives_no_token():
    vx = _vx()
    pw = synth.projector_params(d=256, hidden=384, seed=31)
    out = vx.projector_fwd(dev(synth.frames(2, 3, 256, seed=1)), dev(pw["w1"], torch.bfloat16),
                           dev(pw["w2"], torch.bfloat16))
    assert tuple(out.shape) == (2, 0, 384)


def test_projector_full_size_sampled_tokens():
    # The encoder output of the 4 x 6000-mel workload: [4, 3000, 1280] -> [4, 750, 3072].
    vx = _vx()
    pw = synth.projector_params(seed=8)
    x = synth.frames(4, 3000, 1280, seed=33)
    got = host(vx.projector_fwd(dev(x), dev(pw["w1"], torch.bfloat16), dev(pw["w2"], torch.bfloat16)))
    assert got.shape == (4, 750, 3072)
    for j in (0, 1, 377, 749):
        want = oracle.projector(x[:, 4 * j:4 * j + 4], pw["w1"], pw["w2"])
        compare_bf16(got[:, j:j + 1], want, f"projector token {j}")
