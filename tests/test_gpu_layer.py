"""GPU parity of the encoder layer, RMSNorm, conv stem and whole encoder
against the oracle (bf16 operands, fp32 accumulate / residual): max-abs 3e-2
and relative L2 1e-2.  Structure: transcribe.cpp notes "Voxtral", Voxtral
Realtime 2602 architecture."""
import numpy as np
import pytest
import torch

import oracle
import synth
from test_rounding_floor import C4_MAX_ABS
from gpu_util import cfg_of, compare_bf16, compare_f32, dev, host, layer_params_dev, layer_stack

pytestmark = pytest.mark.gpu

SMALL = synth.LayerDims(d_model=256, n_heads=4, head_dim=64, ffn_hidden=512, window=40)


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def test_rmsnorm_bf16_and_f32():
    vx = _vx()
    rng = np.random.default_rng(0)
    x = rng.standard_normal((37, 1280)).astype(np.float32) * 2
    r = rng.standard_normal((37, 1280)).astype(np.float32)
    g = synth.final_norm_gain(1280, seed=1)
    h = torch.empty(37, 1280, device="cuda")
    y = vx.rms_norm_fwd(dev(x), dev(g, torch.bfloat16), residual=dev(r), h_out=h, out_dtype=torch.float32)
    want = oracle.rms_norm(x.astype(np.float64) + r, g)
    compare_f32(host(h), x.astype(np.float64) + r, "h")
    np.testing.assert_allclose(host(y), want, rtol=2e-5, atol=2e-5)
    yb = vx.rms_norm_fwd(dev(x), dev(g, torch.bfloat16))
    compare_bf16(host(yb), oracle.rms_norm(x, g), "rmsnorm bf16")


@pytest.mark.parametrize("B,T,pos0,gate_up_bias", [(1, 1, 0, False), (2, 100, 0, False), (1, 300, 5, True),
                                                  (3, 129, 0, False)])
def test_small_layer(B, T, pos0, gate_up_bias):
    vx = _vx()
    p = synth.layer_params(SMALL, seed=11, gate_up_bias=gate_up_bias)
    x = synth.frames(B, T, SMALL.d_model, seed=12)
    L = vx.pack_layer(cfg_of(SMALL), layer_params_dev(p))
    y = vx.encoder_layer_fwd(cfg_of(SMALL), L, dev(x), pos0=pos0)
    compare_bf16(host(y), oracle.encoder_layer(x, p, SMALL, pos0=pos0), f"layer B={B} T={T}")


def test_c1_full_layer():
    # One full encoder layer: B=1, T=1500, d 1280, 32x64 heads, F 5120, W 750.
    vx = _vx()
    dims = synth.VOXTRAL_RT
    p = synth.layer_params(dims, seed=1)
    x = synth.frames(1, 1500, dims.d_model, seed=2)
    L = vx.pack_layer(cfg_of(dims), layer_params_dev(p))
    y = vx.encoder_layer_fwd(cfg_of(dims), L, dev(x))
    compare_bf16(host(y), oracle.encoder_layer(x, p, dims), "C1")
    # x == y (in place) gives the same result
    xt = dev(x)
    y2 = vx.encoder_layer_fwd(cfg_of(dims), L, xt, out=xt)
    assert torch.equal(y2, y)


def test_c4_size_layer_last_clip():
    # One encoder layer over the encoder workload's 4 x 3000 frames (M = 12000
    # rows per GEMM), in the walk orders of this size (grouped row panels for
    # the QKV, gate/up and O inputs, N-fastest for the down projection's): the
    # last clip is checked whole against the oracle, the first on a prefix.
    vx = _vx()
    dims = synth.VOXTRAL_RT
    p = synth.layer_params(dims, seed=21)
    x = synth.frames(4, 3000, dims.d_model, seed=22)
    L = vx.pack_layer(cfg_of(dims), layer_params_dev(p))
    y = host(vx.encoder_layer_fwd(cfg_of(dims), L, dev(x)))
    compare_bf16(y[3:], oracle.encoder_layer(x[3:], p, dims), "C4-size layer, clip 3")
    compare_bf16(y[:1, :200], oracle.encoder_layer(x[:1, :200], p, dims), "C4-size layer, clip 0 prefix")


def test_layer_pack_matches_parameters():
    vx = _vx()
    p = synth.layer_params(SMALL, seed=5, gate_up_bias=True)
    L = vx.pack_layer(cfg_of(SMALL), layer_params_dev(p))
    hd, f = SMALL.hd, SMALL.ffn_hidden
    wqkv = host(L.wqkv)
    np.testing.assert_array_equal(wqkv, np.concatenate([p["wq"], p["wk"], p["wv"]]))
    np.testing.assert_array_equal(host(L.bqkv), np.concatenate([p["bq"], np.zeros(hd), p["bv"]]))
    wgu = host(L.wgu).reshape(f // 64, 2, 64, SMALL.d_model)
    np.testing.assert_array_equal(wgu[:, 0].reshape(f, -1), p["wg"])
    np.testing.assert_array_equal(wgu[:, 1].reshape(f, -1), p["wu"])
    bgu = host(L.bgu).reshape(f // 64, 2, 64)
    np.testing.assert_array_equal(bgu[:, 0].reshape(f), p["bg"])
    np.testing.assert_array_equal(bgu[:, 1].reshape(f), p["bu"])


def _conv_dev(conv):
    vx = _vx()
    return (vx.pack_conv_weight(dev(conv["w1"], torch.bfloat16)), dev(conv["b1"], torch.bfloat16),
            vx.pack_conv_weight(dev(conv["w2"], torch.bfloat16)), dev(conv["b2"], torch.bfloat16))


@pytest.mark.parametrize("B,Tm", [(1, 1), (2, 7), (1, 64), (3, 301), (2, 1000)])
def test_conv_stem_small(B, Tm):
    vx = _vx()
    conv = synth.conv_params(seed=3, n_mels=128, d=256)
    mel = synth.mel(B, 128, Tm, seed=4)
    out = vx.conv_stem_fwd(dev(mel), *_conv_dev(conv))
    compare_bf16(host(out), oracle.conv_stem(mel, **conv), f"conv B={B} Tm={Tm}")


def test_conv_stem_c4_full_size_sampled():
    # mel [4, 128, 6000] -> [4, 3000, 1280]; frames checked on a prefix and a
    # tail window of every clip (output t depends on mel frames 2t-4 .. 2t only).
    vx = _vx()
    conv = synth.conv_params(seed=3)
    mel = synth.mel(4, 128, 6000, seed=4)
    out = host(vx.conv_stem_fwd(dev(mel), *_conv_dev(conv)))
    assert out.shape == (4, 3000, 1280)
    compare_bf16(out[:, :200], oracle.conv_stem(mel[:, :, :400], **conv), "C4 stem prefix")
    a = 2 * 2900 - 4   # slice start; outputs t >= 2900 are exact
    tail = oracle.conv_stem(mel[:, :, a:], **conv)[:, 2:]
    compare_bf16(out[:, 2900:], tail, "C4 stem tail")


def test_small_encoder_full():
    vx = _vx()
    dims = SMALL
    conv = synth.conv_params(seed=7, n_mels=128, d=dims.d_model)
    layers = layer_stack(dims, 3, 8)
    g = synth.final_norm_gain(dims.d_model, seed=9)
    mel = synth.mel(2, 128, 333, seed=10)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    out = vx.encoder_fwd(cfg_of(dims), dev(mel), *_conv_dev(conv), Ls, dev(g, torch.bfloat16))
    compare_bf16(host(out), oracle.encoder(mel, conv, layers, g, dims), "small encoder")


def test_c4_full_encoder_prefix():
    # Full streaming-encoder forward, B=4 x 6000 mel frames, 32 layers, final
    # RMSNorm.  Causality makes the first 256 output frames of clip 0 depend
    # only on mel frames < 512, so the oracle runs on that prefix.
    vx = _vx()
    dims = synth.VOXTRAL_RT
    conv = synth.conv_params(seed=3)
    layers = layer_stack(dims, 32, 1)
    g = synth.final_norm_gain(dims.d_model, seed=5)
    mel = synth.mel(4, 128, 6000, seed=4)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    out = host(vx.encoder_fwd(cfg_of(dims), dev(mel), *_conv_dev(conv), Ls, dev(g, torch.bfloat16)))
    assert out.shape == (4, 3000, 1280) and np.all(np.isfinite(out))
    want = oracle.encoder(mel[:1, :, :512], conv, layers, g, dims)
    # 32 layers: rel-L2 keeps the 1e-2 bar; max-abs is bounded by the bf16
    # operand-rounding floor derived in test_rounding_floor.py.
    compare_bf16(out[:1, :256], want, "C4 prefix", max_abs=C4_MAX_ABS)
    # final RMSNorm: every frame's RMS of out / g is ~1
    rms = np.sqrt(np.mean((out / g.astype(np.float64)) ** 2, axis=-1))
    assert np.all(np.abs(rms - 1) < 1e-2)
