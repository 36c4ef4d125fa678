"""Pins of the streaming conv-stem step (conv padding cache) and of the audio
projector of the oracle."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


@pytest.mark.parametrize("chunk", [2, 8])
def test_conv_stem_step_chunks_equal_whole_stream(chunk):
    # Carrying the last two mel frames and the last two conv1 outputs makes
    # chunk-by-chunk output equal to the whole-clip causal conv stem.
    C, d, B, n_chunks = 8, 12, 2, 5
    w = synth.conv_params(seed=11, n_mels=C, d=d)
    mel = synth.mel(B, C, chunk * n_chunks, seed=12).astype(np.float64)
    whole = oracle.conv_stem(mel, **w)
    cx = np.zeros((B, C, 2))
    ch = np.zeros((B, d, 2))
    outs = []
    for s in range(n_chunks):
        o, cx, ch = oracle.conv_stem_step(mel[:, :, s * chunk:(s + 1) * chunk], w["w1"], w["b1"], w["w2"], w["b2"],
                                          cx, ch)
        assert o.shape == (B, chunk // 2, d)
        outs.append(o)
    np.testing.assert_allclose(np.concatenate(outs, axis=1), whole, rtol=1e-12, atol=1e-13)


def test_conv_stem_step_matches_torch_conv1d_on_cached_context():
    # One chunk against torch's conv1d run over [cache | chunk] with no padding.
    C, d, B = 8, 12, 1
    w = synth.conv_params(seed=13, n_mels=C, d=d)
    rng = np.random.default_rng(14)
    mel = rng.standard_normal((B, C, 8))
    cx = rng.standard_normal((B, C, 2))
    ch = rng.standard_normal((B, d, 2))
    out, ncx, nch = oracle.conv_stem_step(mel, w["w1"], w["b1"], w["w2"], w["b2"], cx, ch)
    t = {k: torch.from_numpy(v.astype(np.float64)) for k, v in w.items()}
    h1 = F.gelu(F.conv1d(torch.from_numpy(np.concatenate([cx, mel], 2)), t["w1"], t["b1"]), approximate="none")
    h2 = F.gelu(F.conv1d(torch.cat([torch.from_numpy(ch), h1], 2), t["w2"], t["b2"], stride=2), approximate="none")
    np.testing.assert_allclose(out, h2.permute(0, 2, 1).numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(ncx, mel[:, :, -2:])
    np.testing.assert_allclose(nch, h1[:, :, -2:].numpy(), rtol=1e-12, atol=1e-13)


def test_projector_token_is_four_consecutive_frames_in_time_order():
    # Frame t carries the value t + c / 100 in channel c; with one-hot rows in
    # w1 and w2 = I, token j's hidden unit (r, c) must read frame 4j + r, channel c.
    B, T, d = 1, 13, 3
    x = np.zeros((B, T, d))
    for t in range(T):
        for c in range(d):
            x[0, t, c] = t + c / 100.0
    H = 4 * d
    w1 = np.eye(H)
    w2 = np.eye(H)
    out = oracle.projector(x, w1, w2)
    assert out.shape == (1, 3, H)                  # 13 frames -> 3 tokens, 1 frame dropped
    for j in range(3):
        for r in range(4):
            for c in range(d):
                z = 4 * j + r + c / 100.0
                # GELU(z) for these positive z equals z * Phi(z); Phi(z) ~ 1 beyond z = 8
                expect = z * 0.5 * (1.0 + torch.erf(torch.tensor(z / np.sqrt(2.0), dtype=torch.float64)).item())
                assert abs(out[0, j, r * d + c] - expect) < 1e-12


def test_projector_drops_trailing_frames_and_is_bias_free():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((2, 9, 4))
    w1 = rng.standard_normal((5, 16))
    w2 = rng.standard_normal((5, 5))
    a = oracle.projector(x, w1, w2)
    b = oracle.projector(x[:, :8], w1, w2)
    np.testing.assert_array_equal(a, b)
    assert a.shape == (2, 2, 5)
    np.testing.assert_array_equal(oracle.projector(np.zeros((1, 8, 4)), w1, w2), np.zeros((1, 2, 5)))


def test_projector_against_torch_linear_and_gelu_on_unfolded_frames():
    # torch.unfold builds the tokens independently of the reshape.
    rng = np.random.default_rng(4)
    B, T, d, H = 2, 10, 6, 7
    x = rng.standard_normal((B, T, d))
    w1 = rng.standard_normal((H, 4 * d)) * 0.2
    w2 = rng.standard_normal((H, H)) * 0.2
    xt = torch.from_numpy(x)
    tok = xt.unfold(1, 4, 4)                         # [B, T//4, d, 4]: window of 4 frames along time
    tok = tok.permute(0, 1, 3, 2).reshape(B, T // 4, 4 * d)
    ref = F.linear(F.gelu(F.linear(tok, torch.from_numpy(w1)), approximate="none"), torch.from_numpy(w2))
    np.testing.assert_allclose(oracle.projector(x, w1, w2), ref.numpy(), rtol=1e-12, atol=1e-12)
