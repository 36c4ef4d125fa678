"""Pins of the oracle's encoder layer, streaming step and ring cache.

Structure under test (transcribe.cpp notes "Voxtral", Voxtral Realtime 2602
architecture): pre-norm layer, q/v/o biases, no k bias, SwiGLU MLP with bias on
the down projection; streaming: 4 encoder frames per step (Streaming schedule),
ring cache of W slots (frame f in slot f mod W).
"""
import numpy as np
import pytest

import oracle
import synth

SMALL = synth.LayerDims(d_model=48, n_heads=4, head_dim=16, ffn_hidden=96, window=5)  # hd=64 != d


def _params(seed=1, dims=SMALL, gate_up_bias=False):
    return synth.layer_params(dims, seed=seed, gate_up_bias=gate_up_bias)


def test_zero_branches_leave_residual_plus_biases():
    p = _params()
    p["wo"] = np.zeros_like(p["wo"])
    p["wd"] = np.zeros_like(p["wd"])
    x = synth.frames(2, 13, SMALL.d_model, seed=3).astype(np.float64)
    out = oracle.encoder_layer(x, p, SMALL)
    np.testing.assert_allclose(out, x + p["bo"] + p["bd"], rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("W", [1, 5, 40])
def test_value_path_with_uniform_attention(W):
    # Wq = Wk = 0 and bq = 0 make all scores 0 (uniform attention).  Wv copies
    # the normalised input into the first d value channels and Wo copies them
    # back; with the MLP zeroed, out_t = x_t + mean_{window(t)} RMSNorm(x)_j.
    dims = synth.LayerDims(d_model=64, n_heads=8, head_dim=16, ffn_hidden=96, window=W)
    d, hd = dims.d_model, dims.hd
    p = _params(dims=dims)
    p["wq"][:] = 0; p["bq"][:] = 0; p["wk"][:] = 0
    p["wv"] = np.zeros((hd, d), np.float32); p["wv"][np.arange(d), np.arange(d)] = 1
    p["bv"][:] = 0
    p["wo"] = np.zeros((d, hd), np.float32); p["wo"][np.arange(d), np.arange(d)] = 1
    p["bo"][:] = 0; p["wd"][:] = 0; p["bd"][:] = 0
    T = 17
    x = synth.frames(1, T, d, seed=4).astype(np.float64)
    out = oracle.encoder_layer(x, p, dims)
    y = x / np.sqrt(np.mean(x * x, -1, keepdims=True) + dims.eps) * p["attn_norm_g"]
    for t in range(T):
        lo = max(0, t - W + 1)
        np.testing.assert_allclose(out[0, t], x[0, t] + y[0, lo:t + 1].mean(0), rtol=1e-12, atol=1e-12)


def test_swiglu_orientation():
    # Attention branch off; gate = a * y_c, up = y_c, down writes feature 0 to
    # channel c: out = h + silu(a y_c) y_c e_c with h = x.
    d, f = SMALL.d_model, SMALL.ffn_hidden
    p = _params()
    p["wo"][:] = 0; p["bo"][:] = 0; p["bd"][:] = 0
    c, a = 5, 2.5
    p["wg"] = np.zeros((f, d), np.float32); p["wg"][0, c] = a
    p["wu"] = np.zeros((f, d), np.float32); p["wu"][0, c] = 1
    p["wd"] = np.zeros((d, f), np.float32); p["wd"][c, 0] = 1
    x = synth.frames(1, 6, d, seed=5).astype(np.float64)
    out = oracle.encoder_layer(x, p, SMALL)
    y = x / np.sqrt(np.mean(x * x, -1, keepdims=True) + SMALL.eps) * p["ffn_norm_g"]
    yc = y[..., c]
    want = x.copy()
    want[..., c] += a * yc / (1 + np.exp(-a * yc)) * yc
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_gate_up_bias_is_optional_and_used():
    p = _params(gate_up_bias=True)
    x = synth.frames(1, 8, SMALL.d_model, seed=6).astype(np.float64)
    with_b = oracle.encoder_layer(x, p, SMALL)
    p0 = dict(p, bg=None, bu=None)
    without = oracle.encoder_layer(x, p0, SMALL)
    assert np.max(np.abs(with_b - without)) > 1e-4


def test_layer_is_invariant_to_position_origin():
    # RoPE scores depend only on relative positions, so shifting pos0 leaves
    # the layer output unchanged (fails if RoPE hits only q or only k).
    p = _params()
    x = synth.frames(2, 15, SMALL.d_model, seed=7).astype(np.float64)
    a = oracle.encoder_layer(x, p, SMALL, pos0=0)
    b = oracle.encoder_layer(x, p, SMALL, pos0=1000)
    np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-10)


def test_layer_is_causal():
    p = _params()
    x = synth.frames(1, 20, SMALL.d_model, seed=8).astype(np.float64)
    a = oracle.encoder_layer(x, p, SMALL)
    x2 = x.copy(); x2[:, 12:] += 1.0
    b = oracle.encoder_layer(x2, p, SMALL)
    np.testing.assert_array_equal(a[:, :12], b[:, :12])
    assert np.max(np.abs(a[:, 12] - b[:, 12])) > 1e-3


def test_ring_slots_hold_frames_mod_window():
    # Position-tagged payload: k[s, f] = f (+ head/dim tags) must land in slot f mod W.
    S, T, H, D, W = 2, 13, 2, 3, 5
    tag = np.arange(T)[None, :, None, None] + 1000 * np.arange(S)[:, None, None, None] \
        + 0.01 * np.arange(H)[None, None, :, None] + 0.0001 * np.arange(D)
    rk, rv = oracle.ring_from_sequence(tag, -tag, W)
    for s in range(S):
        for f in range(T - W, T):
            np.testing.assert_array_equal(rk[s, :, f % W], tag[s, f])
            np.testing.assert_array_equal(rv[s, :, f % W], -tag[s, f])


@pytest.mark.parametrize("prefill,steps,n", [(9, 3, 4), (2, 2, 4), (0, 4, 3), (5, 3, 1)])
def test_streaming_equals_whole_sequence(prefill, steps, n):
    # Causality pin: prefill a ring with the first frames, then stream n frames
    # per step through a 2-layer stack; every step must equal the same rows of
    # the whole-sequence forward (ring wraps for prefill + steps * n > W).
    dims = SMALL
    layers = [_params(seed=synth.layer_seed(3, l)) for l in range(2)]
    S, T = 2, prefill + steps * n
    x = synth.frames(S, T, dims.d_model, seed=9).astype(np.float64)
    # whole sequence, and the per-layer K/V of the prefix
    h = x
    rings = []
    for p in layers:
        hp, k, v = oracle.encoder_layer(h[:, :prefill], p, dims, return_kv=True)
        rings.append(oracle.ring_from_sequence(k, v, dims.window))
        h = oracle.encoder_layer(h, p, dims)
    whole = h
    pos = np.full(S, prefill)
    for st in range(steps):
        rows = slice(prefill + st * n, prefill + (st + 1) * n)
        out, rings, pos = oracle.stream_step(x[:, rows], layers, dims, rings, pos)
        np.testing.assert_allclose(out, whole[:, rows], rtol=1e-11, atol=1e-11)
    assert np.all(pos == T)


def test_stream_step_writes_new_frames_into_their_slots():
    dims = SMALL
    p = _params()
    S, T, n = 1, 12, 4
    x = synth.frames(S, T + n, dims.d_model, seed=10).astype(np.float64)
    _, k, v = oracle.encoder_layer(x, p, dims, return_kv=True)
    rk, rv = oracle.ring_from_sequence(k[:, :T], v[:, :T], dims.window)
    _, nk, nv = oracle.stream_step_layer(x[:, T:], p, dims, rk, rv, np.array([T]))
    for t in range(n):
        f = T + t
        np.testing.assert_allclose(nk[0, :, f % dims.window], k[0, f], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(nv[0, :, f % dims.window], v[0, f], rtol=1e-12, atol=1e-12)


def test_value_bias_and_output_projection_orientation():
    # Wq = Wk = Wv = 0: attention output is bv for every frame, so
    # h = x + bv Wo^T + bo exactly (d != H*D catches a transposed Wo).
    p = _params()
    p["wq"][:] = 0; p["wk"][:] = 0; p["wv"][:] = 0
    p["wd"][:] = 0
    x = synth.frames(1, 9, SMALL.d_model, seed=11).astype(np.float64)
    out = oracle.encoder_layer(x, p, SMALL)
    want = x + p["bv"].astype(np.float64) @ p["wo"].astype(np.float64).T + p["bo"] + p["bd"]
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)


def test_query_bias_enters_scores():
    p = _params()
    x = synth.frames(1, 9, SMALL.d_model, seed=12).astype(np.float64)
    a = oracle.encoder_layer(x, p, SMALL)
    p2 = dict(p, bq=p["bq"] * 0)
    assert np.max(np.abs(oracle.encoder_layer(x, p2, SMALL) - a)) > 1e-5


def test_stream_step_final_norm_closed_form():
    # With zero-branch layers a streaming step through L layers adds
    # sum_l (bo_l + bd_l) to the new frames (the ring only feeds the vanished
    # attention branch); final_g then applies the encoder's final RMSNorm:
    #   out = (x + sum b) / sqrt(mean((x + sum b)^2) + eps) * g.
    dims = SMALL
    layers = []
    for l in range(3):
        p = _params(seed=synth.layer_seed(12, l))
        p["wo"] = np.zeros_like(p["wo"])
        p["wd"] = np.zeros_like(p["wd"])
        layers.append(p)
    S, n, P = 2, 4, 7
    x = synth.frames(S, n, dims.d_model, seed=13).astype(np.float64)
    rings = [synth.ring_kv(S, dims.n_heads, dims.window, dims.head_dim, seed=14 + l) for l in range(3)]
    g = synth.final_norm_gain(dims.d_model, seed=15).astype(np.float64)
    raw, _, pos = oracle.stream_step(x, layers, dims, rings, np.full(S, P))
    out, _, _ = oracle.stream_step(x, layers, dims, rings, np.full(S, P), final_g=g)
    h = x + sum(p["bo"].astype(np.float64) + p["bd"].astype(np.float64) for p in layers)
    np.testing.assert_allclose(raw, h, rtol=1e-13, atol=1e-13)
    want = h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + dims.eps) * g
    np.testing.assert_allclose(out, want, rtol=1e-12, atol=1e-12)
    assert np.all(pos == P + n)
