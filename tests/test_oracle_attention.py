"""Pins of the oracle's sliding-window attention to facts outside the oracle.

Window convention under test (transcribe.cpp notes "Voxtral", Voxtral Realtime
2602 architecture: "causal + sliding-window (750)"): query i sees keys j with
i - W < j <= i.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import synth


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_window_one_returns_own_value():
    # W = 1: each query sees only itself, softmax of one score is exactly 1.
    q, k, v = (_rand((2, 11, 3, 8), s) for s in (1, 2, 3))
    o = oracle.swa_attention(q, k, v, window=1)
    np.testing.assert_array_equal(o, v)


@pytest.mark.parametrize("W", [1, 3, 7, 40])
def test_zero_query_gives_mean_of_window(W):
    # q = 0 makes every score 0, so o_i is the plain mean of v over the window.
    T = 23
    v = _rand((1, T, 2, 5), 4)
    q = np.zeros_like(v)
    k = _rand(v.shape, 5)
    o = oracle.swa_attention(q, k, v, window=W)
    c = np.concatenate([np.zeros((1, 1, 2, 5)), np.cumsum(v, axis=1)], axis=1)
    for i in range(T):
        lo = max(0, i - W + 1)
        want = (c[:, i + 1] - c[:, lo]) / (i + 1 - lo)
        np.testing.assert_allclose(o[:, i], want, rtol=1e-12, atol=1e-13)


def test_full_window_equals_torch_causal_sdpa():
    # W >= T reduces to plain causal attention (textbook case, torch fp64 on CPU).
    B, T, H, D = 2, 37, 3, 16
    q, k, v = (_rand((B, T, H, D), s) for s in (6, 7, 8))
    o = oracle.swa_attention(q, k, v, window=T + 5)
    t = [torch.from_numpy(x).permute(0, 2, 1, 3) for x in (q, k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t, is_causal=True)
    np.testing.assert_allclose(o, ref.permute(0, 2, 1, 3).numpy(), rtol=1e-11, atol=1e-12)


def test_window_two_closed_form():
    # W = 2: o_i = sigma(d) v_i + (1 - sigma(d)) v_{i-1}, d = (s_ii - s_i,i-1).
    B, T, H, D = 1, 9, 2, 4
    q, k, v = (_rand((B, T, H, D), s) for s in (9, 10, 11))
    o = oracle.swa_attention(q, k, v, window=2)
    np.testing.assert_allclose(o[:, 0], v[:, 0], rtol=0, atol=1e-15)
    for i in range(1, T):
        d = (np.sum(q[:, i] * k[:, i], -1) - np.sum(q[:, i] * k[:, i - 1], -1)) / math.sqrt(D)
        w = 1.0 / (1.0 + np.exp(-d))
        want = w[..., None] * v[:, i] + (1 - w[..., None]) * v[:, i - 1]
        np.testing.assert_allclose(o[:, i], want, rtol=1e-12, atol=1e-13)


def test_brute_force_loops():
    # Independent scalar loops (math.exp, explicit window test) on a tiny case.
    B, T, H, D, W = 1, 9, 2, 3, 4
    q, k, v = (_rand((B, T, H, D), s) for s in (12, 13, 14))
    o = oracle.swa_attention(q, k, v, window=W)
    for h in range(H):
        for i in range(T):
            js = [j for j in range(T) if j <= i and i - j < W]
            sc = [sum(q[0, i, h, d] * k[0, j, h, d] for d in range(D)) / math.sqrt(D) for j in js]
            mx = max(sc)
            e = [math.exp(s - mx) for s in sc]
            z = sum(e)
            for d in range(D):
                want = sum(e[n] * v[0, j, h, d] for n, j in enumerate(js)) / z
                assert abs(o[0, i, h, d] - want) < 1e-12


def test_window_locality():
    # Keys at j <= i - W never influence o_i; the key at j = i - W + 1 does.
    B, T, H, D, W = 1, 30, 2, 8, 6
    q, k, v = (_rand((B, T, H, D), s) for s in (15, 16, 17))
    base = oracle.swa_attention(q, k, v, window=W)
    i = 20
    k2, v2 = k.copy(), v.copy()
    k2[:, i - W] += 5.0
    v2[:, i - W] -= 3.0
    o2 = oracle.swa_attention(q, k2, v2, window=W)
    np.testing.assert_array_equal(o2[:, i], base[:, i])
    k3 = k.copy()
    k3[:, i - W + 1] += 5.0
    o3 = oracle.swa_attention(q, k3, v, window=W)
    assert np.max(np.abs(o3[:, i] - base[:, i])) > 1e-3


def test_rows_subset_matches_full():
    B, T, H, D, W = 2, 50, 2, 8, 7
    q, k, v = (_rand((B, T, H, D), s) for s in (18, 19, 20))
    full = oracle.swa_attention(q, k, v, window=W)
    rows = [0, 6, 7, 49]
    np.testing.assert_array_equal(oracle.swa_attention_rows(q, k, v, W, rows), full[:, rows])


def test_c0_golden_fixture():
    # Regression pin: the tiny fp32 config's expected output stored by
    # tests/golden/make_golden.py (which calls only oracle/ and synth/).
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "c0_swa_rope_fp32.npz")
    g = np.load(path)
    q, k, v = synth.attention_qkv(1, 64, 2, 64, seed=0)
    pos = np.arange(64)
    o = oracle.swa_attention(oracle.rope(q, pos, 1e6), oracle.rope(k, pos, 1e6), v, window=16)
    np.testing.assert_allclose(o, g["o"], rtol=0, atol=1e-12)
