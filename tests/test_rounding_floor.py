"""Derivation of the 32-layer encoder tolerance (CPU only).

The GPU path rounds every tensor-core operand to bf16.  Two kinds of rounding
are in that list:
  * forced by the configs' "bf16 weights and activations": every activation
    that is a GEMM operand or is stored between kernels -- the RMSNorm outputs
    (QKV and gate/up operands), q/k/v, the attention output (O-projection
    operand), the SwiGLU activation (down-projection operand) and the
    conv-stem hidden frames (conv2 operand);
  * a choice of this implementation: the softmax probabilities P, rounded to
    bf16 so that P V runs on the tensor cores (an fp32 P V on CUDA cores would
    not round them).
This test runs the oracle's float64 arithmetic with those roundings added
(nothing else changed), once with the forced ones only and once with bf16 P as
well, and measures the distance to the plain oracle on the frames that
tests/test_gpu_layer.py::test_c4_full_encoder_prefix compares.  The forced
roundings alone give max-abs 3.8e-2 (bf16 P as well: 3.6e-2): after 32 layers
any implementation with bf16 activations sits above the 3e-2 max-abs bar,
while the relative L2 error stays under 1e-2 (7e-3).
Hence the 32-layer encoder test keeps rel-L2 <= 1e-2 and bounds max-abs by
C4_MAX_ABS below (the floor measured here, 3.6e-2, plus headroom).  The same
holds for the 32-layer streaming step, whose output is the unnormalised
residual stream (values up to about +-7): its floor on the sampled streams of
tests/test_gpu_stream.py::test_c3_full_size_sampled_streams is measured by
the second test and bounded by C3_MAX_ABS.  Every single-layer and attention
test keeps the 3e-2 bar.
"""
import functools

import numpy as np
import pytest

import oracle
import synth

C4_MAX_ABS = 5e-2
C4_FRAMES = 256
C3_MAX_ABS = 1e-1
C3_SAMPLE = (0, 37, 63)
# The streaming config as stated (ring filled by a prefill of 1000 frames,
# then a 4-frame step; tests/test_gpu_stream.py::test_c3_stated_config_prefill_then_step)
# compares 32-layer outputs of streams 0 and 63.  Its floor, computed by
# tests/derive_stream_floor.py (too slow for this suite: 32 whole-sequence
# layers over 1004 frames twice), is max-abs 7.6e-2 / rel 6.4e-3 on the raw
# residual stream (values up to +-11) and 3.0e-2 / 6.4e-3 after the final
# RMSNorm; the bounds below add headroom, rel-L2 stays at 1e-2.
C3_STATED_MAX_ABS = 1e-1
C3_STATED_NORMED_MAX_ABS = 5e-2


@functools.lru_cache(maxsize=1)
def _stack32():
    return [synth.layer_params(synth.VOXTRAL_RT, seed=synth.layer_seed(1, l)) for l in range(32)]


def _r(x):
    return synth.bf16_round(np.asarray(x, dtype=np.float32)).astype(np.float64)


def _layer_bf16_operands(x, p, dims, round_p=True):
    B, T, _ = x.shape
    H, D, W = dims.n_heads, dims.head_dim, dims.window
    pos = np.arange(T)
    f = lambda a: np.asarray(a, dtype=np.float64)
    y0 = _r(oracle.rms_norm(x, p["attn_norm_g"], dims.eps))
    q = _r(oracle.rope((y0 @ f(p["wq"]).T + f(p["bq"])).reshape(B, T, H, D), pos, dims.rope_theta))
    k = _r(oracle.rope((y0 @ f(p["wk"]).T).reshape(B, T, H, D), pos, dims.rope_theta))
    v = _r((y0 @ f(p["wv"]).T + f(p["bv"])).reshape(B, T, H, D))
    a = np.empty((B, T, H, D))
    for i in range(T):
        lo = max(0, i - W + 1)
        s = np.einsum("bhd,bjhd->bhj", q[:, i], k[:, lo:i + 1]) / np.sqrt(D)
        e = np.exp(s - s.max(-1, keepdims=True))
        a[:, i] = np.einsum("bhj,bjhd->bhd", _r(e) if round_p else e, v[:, lo:i + 1]) / e.sum(-1, keepdims=True)
    h = x + _r(a.reshape(B, T, H * D)) @ f(p["wo"]).T + f(p["bo"])
    y1 = _r(oracle.rms_norm(h, p["ffn_norm_g"], dims.eps))
    act = _r(oracle.silu(y1 @ f(p["wg"]).T) * (y1 @ f(p["wu"]).T))
    return h + act @ f(p["wd"]).T + f(p["bd"])


def _stem_bf16_operands(mel, conv):
    f = lambda a: np.asarray(a, dtype=np.float64)
    w1, b1, w2, b2 = f(conv["w1"]), f(conv["b1"]), f(conv["w2"]), f(conv["b2"])
    B, C, Tm = mel.shape
    xp = _r(np.concatenate([np.zeros((B, C, 2)), mel], axis=2))
    h1 = np.zeros((B, w1.shape[0], Tm)) + b1[None, :, None]
    for k in range(3):
        h1 += np.einsum("oc,bct->bot", w1[:, :, k], xp[:, :, k:k + Tm], optimize=True)
    h1 = _r(oracle.gelu(h1))
    To = oracle.conv_out_len(Tm)
    hp = np.concatenate([np.zeros((B, h1.shape[1], 2)), h1], axis=2)
    h2 = np.zeros((B, w2.shape[0], To)) + b2[None, :, None]
    for k in range(3):
        h2 += np.einsum("oc,bct->bot", w2[:, :, k], hp[:, :, k:k + 2 * To - 1:2], optimize=True)
    return np.transpose(oracle.gelu(h2), (0, 2, 1))


@pytest.mark.slow
@pytest.mark.parametrize("round_p", [False, True])
def test_bf16_operand_floor_of_the_32_layer_encoder(round_p):
    dims = synth.VOXTRAL_RT
    layers = _stack32()
    conv = synth.conv_params(seed=3)
    g = synth.final_norm_gain(dims.d_model, seed=5)
    mel = synth.mel(4, 128, 6000, seed=4)[:1, :, :2 * C4_FRAMES].astype(np.float64)
    ref = oracle.encoder(mel, conv, layers, g, dims)
    x = _stem_bf16_operands(mel, conv)
    for p in layers:
        x = _layer_bf16_operands(x, p, dims, round_p)
    out = oracle.rms_norm(x, g, dims.eps)
    err = out - ref
    max_abs = np.abs(err).max()
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    # the floor exceeds the single-layer bar but not the derived one
    assert 3e-2 < max_abs < C4_MAX_ABS, max_abs
    assert rel < 1e-2, rel


def _stream_layer_bf16_operands(x, p, dims, rk, rv, pos):
    """oracle.stream_step_layer with the GPU's bf16 operand roundings added."""
    S, n, _ = x.shape
    H, D, W = dims.n_heads, dims.head_dim, dims.window
    f = lambda a: np.asarray(a, dtype=np.float64)
    y0 = _r(oracle.rms_norm(x, p["attn_norm_g"], dims.eps))
    a = np.empty((S, n, H, D))
    for s in range(S):
        ps = int(pos[s])
        pp = ps + np.arange(n)
        q = _r(oracle.rope((y0[s] @ f(p["wq"]).T + f(p["bq"])).reshape(n, H, D), pp, dims.rope_theta))
        k = _r(oracle.rope((y0[s] @ f(p["wk"]).T).reshape(n, H, D), pp, dims.rope_theta))
        v = _r((y0[s] @ f(p["wv"]).T + f(p["bv"])).reshape(n, H, D))
        for i in range(n):
            fq = ps + i
            fr = range(max(0, fq - W + 1), fq + 1)
            K = np.stack([rk[s, :, fj % W] if fj < ps else k[fj - ps] for fj in fr], axis=1)
            V = np.stack([rv[s, :, fj % W] if fj < ps else v[fj - ps] for fj in fr], axis=1)
            sc = np.einsum("hd,hjd->hj", q[i], K) / np.sqrt(D)
            e = np.exp(sc - sc.max(-1, keepdims=True))
            a[s, i] = np.einsum("hj,hjd->hd", _r(e), V) / e.sum(-1, keepdims=True)
    h = x + _r(a.reshape(S, n, H * D)) @ f(p["wo"]).T + f(p["bo"])
    y1 = _r(oracle.rms_norm(h, p["ffn_norm_g"], dims.eps))
    act = _r(oracle.silu(y1 @ f(p["wg"]).T) * (y1 @ f(p["wu"]).T))
    return h + act @ f(p["wd"]).T + f(p["bd"])


@pytest.mark.slow
def test_bf16_operand_floor_of_the_32_layer_stream_step():
    dims = synth.VOXTRAL_RT
    layers = _stack32()
    rings = [synth.ring_kv(len(C3_SAMPLE), dims.n_heads, dims.window, dims.head_dim, seed=1000 + l)
             for l in range(32)]
    x = synth.frames(64, 4, dims.d_model, seed=3)[list(C3_SAMPLE)].astype(np.float64)
    pos = np.full(len(C3_SAMPLE), 1000)
    ref, _, _ = oracle.stream_step(x, layers, dims, rings, pos)
    h = x
    for p, (rk, rv) in zip(layers, rings):
        h = _stream_layer_bf16_operands(h, p, dims, np.asarray(rk, np.float64), np.asarray(rv, np.float64), pos)
    err = h - ref
    max_abs = np.abs(err).max()
    rel = np.linalg.norm(err) / np.linalg.norm(ref)
    assert 3e-2 < max_abs < C3_MAX_ABS, max_abs
    assert rel < 1e-2, rel
