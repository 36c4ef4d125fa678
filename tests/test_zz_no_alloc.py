"""vx_swa_attn_fwd_noalloc: the attention call for callers that cannot
allocate device memory (real-time audio callbacks, plug-in hosts that own
every allocation, fixed memory budgets).  Its scratch is a static device
array inside libvx; these tests call it through the C ABI and compare it with
vx_swa_attn_fwd (which uses a caller-supplied workspace) on two calls in a
row, and with the float64 oracle, within the tolerances the other GPU tests
use; they also check both sides of its size limit.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import BF16_MAX_ABS, BF16_REL_L2, F32_MAX_ABS, dev, host

pytestmark = pytest.mark.gpu


def _lib():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def _noalloc(vx, q, k, v, o, window, apply_rope=1, theta=1e6, pos0=0):
    dt = 1 if q.dtype == torch.bfloat16 else 0
    B, T, H, D = q.shape
    P = lambda t: C.c_void_p(t.data_ptr())
    return vx.lib.vx_swa_attn_fwd_noalloc(P(q), P(k), P(v), P(o), dt, B, T, H, D, window, apply_rope, theta,
                                          pos0, 0.0, C.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check(got, want, bf16):
    g = host(got)
    w = want if isinstance(want, np.ndarray) else host(want)
    err = np.abs(g - w).max()
    if bf16:
        rel = np.linalg.norm(g - w) / np.linalg.norm(w)
        assert err <= BF16_MAX_ABS and rel <= BF16_REL_L2, (err, rel)
    else:
        assert err <= F32_MAX_ABS, err


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_entry_point_on_two_calls(dtype):
    vx = _lib()
    bf16 = dtype == torch.bfloat16
    shapes = [(2, 700, 8, 300, 0), (1, 1500, 32, 750, 1000)]   # (B, T, H, window, pos0), two calls in a row
    for call, (B, T, H, W, pos0) in enumerate(shapes):
        q, k, v = synth.attention_qkv(B, T, H, 64, seed=500 + call, bf16=bf16)
        q, k, v = (dev(x, dtype) for x in (q, k, v))
        o = torch.empty_like(q)
        assert _noalloc(vx, q, k, v, o, W, pos0=pos0) == 0, vx.lib.vx_last_error()
        ref = vx.swa_attn_fwd(q, k, v, W, pos0=pos0)
        torch.cuda.synchronize()
        _check(o, ref, bf16)
        # and against the oracle on sampled rows (the window's edges, the end)
        rows = sorted({0, 1, W - 1, W, T // 2, T - 1})
        pos = pos0 + np.arange(T)
        qh, kh, vh = (host(x) for x in (q, k, v))
        want = oracle.swa_attention_rows(oracle.rope(qh, pos, 1e6), oracle.rope(kh, pos, 1e6), vh, W, rows)
        _check(o[:, rows], want, bf16)


def test_noalloc_without_rope_and_repeat_is_deterministic():
    vx = _lib()
    q, k, v = synth.attention_qkv(1, 500, 4, 64, seed=7, bf16=True)
    q, k, v = (dev(x, torch.bfloat16) for x in (q, k, v))
    a, b = torch.empty_like(q), torch.empty_like(q)
    assert _noalloc(vx, q, k, v, a, 128, apply_rope=0) == 0
    assert _noalloc(vx, q, k, v, b, 128, apply_rope=0) == 0
    ref = vx.swa_attn_fwd(q, k, v, 128, apply_rope=False)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    _check(a, ref, True)


def test_noalloc_size_limit_both_sides():
    # bf16 with RoPE: 2 * roundup256(B*T*H*128) <= 32 MiB, i.e.
    # B*T*H <= 131072.  B=1, H=32: T = 4096 fits, T = 4097 does not.
    vx = _lib()
    H, W = 32, 750
    q, k, v = synth.attention_qkv(1, 4097, H, 64, seed=9, bf16=True)
    q, k, v = (dev(x, torch.bfloat16) for x in (q, k, v))
    o = torch.empty_like(q)
    assert _noalloc(vx, q, k, v, o, W) == 1
    assert b"static limit" in vx.lib.vx_last_error()
    qs, ks, vs = (x[:, :4096].contiguous() for x in (q, k, v))
    os_ = torch.empty_like(qs)
    assert _noalloc(vx, qs, ks, vs, os_, W) == 0, vx.lib.vx_last_error()
    ref = vx.swa_attn_fwd(qs, ks, vs, W)
    torch.cuda.synchronize()
    _check(os_, ref, True)
    # without RoPE it needs no scratch beyond the status word and runs at any size
    q2 = torch.zeros(2, 4096, 32, 64, dtype=torch.bfloat16, device="cuda")
    o2 = torch.empty_like(q2)
    assert _noalloc(vx, q2, q2, q2, o2, 750, apply_rope=0) == 0
    # fp32 with RoPE: 2 * B*T*H*256 <= 32 MiB, i.e. B*T*H <= 65536; B=1, H=16:
    # T = 4096 fits, 4097 does not
    qf = torch.zeros(1, 4097, 16, 64, dtype=torch.float32, device="cuda")
    of = torch.empty_like(qf)
    assert _noalloc(vx, qf, qf, qf, of, 750) == 1
    qf2 = qf[:, :4096].contiguous()
    assert _noalloc(vx, qf2, qf2, qf2, torch.empty_like(qf2), 750) == 0, vx.lib.vx_last_error()
    torch.cuda.synchronize()
