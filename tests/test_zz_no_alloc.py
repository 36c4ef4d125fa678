"""vx_swa_attn_fwd_noalloc: the attention call for callers that cannot
allocate device memory (real-time audio callbacks, plug-in hosts that own
every allocation, fixed memory budgets).  Its scratch is a static device
array inside libvx; these tests call it through the C ABI and compare it with
vx_swa_attn_fwd (which uses a caller-supplied workspace) on two calls in a
row, within the tolerances the other GPU tests use.

This file is named to be collected last, so a run that stops at the first
failure has already run every other test."""
import ctypes as C

import numpy as np
import pytest
import torch

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
    g, w = host(got), host(want)
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


def test_noalloc_rejects_sizes_beyond_its_static_scratch():
    vx = _lib()
    # bf16: B*T*H must stay <= 131072; 2 x 4096 x 32 = 262144 is too large
    q = torch.zeros(2, 4096, 32, 64, dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    assert _noalloc(vx, q, q, q, o, 750) == 1
    assert b"static limit" in vx.lib.vx_last_error()
    # without RoPE it needs no scratch and runs
    assert _noalloc(vx, q, q, q, o, 750, apply_rope=0) == 0
    torch.cuda.synchronize()
