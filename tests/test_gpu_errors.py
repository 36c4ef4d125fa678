"""Failure detection on the GPU without faulting it: a bounded in-kernel wait
that runs out reports VX_ERR_DEVICE_TIMEOUT through the workspace status word
and leaves the context usable; argument errors are rejected on the host."""
import ctypes as C

import numpy as np
import pytest
import torch

import synth
from gpu_util import compare_f32, dev, host

pytestmark = pytest.mark.gpu


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def test_bounded_wait_reports_timeout_and_context_survives():
    vx = _vx()
    ws = vx.Workspace(1 << 20)
    vx.status_reset(ws)
    assert vx.status_check(ws) == 0
    vx.selftest_wait_timeout(ws, 2_000_000)       # 2 ms limit on a barrier nothing arrives on
    assert vx.status_check(ws) == 4               # VX_ERR_DEVICE_TIMEOUT
    assert "expired" in vx.lib.vx_last_error().decode()
    vx.status_reset(ws)
    assert vx.status_check(ws) == 0
    # the context still works
    q, k, v = synth.attention_qkv(1, 64, 2, 64, seed=0)
    o = vx.swa_attn_fwd(dev(q), dev(k), dev(v), window=16, ws=ws)
    assert vx.status_check(ws) == 0
    assert np.all(np.isfinite(host(o)))


def test_regular_calls_leave_status_clear():
    vx = _vx()
    ws = vx.Workspace(1 << 20)
    vx.status_reset(ws)
    q, k, v = synth.attention_qkv(2, 300, 4, 64, seed=1, bf16=True)
    vx.swa_attn_fwd(*(dev(t, torch.bfloat16) for t in (q, k, v)), window=100, ws=ws)
    assert vx.status_check(ws) == 0


def test_argument_errors_are_reported():
    vx = _vx()
    lib = vx.lib
    q = torch.zeros(1, 8, 2, 64, device="cuda")
    ws = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    P = lambda t: C.c_void_p(t.data_ptr())
    s = torch.cuda.current_stream().cuda_stream
    # head_dim != 64 -> unsupported
    assert lib.vx_swa_attn_fwd(P(q), P(q), P(q), P(q), 0, 1, 8, 2, 32, 4, 0, 1e6, 0, 0.0, P(ws), ws.numel(), s) == 2
    # workspace too small
    assert lib.vx_swa_attn_fwd(P(q), P(q), P(q), P(q), 0, 1, 8, 2, 64, 4, 1, 1e6, 0, 0.0, P(ws), 16, s) == 1
    assert "workspace too small" in lib.vx_last_error().decode()
    # misaligned workspace
    assert lib.vx_swa_attn_fwd(P(q), P(q), P(q), P(q), 0, 1, 8, 2, 64, 4, 0, 1e6, 0, 0.0,
                               C.c_void_p(ws.data_ptr() + 8), ws.numel() - 8, s) == 1
    # window 0
    assert lib.vx_swa_attn_fwd(P(q), P(q), P(q), P(q), 0, 1, 8, 2, 64, 0, 0, 1e6, 0, 0.0, P(ws), ws.numel(), s) == 1
    # bad stream-step frame count
    cfg = vx.LayerCfg(d_model=256, n_heads=4, head_dim=64, ffn_hidden=512, window=16)
    ring = vx.KVRing(cfg, 1, 1)
    with pytest.raises(vx.VxError):
        vx.stream_step(cfg, [], ring, torch.zeros(1, 4, 256, device="cuda"))


def test_fp32_path_equals_itself_after_timeout():
    # A timeout in one workspace does not leak into calls on another.
    vx = _vx()
    ws_a, ws_b = vx.Workspace(1 << 20), vx.Workspace(1 << 20)
    vx.status_reset(ws_a); vx.status_reset(ws_b)
    vx.selftest_wait_timeout(ws_a, 1_000_000)
    q, k, v = synth.attention_qkv(1, 64, 2, 64, seed=0)
    o = vx.swa_attn_fwd(dev(q), dev(k), dev(v), window=16, ws=ws_b)
    assert vx.status_check(ws_a) == 4 and vx.status_check(ws_b) == 0
    o2 = vx.swa_attn_fwd(dev(q), dev(k), dev(v), window=16, ws=ws_b)
    compare_f32(host(o), host(o2))
