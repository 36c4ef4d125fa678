"""CPU checks of the C-ABI library: it loads, exports every entry point that
include/vx.h declares, and rejects bad arguments on the host (no GPU needed:
these paths return before any CUDA call)."""
import ctypes as C
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "vx.h")).read()
    return sorted(set(re.findall(r"^VX_API\s+[\w\s\*]*?\b(vx_\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_four_operations():
    names = _declared()
    for n in ("vx_swa_attn_fwd", "vx_encoder_layer_fwd", "vx_stream_step", "vx_conv_stem_fwd"):
        assert n in names


def test_library_exports_every_declared_symbol():
    import sliding_window_attention_tcgen05_b200 as vx
    lib = C.CDLL(vx.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_declared()) == set(vx._lib.SIGNATURES), "binding signatures drift from the header"


def test_workspace_queries_are_host_only():
    import sliding_window_attention_tcgen05_b200 as vx
    lib = vx.lib
    c = vx.VOXTRAL_RT.c()
    assert lib.vx_encoder_layer_workspace(C.byref(c), 1, 1500) > 1500 * 1280 * 4
    assert lib.vx_stream_step_workspace(C.byref(c), 64, 4) > 256 * 6144 * 2
    assert lib.vx_conv_stem_workspace(4, 128, 6000, 1280) >= 4 * 6002 * (128 + 1280) * 2
    assert lib.vx_swa_attn_workspace(1, 8, 6000, 32, 64, 1) >= 2 * 8 * 6000 * 32 * 64 * 2
    assert lib.vx_swa_attn_workspace(1, 8, 6000, 32, 64, 0) == 1024


def test_null_arguments_are_rejected_without_a_gpu():
    import sliding_window_attention_tcgen05_b200 as vx
    lib = vx.lib
    st = lib.vx_swa_attn_fwd(None, None, None, None, 1, 1, 8, 1, 64, 4, 1, 1e6, 0, 0.0, None, 0, None)
    assert st == 1
    assert b"null" in lib.vx_last_error()
    c = vx.VOXTRAL_RT.c()
    assert lib.vx_encoder_layer_fwd(C.byref(c), None, None, None, 1, 1, 0, None, 0, None) == 1
    bad = vx.LayerCfg(head_dim=128).c()
    assert lib.vx_encoder_layer_fwd(C.byref(bad), None, None, None, 1, 1, 0, None, 0, None) == 2
    assert lib.vx_conv_stem_fwd(None, None, None, None, None, None, 1, 128, 10, 1280, None, 0, None) == 1
    assert lib.vx_stream_step(C.byref(c), None, None, None, None, 4, None, None, 0, None) == 1


def test_package_has_no_cpu_fallback():
    # The binding only marshals arguments into libvx: no torch compute ops and
    # no import of the oracle.
    pkg = os.path.join(ROOT, "sliding_window_attention_tcgen05_b200")
    for fn in ("api.py", "_lib.py", "__init__.py"):
        src = open(os.path.join(pkg, fn)).read()
        assert "oracle" not in src
        for op in ("torch.matmul", "torch.nn.functional", "softmax", "einsum", "@ "):
            assert op not in src, (fn, op)
