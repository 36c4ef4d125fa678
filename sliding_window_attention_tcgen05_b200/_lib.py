"""ctypes declarations of libvx (include/vx.h).  Argument marshalling only.

Loading fails loudly when libvx.so has not been built: there is no other
implementation of these operations in this package.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libvx.so")

VX_OK, VX_ERR_INVALID_ARG, VX_ERR_UNSUPPORTED, VX_ERR_CUDA, VX_ERR_DEVICE_TIMEOUT = range(5)
VX_F32, VX_BF16 = 0, 1
STATUS_NAMES = {0: "VX_OK", 1: "VX_ERR_INVALID_ARG", 2: "VX_ERR_UNSUPPORTED", 3: "VX_ERR_CUDA",
                4: "VX_ERR_DEVICE_TIMEOUT"}


class VxLayerCfg(C.Structure):
    _fields_ = [("d_model", C.c_int), ("n_heads", C.c_int), ("head_dim", C.c_int),
                ("ffn_hidden", C.c_int), ("window", C.c_int), ("rope_theta", C.c_float),
                ("eps", C.c_float)]


class VxLayerParams(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm_g", "wq", "wk", "wv", "bq", "bv", "wo", "bo",
                                           "ffn_norm_g", "wg", "wu", "bg", "bu", "wd", "bd")]


class VxLayerWeights(C.Structure):
    _fields_ = [(n, C.c_void_p) for n in ("attn_norm_g", "wqkv", "bqkv", "wo", "bo", "ffn_norm_g",
                                           "wgu", "bgu", "wd", "bd")]


class VxKvRing(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("pos", C.c_void_p), ("n_layers", C.c_int),
                ("n_streams", C.c_int), ("window", C.c_int)]


# name -> (restype, argtypes); this list is the exported ABI of include/vx.h.
_P, _I, _F, _S, _U64, _I64 = C.c_void_p, C.c_int, C.c_float, C.c_size_t, C.c_uint64, C.c_int64
_CFG, _W, _R = C.POINTER(VxLayerCfg), C.POINTER(VxLayerWeights), C.POINTER(VxKvRing)
SIGNATURES = {
    "vx_last_error": (C.c_char_p, []),
    "vx_version": (C.c_char_p, []),
    "vx_set_wait_timeout_ns": (None, [_U64]),
    "vx_trace_enable": (None, [_I]),
    "vx_trace_read": (_I, [C.c_char_p, _S]),
    "vx_launch_count": (_U64, []),
    "vx_status_reset": (_I, [_P, _P]),
    "vx_status_check": (_I, [_P, _P]),
    "vx_pack_layer": (_I, [_CFG, C.POINTER(VxLayerParams), _P, _P, _P, _P, _P]),
    "vx_pack_conv_weight": (_I, [_P, _P, _I, _I, _P]),
    "vx_swa_attn_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I64, _F, _P, _S, _P]),
    "vx_swa_attn_workspace": (_S, [_I, _I, _I, _I, _I, _I]),
    "vx_swa_attn_fwd_noalloc": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _F, _I64, _F, _P]),
    "vx_rms_norm_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _F, _P, _S, _P]),
    "vx_encoder_layer_fwd": (_I, [_CFG, _W, _P, _P, _I, _I, _I64, _P, _S, _P]),
    "vx_encoder_layer_workspace": (_S, [_CFG, _I, _I]),
    "vx_conv_stem_fwd": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "vx_conv_stem_workspace": (_S, [_I, _I, _I, _I]),
    "vx_conv_stem_step": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "vx_conv_stem_step_workspace": (_S, [_I, _I, _I, _I]),
    "vx_projector_fwd": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P, _S, _P]),
    "vx_projector_workspace": (_S, [_I, _I, _I, _I]),
    "vx_log_mel_fwd": (_I, [_P, _P, _I, _I, _I, _P, _S, _P]),
    "vx_log_mel_workspace": (_S, [_I, _I]),
    "vx_encoder_fwd": (_I, [_CFG, _P, _I, _I, _I, _P, _P, _P, _P, _W, _I, _P, _P, _P, _S, _P]),
    "vx_encoder_workspace": (_S, [_CFG, _I, _I, _I]),
    "vx_stream_prefill": (_I, [_CFG, _W, _R, _P, _P, _I, _P, _P, _S, _P]),
    "vx_stream_step": (_I, [_CFG, _W, _R, _P, _P, _I, _P, _P, _S, _P]),
    "vx_stream_step_workspace": (_S, [_CFG, _I, _I]),
    "vx_selftest_wait_timeout": (_I, [_P, _S, _U64, _P]),
}


def load(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libvx.so not found at {path}; build it with "
            "`python sliding_window_attention_tcgen05_b200/build.py` (nvcc, sm_100a)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = load()


class VxError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = lib.vx_last_error().decode(errors="replace")
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


def check(status: int, where: str) -> None:
    if status != VX_OK:
        raise VxError(status, where)
