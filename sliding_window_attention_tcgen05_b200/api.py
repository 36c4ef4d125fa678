"""PyTorch-facing wrappers of the libvx entry points (argument marshalling only).

Tensors are CUDA torch tensors; bf16 data is ``torch.bfloat16``.  Every call
is enqueued on the current torch CUDA stream.  Workspaces are plain uint8
device tensors, sized by the library's own vx_*_workspace queries.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import torch

from ._lib import VX_BF16, VX_F32, VxKvRing, VxLayerCfg, VxLayerParams, VxLayerWeights, check, lib


@dataclass(frozen=True)
class LayerCfg:
    """Shape of one encoder layer (mirrors vx_layer_cfg)."""

    d_model: int = 1280
    n_heads: int = 32
    head_dim: int = 64
    ffn_hidden: int = 5120
    window: int = 750
    rope_theta: float = 1e6
    eps: float = 1e-5

    @property
    def hd(self) -> int:
        return self.n_heads * self.head_dim

    def c(self) -> VxLayerCfg:
        return VxLayerCfg(self.d_model, self.n_heads, self.head_dim, self.ffn_hidden, self.window,
                          self.rope_theta, self.eps)


VOXTRAL_RT = LayerCfg()


def _stream() -> C.c_void_p:
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return C.c_void_p(t.data_ptr())


class Workspace:
    """A device scratch buffer; grows on demand, never shrinks."""

    def __init__(self, nbytes: int = 0, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)

    def get(self, nbytes: int):
        if self.buf.numel() < nbytes:
            self.buf = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        return C.c_void_p(self.buf.data_ptr()), C.c_size_t(self.buf.numel())

    def ptr(self):
        return C.c_void_p(self.buf.data_ptr())


_default_ws: dict = {}


def _ws(ws: Workspace | None, nbytes: int, device) -> Workspace:
    if ws is None:
        key = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
        ws = _default_ws.get(key)
        if ws is None:
            ws = _default_ws[key] = Workspace(256, device=torch.device("cuda", key))
    ws.get(nbytes)
    return ws


def set_wait_timeout_ns(ns: int) -> None:
    lib.vx_set_wait_timeout_ns(int(ns))


def status_reset(ws: Workspace) -> None:
    check(lib.vx_status_reset(ws.ptr(), _stream()), "vx_status_reset")


def status_check(ws: Workspace) -> int:
    """Synchronises the current stream; returns the status code (0 or VX_ERR_DEVICE_TIMEOUT)."""
    return lib.vx_status_check(ws.ptr(), _stream())


def selftest_wait_timeout(ws: Workspace, timeout_ns: int) -> None:
    p, n = ws.get(256)
    check(lib.vx_selftest_wait_timeout(p, n, int(timeout_ns), _stream()), "vx_selftest_wait_timeout")


# ---------------------------------------------------------------- attention

def swa_attn_fwd(q, k, v, window: int, apply_rope: bool = True, rope_theta: float = 1e6, pos0: int = 0,
                 scale: float = 0.0, out=None, ws: Workspace | None = None):
    """Causal sliding-window attention, q/k/v/out [B, T, H, 64] (fp32 or bf16)."""
    B, T, H, D = q.shape
    if q.dtype == torch.float32:
        dt = VX_F32
    elif q.dtype == torch.bfloat16:
        dt = VX_BF16
    else:
        raise TypeError("q/k/v must be float32 or bfloat16")
    if out is None:
        out = torch.empty_like(q)
    need = lib.vx_swa_attn_workspace(dt, B, T, H, D, int(apply_rope))
    ws = _ws(ws, need, q.device)
    p, n = ws.get(need)
    check(lib.vx_swa_attn_fwd(_p(q), _p(k), _p(v), _p(out), dt, B, T, H, D, window, int(apply_rope),
                              rope_theta, pos0, scale, p, n, _stream()), "vx_swa_attn_fwd")
    return out


def rms_norm_fwd(x, g, eps=1e-5, residual=None, h_out=None, out_dtype=torch.bfloat16, out=None,
                 ws: Workspace | None = None):
    d = x.shape[-1]
    M = x.numel() // d
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype, device=x.device)
    dt = VX_BF16 if out.dtype == torch.bfloat16 else VX_F32
    ws = _ws(ws, 256, x.device)
    p, n = ws.get(256)
    check(lib.vx_rms_norm_fwd(_p(x), _p(residual), _p(g), _p(h_out), _p(out), dt, M, d, eps, p, n, _stream()),
          "vx_rms_norm_fwd")
    return out


# ------------------------------------------------------------------ weights

class PackedLayer:
    """A layer's parameters in the kernels' layout; keeps its tensors alive."""

    def __init__(self, cfg: LayerCfg, params: dict):
        dev = params["wq"].device
        hd, f, d = cfg.hd, cfg.ffn_hidden, cfg.d_model
        self.t = {k: v for k, v in params.items() if v is not None}
        self.wqkv = torch.empty(3 * hd, d, dtype=torch.bfloat16, device=dev)
        self.bqkv = torch.empty(3 * hd, dtype=torch.bfloat16, device=dev)
        self.wgu = torch.empty(2 * f, d, dtype=torch.bfloat16, device=dev)
        self.bgu = torch.empty(2 * f, dtype=torch.bfloat16, device=dev)
        pr = VxLayerParams(*[_p(params.get(n)) for n, _ in VxLayerParams._fields_])
        check(lib.vx_pack_layer(C.byref(cfg.c()), C.byref(pr), _p(self.wqkv), _p(self.bqkv), _p(self.wgu),
                                _p(self.bgu), _stream()), "vx_pack_layer")
        self.w = VxLayerWeights(_p(params["attn_norm_g"]), _p(self.wqkv), _p(self.bqkv), _p(params["wo"]),
                                _p(params["bo"]), _p(params["ffn_norm_g"]), _p(self.wgu), _p(self.bgu),
                                _p(params["wd"]), _p(params["bd"]))


def pack_layer(cfg: LayerCfg, params: dict) -> PackedLayer:
    """params: bf16 CUDA tensors named as vx_layer_params (bg/bu may be None)."""
    return PackedLayer(cfg, params)


def pack_conv_weight(w):
    """Conv1d weight [out, in, 3] bf16 -> [out, 3, in] bf16."""
    O, Cin, K = w.shape
    assert K == 3
    out = torch.empty(O, 3, Cin, dtype=torch.bfloat16, device=w.device)
    check(lib.vx_pack_conv_weight(_p(w), _p(out), O, Cin, _stream()), "vx_pack_conv_weight")
    return out


def _weights_array(layers):
    arr = (VxLayerWeights * len(layers))()
    for i, L in enumerate(layers):
        arr[i] = L.w
    return arr


# -------------------------------------------------------------------- layer

def encoder_layer_fwd(cfg: LayerCfg, layer: PackedLayer, x, pos0: int = 0, out=None, ws: Workspace | None = None):
    """x: [B, T, d] fp32 -> [B, T, d] fp32."""
    B, T, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    c = cfg.c()
    need = lib.vx_encoder_layer_workspace(C.byref(c), B, T)
    ws = _ws(ws, need, x.device)
    p, n = ws.get(need)
    check(lib.vx_encoder_layer_fwd(C.byref(c), C.byref(layer.w), _p(x), _p(out), B, T, pos0, p, n, _stream()),
          "vx_encoder_layer_fwd")
    return out


def conv_stem_fwd(mel, w1p, b1, w2p, b2, out=None, ws: Workspace | None = None):
    """mel [B, n_mels, Tm] fp32 -> [B, (Tm-1)//2+1, d] fp32 (packed conv weights)."""
    B, nm, Tm = mel.shape
    d = w1p.shape[0]
    To = (Tm - 1) // 2 + 1
    if out is None:
        out = torch.empty(B, To, d, dtype=torch.float32, device=mel.device)
    need = lib.vx_conv_stem_workspace(B, nm, Tm, d)
    ws = _ws(ws, need, mel.device)
    p, n = ws.get(need)
    check(lib.vx_conv_stem_fwd(_p(mel), _p(w1p), _p(b1), _p(w2p), _p(b2), _p(out), B, nm, Tm, d, p, n,
                               _stream()), "vx_conv_stem_fwd")
    return out


class ConvCache:
    """Conv padding cache of one set of streams for conv_stem_step: the last
    two mel frames ([S, 2, n_mels] bf16) and conv1 outputs ([S, 2, d] bf16)."""

    def __init__(self, S: int, n_mels: int, d: int, device="cuda"):
        self.x = torch.zeros(S, 2, n_mels, dtype=torch.bfloat16, device=device)
        self.h1 = torch.zeros(S, 2, d, dtype=torch.bfloat16, device=device)

    def reset(self):
        self.x.zero_()
        self.h1.zero_()


def conv_stem_step(mel_new, w1p, b1, w2p, b2, cache: ConvCache, out=None, ws: Workspace | None = None):
    """One streaming chunk: mel_new [S, n_mels, n_new] fp32 -> [S, n_new // 2, d] fp32; updates cache."""
    S, nm, n = mel_new.shape
    d = w1p.shape[0]
    if out is None:
        out = torch.empty(S, n // 2, d, dtype=torch.float32, device=mel_new.device)
    need = lib.vx_conv_stem_step_workspace(S, nm, n, d)
    ws = _ws(ws, need, mel_new.device)
    p, nb = ws.get(need)
    check(lib.vx_conv_stem_step(_p(mel_new), _p(w1p), _p(b1), _p(w2p), _p(b2), _p(cache.x), _p(cache.h1), _p(out),
                                S, nm, n, d, p, nb, _stream()), "vx_conv_stem_step")
    return out


def log_mel_fwd(audio, center: bool = True, out=None, ws: Workspace | None = None):
    """Streaming log-mel frontend: audio [B, N] fp32 at 16 kHz -> [B, 128, F] fp32."""
    B, N = audio.shape
    F = N // 160 if center else (1 + (N - 400) // 160 if N >= 400 else 0)
    if out is None:
        out = torch.empty(B, 128, F, dtype=torch.float32, device=audio.device)
    need = lib.vx_log_mel_workspace(B, N)
    ws = _ws(ws, need, audio.device)
    p, n = ws.get(need)
    check(lib.vx_log_mel_fwd(_p(audio), _p(out), B, N, int(center), p, n, _stream()), "vx_log_mel_fwd")
    return out


def projector_fwd(x, w1, w2, out=None, ws: Workspace | None = None):
    """Audio projector: x [B, T, d] fp32 -> [B, T // 4, hidden] fp32 (w1 [hidden, 4d], w2 [hidden, hidden] bf16)."""
    B, T, d = x.shape
    hidden = w1.shape[0]
    if out is None:
        out = torch.empty(B, T // 4, hidden, dtype=torch.float32, device=x.device)
    need = lib.vx_projector_workspace(B, T, d, hidden)
    ws = _ws(ws, need, x.device)
    p, n = ws.get(need)
    check(lib.vx_projector_fwd(_p(x), _p(w1), _p(w2), _p(out), B, T, d, hidden, p, n, _stream()), "vx_projector_fwd")
    return out


def encoder_fwd(cfg: LayerCfg, mel, w1p, b1, w2p, b2, layers, final_g, out=None, ws: Workspace | None = None):
    B, nm, Tm = mel.shape
    To = (Tm - 1) // 2 + 1
    if out is None:
        out = torch.empty(B, To, cfg.d_model, dtype=torch.float32, device=mel.device)
    c = cfg.c()
    need = lib.vx_encoder_workspace(C.byref(c), B, nm, Tm)
    ws = _ws(ws, need, mel.device)
    p, n = ws.get(need)
    arr = _weights_array(layers)
    check(lib.vx_encoder_fwd(C.byref(c), _p(mel), B, nm, Tm, _p(w1p), _p(b1), _p(w2p), _p(b2), arr, len(layers),
                             _p(final_g), _p(out), p, n, _stream()), "vx_encoder_fwd")
    return out


# ---------------------------------------------------------------- streaming

class KVRing:
    """Per-layer ring K/V cache: k, v [L, S, H, W, 64] bf16 and pos [S] int64."""

    def __init__(self, cfg: LayerCfg, n_layers: int, n_streams: int, device=None):
        device = torch.device(device or "cuda")
        shape = (n_layers, n_streams, cfg.n_heads, cfg.window, cfg.head_dim)
        self.k = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.v = torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.pos = torch.zeros(n_streams, dtype=torch.int64, device=device)
        self.n_layers, self.n_streams, self.window = n_layers, n_streams, cfg.window

    def c(self) -> VxKvRing:
        return VxKvRing(_p(self.k), _p(self.v), _p(self.pos), self.n_layers, self.n_streams, self.window)


def stream_prefill(cfg: LayerCfg, layers, ring: KVRing, x, final_g=None, out=None, ws: Workspace | None = None):
    """x: [S, T, d] fp32 -> [S, T, d] fp32; fills the ring and sets pos = T."""
    S, T, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    c = cfg.c()
    need = lib.vx_encoder_layer_workspace(C.byref(c), S, T)
    ws = _ws(ws, need, x.device)
    p, n = ws.get(need)
    r = ring.c()
    check(lib.vx_stream_prefill(C.byref(c), _weights_array(layers), C.byref(r), _p(x), _p(out), T, _p(final_g),
                                p, n, _stream()), "vx_stream_prefill")
    return out


def stream_step(cfg: LayerCfg, layers, ring: KVRing, x_new, final_g=None, out=None, ws: Workspace | None = None):
    """x_new: [S, n_new, d] fp32 -> [S, n_new, d] fp32; advances pos by n_new."""
    S, n_new, d = x_new.shape
    if out is None:
        out = torch.empty_like(x_new)
    c = cfg.c()
    need = lib.vx_stream_step_workspace(C.byref(c), S, n_new)
    ws = _ws(ws, need, x_new.device)
    p, n = ws.get(need)
    r = ring.c()
    check(lib.vx_stream_step(C.byref(c), _weights_array(layers), C.byref(r), _p(x_new), _p(out), n_new,
                             _p(final_g), p, n, _stream()), "vx_stream_step")
    return out
