#!/usr/bin/env python
"""Throughput of the Voxtral Realtime encoder hot path on B200, one JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl vx|reference]

Workload (one "step"): one full encoder layer over one clip of 1500 frames
(d 1280, 32 heads x 64, SwiGLU 5120, causal window 750, RoPE theta 1e6), bf16
operands with fp32 accumulation and an fp32 residual stream: RMSNorm -> QKV
GEMM + RoPE -> sliding-window attention -> O-proj + residual -> RMSNorm ->
gate/up GEMM + SwiGLU -> down GEMM + residual, all in libvx's sm_100a kernels.
Inputs are synthetic and seeded, resident in HBM before the timed region; L2
is flushed (a 256 MiB write) between timed steps, outside the step's events.

`value` is encoder frames/s over all ranks (each rank runs an independent
replica: the path shards by clip with no collective).  `e2e` repeats the
measurement through the same public call with the input copied from pinned
host memory and the output copied back inside the timed region.
`roofline` reports the dominant kernel, timed live with CUDA events on its
launch stream (libvx's trace mode).  On one GPU the line also carries
`components`: the attention-only sweep (TFLOP/s), the 32-layer streaming step
(GB/s) and the full 32-layer encoder (frames/s).  `cpu_baseline` times the
float64 oracle on this host's cores on a bounded sample of the same workload.

`--impl reference` times that oracle alone (the reference arm of this build:
the pages ship no runnable reference), printing the same line with
"impl": "reference".
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import subprocess
import sys
import tempfile
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "encoder frames/sec (1 B200); SWA TFLOP/s & % bf16 peak; stream-step GB/s"
UNIT = "frames/s"
C1 = dict(B=1, T=1500, d=1280, H=32, D=64, F=5120, W=750)
WORKLOAD = ("one encoder layer (C1): B=1 clip x T=1500 frames, d_model 1280, 32 heads x 64, SwiGLU 5120, "
            "causal window 750, RoPE theta 1e6; bf16 operands, fp32 accumulate and residual")
L2_FLUSH_BYTES = 256 << 20


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description="Voxtral Realtime encoder hot-path benchmark")
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=("vx", "reference"), default="vx")
    ap.add_argument("--no-components", action="store_true", help="skip the C2/C3/C4 component timings")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--components-only", default="", help="comma list of c0,c2,c3,c4,next (profiling runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-copy end-to-end pass (profiling runs)")
    ap.add_argument("--no-trace", action="store_true", help="skip the traced per-kernel pass (profiling runs)")
    ap.add_argument("--c3-layers", type=int, default=32, help="layers of the streaming-step component (profiling runs)")
    return ap.parse_args(argv)


# ------------------------------------------------------------ distribution

def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def reduce_max(value: float, device=None) -> float:
    """Max of a scalar over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples (200 ms) of the benchmark GPU; summarised over a window."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.p = subprocess.Popen(["nvidia-smi", "-i", gpu_id, f"--query-gpu={self.FIELDS}",
                                       "--format=csv,noheader,nounits", "-lms", "200"],
                                      stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.p = None

    def stop(self):
        if self.p is not None:
            self.p.terminate()
            try:
                self.p.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.p.kill()
        self.f.flush()

    def summary(self, t0: float, t1: float):
        self.f.seek(0)
        rows = []
        for line in self.f.read().splitlines():
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        inside = [r for r in rows if t0 - 0.25 <= r[0] <= t1 + 0.25] or rows[-3:]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in inside for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": float(np.median([r[1] for r in inside])), "sm_max_mhz": inside[0][2],
                "reasons": reasons, "samples": len(inside)}


# ---------------------------------------------------------------- workload

def make_layer(vx, torch, seed=1, device="cuda"):
    """Random-init bf16 layer weights of the C1 shape (synth distributions), packed."""
    import synth
    cfg = vx.VOXTRAL_RT
    p = synth.layer_params(synth.VOXTRAL_RT, seed=seed)
    t = {k: (None if v is None else torch.from_numpy(v).to(device).to(torch.bfloat16)) for k, v in p.items()}
    return cfg, vx.pack_layer(cfg, t)


def device_layers(vx, torch, n, seed, device):
    """n layers drawn on the device (torch RNG; distributions of synth.layer_params)."""
    cfg = vx.VOXTRAL_RT
    g = torch.Generator(device=device).manual_seed(seed)
    d, hd, f = cfg.d_model, cfg.hd, cfg.ffn_hidden

    def nrm(shape, std, mean=0.0):
        return (torch.randn(shape, generator=g, device=device) * std + mean).to(torch.bfloat16)

    layers = []
    for _ in range(n):
        p = {"attn_norm_g": nrm((d,), 0.02, 1.0), "wq": nrm((hd, d), 0.02), "wk": nrm((hd, d), 0.02),
             "wv": nrm((hd, d), 0.02), "bq": nrm((hd,), 0.01), "bv": nrm((hd,), 0.01),
             "wo": nrm((d, hd), 0.02), "bo": nrm((d,), 0.01), "ffn_norm_g": nrm((d,), 0.02, 1.0),
             "wg": nrm((f, d), 0.02), "wu": nrm((f, d), 0.02), "wd": nrm((d, f), 0.02), "bd": nrm((d,), 0.01),
             "bg": None, "bu": None}
        layers.append(vx.pack_layer(cfg, p))
    return cfg, layers


def gemm_flops(M, d=1280, hd=2048, F=5120):
    return {"gemm_qkv_rope": 2 * M * d * 3 * hd, "gemm_o_residual": 2 * M * hd * d,
            "gemm_gate_up_swiglu": 2 * M * d * 2 * F, "gemm_down_residual": 2 * M * F * d}


def attended_pairs(T, W):
    return sum(min(i + 1, W) for i in range(T))


def attn_flops(B, T, H, D, W):
    return 4 * D * H * B * attended_pairs(T, W)      # QK^T and PV, 2 flops per MAC


def layer_flops(B, T, W=750):
    M = B * T
    return sum(gemm_flops(M).values()) + attn_flops(B, T, 32, 64, W)


def kernel_work(name, B, T):
    """(amount, unit, bound) of algorithmic work of one launch in the C1 layer."""
    M = B * T
    if name in gemm_flops(M):
        return gemm_flops(M)[name], "flop", "tensor"
    if name == "swa_attn_tc":
        return attn_flops(B, T, 32, 64, 750), "flop", "tensor"
    if name == "rmsnorm":
        return M * 1280 * (4 + 2) + 1280 * 2, "byte", "hbm"
    return None, None, None


def src_digest(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "sliding_window_attention_tcgen05_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


KERNEL_SRC = {"gemm_qkv_rope": ("gemm.cu", "vx_common.cuh"), "gemm_o_residual": ("gemm.cu", "vx_common.cuh"),
              "gemm_gate_up_swiglu": ("gemm.cu", "vx_common.cuh"), "gemm_down_residual": ("gemm.cu", "vx_common.cuh"),
              "swa_attn_tc": ("attn.cu", "vx_common.cuh"), "rmsnorm": ("misc.cu",), "ring_attn": ("stream.cu",)}


def ncu_traffic(kernel, workload):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current source of that kernel; else None."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            db = json.load(f)
    except (OSError, ValueError):
        return None
    e = db.get(f"{kernel}@{workload}")
    if not e or e.get("src") != src_digest(*KERNEL_SRC.get(kernel, ())):
        return None
    return e.get("dram_bytes_per_launch")


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return p["hbm_gbs"], p["bf16_tflops"], p.get("bf16_tflops_sustained", p["bf16_tflops"]), "measured"
    except (OSError, ValueError, KeyError):
        return 6650.0, 1590.0, 1400.0, "fallback"


# -------------------------------------------------------------- timed loops

def timed_steps(torch, step, K, flush, stream):
    """K steps, each bracketed by CUDA events on `stream`; L2 flushed between
    steps outside the events.  Returns (mean ms per step, wall t0, wall t1)."""
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0 = time.time()
    for a, b in ev:
        flush()
        a.record(stream)
        step()
        b.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    return sum(a.elapsed_time(b) for a, b in ev) / K, t0, t1


def traced_kernels(vx, torch, step, K, flush):
    """Per-kernel mean duration (ms) over K traced steps, keyed by kernel name."""
    import ctypes
    vx.lib.vx_trace_enable(1)
    acc = {}
    try:
        for _ in range(K):
            flush()
            step()
            buf = ctypes.create_string_buffer(1 << 16)
            vx.lib.vx_trace_read(buf, len(buf))
            for line in buf.value.decode().splitlines():
                name, ms = line.rsplit(" ", 1)
                acc.setdefault(name, []).append(float(ms))
    finally:
        vx.lib.vx_trace_enable(0)
    # launches per step of each name -> mean per launch and per step
    return {k: {"ms_per_launch": float(np.mean(v)), "launches_per_step": len(v) / K,
                "ms_per_step": float(np.sum(v)) / K} for k, v in acc.items()}


# ------------------------------------------------------------- components

def component_c0(vx, torch, flush, hbm, tf):
    """The tiny fp32 case: q, k, v [1, 64, 2, 64] (seed 0, drawn in that order),
    window 16, RoPE theta 1e6 at pos0 0, through the public fp32 attention call
    (RoPE kernel + CUDA-core attention kernel); latency per call, L2 flushed
    between calls outside the events."""
    import synth
    q, k, v = (torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
               for a in synth.attention_qkv(1, 64, 2, 64, seed=0))
    o = torch.empty_like(q)
    ws = vx.Workspace(vx.lib.vx_swa_attn_workspace(0, 1, 64, 2, 64, 1))
    step = lambda: vx.swa_attn_fwd(q, k, v, 16, apply_rope=True, rope_theta=1e6, pos0=0, out=o, ws=ws)
    for _ in range(5):
        step()
    ms, _, _ = timed_steps(torch, step, 200, flush, torch.cuda.current_stream())
    tr = traced_kernels(vx, torch, step, 20, flush)
    fl = attn_flops(1, 64, 2, 64, 16)
    return {"us_per_call": ms * 1e3, "kernels_us": {k2: v2["ms_per_launch"] * 1e3 for k2, v2 in tr.items()},
            "mflop": fl / 1e6, "note": "launch-latency bound: 0.46 MFLOP"}


def component_c2(vx, torch, flush, hbm, tf):
    out = {}
    g = torch.Generator(device="cuda").manual_seed(20)
    for T in (1500, 3000, 6000):
        q, k, v = (torch.randn(8, T, 32, 64, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
        o = torch.empty_like(q)
        ws = vx.Workspace(vx.lib.vx_swa_attn_workspace(1, 8, T, 32, 64, 1))
        step = lambda: vx.swa_attn_fwd(q, k, v, 750, out=o, ws=ws)
        for _ in range(3):
            step()
        tr = traced_kernels(vx, torch, step, 10, flush)
        ms, _, _ = timed_steps(torch, step, 10, flush, torch.cuda.current_stream())
        fl = attn_flops(8, T, 32, 64, 750)
        ka = tr["swa_attn_tc"]["ms_per_launch"]
        out[f"T{T}"] = {"ms_per_call": ms, "attn_kernel_ms": ka, "rope_ms": tr.get("rope", {}).get("ms_per_step"),
                        "gflop": fl / 1e9, "kernel_tflops": fl / ka / 1e9, "kernel_frac_of_measured_peak": fl / ka / 1e9 / tf,
                        "call_tflops": fl / ms / 1e9}
        del q, k, v, o, ws
    return out


def component_c3(vx, torch, flush, hbm, tf, L=32):
    cfg, layers = device_layers(vx, torch, L, 300, "cuda")
    S, n, P = 64, 4, 1000
    ring = vx.KVRing(cfg, L, S)
    g = torch.Generator(device="cuda").manual_seed(301)
    ring.k.normal_(generator=g)
    ring.v.normal_(generator=g)
    ring.pos.fill_(P)
    x = torch.randn(S, n, cfg.d_model, generator=g, device="cuda")
    y = torch.empty_like(x)
    ws = vx.Workspace(vx.lib.vx_stream_step_workspace(__import__("ctypes").byref(cfg.c()), S, n))
    step = lambda: vx.stream_step(cfg, layers, ring, x, out=y, ws=ws)
    for _ in range(3):
        step()
    tr = traced_kernels(vx, torch, step, 5, lambda: None)
    ms, _, _ = timed_steps(torch, step, 10, lambda: None, torch.cuda.current_stream())
    # CUDA-graph replay of the whole 32-layer step (launch overhead removed)
    gr = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(gr, stream=s):
            step()
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(3):
        gr.replay()
    ms_g, _, _ = timed_steps(torch, gr.replay, 10, lambda: None, torch.cuda.current_stream())
    kv_read = 749 * 64 * 2 * 2 * 32 * S * L            # bytes: 749 slots x 64 x bf16 x (K,V) x heads x streams x layers
    w_read = L * 30146560 * 2
    kv_write = 4 * 64 * 2 * 2 * 32 * S * L
    io = 2 * S * n * 1280 * 4
    total = kv_read + w_read + kv_write + io
    ring_ms = tr["ring_attn"]["ms_per_launch"]
    ring_bytes = (749 + 4) * 64 * 2 * 2 * 32 * S + 4 * 64 * 2 * 2 * 32 * S
    del gr
    return {"ms_per_step_eager": ms, "ms_per_step_graph": ms_g, "bytes_per_step": total,
            "gbs_graph": total / ms_g / 1e6, "frac_of_measured_hbm": total / ms_g / 1e6 / hbm,
            "frames_per_s_graph": S * n / ms_g * 1e3,
            "ring_attn_ms_per_launch": ring_ms, "ring_attn_gbs": ring_bytes / ring_ms / 1e6,
            "kernel_ms_per_step": {k: v["ms_per_step"] for k, v in tr.items()}}


def component_c4(vx, torch, flush, hbm, tf):
    cfg, layers = device_layers(vx, torch, 32, 400, "cuda")
    g = torch.Generator(device="cuda").manual_seed(401)

    def nrm(shape, std):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    w1p = vx.pack_conv_weight(nrm((1280, 128, 3), 0.02))
    w2p = vx.pack_conv_weight(nrm((1280, 1280, 3), 0.02))
    b1, b2, fg = nrm((1280,), 0.01), nrm((1280,), 0.01), (1 + nrm((1280,), 0.02).float()).to(torch.bfloat16)
    mel = torch.randn(4, 128, 6000, generator=g, device="cuda")
    out = torch.empty(4, 3000, 1280, device="cuda")
    ws = vx.Workspace(vx.lib.vx_encoder_workspace(__import__("ctypes").byref(cfg.c()), 4, 128, 6000))
    step = lambda: vx.encoder_fwd(cfg, mel, w1p, b1, w2p, b2, layers, fg, out=out, ws=ws)
    for _ in range(2):
        step()
    tr = traced_kernels(vx, torch, step, 2, lambda: None)
    ms, _, _ = timed_steps(torch, step, 5, lambda: None, torch.cuda.current_stream())
    stem = 2 * 4 * 6000 * 1280 * 128 * 3 + 2 * 4 * 3000 * 1280 * 1280 * 3
    fl = stem + 32 * layer_flops(4, 3000)
    return {"ms_per_forward": ms, "frames_per_s": 12000 / ms * 1e3, "tflop_per_forward": fl / 1e12,
            "tflops": fl / ms / 1e9, "frac_of_measured_peak": fl / ms / 1e9 / tf,
            "kernel_ms_per_forward": {k: v["ms_per_step"] for k, v in tr.items()}}


# Log-mel frontend arithmetic per 10 ms frame: window (400 mul), the 201-bin
# DFT as 2 x 400 FMAs per bin, power (3 flop per bin) and the dense
# 128 x 201 filterbank product; its bound is the fp32 CUDA-core rate:
# 148 SMs x 128 fp32 lanes x 2 flop x 1.965 GHz.
LOG_MEL_FLOP_PER_FRAME = 400 + 201 * 400 * 4 + 201 * 3 + 128 * 201 * 2
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def component_next(vx, torch, flush, hbm, tf):
    """The widened rows: the streaming conv-stem step (64 streams x 8 mel frames
    -> 4 frames, warm padding cache), the audio projector on the encoder
    output of the 4 x 6000-mel workload ([4, 3000, 1280] -> [4, 750, 3072])
    and the log-mel frontend producing that workload's input (4 x 60 s)."""
    g = torch.Generator(device="cuda").manual_seed(501)

    def nrm(shape, std):
        return (torch.randn(shape, generator=g, device="cuda") * std).to(torch.bfloat16)

    w1p = vx.pack_conv_weight(nrm((1280, 128, 3), 0.02))
    w2p = vx.pack_conv_weight(nrm((1280, 1280, 3), 0.02))
    b1, b2 = nrm((1280,), 0.01), nrm((1280,), 0.01)
    S = 64
    cache = vx.ConvCache(S, 128, 1280)
    mel = torch.randn(S, 128, 8, generator=g, device="cuda")
    y = torch.empty(S, 4, 1280, device="cuda")
    ws = vx.Workspace(vx.lib.vx_conv_stem_step_workspace(S, 128, 8, 1280))
    step = lambda: vx.conv_stem_step(mel, w1p, b1, w2p, b2, cache, out=y, ws=ws)
    for _ in range(3):
        step()
    ms_c, _, _ = timed_steps(torch, step, 50, lambda: None, torch.cuda.current_stream())
    conv_flop = 2 * S * 8 * 1280 * 128 * 3 + 2 * S * 4 * 1280 * 1280 * 3
    conv_bytes = (1280 * 128 * 3 + 1280 * 1280 * 3) * 2 + S * 128 * 8 * 4 + S * 4 * 1280 * 4
    w1 = nrm((3072, 5120), 0.02)
    w2 = nrm((3072, 3072), 0.02)
    x = torch.randn(4, 3000, 1280, generator=g, device="cuda")
    out = torch.empty(4, 750, 3072, device="cuda")
    wsp = vx.Workspace(vx.lib.vx_projector_workspace(4, 3000, 1280, 3072))
    proj = lambda: vx.projector_fwd(x, w1, w2, out=out, ws=wsp)
    for _ in range(3):
        proj()
    ms_p, _, _ = timed_steps(torch, proj, 20, flush, torch.cuda.current_stream())
    proj_flop = 2 * 3000 * 5120 * 3072 + 2 * 3000 * 3072 * 3072
    audio = torch.randn(4, 960000, generator=g, device="cuda") * 0.1
    melo = torch.empty(4, 128, 6000, device="cuda")
    wsm = vx.Workspace(vx.lib.vx_log_mel_workspace(4, 960000))
    lm = lambda: vx.log_mel_fwd(audio, True, out=melo, ws=wsm)
    for _ in range(3):
        lm()
    ms_m, _, _ = timed_steps(torch, lm, 20, flush, torch.cuda.current_stream())
    return {"conv_step_64x8": {"ms_per_step": ms_c, "frames_per_s": S * 4 / ms_c * 1e3,
                               "gbs": conv_bytes / ms_c / 1e6, "tflops": conv_flop / ms_c / 1e9},
            "log_mel_4x60s": {"ms_per_call": ms_m, "mel_frames_per_s": 24000 / ms_m * 1e3,
                              "gbs": (4 * 960000 * 4 + 4 * 128 * 6000 * 4) / ms_m / 1e6,
                              "tflops_fp32": 24000 * LOG_MEL_FLOP_PER_FRAME / ms_m / 1e9,
                              "frac_of_fp32_alu_peak": 24000 * LOG_MEL_FLOP_PER_FRAME / ms_m / 1e9 / FP32_ALU_TFLOPS},
            "projector_4x3000": {"ms_per_call": ms_p, "tokens_per_s": 3000 / ms_p * 1e3,
                                 "tflops": proj_flop / ms_p / 1e9, "frac_of_measured_peak": proj_flop / ms_p / 1e9 / tf}}


# ------------------------------------------------------------- cpu legs

def oracle_sample(frames: int):
    """One oracle encoder layer over the first `frames` frames of the C1 input
    (causal, so those outputs are exact); returns seconds."""
    import oracle
    import synth
    p = synth.layer_params(synth.VOXTRAL_RT, seed=1)
    x = synth.frames(1, C1["T"], C1["d"], seed=2)[:, :frames]
    t = time.perf_counter()
    oracle.encoder_layer(x, p, synth.VOXTRAL_RT)
    return time.perf_counter() - t


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        return max(i.get("num_threads", 1) for i in threadpool_info()) or os.cpu_count()
    except Exception:
        return os.cpu_count()


def cpu_baseline(budget_s=12.0):
    """The oracle as it stands on this host: full C1 layers repeated until ~budget_s."""
    n, total = 0, 0.0
    while total < budget_s and n < 20:
        total += oracle_sample(C1["T"])
        n += 1
    return {"value": n * C1["T"] / total, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": f"{n} full C1 layer(s) ({n} x {C1['T']} frames) of the float64 numpy oracle, "
                      f"{total:.1f} s of CPU time on {os.cpu_count()} host cores"}


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    frames = 375   # a quarter of the C1 clip per step (causal: exact outputs for those frames)
    for _ in range(args.warmup):
        oracle_sample(frames)
    t = [oracle_sample(frames) for _ in range(args.steps)]
    ms = 1e3 * float(np.mean(t))
    value = frames / (ms / 1e3)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": C1["B"], "T": C1["T"], "parallelism": "replicas",
                       "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": f"first {frames} frames of the C1 clip per step, float64 numpy oracle"},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ main

def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import sliding_window_attention_tcgen05_b200 as vx

    rank, world, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=device)
    hbm, tf_burst, tf_sust, peak_kind = peaks()

    flush_buf = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    flush = lambda: flush_buf.zero_()
    stream = torch.cuda.current_stream()

    comps_only = [c for c in args.components_only.split(",") if c]
    if comps_only:
        out = {}
        for c in comps_only:
            if c == "c3":
                out[c] = component_c3(vx, torch, flush, hbm, tf_burst, L=args.c3_layers)
            else:
                out[c] = {"c0": component_c0, "c2": component_c2, "c4": component_c4,
                          "next": component_next}[c](vx, torch, flush, hbm, tf_burst)
        if rank == 0:
            print(json.dumps({"components": out}), flush=True)
        return 0

    B, T, d = C1["B"], C1["T"], C1["d"]
    cfg, L = make_layer(vx, torch, device=device)
    g = torch.Generator(device=device).manual_seed(2 + rank)
    x = torch.randn(B, T, d, generator=g, device=device)
    y = torch.empty_like(x)
    ws = vx.Workspace(vx.lib.vx_encoder_layer_workspace(__import__("ctypes").byref(cfg.c()), B, T), device=device)
    step = lambda: vx.encoder_layer_fwd(cfg, L, x, out=y, ws=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    gpu_uuid = str(torch.cuda.get_device_properties(device).uuid)
    sampler = ClockSampler(gpu_uuid if gpu_uuid.startswith("GPU-") else f"GPU-{gpu_uuid}")
    time.sleep(0.3)
    barrier(device)
    torch.cuda.synchronize()
    n0 = vx.lib.vx_launch_count()
    ms_local, t0, t1 = timed_steps(torch, step, args.steps, flush, stream)
    launches = vx.lib.vx_launch_count() - n0
    torch.cuda.synchronize()
    barrier(device)
    ms = reduce_max(ms_local, device)
    frames_all = reduce_sum(B * T, device)
    value = frames_all / (ms / 1e3)

    # End to end through the public call from pinned host buffers: every step
    # copies its input in (H2D), runs the layer and reads its output back (D2H).
    # Like a server fed a stream of clips, the copies of neighbouring steps run
    # on their own streams (two device buffers each way), overlapping the
    # layer; the L2 flush before each step's layer is inside the timed region.
    xh = torch.empty(B, T, d, dtype=torch.float32, pin_memory=True)
    xh.copy_(x.cpu())
    yh = torch.empty_like(xh, pin_memory=True)
    xs = [x, torch.empty_like(x)]
    ys = [y, torch.empty_like(y)]
    s_in, s_out = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)

    def e2e_run(K):
        ev_in = [torch.cuda.Event() for _ in range(K)]
        ev_comp = [torch.cuda.Event() for _ in range(K)]
        ev_out = [torch.cuda.Event() for _ in range(K)]
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(K):
            bb = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_comp[i - 2])      # the layer of step i-2 has read xs[bb]
                xs[bb].copy_(xh, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])         # ys[bb] of step i-2 is on the host
            flush()
            vx.encoder_layer_fwd(cfg, L, xs[bb], out=ys[bb], ws=ws)
            ev_comp[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_comp[i])
                yh.copy_(ys[bb], non_blocking=True)
                ev_out[i].record(s_out)
        stream.wait_stream(s_out)
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / K

    ms_e2e = float("nan")
    if not args.no_e2e:
        e2e_run(3)
        barrier(device)
        ms_e2e = reduce_max(e2e_run(max(20, min(args.steps, 200))), device)
    sampler.stop()
    clocks = sampler.summary(t0, t1)

    # dominant kernel, timed live per launch (trace mode), and its roofline
    tr = traced_kernels(vx, torch, step, 0 if args.no_trace else 50, flush)
    if not tr:
        tr = {"none": {"ms_per_launch": float("nan"), "launches_per_step": 0, "ms_per_step": 0.0}}
    dom = max(tr, key=lambda k: tr[k]["ms_per_step"])
    work, wunit, bound = kernel_work(dom, B, T)
    if work is None:
        roof = {"bound": None, "achieved": None, "peak": None, "unit": None, "frac": None}
    elif bound == "tensor":
        achieved = work / (tr[dom]["ms_per_launch"] / 1e3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                "frac": achieved / tf_burst, "peak_kind": f"{peak_kind} bf16 dense (burst)"}
    else:
        achieved = work / (tr[dom]["ms_per_launch"] / 1e3) / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                "peak_kind": f"{peak_kind} HBM copy"}
    roof.update({"kernel": dom, "work_per_launch": work, "work_unit": wunit,
                 "ms_per_launch": tr[dom]["ms_per_launch"], "traffic": ncu_traffic(dom, "C1")})
    per_kernel = {k: {"ms_per_launch": v["ms_per_launch"], "launches_per_step": v["launches_per_step"]}
                  for k, v in tr.items()}
    for k, v in per_kernel.items():
        w, u, b = kernel_work(k, B, T)
        if w is not None:
            v["tflops" if u == "flop" else "gbs"] = w / (v["ms_per_launch"] / 1e3) / (1e12 if u == "flop" else 1e9)

    comps = None
    if world == 1 and not args.no_components:
        comps = {}
        for name, fn in (("swa_c0", component_c0), ("swa_c2", component_c2), ("stream_step_c3", component_c3),
                         ("encoder_c4", component_c4), ("next_rows", component_next)):
            try:
                comps[name] = fn(vx, torch, flush, hbm, tf_burst)
            except Exception as e:   # report, never hide
                comps[name] = {"error": repr(e)}
            torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": WORKLOAD, "B": B, "T": T, "parallelism": f"replicas x{world}",
                       "l2": "flushed between timed steps (256 MiB write outside the step events)"},
            "layer_tflops": layer_flops(B, T) / (ms / 1e3) / 1e12,
            "layer_frac_of_measured_peak": layer_flops(B, T) / (ms / 1e3) / 1e12 / tf_burst,
            "e2e": {"value": frames_all / (ms_e2e / 1e3), "unit": UNIT,
                    "h2d_bytes_per_step": B * T * d * 4, "d2h_bytes_per_step": B * T * d * 4,
                    "method": "pinned host buffers; H2D, layer (after a 256 MiB L2 flush) and D2H of consecutive "
                              "steps on three streams with two device buffers each way; timed over the whole run"},
            "gpu_launches": int(launches),
            "roofline": roof,
            "kernels": per_kernel,
            "clocks": clocks,
            "cpu_baseline": cpu,
            "components": comps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        barrier(device)
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
