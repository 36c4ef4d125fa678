"""CPU tests of bench.py's host logic: the max/sum reductions over ranks (gloo,
world size 2), the algorithmic work counts, and the reference arm's line."""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.reduce_max(1.0 + rank)            # rank 1 is the slow one
        frames = bench.reduce_sum(1500)
        q.put((rank, ms, frames))
    finally:
        dist.destroy_process_group()


def test_reductions_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    ps = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    res = sorted(q.get(timeout=120) for _ in ps)
    for p in ps:
        p.join(timeout=60)
    assert [r[1] for r in res] == [2.0, 2.0]          # max over ranks
    assert [r[2] for r in res] == [3000.0, 3000.0]    # whole-job frames
    # value = all ranks' frames / max-over-ranks time
    assert 3000.0 / (2.0 / 1e3) == pytest.approx(1.5e6)


def test_reductions_without_process_group_are_identity():
    assert bench.reduce_max(3.5) == 3.5
    assert bench.reduce_sum(7) == 7.0


def test_algorithmic_work_counts():
    # attended pairs for T >= W: W(W+1)/2 + (T-W)W
    assert bench.attended_pairs(1500, 750) == 844125
    assert bench.attended_pairs(6000, 750) == 4219125
    assert bench.attended_pairs(10, 750) == 55
    # C1 layer: 90.44 GFLOP of GEMMs + 6.92 GFLOP of attention
    assert sum(bench.gemm_flops(1500).values()) == 2 * 1500 * 30146560
    assert bench.layer_flops(1, 1500) == pytest.approx(97.35e9, rel=1e-3)
    assert bench.attn_flops(8, 6000, 32, 64, 750) == pytest.approx(276.50e9, rel=1e-3)
    # the encoder workload: stem 141.6 GFLOP + 32 layers of 4 x 3000 frames = 25.36 TFLOP
    assert sum(bench.stem_flops(4, 6000).values()) == pytest.approx(141.6e9, rel=1e-3)
    assert bench.encoder_flops(4, 6000) == pytest.approx(25.36e12, rel=1e-3)


def test_attention_tile_counts():
    # key tiles of 128 visited per (clip, head): 63 / 147 / 308 of 144 / 576 / 2209
    for T, visited, total in ((1500, 63, 144), (3000, 147, 576), (6000, 308, 2209)):
        t = bench.attn_tiles(T, 750)
        assert (t["visited"], t["all_tiles"]) == (visited, total)
        assert 0.8 < t["useful_frac"] < 0.85
    # a window covering the clip visits the whole causal triangle
    t = bench.attn_tiles(1000, 2000)
    assert t["visited"] == t["causal_tiles"] == 8 * 9 // 2


def test_rmsnorm_trace_names_count_their_bytes():
    M = 1500
    w = lambda name: bench.kernel_work(name, {"M": M})[0] - 1280 * 2
    assert w("rmsnorm_p0_y16") == M * 1280 * (4 + 2)            # x in, bf16 y out
    assert w("rmsnorm_p2_h_y16") == M * 1280 * (4 + 8 + 4 + 2)  # + two partial sums in, h out
    assert w("rmsnorm_p1_h") == M * 1280 * (4 + 4 + 4)          # a reduction only
    assert w("rmsnorm_p0_y32") == M * 1280 * (4 + 4)            # the final norm
    assert bench.kernel_work("gemm_conv2_gelu", {"stem": (4, 6000)})[0] == 2 * 4 * 3000 * 1280 * 3 * 1280


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    j = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "config", "cpu_baseline", "e2e"):
        assert key in j
    assert j["impl"] == "reference" and j["value"] > 0 and j["e2e"]["h2d_bytes_per_step"] == 0
    assert j["cpu_baseline"]["kind"] == "oracle"
