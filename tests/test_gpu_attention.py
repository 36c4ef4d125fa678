"""GPU parity of vx_swa_attn_fwd against the oracle (same seeded inputs).

fp32 path (CUDA cores): max-abs 1e-4.  bf16 path (tcgen05): max-abs 3e-2 and
relative L2 1e-2.  Operation: causal sliding-window attention with RoPE
(transcribe.cpp notes "Voxtral", Voxtral Realtime 2602 architecture)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import compare_bf16, compare_f32, dev, host

pytestmark = pytest.mark.gpu


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def _oracle_rows(q, k, v, W, rows, pos0=0, theta=1e6):
    T = q.shape[1]
    pos = pos0 + np.arange(T)
    return oracle.swa_attention_rows(oracle.rope(q, pos, theta), oracle.rope(k, pos, theta), v, W, rows)


def test_c0_tiny_fp32():
    # B=1, T=64, 2 heads, head_dim 64, window 16, RoPE theta 1e6, seed 0.
    q, k, v = synth.attention_qkv(1, 64, 2, 64, seed=0)
    o = _vx().swa_attn_fwd(dev(q), dev(k), dev(v), window=16)
    want = _oracle_rows(q, k, v, 16, range(64))
    compare_f32(host(o), want, "C0")
    g = np.load(__import__("os").path.join(__import__("os").path.dirname(__file__), "golden", "c0_swa_rope_fp32.npz"))
    compare_f32(host(o), g["o"], "C0 golden")


@pytest.mark.parametrize("T,W,pos0", [(1, 1, 0), (5, 3, 7), (100, 1, 0), (200, 64, 1000), (333, 750, 0)])
def test_fp32_edge_shapes(T, W, pos0):
    q, k, v = synth.attention_qkv(2, T, 3, 64, seed=T + W)
    o = _vx().swa_attn_fwd(dev(q), dev(k), dev(v), window=W, pos0=pos0)
    compare_f32(host(o), _oracle_rows(q, k, v, W, range(T), pos0), f"fp32 T={T} W={W}")


@pytest.mark.parametrize("T,W", [(1, 1), (64, 16), (127, 5), (128, 128), (129, 128), (300, 1),
                                 (300, 100), (513, 200), (1000, 750), (700, 2000)])
def test_bf16_small_shapes(T, W):
    B, H = 2, 3
    q, k, v = synth.attention_qkv(B, T, H, 64, seed=100 + T + W, bf16=True)
    o = _vx().swa_attn_fwd(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), window=W)
    compare_bf16(host(o), _oracle_rows(q, k, v, W, range(T)), f"bf16 T={T} W={W}")


def test_bf16_without_rope_matches_plain_window_attention():
    B, T, H, W = 1, 400, 2, 100
    q, k, v = synth.attention_qkv(B, T, H, 64, seed=7, bf16=True)
    o = _vx().swa_attn_fwd(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), window=W,
                           apply_rope=False)
    compare_bf16(host(o), oracle.swa_attention(q, k, v, W), "bf16 no-rope")


@pytest.mark.parametrize("T", [1500, 3000, 6000])
def test_c2_full_size_sampled_rows(T):
    # Attention-only sweep: B=8, 32 heads, head_dim 64, window 750, RoPE 1e6.
    B, H, W = 8, 32, 750
    q, k, v = synth.attention_qkv(B, T, H, 64, seed=20 + T // 1500, bf16=True)
    vx = _vx()
    ws = vx.Workspace()
    o = vx.swa_attn_fwd(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), window=W, ws=ws)
    assert vx.status_check(ws) == 0   # no bounded wait ran out
    rng = np.random.default_rng(T)
    rows = sorted(set([0, 1, 127, 128, 749, 750, 751, 1023, T - 129, T - 1] +
                      list(rng.integers(0, T, 6))))
    want = _oracle_rows(q, k, v, W, rows)
    got = host(o)[:, rows]
    compare_bf16(got, want, f"C2 T={T}")


def test_bf16_deterministic():
    q, k, v = synth.attention_qkv(2, 700, 4, 64, seed=3, bf16=True)
    args = [dev(x, torch.bfloat16) for x in (q, k, v)]
    a = _vx().swa_attn_fwd(*args, window=300)
    b = _vx().swa_attn_fwd(*args, window=300)
    assert torch.equal(a, b)


def test_bf16_many_items_per_cta_with_single_tile_query_tiles():
    # More pair items (two neighbouring query tiles of one clip and head) than
    # SMs, with short items (the first query tiles of each head see one or two
    # 64-key tiles): every CTA of the persistent kernel walks several items.
    B, T, H, W = 4, 256, 48, 100
    q, k, v = synth.attention_qkv(B, T, H, 64, seed=11, bf16=True)
    args = [dev(x, torch.bfloat16) for x in (q, k, v)]
    vx = _vx()
    ws = vx.Workspace()
    o = host(vx.swa_attn_fwd(*args, window=W, ws=ws))
    assert vx.status_check(ws) == 0   # no bounded wait ran out
    rows = [0, 1, 127, 128, 129, 200, 255]
    compare_bf16(o[:, rows], _oracle_rows(q, k, v, W, rows), "bf16 many items")


def test_bf16_item_pairs_with_odd_item_count():
    # 5 query tiles per head: every third pair item has a single query tile,
    # so its second softmax warpgroup idles for that item while the K/V ring
    # and the MUFU turn-taking continue across items.
    B, T, H, W = 1, 640, 255, 300
    q, k, v = synth.attention_qkv(B, T, H, 64, seed=12, bf16=True)
    args = [dev(x, torch.bfloat16) for x in (q, k, v)]
    vx = _vx()
    ws = vx.Workspace()
    o = host(vx.swa_attn_fwd(*args, window=W, ws=ws))
    assert vx.status_check(ws) == 0
    rows = [0, 127, 128, 383, 384, 639]
    compare_bf16(o[:, rows], _oracle_rows(q, k, v, W, rows), "bf16 odd item pairs")


def test_bf16_running_max_grows_across_tiles():
    # Scores that grow along the keys (k_j = 0.05 j e_0, q = 8 e_0, no RoPE:
    # s_j = 0.05 j, +3.2 per 64-key tile) make the running maximum rise by
    # more than the rescale slack (2^8) every few tiles, so O and the row sum
    # are rescaled in place many times; W >= T keeps every key in the window.
    B, T, H, W = 1, 700, 2, 700
    q = np.zeros((B, T, H, 64), np.float32)
    k = np.zeros((B, T, H, 64), np.float32)
    q[..., 0] = 8.0
    k[..., 0] = (0.05 * np.arange(T, dtype=np.float32))[None, :, None]
    v = synth.attention_qkv(B, T, H, 64, seed=13, bf16=True)[2]
    q, k = synth.bf16_round(q), synth.bf16_round(k)
    o = _vx().swa_attn_fwd(dev(q, torch.bfloat16), dev(k, torch.bfloat16), dev(v, torch.bfloat16), window=W,
                           apply_rope=False)
    compare_bf16(host(o), oracle.swa_attention(q, k, v, W), "bf16 growing max")
