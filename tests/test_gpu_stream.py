"""GPU parity of the streaming path (vx_stream_prefill / vx_stream_step)
against the oracle, the whole-sequence path and the ring-slot rule.

Streaming schedule: 4 encoder frames per step (transcribe.cpp notes
"Voxtral", Voxtral Realtime 2602 architecture); cache: W-slot ring, frame f in
slot f mod W (replacing the append-only buffer of the Core AI port, model card
"Voxtral Mini 4B Realtime -- Core AI", Usage)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from test_rounding_floor import C3_MAX_ABS, C3_SAMPLE, C3_STATED_MAX_ABS, C3_STATED_NORMED_MAX_ABS
from gpu_util import cfg_of, compare_bf16, dev, host, layer_params_dev, layer_stack

pytestmark = pytest.mark.gpu

SMALL = synth.LayerDims(d_model=256, n_heads=4, head_dim=64, ffn_hidden=512, window=16)


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


def _oracle_rings(x, layers, dims, T):
    """Per-layer oracle rings after the first T frames of x [S, *, d]."""
    rings = []
    h = np.asarray(x[:, :T], dtype=np.float64)
    for p in layers:
        h2, k, v = oracle.encoder_layer(h, p, dims, return_kv=True)
        rings.append(oracle.ring_from_sequence(k, v, dims.window))
        h = h2
    return rings


@pytest.mark.parametrize("prefill,n_new,steps", [(21, 4, 3), (5, 4, 3), (16, 1, 5), (40, 3, 2), (2, 2, 4)])
def test_small_stream_matches_oracle_and_whole_sequence(prefill, n_new, steps):
    vx = _vx()
    dims = SMALL
    layers = layer_stack(dims, 2, 31)
    S = 3
    T = prefill + n_new * steps
    x = synth.frames(S, T, dims.d_model, seed=32)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    ring = vx.KVRing(cfg_of(dims), 2, S)
    vx.stream_prefill(cfg_of(dims), Ls, ring, dev(x[:, :prefill]))
    assert torch.all(ring.pos == prefill)
    whole_gpu = host(vx.stream_prefill(cfg_of(dims), Ls, vx.KVRing(cfg_of(dims), 2, S), dev(x)))
    rings = _oracle_rings(x, layers, dims, prefill)
    pos = np.full(S, prefill)
    for st in range(steps):
        rows = slice(prefill + st * n_new, prefill + (st + 1) * n_new)
        got = host(vx.stream_step(cfg_of(dims), Ls, ring, dev(x[:, rows])))
        want, rings, pos = oracle.stream_step(x[:, rows], layers, dims, rings, pos)
        compare_bf16(got, want, f"step {st}")
        compare_bf16(got, whole_gpu[:, rows], f"step {st} vs whole-sequence GPU")
    assert torch.all(ring.pos == T)


@pytest.mark.parametrize("window,S,prefill,n_new", [(16, 600, 21, 1), (16, 600, 21, 8), (200, 300, 230, 4),
                                                     (200, 160, 37, 3)])
def test_many_items_per_ring_cta(window, S, prefill, n_new):
    # More (stream, head) items than the ring kernel keeps resident (a few CTAs
    # per SM), so each CTA walks several items through one stage ring, items of
    # one chunk (W = 16) or of several with a ragged last one (W = 200, wrapped
    # or not).  Every stream must equal the whole-sequence output, and sampled
    # streams the oracle.
    vx = _vx()
    dims = synth.LayerDims(d_model=256, n_heads=4, head_dim=64, ffn_hidden=512, window=window)
    layers = layer_stack(dims, 1, 71)
    steps = 2
    T = prefill + n_new * steps
    x = synth.frames(S, T, dims.d_model, seed=72)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    ring = vx.KVRing(cfg_of(dims), 1, S)
    vx.stream_prefill(cfg_of(dims), Ls, ring, dev(x[:, :prefill]))
    whole_gpu = host(vx.stream_prefill(cfg_of(dims), Ls, vx.KVRing(cfg_of(dims), 1, S), dev(x)))
    sample = [0, S // 2 + 1, S - 1]
    xs = x[sample]
    rings = _oracle_rings(xs, layers, dims, prefill)
    pos = np.full(len(sample), prefill)
    for st in range(steps):
        rows = slice(prefill + st * n_new, prefill + (st + 1) * n_new)
        got = host(vx.stream_step(cfg_of(dims), Ls, ring, dev(x[:, rows])))
        compare_bf16(got, whole_gpu[:, rows], f"step {st} vs whole-sequence GPU")
        want, rings, pos = oracle.stream_step(xs[:, rows], layers, dims, rings, pos)
        compare_bf16(got[sample], want, f"step {st} vs oracle")
    assert torch.all(ring.pos == T)


def test_ring_slots_bit_exact_across_wrap():
    # Layer 0's K/V depend only on the layer input, so after [prefill T, step 4]
    # the layer-0 ring must equal, bit for bit, the ring after prefill T + 4;
    # T + 4 > W makes the step wrap around slot W - 1 -> 0.
    vx = _vx()
    dims = SMALL
    layers = layer_stack(dims, 2, 41)
    S, T, n = 2, 30, 4   # frames 30..33 -> slots 14, 15, 0, 1
    x = synth.frames(S, T + n, dims.d_model, seed=42)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    a = vx.KVRing(cfg_of(dims), 2, S)
    vx.stream_prefill(cfg_of(dims), Ls, a, dev(x[:, :T]))
    vx.stream_step(cfg_of(dims), Ls, a, dev(x[:, T:]))
    b = vx.KVRing(cfg_of(dims), 2, S)
    vx.stream_prefill(cfg_of(dims), Ls, b, dev(x))
    assert torch.equal(a.k[0], b.k[0]) and torch.equal(a.v[0], b.v[0])
    assert torch.equal(a.pos, b.pos)


def test_ring_holds_frame_f_in_slot_f_mod_w():
    # Prefill T frames: slot f mod W of layer 0 holds the K/V of frame f for
    # the last W frames; compared against the oracle's K/V of those frames.
    vx = _vx()
    dims = SMALL
    layers = layer_stack(dims, 1, 51)
    S, T, W = 2, 37, dims.window
    x = synth.frames(S, T, dims.d_model, seed=52)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    r = vx.KVRing(cfg_of(dims), 1, S)
    vx.stream_prefill(cfg_of(dims), Ls, r, dev(x))
    _, k, v = oracle.encoder_layer(x, layers[0], dims, return_kv=True)
    rk, rv = host(r.k[0]), host(r.v[0])
    for f in range(T - W, T):
        compare_bf16(rk[:, :, f % W], k[:, f], f"K frame {f}")
        compare_bf16(rv[:, :, f % W], v[:, f], f"V frame {f}")


def test_step_from_empty_ring():
    # pos = 0: the first step attends only to its own frames.
    vx = _vx()
    dims = SMALL
    layers = layer_stack(dims, 2, 61)
    S = 2
    x = synth.frames(S, 4, dims.d_model, seed=62)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    ring = vx.KVRing(cfg_of(dims), 2, S)
    got = host(vx.stream_step(cfg_of(dims), Ls, ring, dev(x)))
    h = x.astype(np.float64)
    for p in layers:
        h = oracle.encoder_layer(h, p, dims)
    compare_bf16(got, h, "first step")


def test_c3_full_size_sampled_streams():
    # 32 layers, 64 streams, 4 new frames each, ring wrapped at pos = 1000.
    # Ring contents are seeded inputs (synth.ring_kv) for the sampled streams
    # and arbitrary for the others (streams are independent).
    vx = _vx()
    dims = synth.VOXTRAL_RT
    L, S, n, P = 32, 64, 4, 1000
    layers = layer_stack(dims, L, 1)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    ring = vx.KVRing(cfg_of(dims), L, S)
    gen = torch.Generator(device="cuda").manual_seed(0)
    ring.k.normal_(generator=gen)
    ring.v.normal_(generator=gen)
    ring.pos.fill_(P)
    sample = list(C3_SAMPLE)
    host_rings = []
    for l in range(L):
        k, v = synth.ring_kv(len(sample), dims.n_heads, dims.window, dims.head_dim, seed=1000 + l)
        ring.k[l, sample] = dev(k, torch.bfloat16)
        ring.v[l, sample] = dev(v, torch.bfloat16)
        host_rings.append((k, v))
    x = synth.frames(S, n, dims.d_model, seed=3)
    got = host(vx.stream_step(cfg_of(dims), Ls, ring, dev(x)))
    assert np.all(np.isfinite(got))
    want, new_rings, _ = oracle.stream_step(x[sample], layers, dims, host_rings, np.full(len(sample), P))
    # 32 layers of unnormalised residual stream: rel-L2 keeps the 1e-2 bar;
    # max-abs is bounded by the bf16 operand floor (test_rounding_floor.py).
    compare_bf16(got[sample], want, "C3 sampled streams", max_abs=C3_MAX_ABS)
    assert torch.all(ring.pos == P + n)
    # the step wrote the 4 new frames' K/V into slots (1000 + t) mod 750 = 250..253
    for l in (0, 31):
        compare_bf16(host(ring.k[l, sample][:, :, 250:254]), new_rings[l][0][:, :, 250:254], f"ring K layer {l}")


def test_cuda_graph_replay_of_a_step():
    # vx_stream_step only enqueues kernels, so a step can be captured and replayed.
    vx = _vx()
    dims = SMALL
    layers = layer_stack(dims, 2, 71)
    S = 2
    x = synth.frames(S, 16 + 8, dims.d_model, seed=72)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    ring_a = vx.KVRing(cfg_of(dims), 2, S)
    ring_b = vx.KVRing(cfg_of(dims), 2, S)
    for r in (ring_a, ring_b):
        vx.stream_prefill(cfg_of(dims), Ls, r, dev(x[:, :16]))
    ws = vx.Workspace(1 << 24)
    xin = dev(x[:, 16:20])
    out = torch.empty_like(xin)
    vx.stream_step(cfg_of(dims), Ls, ring_a, xin, out=out, ws=ws)   # warm up (sets kernel attributes)
    ref1 = out.clone()
    # replay on ring_b: two graph launches = two steps
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            vx.stream_step(cfg_of(dims), Ls, ring_b, xin, out=out, ws=ws)
    torch.cuda.current_stream().wait_stream(s)
    # capture does not execute: ring_b is still at pos 16
    assert torch.all(ring_b.pos == 16)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, ref1)
    xin.copy_(dev(x[:, 20:24]))
    g.replay()
    vx.stream_step(cfg_of(dims), Ls, ring_a, xin)   # second eager step on ring_a
    torch.cuda.synchronize()
    assert torch.all(ring_b.pos == 24) and torch.equal(ring_a.k, ring_b.k)


def test_c3_stated_config_prefill_then_step():
    # The streaming config as stated: 32 layers of the one-layer shape, 64
    # streams, the ring filled by vx_stream_prefill from 1000 seeded frames
    # per stream (so it has wrapped: frames 250..999 in slots f mod 750),
    # then one 4-frame step at positions 1000..1003.  The step must equal
    # (i) the GPU whole-sequence output of frames 1000..1003 (a prefill over
    # all 1004 frames) and (ii) the oracle over those 1004 frames x 32 layers
    # (streams 0 and 63).  Raw outputs are the unnormalised residual stream;
    # with the final RMSNorm (final_g) they are the encoder's output.
    vx = _vx()
    dims = synth.VOXTRAL_RT
    L, S, n, P = 32, 64, 4, 1000
    layers = layer_stack(dims, L, 1)
    Ls = [vx.pack_layer(cfg_of(dims), layer_params_dev(p)) for p in layers]
    cfg = cfg_of(dims)
    g = synth.final_norm_gain(dims.d_model, seed=5)
    gd = dev(g, torch.bfloat16)
    x = synth.frames(S, P + n, dims.d_model, seed=7)
    xd = dev(x)
    ring = vx.KVRing(cfg, L, S)
    ws = vx.Workspace()
    out = {}
    for fg in (None, gd):
        vx.stream_prefill(cfg, Ls, ring, xd[:, :P].contiguous(), ws=ws)
        assert torch.all(ring.pos == P)
        out[fg is None] = host(vx.stream_step(cfg, Ls, ring, xd[:, P:].contiguous(), final_g=fg, ws=ws))
        assert torch.all(ring.pos == P + n)
    whole = host(vx.stream_prefill(cfg, Ls, ring, xd, ws=ws)[:, P:])
    whole_n = host(vx.stream_prefill(cfg, Ls, ring, xd, final_g=gd, ws=ws)[:, P:])
    del ring, ws
    torch.cuda.empty_cache()
    raw, normed = out[True], out[False]
    compare_bf16(raw, whole, "C3 stated: step vs GPU whole sequence (raw)", max_abs=C3_STATED_MAX_ABS)
    compare_bf16(normed, whole_n, "C3 stated: step vs GPU whole sequence (final norm)", max_abs=C3_STATED_NORMED_MAX_ABS)
    # the oracle over 1004 frames x 32 layers for two streams
    sample = [0, 63]
    h = np.asarray(x[sample], dtype=np.float64)
    for p in layers:
        h = oracle.encoder_layer(h, p, dims)
    want = h[:, P:]
    compare_bf16(raw[sample], want, "C3 stated: step vs oracle (raw)", max_abs=C3_STATED_MAX_ABS)
    compare_bf16(normed[sample], oracle.rms_norm(want, g, dims.eps), "C3 stated: step vs oracle (final norm)",
                 max_abs=C3_STATED_NORMED_MAX_ABS)
