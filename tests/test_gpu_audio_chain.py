"""The streaming chain from audio to encoder frames, against the whole-clip
path and the oracle.

The pages' streaming mode (Core AI card "Voxtral Mini 4B Realtime -- Core
AI", sections "What this is" and "Streaming"): one batched first chunk of 312
mel frames, then chunks of 8 mel frames (4 encoder frames, 80 ms) through the
streaming encoder.  The transcribe.cpp notes "Voxtral", section "Notes", leave
open whether the realtime encoder's offline path equals the streaming one
(fixed frontend maximum, causal convolutions); this test checks it.

Per stream:
  audio -> vx_log_mel_fwd: a centred first chunk (frames 0..311), then
           uncentred 8-frame chunks continuing the centred frame grid (the
           samples from 160 t0 - 200 on)
        -> vx_conv_stem_step: the 312 mel frames, then 8 per chunk, through the
           conv padding cache
        -> vx_stream_prefill over the first 156 encoder frames (ring filled),
           then vx_stream_step with 4 frames per chunk, final RMSNorm applied.
Whole clip: vx_log_mel_fwd over all the audio -> vx_encoder_fwd."""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_util import cfg_of, compare_bf16, dev, host, layer_params_dev, layer_stack
from test_rounding_floor import C4_MAX_ABS

pytestmark = pytest.mark.gpu

FIRST, CHUNK = 312, 8


def _vx():
    import sliding_window_attention_tcgen05_b200 as vx
    return vx


@pytest.mark.parametrize("full", [False, True])
def test_audio_to_stream_chain_equals_whole_clip_and_oracle(full):
    vx = _vx()
    if full:   # the encoder of the pages: 32 layers, window 750 (no wrap at 180 frames)
        dims, n_layers, n_chunks, bar = synth.VOXTRAL_RT, 32, 6, C4_MAX_ABS
    else:      # a small stack with window 16: the ring wraps during the prefill and every step
        dims, n_layers, n_chunks, bar = synth.LayerDims(d_model=256, n_heads=4, head_dim=64, ffn_hidden=512,
                                                        window=16), 2, 6, 3e-2
    S, d = 2, dims.d_model
    cfg = cfg_of(dims)
    F = FIRST + CHUNK * n_chunks                       # mel frames compared
    N = 160 * F + 200                                  # frame F-1 lies wholly inside the audio
    x = synth.audio(S, N, seed=11)
    layers = layer_stack(dims, n_layers, 13)
    Ls = [vx.pack_layer(cfg, layer_params_dev(p)) for p in layers]
    conv = synth.conv_params(seed=14, n_mels=128, d=d)
    w1p = vx.pack_conv_weight(dev(conv["w1"], torch.bfloat16))
    w2p = vx.pack_conv_weight(dev(conv["w2"], torch.bfloat16))
    b1, b2 = dev(conv["b1"], torch.bfloat16), dev(conv["b2"], torch.bfloat16)
    g = synth.final_norm_gain(d, seed=15)
    gd = dev(g, torch.bfloat16)
    xd = dev(x)

    # streaming chain
    cache = vx.ConvCache(S, 128, d)
    ring = vx.KVRing(cfg, n_layers, S)
    mel0 = vx.log_mel_fwd(xd[:, :160 * FIRST + 200].contiguous(), center=True)[:, :, :FIRST].contiguous()
    h0 = vx.conv_stem_step(mel0, w1p, b1, w2p, b2, cache)
    outs = [host(vx.stream_prefill(cfg, Ls, ring, h0, final_g=gd))]
    for c in range(n_chunks):
        t0 = FIRST + CHUNK * c
        seg = xd[:, 160 * t0 - 200:160 * (t0 + CHUNK - 1) + 200].contiguous()
        mel = vx.log_mel_fwd(seg, center=False)
        assert mel.shape == (S, 128, CHUNK)
        hc = vx.conv_stem_step(mel, w1p, b1, w2p, b2, cache)
        outs.append(host(vx.stream_step(cfg, Ls, ring, hc, final_g=gd)))
    streamed = np.concatenate(outs, axis=1)
    assert streamed.shape == (S, F // 2, d)
    assert torch.all(ring.pos == F // 2)

    # whole clip through the offline path
    mel_all = vx.log_mel_fwd(xd, center=True)[:, :, :F].contiguous()
    whole = host(vx.encoder_fwd(cfg, mel_all, w1p, b1, w2p, b2, Ls, gd))
    compare_bf16(streamed, whole, f"audio chain vs whole clip ({'full' if full else 'small'})", max_abs=bar)

    # the oracle over the whole clip
    mel_o = oracle.log_mel(x, center=True)[:, :, :F]
    want = oracle.encoder(mel_o, conv, layers, g, dims)
    compare_bf16(streamed, want, f"audio chain vs oracle ({'full' if full else 'small'})", max_abs=bar)
