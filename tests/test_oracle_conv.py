"""Pins of the oracle's causal conv stem (left-pad-only Conv1d 128->1280 k3 s1,
GELU, Conv1d 1280->1280 k3 s2, GELU) against torch's conv1d in float64."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth


def _small_conv(seed, c_in=8, d=12):
    return synth.conv_params(seed=seed, n_mels=c_in, d=d)


@pytest.mark.parametrize("Tm", [1, 2, 7, 16, 33])
def test_conv_stem_matches_torch_conv1d_on_left_padded_input(Tm):
    w = _small_conv(1)
    mel = synth.mel(2, 8, Tm, seed=2).astype(np.float64)
    out = oracle.conv_stem(mel, **w)
    x = torch.from_numpy(mel)
    t = {k: torch.from_numpy(v.astype(np.float64)) for k, v in w.items()}
    h = F.gelu(F.conv1d(F.pad(x, (2, 0)), t["w1"], t["b1"]), approximate="none")
    h = F.gelu(F.conv1d(F.pad(h, (2, 0)), t["w2"], t["b2"], stride=2), approximate="none")
    assert out.shape == (2, oracle.conv_out_len(Tm), 12)
    np.testing.assert_allclose(out, h.permute(0, 2, 1).numpy(), rtol=1e-12, atol=1e-13)


def test_conv_output_length():
    assert oracle.conv_out_len(6000) == 3000
    assert oracle.conv_out_len(8) == 4        # one 8-mel streaming chunk -> 4 frames
    assert oracle.conv_out_len(312) == 156    # the batched first chunk -> 156 frames
    assert oracle.conv_out_len(7) == 4


def test_conv_stem_is_causal():
    # Output frame t reads mel frames <= 2t only.
    w = _small_conv(3)
    mel = synth.mel(1, 8, 30, seed=4).astype(np.float64)
    base = oracle.conv_stem(mel, **w)
    t = 6
    m2 = mel.copy(); m2[..., 2 * t + 1:] += 1.0
    np.testing.assert_array_equal(oracle.conv_stem(m2, **w)[:, :t + 1], base[:, :t + 1])
    m3 = mel.copy(); m3[..., 2 * t] += 1.0
    assert np.max(np.abs(oracle.conv_stem(m3, **w)[:, t] - base[:, t])) > 1e-4


def _zero_branch_layers(dims, n, seed):
    """Layers whose O and down projections are zero: each layer then adds
    exactly bo + bd to the residual stream (attention and MLP branches vanish)."""
    layers = []
    for l in range(n):
        p = synth.layer_params(dims, seed=synth.layer_seed(seed, l))
        p["wo"] = np.zeros_like(p["wo"])
        p["wd"] = np.zeros_like(p["wd"])
        layers.append(p)
    return layers


def test_encoder_is_stem_then_each_layer_once_then_final_norm():
    # With zero-branch layers the encoder is, in closed form,
    #   RMSNorm(stem(mel) + sum_l (bo_l + bd_l); g),
    # the stem taken from torch's conv1d on the left-padded input.  A dropped,
    # repeated or reordered-with-the-norm layer changes the bias sum or the
    # normalisation, so it fails here.
    dims = synth.LayerDims(d_model=12, n_heads=2, head_dim=6, ffn_hidden=20, window=3)
    conv = _small_conv(5)
    layers = _zero_branch_layers(dims, 3, 6)
    g = synth.final_norm_gain(12, seed=7)
    mel = synth.mel(1, 8, 14, seed=8).astype(np.float64)
    out = oracle.encoder(mel, conv, layers, g, dims)
    t = {k: torch.from_numpy(v.astype(np.float64)) for k, v in conv.items()}
    h = F.gelu(F.conv1d(F.pad(torch.from_numpy(mel), (2, 0)), t["w1"], t["b1"]), approximate="none")
    h = F.gelu(F.conv1d(F.pad(h, (2, 0)), t["w2"], t["b2"], stride=2), approximate="none")
    x = h.permute(0, 2, 1).numpy() + sum(p["bo"].astype(np.float64) + p["bd"].astype(np.float64) for p in layers)
    # out / g is x scaled per frame by 1 / sqrt(mean(x^2) + eps)
    scale = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + dims.eps)
    np.testing.assert_allclose(out / g.astype(np.float64), x * scale, rtol=1e-12, atol=1e-12)
    # and with one layer fewer the result differs
    assert np.max(np.abs(oracle.encoder(mel, conv, layers[:2], g, dims) - out)) > 1e-3
