"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and bench.py.

This module holds none of the encoder's arithmetic.  It only draws numbers from
numpy's ``default_rng`` (PCG64) in a fixed, documented order and rounds them to
bfloat16 (round to nearest, ties to even), the storage type the GPU path reads.
Both sides consume exactly these values: the oracle upcasts them to float64,
the CUDA path receives the bf16 bit patterns (or float32 for fp32 inputs).

Distributions follow the workloads of the Voxtral Realtime encoder layer:
activations ~ N(0, 1), projection and conv weights ~ N(0, 0.02),
biases ~ N(0, 0.01), RMSNorm gains 1 + N(0, 0.02).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class LayerDims:
    """Shape of one Voxtral Realtime encoder layer (defaults: the 2602 encoder)."""

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


VOXTRAL_RT = LayerDims()

# Order in which layer_params draws its tensors (one generator, one pass).
LAYER_DRAW_ORDER = ("attn_norm_g", "wq", "wk", "wv", "bq", "bv", "wo", "bo",
                    "ffn_norm_g", "wg", "wu", "wd", "bd", "bg", "bu")


def bf16_round(a) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).reshape(a.shape)


def bf16_bits(a) -> np.ndarray:
    """bfloat16 bit patterns (uint16) of float32 values, rounding to nearest even."""
    r = bf16_round(a)
    return (r.view(np.uint32) >> 16).astype(np.uint16)


def from_bf16_bits(u) -> np.ndarray:
    """float32 values of bfloat16 bit patterns."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32)


def _normal(rng, shape, std=1.0, mean=0.0):
    x = rng.standard_normal(shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    if mean != 0.0:
        x += np.float32(mean)
    return x


def attention_qkv(B, T, H, D, seed=0, bf16=False):
    """q, k, v ~ N(0,1) of shape [B, T, H, D], drawn in the order q, k, v."""
    rng = np.random.default_rng(seed)
    out = [_normal(rng, (B, T, H, D)) for _ in range(3)]
    if bf16:
        out = [bf16_round(x) for x in out]
    return tuple(out)


def layer_params(dims: LayerDims = VOXTRAL_RT, seed=1, gate_up_bias=False):
    """One encoder layer's parameters as bf16-exact float32 arrays.

    Linear weights use PyTorch's [out, in] order.  Tensors are drawn from one
    generator in LAYER_DRAW_ORDER; bg/bu are drawn only when gate_up_bias is set
    (otherwise they are None: the layer has bias on the down projection only).
    """
    d, hd, f = dims.d_model, dims.hd, dims.ffn_hidden
    rng = np.random.default_rng(seed)
    shapes = {
        "attn_norm_g": ((d,), 0.02, 1.0), "wq": ((hd, d), 0.02, 0.0),
        "wk": ((hd, d), 0.02, 0.0), "wv": ((hd, d), 0.02, 0.0),
        "bq": ((hd,), 0.01, 0.0), "bv": ((hd,), 0.01, 0.0),
        "wo": ((d, hd), 0.02, 0.0), "bo": ((d,), 0.01, 0.0),
        "ffn_norm_g": ((d,), 0.02, 1.0), "wg": ((f, d), 0.02, 0.0),
        "wu": ((f, d), 0.02, 0.0), "wd": ((d, f), 0.02, 0.0),
        "bd": ((d,), 0.01, 0.0), "bg": ((f,), 0.01, 0.0), "bu": ((f,), 0.01, 0.0),
    }
    p = {}
    for name in LAYER_DRAW_ORDER:
        if name in ("bg", "bu") and not gate_up_bias:
            p[name] = None
            continue
        shape, std, mean = shapes[name]
        p[name] = bf16_round(_normal(rng, shape, std, mean))
    return p


def layer_seed(base_seed: int, layer: int) -> int:
    """Seed of layer `layer` in a multi-layer stack drawn from `base_seed`."""
    return base_seed * 1000 + layer


def frames(B, T, d=1280, seed=2):
    """Layer input activations ~ N(0,1), float32 [B, T, d] (the residual stream is fp32)."""
    rng = np.random.default_rng(seed)
    return _normal(rng, (B, T, d))


def conv_params(seed=3, n_mels=128, d=1280):
    """Causal conv stem parameters, PyTorch Conv1d order [out, in, k]; bf16-exact.

    Drawn in the order w1, b1, w2, b2; weights ~ N(0, 0.02), biases ~ N(0, 0.01).
    """
    rng = np.random.default_rng(seed)
    w1 = bf16_round(_normal(rng, (d, n_mels, 3), 0.02))
    b1 = bf16_round(_normal(rng, (d,), 0.01))
    w2 = bf16_round(_normal(rng, (d, d, 3), 0.02))
    b2 = bf16_round(_normal(rng, (d,), 0.01))
    return {"w1": w1, "b1": b1, "w2": w2, "b2": b2}


def mel(B, n_mels, Tm, seed=4):
    """Log-mel features ~ N(0,1), float32 [B, n_mels, Tm]."""
    rng = np.random.default_rng(seed)
    return _normal(rng, (B, n_mels, Tm))


def projector_params(d=1280, hidden=3072, factor=4, seed=8):
    """Audio projector weights (no biases): w1 [hidden, factor*d], w2 [hidden, hidden],
    drawn in that order ~ N(0, 0.02), bf16-exact."""
    rng = np.random.default_rng(seed)
    w1 = bf16_round(_normal(rng, (hidden, factor * d), 0.02))
    w2 = bf16_round(_normal(rng, (hidden, hidden), 0.02))
    return {"w1": w1, "w2": w2}


def final_norm_gain(d=1280, seed=5):
    """Final encoder RMSNorm gain, 1 + N(0, 0.02), bf16-exact."""
    rng = np.random.default_rng(seed)
    return bf16_round(_normal(rng, (d,), 0.02, 1.0))


def ring_kv(S, H, W, D, seed=6):
    """Synthetic contents of one layer's ring cache: K and V ~ N(0,1), bf16-exact,
    each [S, H, W, D], drawn in the order K, V."""
    rng = np.random.default_rng(seed)
    k = bf16_round(_normal(rng, (S, H, W, D)))
    v = bf16_round(_normal(rng, (S, H, W, D)))
    return k, v


def audio(B, N, seed=9, std=0.1):
    """16 kHz audio samples ~ N(0, std^2) (white noise), float32 [B, N]."""
    rng = np.random.default_rng(seed)
    return _normal(rng, (B, N), std)
