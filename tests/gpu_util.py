"""Helpers of the GPU parity tests: device copies of synth inputs and the
comparison rules (bf16 paths: max-abs 3e-2 and relative L2 1e-2; fp32
paths: max-abs 1e-4)."""
from __future__ import annotations

import functools

import numpy as np
import torch

import synth

BF16_MAX_ABS = 3e-2
BF16_REL_L2 = 1e-2
F32_MAX_ABS = 1e-4


def dev(a, dtype=torch.float32):
    """numpy (bf16-exact for bf16) -> CUDA tensor of dtype (exact)."""
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to("cuda").to(dtype)


def host(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def _log(what, **kv):
    """Appends measured errors to $VX_PARITY_LOG (one JSON line per check)."""
    import json
    import os
    path = os.environ.get("VX_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"check": what, **kv}) + "\n")


def compare_bf16(got, want, what="", max_abs=BF16_MAX_ABS, rel_l2=BF16_REL_L2):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    max_abs_bar = max_abs
    err = np.abs(got - want)
    max_abs = float(err.max()) if err.size else 0.0
    rel = float(np.linalg.norm(got - want) / max(np.linalg.norm(want), 1e-30))
    _log(what, max_abs=max_abs, rel_l2=rel, bar_max_abs=max_abs_bar, bar_rel_l2=rel_l2)
    assert max_abs <= max_abs_bar and rel <= rel_l2, f"{what}: max_abs={max_abs:.3e} rel_l2={rel:.3e}"
    return max_abs, rel


def compare_f32(got, want, what=""):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape
    max_abs = float(np.abs(got - want).max())
    _log(what, max_abs=max_abs, bar_max_abs=F32_MAX_ABS)
    assert max_abs <= F32_MAX_ABS, f"{what}: max_abs={max_abs:.3e}"
    return max_abs


def layer_params_dev(params):
    return {k: (None if v is None else dev(v, torch.bfloat16)) for k, v in params.items()}


@functools.lru_cache(maxsize=4)
def layer_stack(dims: synth.LayerDims, n_layers: int, base_seed: int):
    """Host parameters of a stack of layers drawn with synth.layer_seed."""
    return tuple(synth.layer_params(dims, seed=synth.layer_seed(base_seed, l)) for l in range(n_layers))


def cfg_of(dims: synth.LayerDims):
    import sliding_window_attention_tcgen05_b200 as vx
    return vx.LayerCfg(dims.d_model, dims.n_heads, dims.head_dim, dims.ffn_hidden, dims.window,
                       dims.rope_theta, dims.eps)
