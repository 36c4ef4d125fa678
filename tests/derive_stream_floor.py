"""Derives the bf16 rounding floor of the streaming config as stated (CPU,
float64, several minutes; run by hand, not collected by pytest):

    python tests/derive_stream_floor.py

32 layers of the one-layer shape, streams 0 and 63 of the 64, frames
0..1003 (the 1000-frame prefill and the 4-frame step together equal the
whole-sequence forward, by causality): the oracle, and the oracle with the
GPU's bf16 operand roundings added (tests/test_rounding_floor.py), compared on
frames 1000..1003, raw and after the final RMSNorm.  The numbers it prints
are the ones recorded beside C3_STATED_MAX_ABS in tests/test_rounding_floor.py."""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, HERE)
sys.path.insert(0, os.path.dirname(HERE))

import oracle  # noqa: E402
import synth  # noqa: E402
import test_rounding_floor as F  # noqa: E402


def main():
    dims = synth.VOXTRAL_RT
    layers = F._stack32()
    x = synth.frames(64, 1004, dims.d_model, seed=7)[[0, 63]].astype(np.float64)
    ref, h = x, x
    for p in layers:
        ref = oracle.encoder_layer(ref, p, dims)
        h = F._layer_bf16_operands(h, p, dims, True)
    g = synth.final_norm_gain(dims.d_model, seed=5).astype(np.float64)
    for name, a, b in (("raw", h, ref), ("final norm", oracle.rms_norm(h, g), oracle.rms_norm(ref, g))):
        e = a[:, 1000:] - b[:, 1000:]
        print(f"{name}: max_abs {np.abs(e).max():.3e}  rel_l2 {np.linalg.norm(e) / np.linalg.norm(b[:, 1000:]):.3e}  "
              f"max |value| {np.abs(b[:, 1000:]).max():.2f}")


if __name__ == "__main__":
    main()
