"""Writes the stored expected values under tests/golden/.

Calls only oracle/ and synth/ (never the CUDA path).  Run from the repo root:
    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
import synth   # noqa: E402

HERE = os.path.dirname(os.path.abspath(__file__))


def c0_tiny_swa_rope_fp32():
    # Tiny causal sliding-window attention with RoPE: B=1, T=64, 2 heads,
    # head_dim 64, window 16, theta 1e6, q/k/v ~ N(0,1) from seed 0 (q, k, v order).
    q, k, v = synth.attention_qkv(1, 64, 2, 64, seed=0)
    pos = np.arange(64)
    o = oracle.swa_attention(oracle.rope(q, pos, 1e6), oracle.rope(k, pos, 1e6), v, window=16)
    np.savez_compressed(os.path.join(HERE, "c0_swa_rope_fp32.npz"), o=o)


if __name__ == "__main__":
    c0_tiny_swa_rope_fp32()
    print("wrote", HERE)
