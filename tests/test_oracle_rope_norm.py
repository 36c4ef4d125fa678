"""Pins of the oracle's RoPE (theta 1e6, head_dim 64, split-halves pairing) and
RMSNorm (eps 1e-5) to closed forms and invariants."""
import math

import numpy as np
import pytest

import oracle


def test_rope_position_zero_is_identity():
    x = np.random.default_rng(0).standard_normal((5, 3, 64))
    y = oracle.rope(x, np.zeros(5), 1e6)
    np.testing.assert_array_equal(y, x)


def test_rope_preserves_norm():
    x = np.random.default_rng(1).standard_normal((40, 4, 64))
    pos = np.arange(1000, 1040)
    y = oracle.rope(x, pos, 1e6)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)


@pytest.mark.parametrize("m", [0, 1, 7, 31])
def test_rope_basis_vectors(m):
    # e_m at position p goes to cos(a) e_m + sin(a) e_{m+32}; e_{m+32} goes to
    # -sin(a) e_m + cos(a) e_{m+32}, with a = p * 1e6^(-2m/64).
    D, p = 64, 1234.0
    a = p * (1e6 ** (-2.0 * m / D))
    e = np.zeros((1, 1, D)); e[..., m] = 1.0
    y = oracle.rope(e, np.array([p]), 1e6)[0, 0]
    want = np.zeros(D); want[m] = math.cos(a); want[m + 32] = math.sin(a)
    np.testing.assert_allclose(y, want, atol=1e-12)
    e2 = np.zeros((1, 1, D)); e2[..., m + 32] = 1.0
    y2 = oracle.rope(e2, np.array([p]), 1e6)[0, 0]
    want2 = np.zeros(D); want2[m] = -math.sin(a); want2[m + 32] = math.cos(a)
    np.testing.assert_allclose(y2, want2, atol=1e-12)


def test_rope_scores_depend_only_on_relative_position():
    rng = np.random.default_rng(2)
    q = rng.standard_normal((1, 1, 64))
    k = rng.standard_normal((1, 1, 64))
    def score(pq, pk):
        return float(np.sum(oracle.rope(q, np.array([pq]), 1e6) * oracle.rope(k, np.array([pk]), 1e6)))
    base = score(10, 3)
    for shift in (1, 77, 1000, 5000):
        assert abs(score(10 + shift, 3 + shift) - base) < 1e-9
    assert abs(score(11, 3) - base) > 1e-6


def test_rmsnorm_unit_gain_gives_unit_rms():
    x = np.random.default_rng(3).standard_normal((7, 1280)) * 3.0
    y = oracle.rms_norm(x, np.ones(1280), eps=1e-5)
    ms = np.mean(x * x, axis=-1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=-1)), np.sqrt(ms / (ms + 1e-5)), rtol=1e-13)


def test_rmsnorm_constant_vector():
    c, g = 0.37, np.linspace(0.5, 1.5, 1280)
    y = oracle.rms_norm(np.full((1, 1280), c), g, eps=1e-5)
    np.testing.assert_allclose(y[0], c / math.sqrt(c * c + 1e-5) * g, rtol=1e-14)


def test_silu_and_gelu_special_values():
    z = np.array([0.0, 30.0, -30.0, 1.0])
    np.testing.assert_allclose(oracle.silu(z), [0.0, 30.0, -30.0 * math.exp(-30.0) / (1 + math.exp(-30.0)),
                                                1.0 / (1.0 + math.exp(-1.0))], rtol=1e-12, atol=1e-30)
    # GELU(1) = Phi(1) = 0.8413447460685429 (standard normal CDF at 1).
    np.testing.assert_allclose(oracle.gelu(np.array([0.0, 1.0, -1.0])),
                               [0.0, 0.8413447460685429, -1.0 + 0.8413447460685429], rtol=1e-14)
