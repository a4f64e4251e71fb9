"""Pins for the oracle's gated-LoRA linear (CPU only)."""
from fractions import Fraction

import numpy as np

from oracle.gated_linear import gated_linear


def _rand(seed, M=7, K=11, N=5, r=3):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((M, K)), rng.standard_normal((N, K)), rng.standard_normal((r, K)),
            rng.standard_normal((N, r)))


def test_brute_force_exact_on_integers():
    """Triple loops in exact rationals on small asymmetric integer inputs."""
    rng = np.random.default_rng(1)
    M, K, N, r = 3, 5, 4, 2
    x = rng.integers(-4, 5, (M, K))
    W = rng.integers(-4, 5, (N, K))
    A = rng.integers(-4, 5, (r, K))
    Bl = rng.integers(-4, 5, (N, r))
    g = np.array([0, 1, 1], np.uint8)
    s = Fraction(3, 4)
    y = gated_linear(x, W, A, Bl, g, float(s))
    for m in range(M):
        for n in range(N):
            base = sum(int(x[m, kk]) * int(W[n, kk]) for kk in range(K))
            lora = 0
            for j in range(r):
                t = sum(int(x[m, kk]) * int(A[j, kk]) for kk in range(K))
                lora += t * int(Bl[n, j])
            ref = base + s * int(g[m]) * lora
            assert Fraction(y[m, n]) == ref


def test_gate_zero_is_base_matmul():
    x, W, A, Bl = _rand(2)
    y = gated_linear(x, W, A, Bl, np.zeros(7, np.uint8), 1.0)
    assert np.array_equal(y, x @ W.T)


def test_gate_one_is_merged_weight():
    """Adapter on everywhere == one linear with the merged weight W + s Bl A."""
    x, W, A, Bl = _rand(3)
    s = 0.37
    y = gated_linear(x, W, A, Bl, np.ones(7, np.uint8), s)
    merged = x @ (W + s * Bl @ A).T
    np.testing.assert_allclose(y, merged, rtol=1e-12, atol=1e-12)


def test_zero_adapter_or_zero_scale_is_gate_independent():
    x, W, A, Bl = _rand(4)
    g = np.array([0, 1, 0, 1, 1, 0, 1], np.uint8)
    ref = gated_linear(x, W, A, Bl, np.zeros(7, np.uint8), 1.0)
    assert np.array_equal(gated_linear(x, W, A, np.zeros_like(Bl), g, 1.0), ref)
    assert np.array_equal(gated_linear(x, W, A, Bl, g, 0.0), ref)


def test_gate_is_per_row():
    x, W, A, Bl = _rand(5)
    g = np.array([0, 1, 0, 1, 1, 0, 1], np.uint8)
    y = gated_linear(x, W, A, Bl, g, 0.5)
    on = gated_linear(x, W, A, Bl, np.ones(7, np.uint8), 0.5)
    off = gated_linear(x, W, A, Bl, np.zeros(7, np.uint8), 0.5)
    for m in range(7):
        np.testing.assert_array_equal(y[m], (on if g[m] else off)[m])
