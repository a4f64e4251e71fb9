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


# ---------------------------------------------------------------- adapter backward (NEXT f4)

def _bw_case(M=7, K=6, N=5, r=3, seed=0):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(M, K)), rng.normal(size=(N, K)), rng.normal(size=(r, K)),
            rng.normal(size=(N, r)), (rng.random(M) < 0.5).astype(np.uint8), 0.8,
            rng.normal(size=(M, N)))


def test_adapter_grads_match_finite_differences():
    from oracle.gated_linear import gated_linear_adapter_grads
    x, W, A, Bl, g, s, dy = _bw_case()
    dA, dBl = gated_linear_adapter_grads(x, A, Bl, g, s, dy)
    f = lambda A_, Bl_: float((dy * gated_linear(x, W, A_, Bl_, g, s)).sum())
    h = 1e-6
    for P, G, name in ((A, dA, "A"), (Bl, dBl, "Bl")):
        num = np.zeros_like(P)
        for idx in np.ndindex(P.shape):
            e = np.zeros_like(P)
            e[idx] = h
            num[idx] = ((f(A + e, Bl) - f(A - e, Bl)) if name == "A" else
                        (f(A, Bl + e) - f(A, Bl - e))) / (2 * h)
        np.testing.assert_allclose(G, num, rtol=1e-6, atol=1e-8)


def test_adapter_grads_special_cases():
    """Gate 0 everywhere or scale 0: no gradient; gate 1 everywhere: the merged-weight
    form y = x (W + s Bl A)^T gives dBl = s dy^T x A^T and dA = s Bl^T dy^T x."""
    from oracle.gated_linear import gated_linear_adapter_grads
    x, W, A, Bl, g, s, dy = _bw_case(seed=1)
    for gate, scale in ((np.zeros_like(g), s), (g, 0.0)):
        dA, dBl = gated_linear_adapter_grads(x, A, Bl, gate, scale, dy)
        assert not dA.any() and not dBl.any()
    ones = np.ones_like(g)
    dA, dBl = gated_linear_adapter_grads(x, A, Bl, ones, s, dy)
    np.testing.assert_allclose(dBl, s * dy.T @ x @ A.T, rtol=1e-12)
    np.testing.assert_allclose(dA, s * Bl.T @ dy.T @ x, rtol=1e-12)
    # only gate-1 rows count: the gradient equals that of the gate-1 rows alone
    keep = g.astype(bool)
    dA1, dBl1 = gated_linear_adapter_grads(x[keep], A, Bl, ones[keep], s, dy[keep])
    dA, dBl = gated_linear_adapter_grads(x, A, Bl, g, s, dy)
    np.testing.assert_allclose(dA, dA1, rtol=1e-12)
    np.testing.assert_allclose(dBl, dBl1, rtol=1e-12)
