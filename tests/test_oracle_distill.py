"""Pins of the distillation-loss oracle (oracle/distill.py) against what the mathematics fixes."""
import numpy as np
import pytest

from oracle import distill as D
from oracle import sampling as S


def _pair(rows, V, seed, scale=2.0):
    rng = np.random.default_rng(seed)
    zt = rng.normal(0, scale, (rows, V))
    zs = zt + rng.normal(0, 1.0, (rows, V))
    return zt, zs


def test_zero_at_equal_distributions():
    zt, _ = _pair(4, 50, 0)
    kl, tv = D.distill_losses(zt, zt + 3.0)        # a shift of the logits is the same q
    assert np.allclose(kl, 0, atol=1e-14) and np.allclose(tv, 0, atol=1e-14)
    assert np.abs(D.distill_grad(zt, zt, 0.7, 0.3)).max() < 1e-15


def test_closed_forms_on_two_tokens():
    """V = 2: p = (a, 1-a), q = (b, 1-b): KL = a log(a/b) + (1-a) log((1-a)/(1-b)), TV = |a-b|."""
    for zt0, zs0, T in ((0.3, -1.1, 1.0), (2.0, 0.5, 0.7), (-1.5, 1.5, 2.0)):
        zt, zs = np.array([[zt0, 0.0]]), np.array([[zs0, 0.0]])
        a, b = 1 / (1 + np.exp(-zt0 / T)), 1 / (1 + np.exp(-zs0 / T))
        kl, tv = D.distill_losses(zt, zs, T)
        assert kl[0] == pytest.approx(a * np.log(a / b) + (1 - a) * np.log((1 - a) / (1 - b)), rel=1e-12)
        assert tv[0] == pytest.approx(abs(a - b), rel=1e-12)


def test_tv_identity_pinsker_and_acceptance_rate():
    """TV = 1 - sum min(p, q) (so 1 - TV is the accept probability of one speculative test with
    target p and proposal q, as the verification oracle computes it), and TV <= sqrt(KL / 2)."""
    zt, zs = _pair(16, 300, 1)
    kl, tv = D.distill_losses(zt, zs)
    p, q = S.softmax_t(zt, 1.0), S.softmax_t(zs, 1.0)
    np.testing.assert_allclose(tv, 1 - np.minimum(p, q).sum(axis=-1), rtol=0, atol=1e-14)
    resid = np.array([S.residual_weights(p[i], q[i]).sum() for i in range(len(p))])
    np.testing.assert_allclose(1 - tv, 1 - resid, atol=1e-14)     # accept prob = 1 - residual mass
    assert np.all(tv <= np.sqrt(kl / 2) + 1e-15)


def test_gradient_matches_finite_differences():
    """Central differences of the objective (fp64) against the analytic gradient, away
    from the kinks of |p - q| (no entry with p = q)."""
    zt, zs = _pair(3, 12, 2)
    for alpha, beta, T in ((1.0, 0.0, 1.0), (0.0, 1.0, 1.0), (0.6, 0.4, 0.7)):
        g = D.distill_grad(zt, zs, alpha, beta, T)
        h = 1e-6
        num = np.zeros_like(zs)
        for i in range(zs.shape[0]):
            for v in range(zs.shape[1]):
                e = np.zeros_like(zs)
                e[i, v] = h
                num[i, v] = (D.distill_objective(zt, zs + e, alpha, beta, T)
                             - D.distill_objective(zt, zs - e, alpha, beta, T)) / (2 * h)
        np.testing.assert_allclose(g, num, rtol=1e-5, atol=1e-9)


def test_gradient_is_shift_free_and_catches_planted_mistakes():
    """Each row's gradient sums to zero (the loss ignores a constant shift of the logits);
    a sign slip or a dropped term in the TV gradient breaks the finite-difference check."""
    zt, zs = _pair(5, 40, 3)
    g = D.distill_grad(zt, zs, 0.5, 0.5, 0.9)
    assert np.abs(g.sum(axis=-1)).max() < 1e-15
    p, q = S.softmax_t(zt, 1.0), S.softmax_t(zs, 1.0)
    s = np.sign(q - p)
    good = q * (s - (s * q).sum(-1, keepdims=True)) / 2 / len(zs)
    bad_sign = q * (-s - (-s * q).sum(-1, keepdims=True)) / 2 / len(zs)
    bad_drop = q * s / 2 / len(zs)
    h, i, v = 1e-6, 1, 7
    e = np.zeros_like(zs)
    e[i, v] = h
    num = (D.distill_objective(zt, zs + e, 0, 1) - D.distill_objective(zt, zs - e, 0, 1)) / (2 * h)
    assert good[i, v] == pytest.approx(num, rel=1e-5)
    assert bad_sign[i, v] != pytest.approx(num, rel=1e-3)
    assert bad_drop[i, v] != pytest.approx(num, rel=1e-3)
