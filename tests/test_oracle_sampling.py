"""Pins for the oracle's sampler and verification (CPU only).

The key pin is exact: on V=8, k=2 the law of the emitted tokens, summed over
every draft and integrated over the accept/residual randomness in rational
arithmetic, equals p_1 x p_2 (x p_3 with the bonus row) — the "lossless"
property (ainews page: same sampling distribution as the base AR model;
hyper.ai page, section "方法": first token from theta_AR, longest accepted
prefix). It runs the oracle's own accept and residual helpers on Fractions.
"""
from fractions import Fraction
from itertools import product

import numpy as np
import pytest
from scipy import special, stats

from oracle import philox
from oracle import sampling as S


# ---------------------------------------------------------------- softmax, inverse CDF

def test_softmax_matches_library_and_temperature():
    z = np.random.default_rng(0).standard_normal((3, 50)) * 4
    for T in (1.0, 0.7, 2.5):
        np.testing.assert_allclose(S.softmax_t(z, T), special.softmax(z / T, axis=-1), rtol=1e-13)
    np.testing.assert_allclose(S.softmax_t(z + 123.0, 0.7), S.softmax_t(z, 0.7), rtol=1e-12)
    with pytest.raises(ValueError):
        S.softmax_t(z, 0.0)


def test_inverse_cdf_brute_force():
    """Every threshold on a grid, checked against the definition by a linear walk."""
    w = [Fraction(0), Fraction(3), Fraction(0), Fraction(1), Fraction(4), Fraction(0)]
    total = sum(w)
    for num in range(0, 64):
        u = Fraction(num, 64)
        t = u * total
        run, expect = Fraction(0), None
        for v, wv in enumerate(w):
            run += wv
            if run > t:
                expect = v
                break
        assert S.inverse_cdf(np.array(w, dtype=object), u) == expect
        assert S.inverse_cdf(np.array([float(x) for x in w]), float(u)) == expect
    # u = 0 skips leading zero weights; ids with zero weight are never returned
    assert S.inverse_cdf(np.array([0.0, 0.0, 2.0, 1.0]), 0.0) == 2


def test_inverse_cdf_rounding_fallback():
    w = np.array([0.5, 0.5, 0.0])
    assert S.inverse_cdf(w, 1.0) == 1      # threshold == total -> last positive id


def test_residual_and_threshold_generic():
    p = np.array([Fraction(1, 2), Fraction(1, 4), Fraction(1, 4)], dtype=object)
    q = np.array([Fraction(1, 4), Fraction(1, 2), Fraction(1, 4)], dtype=object)
    assert list(S.residual_weights(p, q)) == [Fraction(1, 4), 0, 0]
    assert S.accept_threshold(Fraction(1, 4), Fraction(1, 2)) == Fraction(1, 2)
    assert S.accept_threshold(Fraction(1, 2), Fraction(1, 4)) == 1
    assert S.accept_threshold(Fraction(1, 2), 0) == 1


# ---------------------------------------------------------------- exact enumeration

def _dist(weights):
    t = sum(weights)
    return np.array([Fraction(w, t) for w in weights], dtype=object)


# Small-integer weights: q > p and q < p cases, a token with p = 0 < q, one with q = 0 < p.
P_ROWS = [_dist([5, 1, 0, 3, 2, 7, 1, 1]), _dist([1, 1, 4, 2, 0, 6, 2, 3]), _dist([2, 3, 1, 1, 4, 1, 5, 3])]
Q_ROWS = [_dist([2, 4, 3, 3, 0, 3, 2, 3]), _dist([3, 1, 1, 2, 5, 2, 1, 1])]


def _emitted_law(p_rows, q_rows, K):
    """Exact law of the first K emitted tokens under the Psi-Spec linear step.

    Drafts d ~ prod q_j; accept d_j with probability accept_threshold; at the
    first rejection j emit r ~ residual_weights / Z; if all k drafts pass and a
    (k+1)-th AR row is present emit the bonus from it. Positions after the
    step come from p (the next step starts with a token from theta_AR), which
    with independent positions means the product of the remaining p rows.
    """
    k = len(q_rows)
    V = len(p_rows[0])
    law = {}

    def add(prefix, mass):
        rest = list(range(len(prefix), K))
        for tail in product(range(V), repeat=len(rest)):
            w = mass
            for j, t in zip(rest, tail):
                w *= p_rows[j][t]
            if w:
                key = tuple(prefix) + tail
                law[key] = law.get(key, 0) + w

    for d in product(range(V), repeat=k):
        mass = Fraction(1)
        for j in range(k):
            mass *= q_rows[j][d[j]]
        if mass == 0:
            continue
        for j in range(k):
            a = S.accept_threshold(p_rows[j][d[j]], q_rows[j][d[j]])
            rej = mass * (1 - a)
            if rej:
                R = S.residual_weights(p_rows[j], q_rows[j])
                Z = sum(R)
                for r in range(V):
                    if R[r]:
                        add(list(d[:j]) + [r], rej * R[r] / Z)
            mass *= a
        if K == k + 1:
            for b in range(V):
                if p_rows[k][b]:
                    add(list(d) + [b], mass * p_rows[k][b])
        else:
            add(list(d), mass)
    return law


def _product_law(p_rows, K):
    V = len(p_rows[0])
    law = {}
    for t in product(range(V), repeat=K):
        w = Fraction(1)
        for j in range(K):
            w *= p_rows[j][t[j]]
        if w:
            law[t] = w
    return law


def test_exact_enumeration_lossless_k2():
    law = _emitted_law(P_ROWS[:2], Q_ROWS, K=2)
    assert sum(law.values()) == 1
    assert law == _product_law(P_ROWS[:2], 2)


def test_exact_enumeration_lossless_with_bonus():
    law = _emitted_law(P_ROWS, Q_ROWS, K=3)
    assert law == _product_law(P_ROWS, 3)


@pytest.mark.parametrize("mutant", ["inverted_ratio", "residual_sign", "residual_q"])
def test_enumeration_catches_planted_mistakes(monkeypatch, mutant):
    """A plausible mistake in the oracle's helpers breaks the exact pin."""
    if mutant == "inverted_ratio":
        monkeypatch.setattr(S, "accept_threshold",
                            lambda p, q: 1 if p == 0 or q / p >= 1 else q / p)
    elif mutant == "residual_sign":
        orig = S.residual_weights
        monkeypatch.setattr(S, "residual_weights", lambda p, q: orig(q, p))
    else:
        monkeypatch.setattr(S, "residual_weights", lambda p, q: np.asarray(p) * 1)
    assert _emitted_law(P_ROWS[:2], Q_ROWS, K=2) != _product_law(P_ROWS[:2], 2)


# ---------------------------------------------------------------- sampled behaviour

def _small_logits(seed, B, k, V, sigma, k_p=None):
    rng = np.random.default_rng(seed)
    k_p = k if k_p is None else k_p
    ar = rng.standard_normal((B, k_p, V)) * 1.5
    q = ar[:, :k] + rng.standard_normal((B, k, V)) * sigma
    return ar, q


def test_zero_adapter_accepts_every_block():
    """Bl = 0 makes q == p: every draft is accepted, n = k, at any seed."""
    for seed in range(5):
        ar, _ = _small_logits(seed, 16, 6, 40, 0.0)
        for T in (1.0, 0.7):
            d = S.draft_sample(ar, T, seed, 3)
            res = S.psi_verify(ar, ar, d, T, seed, 3)
            assert np.all(res["accepted_len"] == 6)
            assert np.all(res["out_count"] == 6)
            assert np.array_equal(res["out_tokens"][:, :6], d)


def test_bonus_row_adds_one_token_when_all_accepted():
    ar, _ = _small_logits(1, 8, 4, 30, 0.0, k_p=5)
    d = S.draft_sample(ar[:, :4], 1.0, 9, 0)
    res = S.psi_verify(ar, ar[:, :4], d, 1.0, 9, 0)
    assert np.all(res["out_count"] == 5)
    assert np.all((res["out_tokens"][:, 4] >= 0) & (res["out_tokens"][:, 4] < 30))


def test_draft_sampler_chi_square():
    V, T = 8, 0.7
    rng = np.random.default_rng(3)
    z = rng.standard_normal(V) * 2
    B, k = 2500, 8
    logits = np.broadcast_to(z, (B, k, V))
    d = S.draft_sample(logits, T, 11, 0)
    counts = np.bincount(d.ravel(), minlength=V)
    expect = S.softmax_t(z, T) * d.size
    assert stats.chisquare(counts, expect).pvalue > 1e-3


def test_acceptance_closed_forms():
    """P(accept at j) = sum_v min(p_j, q_j); E[n] = sum_j prod_{i<=j} alpha_i (4 sigma)."""
    B, k, V, T, seed = 20000, 3, 6, 1.0, 21
    rng = np.random.default_rng(8)
    ar = rng.standard_normal((k, V)) * 1.5
    qz = ar + rng.standard_normal((k, V)) * 1.0
    p, q = S.softmax_t(ar, T), S.softmax_t(qz, T)
    alpha = np.minimum(p, q).sum(axis=1)
    P = np.broadcast_to(ar, (B, k, V))
    Q = np.broadcast_to(qz, (B, k, V))
    d = S.draft_sample(Q, T, seed, 0)
    res = S.psi_verify(P, Q, d, T, seed, 0)
    n = res["accepted_len"]
    # first position: empirical accept rate vs alpha_0
    acc0 = np.mean(n >= 1)
    sd0 = np.sqrt(alpha[0] * (1 - alpha[0]) / B)
    assert abs(acc0 - alpha[0]) < 4 * sd0
    expect_n = sum(np.prod(alpha[: j + 1]) for j in range(k))
    sd_n = n.std() / np.sqrt(B)
    assert abs(n.mean() - expect_n) < 4 * sd_n
    # conditional rejection law at position 0: residual max(p-q,0)/Z
    rej0 = n == 0
    toks = res["out_tokens"][rej0, 0]
    R = np.maximum(p[0] - q[0], 0)
    R /= R.sum()
    keep = R > 0
    counts = np.bincount(toks, minlength=V)
    assert counts[~keep].sum() == 0
    assert stats.chisquare(counts[keep], R[keep] * rej0.sum()).pvalue > 1e-3


def test_emitted_first_token_follows_p():
    """Marginal of the first emitted token is p_0 (sampled check of losslessness)."""
    B, k, V, T, seed = 20000, 2, 6, 0.7, 5
    rng = np.random.default_rng(2)
    ar = rng.standard_normal((k, V)) * 1.5
    qz = ar + rng.standard_normal((k, V)) * 1.5
    P = np.broadcast_to(ar, (B, k, V))
    Q = np.broadcast_to(qz, (B, k, V))
    d = S.draft_sample(Q, T, seed, 0)
    res = S.psi_verify(P, Q, d, T, seed, 0)
    counts = np.bincount(res["out_tokens"][:, 0], minlength=V)
    assert stats.chisquare(counts, S.softmax_t(ar[0], T) * B).pvalue > 1e-3


def test_counter_layout_and_offset():
    """Sharded batches reproduce the unsharded draws when given the sequence offset."""
    ar, qz = _small_logits(4, 6, 4, 32, 1.0)
    d = S.draft_sample(qz, 1.0, 77, 2)
    full = S.psi_verify(ar, qz, d, 1.0, 77, 2)
    lo = S.psi_verify(ar[:3], qz[:3], d[:3], 1.0, 77, 2)
    hi = S.psi_verify(ar[3:], qz[3:], d[3:], 1.0, 77, 2, seq_offset=3)
    assert np.array_equal(np.concatenate([lo["out_tokens"], hi["out_tokens"]]), full["out_tokens"])
    d_hi = S.draft_sample(qz[3:], 1.0, 77, 2, seq_offset=3)
    assert np.array_equal(d_hi, d[3:])
    # the accept uniforms are the Philox stream-1 draws at index b*k + j
    diag = full["diags"][5]
    np.testing.assert_array_equal(diag["u_accept"],
                                  [philox.uniform_scalar(77, 2, 1, 5 * 4 + j) for j in range(4)])
