"""Pins for the sharded-vocabulary verification and draft (oracle/vocab_parallel.py).

In exact arithmetic the sharded steps (per-shard partials, exchange, merge,
owner draw) give what the unsharded verification gives; in float64 only the
order of sums differs, so on these inputs the results must be identical to
sampling.psi_verify / sampling.draft_sample (themselves pinned by exact
enumeration). Planted slips in the exchange logic must break the equality."""
import numpy as np
import pytest

import workloads as W
from oracle import sampling as S
from oracle import vocab_parallel as VP


def _case(B, k, V, k_p, seed, sigma=1.0, ar_std=3.0):
    c = W.logits_case(B, k, V, k_p=k_p, ar_std=ar_std, sigma=sigma, seed=seed, dtype="f32",
                      threads=1)
    return c.p_logits.astype(np.float64), c.q_logits.astype(np.float64)


def test_shard_bounds_cover_the_vocabulary_in_order():
    for V, G in [(1000, 1), (1000, 3), (1001, 5), (151936, 8), (20, 8)]:
        b = VP.shard_bounds(V, G)
        assert len(b) == G and b[0][0] == 0 and b[-1][1] == V
        assert all(b[i][1] == b[i + 1][0] for i in range(G - 1))
        assert all((hi - lo) % 8 == 0 for lo, hi in b if hi < V)


@pytest.mark.parametrize("G", [1, 2, 3, 5])
@pytest.mark.parametrize("V,k,k_p,T", [(1000, 4, 4, 1.0), (1001, 4, 5, 0.7), (777, 8, 9, 1.0)])
def test_sharded_verification_equals_unsharded(G, V, k, k_p, T):
    B = 12
    p, q = _case(B, k, V, k_p, seed=G * 100 + V)
    d = S.draft_sample(q, T, 3, 1)
    bounds = VP.shard_bounds(V, G)
    got = VP.vp_psi_verify(VP.split(p, bounds), VP.split(q, bounds), bounds, d, T, 7, 2, 5)
    want = S.psi_verify(p, q, d, T, 7, 2, 5)
    for key in ("accepted_len", "out_tokens", "out_count"):
        np.testing.assert_array_equal(got[key], want[key])
    # the cases reach both residual and (when k_p = k + 1) bonus draws
    assert np.any(want["accepted_len"] < k)


@pytest.mark.parametrize("G", [1, 2, 4, 7])
def test_sharded_draft_equals_unsharded(G):
    B, k, V = 6, 5, 2003
    _, q = _case(B, k, V, k, seed=G)
    bounds = VP.shard_bounds(V, G)
    for T in (1.0, 0.7):
        np.testing.assert_array_equal(VP.vp_draft_sample(VP.split(q, bounds), bounds, T, 9, 4, 2),
                                      S.draft_sample(q, T, 9, 4, 2))


def test_equal_distributions_accept_every_block_sharded():
    B, k, V = 8, 6, 500
    p, _ = _case(B, k, V, k + 1, seed=11)
    bounds = VP.shard_bounds(V, 3)
    d = S.draft_sample(p[:, :k], 1.0, 1, 0)
    got = VP.vp_psi_verify(VP.split(p, bounds), VP.split(p[:, :k], bounds), bounds, d, 1.0, 2, 0)
    assert np.all(got["accepted_len"] == k) and np.all(got["out_count"] == k + 1)


@pytest.mark.parametrize("slip", ["owner_first", "local_normaliser", "id_from_first_shard"])
def test_planted_slips_break_the_equality(monkeypatch, slip):
    orig_owner, orig_merge = VP.owner, VP.merge
    if slip == "owner_first":           # the first shard with mass draws, whatever the threshold
        def owner(masses, u):
            own, t, Z = orig_owner(masses, u)
            g = int(np.nonzero(np.asarray(masses) > 0)[0][0])
            return g, u * Z, Z
        monkeypatch.setattr(VP, "owner", owner)
    elif slip == "local_normaliser":    # each shard's own sum taken as the row's normaliser
        def merge(parts):
            M, S_, z = orig_merge(parts)
            return M, np.asarray(parts)[0, :, 1] * np.exp(np.asarray(parts)[0, :, 0] - M), z
        monkeypatch.setattr(VP, "merge", merge)
    else:                                # the drafted token's logit looked up in shard 0 only
        def merge(parts):
            M, S_, _ = orig_merge(parts)
            return M, S_, np.asarray(parts, dtype=np.float64)[0, :, 2]
        monkeypatch.setattr(VP, "merge", merge)
    B, k, V = 16, 6, 1000
    p, q = _case(B, k, V, k + 1, seed=21)
    d = S.draft_sample(q, 1.0, 3, 1)
    bounds = VP.shard_bounds(V, 3)
    got = VP.vp_psi_verify(VP.split(p, bounds), VP.split(q, bounds), bounds, d, 1.0, 7, 2)
    want = S.psi_verify(p, q, d, 1.0, 7, 2)
    assert not (np.array_equal(got["out_tokens"], want["out_tokens"])
                and np.array_equal(got["accepted_len"], want["accepted_len"]))
