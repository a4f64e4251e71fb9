"""Pins of the tree-sampler oracle (oracle/tree.py) against what the mathematics fixes.

* one candidate: exactly the linear verification (its own pins in test_oracle_sampling.py);
* exact enumeration in rationals over every candidate draw: the emitted tokens
  follow the AR law, prefix by prefix, with and without the bonus token; the
  enumeration runs the oracle's own per-node arithmetic (node_tests), and
  planted mistakes in that arithmetic are caught;
* the Philox-driven walk against the exact law conditional on fixed candidates (chi-square);
* special cases and closed forms.
"""
import itertools
from fractions import Fraction

import numpy as np
import pytest

from oracle import sampling, tree

F = Fraction


# ---------------------------------------------------------------- one candidate = linear

@pytest.mark.parametrize("k,T,bonus", [(1, 1.0, False), (3, 0.7, True), (6, 1.0, True)])
def test_one_candidate_is_the_linear_verification(k, T, bonus):
    rng = np.random.default_rng(k)
    B, V = 40, 64
    pl = rng.normal(0, 2, (B, k + 1, V))
    ql = pl[:, :k] + rng.normal(0, 1.0, (B, k, V))
    c = tree.tree_candidates(ql, 1, T, seed=11, step=3, seq_offset=5)
    d = sampling.draft_sample(ql, T, 11, 3, seq_offset=5)
    np.testing.assert_array_equal(c[:, 0, :], d)
    p_rows = pl if bonus else pl[:, :k]
    lens = []
    for b in range(B):
        lin = sampling.verify_sequence(p_rows[b], ql[b], d[b], T, 17, 4, b + 5)
        # the one-candidate trie is a chain of k + 1 nodes: the AR rows in order
        tr = tree.tree_verify_sequence(pl[b], ql[b], c[b], T, 17, 4, b + 5, bonus=bonus)
        assert tr["accepted_len"] == lin["accepted_len"]
        assert tr["tokens"] == lin["tokens"]
        lens.append(lin["accepted_len"])
    assert len(set(lens)) > 1          # the cases reach different rejection points


# ---------------------------------------------------------------- trie

def test_trie_numbering_and_structure():
    rng = np.random.default_rng(2)
    for _ in range(50):
        N, k = rng.integers(1, 6), rng.integers(1, 5)
        c = rng.integers(0, 3, (N, k))
        node_of, parent, token, depth = tree.trie(c)
        prefixes = {(): 0}
        next_id = 1
        for i in range(N):
            for j in range(k):
                pre = tuple(c[i, :j + 1])
                if pre not in prefixes:        # first visit in walk order gets the next id
                    prefixes[pre] = next_id
                    next_id += 1
                n = node_of[i, j + 1]
                assert n == prefixes[pre]
                assert parent[n] == node_of[i, j] and token[n] == c[i, j] and depth[n] == j + 1
        assert len(parent) == len(prefixes) and parent[0] == -1 and node_of[:, 0].tolist() == [0] * N


# ---------------------------------------------------------------- exact enumeration

def _rand_dist(rng, V, zero=None):
    w = [F(int(x)) for x in rng.integers(1, 6, V)]
    if zero is not None:
        w[zero] = F(0)
    s = sum(w)
    return np.array([x / s for x in w], dtype=object)


def _ar_table(rng, V, depth):
    """An AR model: a distribution for every prefix of length < depth (some with a zero)."""
    tab = {}
    for L in range(depth):
        for pre in itertools.product(range(V), repeat=L):
            tab[pre] = _rand_dist(rng, V, zero=int(rng.integers(0, V)) if rng.random() < 0.3 else None)
    return tab


def _tree_law(tab, q, N, k, V, bonus, tests=tree.node_tests):
    """Exact law of the emitted block, filled up to L = k (+1) tokens from the AR model
    (the next step starts from the AR weights), over all candidate draws and uniforms."""
    L = k + 1 if bonus else k
    law = {}

    def fill(pre, prob):
        if len(pre) == L:
            law[pre] = law.get(pre, F(0)) + prob
            return
        for x in range(V):
            if tab[pre][x]:
                fill(pre + (x,), prob * tab[pre][x])

    def walk(c, pre, live, prob):
        j = len(pre)
        if j == k:
            if bonus:
                for x in range(V):
                    if tab[pre][x]:
                        fill(pre + (x,), prob * tab[pre][x])
            else:
                fill(pre, prob)
            return
        ths, w = tests(tab[pre], q[j], [c[i][j] for i in live])
        rest = prob
        for t, i in enumerate(live):
            x = c[i][j]
            th = F(ths[t])
            walk(c, pre + (x,), [i2 for i2 in live if c[i2][j] == x], rest * th)
            rest *= 1 - th
        z = sum(w)
        for y in range(V):
            if w[y]:
                fill(pre + (y,), rest * w[y] / z)

    for flat in itertools.product(range(V), repeat=N * k):
        c = [flat[i * k:(i + 1) * k] for i in range(N)]
        pc = F(1)
        for i in range(N):
            for j in range(k):
                pc *= q[j][c[i][j]]
        if pc:
            walk(c, (), list(range(N)), pc)
    return {seq: pr for seq, pr in law.items() if pr}


def _ar_law(tab, V, L):
    law = {}
    for seq in itertools.product(range(V), repeat=L):
        pr = F(1)
        for j in range(L):
            pr *= tab[seq[:j]][seq[j]]
        if pr:
            law[seq] = pr
    return law


@pytest.mark.parametrize("V,k,N,bonus", [(3, 2, 2, False), (3, 1, 3, False), (2, 3, 2, False),
                                         (3, 2, 2, True), (4, 1, 2, True)])
def test_exact_enumeration_lossless(V, k, N, bonus):
    rng = np.random.default_rng(V * 100 + k * 10 + N)
    tab = _ar_table(rng, V, k + 1)
    q = [_rand_dist(rng, V, zero=0 if j == 0 else None) for j in range(k)]
    law = _tree_law(tab, q, N, k, V, bonus)
    assert law == _ar_law(tab, V, k + 1 if bonus else k)


def test_enumeration_catches_planted_mistakes():
    """Each plausible slip in the per-node arithmetic changes the exact law."""
    V, k, N = 3, 2, 2
    rng = np.random.default_rng(7)
    tab = _ar_table(rng, V, k)
    q = [_rand_dist(rng, V) for _ in range(k)]
    target = _ar_law(tab, V, k)

    def no_residual_update(r, qq, toks):   # every candidate tested against p itself
        ths = [sampling.accept_threshold(r[x], qq[x]) for x in toks]
        return ths, sampling.residual_weights(r, qq)

    def flipped_residual(r, qq, toks):      # max(q - r, 0) instead of max(r - q, 0)
        ths, _ = tree.node_tests(r, qq, toks)
        return ths, sampling.residual_weights(qq, r)

    def draw_from_p(r, qq, toks):           # after all rejections, draw from p
        ths, _ = tree.node_tests(r, qq, toks)
        return ths, np.asarray(r)

    def ratio_inverted(r, qq, toks):        # min(1, q/p)
        ths, w = tree.node_tests(r, qq, toks)
        return [sampling.accept_threshold(qq[x], r[x]) for x in toks], w

    for bad in (no_residual_update, flipped_residual, draw_from_p, ratio_inverted):
        assert _tree_law(tab, q, N, k, V, False, tests=bad) != target, bad.__name__


# ---------------------------------------------------------------- the Philox walk

def test_walk_matches_the_exact_conditional_law():
    """Fixed candidates (with a shared first token), many (seed, step) pairs: the
    frequencies of the oracle's emitted blocks follow the exact law given those
    candidates (chi-square)."""
    from scipy import stats
    V, k, N, T = 4, 2, 3, 1.0
    rng = np.random.default_rng(5)
    pl_root = rng.normal(0, 1, V)
    pl_child = {x: rng.normal(0, 1, V) for x in range(V)}
    ql = rng.normal(0, 1, (k, V))
    c = np.array([[1, 2], [1, 0], [3, 3]])
    node_of, parent, token, depth = tree.trie(c)
    rows = []
    for n in range(len(parent)):
        rows.append(pl_root if depth[n] == 0 else pl_child[int(token[n])] if depth[n] == 1
                    else rng.normal(0, 1, V))
    p_nodes = np.stack(rows)
    # exact law given c, in float64 through the oracle's node arithmetic
    p = {(): sampling.softmax_t(pl_root, T)}
    for x in range(V):
        p[(x,)] = sampling.softmax_t(pl_child[x], T)
    q = sampling.softmax_t(ql, T)
    law = {}

    def walk(pre, live, prob):
        j = len(pre)
        if j == k:
            law[pre] = law.get(pre, 0.0) + prob
            return
        ths, w = tree.node_tests(p[pre], q[j], [c[i, j] for i in live])
        rest = prob
        for t, i in enumerate(live):
            x = int(c[i, j])
            walk(pre + (x,), [i2 for i2 in live if c[i2, j] == x], rest * ths[t])
            rest *= 1 - ths[t]
        for y in range(V):
            law[pre + (y,)] = law.get(pre + (y,), 0.0) + rest * w[y] / w.sum()

    walk((), list(range(N)), 1.0)
    n = 20000
    counts = {}
    for s in range(n):
        r = tree.tree_verify_sequence(p_nodes, ql, c, T, seed=s, step=s // 7, b_global=s % 3)
        key = tuple(r["tokens"])
        counts[key] = counts.get(key, 0) + 1
    keys = sorted(law)
    exp = np.array([law[kk] * n for kk in keys])
    obs = np.array([counts.get(kk, 0) for kk in keys])
    assert sum(counts.values()) == obs.sum()          # no block outside the support
    big = exp >= 5
    obs_b = np.append(obs[big], obs[~big].sum())
    exp_b = np.append(exp[big], exp[~big].sum())
    if exp_b[-1] == 0:
        obs_b, exp_b = obs_b[:-1], exp_b[:-1]
    assert stats.chisquare(obs_b, exp_b).pvalue > 1e-3


# ---------------------------------------------------------------- special cases, closed forms

def test_zero_adapter_accepts_every_block():
    """q_j equal to the AR law at every node of depth j: every block is accepted."""
    rng = np.random.default_rng(3)
    V, k, N = 32, 4, 3
    ql = rng.normal(0, 2, (k, V))
    for s in range(30):
        c = tree.tree_candidates(ql[None], N, 1.0, seed=s, step=1)[0]
        node_of, parent, token, depth = tree.trie(c)
        p_nodes = np.stack([ql[min(int(depth[n]), k - 1)] for n in range(len(parent))])
        r = tree.tree_verify_sequence(p_nodes, ql, c, 1.0, seed=s + 100, step=2, b_global=0)
        assert r["accepted_len"] == k and r["tokens"] == c[0].tolist()


def test_rejection_probability_closed_form():
    """One position, N i.i.d. candidates: P(all rejected) = prod_i Z_i, with Z_i the
    residual mass of the i-th test (each Z_i = 1 - sum(min(r_i, q)))."""
    V, N = 16, 3
    rng = np.random.default_rng(9)
    pl, ql = rng.normal(0, 1.5, V), rng.normal(0, 1.5, V)
    p, q = sampling.softmax_t(pl, 1.0), sampling.softmax_t(ql, 1.0)
    zs, r = [], p
    for _ in range(N):
        w = sampling.residual_weights(r, q)
        zs.append(w.sum())
        r = w / w.sum()
    p_rej = float(np.prod(zs))
    n, rej = 30000, 0
    c_all = tree.tree_candidates(np.tile(ql, (n, 1, 1)), N, 1.0, seed=4, step=0)
    for b in range(n):
        node_of, parent, _, _ = tree.trie(c_all[b])
        p_nodes = np.tile(pl, (len(parent), 1))
        rej += tree.tree_verify_sequence(p_nodes, ql[None], c_all[b], 1.0, 8, 0, b)["accepted_len"] == 0
    sd = np.sqrt(p_rej * (1 - p_rej) / n)
    assert abs(rej / n - p_rej) < 4 * sd
