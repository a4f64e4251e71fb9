"""Psi-Spec tree sampler: verification of several drafted blocks laid out as a prefix tree.

Oracle; test infrastructure only (see the package docstring).

What the pages fix (hyper.ai page, section "方法", the Psi-Spec paragraph; the
ainews page, the Psi-Spec paragraph): at low batch sizes the tree sampler draws
several candidate blocks from the draft path, verifies them at once as a prefix
tree, and keeps the output distribution equal to the base AR distribution
(lossless); the first token of each block comes from the AR weights, as in the
linear sampler. The pages give no acceptance rule for several candidates.

Reading taken here (the plainest one that keeps the output law exact, and the
one that reduces to the linear verification for one candidate):
  * candidate i of a sequence draws its token at position j from the draft
    marginal q_j, independently over i and j (the linear sampler, N times);
  * the candidates form a trie; the AR distribution p at a trie node is the
    distribution of the next token after that node's prefix;
  * the walk starts at the root. At a node of depth j the live candidates
    (those whose prefix is the accepted path) are tried in index order:
    candidate i with token x is accepted iff u < min(1, r_i(x) / q_j(x)),
    where r_1 = p(node) and, after each rejection, r_{i+1} = max(r_i - q_j, 0)
    normalised (the residual of a single speculative-sampling step). On
    acceptance the walk moves to the child x, and the candidates with token x
    at depth j stay live; if every live candidate is rejected, a token is
    drawn from the last residual and the block ends. If all k positions are
    accepted and the AR rows of the leaves are given, a bonus token is drawn
    from p(leaf).
  Why this is exact: one test with target r and proposal q emits x with
  probability min(q(x), r(x)) and rejects with probability
  Z = sum(max(r - q, 0)); a further step that emits x ~ max(r - q, 0) / Z
  makes the total min(q, r) + max(r - q, 0) = r. By induction over the live
  candidates the token at each node follows p(node); the candidates' tokens at
  the next depth are independent of everything that decided this one, so the
  same holds one level down.
  If rounding makes a residual mass zero, the target stays unchanged (exactly
  r = q there, which accepts every candidate).

Uniforms (Philox4x32-10, see philox.py), b = global sequence id, N candidates:
  candidate tokens   stream 0, index (b N + i) k + j   (= the linear draft for N = 1)
  accept test        stream 1, index (b k + j) N + i   (= the linear accept for N = 1)
  residual draw      stream 2, index b k + j
  bonus draw         stream 3, index b k + k
Trie node numbering: nodes are numbered in order of first visit when the
candidates are walked from the root in index order; node 0 is the root.
"""
from __future__ import annotations

import numpy as np

from . import philox
from .sampling import (accept_threshold, as_f64, cdf_margin, inverse_cdf, residual_weights,
                       softmax_t)


def tree_candidates(q_logits, N: int, T: float, seed: int, step: int, seq_offset: int = 0):
    """N candidate blocks per sequence: c[b,i,j] ~ softmax(z_q[b,j] / T), stream 0.

    q_logits [B,k,V]; returns int32 [B,N,k].
    """
    q_logits = as_f64(q_logits)
    B, k, V = q_logits.shape
    c = np.empty((B, N, k), dtype=np.int32)
    for b in range(B):
        q = softmax_t(q_logits[b], T)
        bg = b + seq_offset
        idx = (np.uint64(bg) * np.uint64(N) + np.arange(N, dtype=np.uint64)[:, None]) * np.uint64(k) \
            + np.arange(k, dtype=np.uint64)[None, :]
        u = philox.uniforms(seed, step, philox.STREAM_DRAFT, idx)
        for i in range(N):
            for j in range(k):
                c[b, i, j] = inverse_cdf(q[j], u[i, j])
    return c


def trie(cands):
    """Trie of the candidate blocks cands [N,k].

    Returns (node_of [N,k+1] int32: the node reached by candidate i after j
    tokens, node_of[:,0] = 0; parent [n] int32, -1 for the root; token [n]
    int32, the token that leads into the node, -1 for the root; depth [n]).
    """
    cands = np.asarray(cands)
    N, k = cands.shape
    children = [{}]
    parent, token, depth = [-1], [-1], [0]
    node_of = np.zeros((N, k + 1), dtype=np.int32)
    for i in range(N):
        node = 0
        for j in range(k):
            x = int(cands[i, j])
            nxt = children[node].get(x)
            if nxt is None:
                nxt = len(parent)
                children[node][x] = nxt
                children.append({})
                parent.append(node)
                token.append(x)
                depth.append(j + 1)
            node = nxt
            node_of[i, j + 1] = node
    return (node_of, np.asarray(parent, np.int32), np.asarray(token, np.int32),
            np.asarray(depth, np.int32))


def node_tests(r, q, tokens):
    """The test chain at one node: target r (= p of the node), proposal q, the
    live candidates' tokens in order.

    Returns (thresholds, weights): candidate i is accepted iff its uniform is
    below thresholds[i] (when all before it were rejected); `weights` are the
    unnormalised draw weights once every candidate was rejected (the last
    residual max(r - q, 0), or the unchanged target if that mass is zero).
    With one candidate these are exactly the linear verification's residual
    weights. Generic over float and fractions.Fraction arrays.
    """
    r = np.asarray(r)
    q = np.asarray(q)
    ths, weights = [], r
    for x in tokens:
        ths.append(accept_threshold(r[int(x)], q[int(x)]))
        w = residual_weights(r, q)
        z = w.sum()
        if z > 0:
            r, weights = w / z, w
        else:
            weights = r
    return ths, weights


def tree_verify_sequence(p_logits, q_logits, cands, T: float, seed: int, step: int,
                         b_global: int, bonus: bool = False):
    """Verify one sequence's candidate trie.

    p_logits [n_nodes, V]: AR logits of every trie node (numbering of `trie`);
    the rows of depth-k nodes are read only when `bonus`. q_logits [k,V],
    cands [N,k]. Returns a dict: accepted_len n, tokens (the n accepted ones
    plus the residual or bonus token), path (trie nodes visited), draw kind,
    and for comparisons with a lower-precision implementation: test_margin
    (smallest |u - threshold| over the tests taken) and draw_margin (distance
    of the draw's threshold to the nearest CDF edge of the drawn token, / Z).
    """
    p_logits, q_logits = as_f64(p_logits), as_f64(q_logits)
    cands = np.asarray(cands)
    N, k = cands.shape
    node_of, parent, _, _ = trie(cands)
    if p_logits.shape[0] != len(parent):
        raise ValueError(f"p_logits has {p_logits.shape[0]} rows, the trie {len(parent)} nodes")
    q = softmax_t(q_logits, T)
    node, live, tokens, path = 0, list(range(N)), [], [0]
    margin = np.inf
    for j in range(k):
        r = softmax_t(p_logits[node], T)
        ths, resid = node_tests(r, q[j], [cands[i, j] for i in live])
        idx = (np.uint64(b_global * k + j) * np.uint64(N) + np.asarray(live, np.uint64))
        u1 = philox.uniforms(seed, step, philox.STREAM_ACCEPT, idx)
        hit = next((t for t in range(len(live)) if u1[t] < ths[t]), None)
        taken = len(live) if hit is None else hit + 1
        margin = min([margin] + [abs(float(u1[t]) - float(ths[t])) for t in range(taken)])
        if hit is None:
            u2 = philox.uniforms(seed, step, philox.STREAM_RESIDUAL, b_global * k + j)
            v = inverse_cdf(resid, u2)
            tokens.append(v)
            return dict(accepted_len=j, tokens=tokens, path=path, draw="residual",
                        test_margin=margin, draw_margin=cdf_margin(resid, u2, v))
        x = int(cands[live[hit], j])
        tokens.append(x)
        node = int(node_of[live[hit], j + 1])
        path.append(node)
        live = [i for i in live if int(cands[i, j]) == x]
    if bonus:
        u3 = philox.uniforms(seed, step, philox.STREAM_BONUS, b_global * k + k)
        w = softmax_t(p_logits[node], T)
        v = inverse_cdf(w, u3)
        tokens.append(v)
        return dict(accepted_len=k, tokens=tokens, path=path, draw="bonus",
                    test_margin=margin, draw_margin=cdf_margin(w, u3, v))
    return dict(accepted_len=k, tokens=tokens, path=path, draw=None, test_margin=margin,
                draw_margin=np.inf)
