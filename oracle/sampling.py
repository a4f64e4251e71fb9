"""Psi-Spec linear sampler and lossless verification (oracle; test infrastructure).

What the method computes (hyper.ai page, section "方法", the Psi-Spec
paragraph; ainews page, the Psi-Spec paragraph):
  * the draft path proposes one block of k tokens drawn from its per-position
    marginal distributions q_j (the linear sampler);
  * the block is checked by rejection sampling against the base AR
    distributions p_j, and the longest accepted prefix is kept;
  * "lossless" means the emitted tokens follow p exactly in distribution.
Position convention: the AR model reads the distribution of token l from its
output at position l-1 (same section, the factorisation with the shift).

The textbook steps used where the pages stop (speculative sampling:
Leviathan, Kalman & Matias 2023; Chen et al. 2023):
  accept d_j iff u1 < min(1, p_j(d_j) / q_j(d_j));
  n = index of the first rejection (k if none);
  if n < k, emit d_0..d_{n-1} and r ~ max(p_n - q_n, 0) / Z;
  if n = k and an extra AR row p_k exists, emit the bonus b ~ p_k.
Readings fixed here (the pages are silent): temperature T divides both p and q
logits; a categorical draw with weights w and uniform u returns the smallest
vocab id v whose inclusive cumulative weight (ascending id) exceeds u * sum(w);
if the residual mass Z is zero the residual draw falls back to p_n.

All arithmetic is float64. The generic helpers (`accept_threshold`,
`residual_weights`, `inverse_cdf`) also work on numpy object arrays of
fractions.Fraction, which the exact-enumeration pin uses.
"""
from __future__ import annotations

import numpy as np

from . import philox


# ---------------------------------------------------------------- generic helpers

def as_f64(a):
    """Widen float arrays, or bf16 bit patterns held as uint16, to float64 (exact)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def softmax_t(z, T: float):
    """softmax(z / T) along the last axis, float64, max-subtracted."""
    if not T > 0:
        raise ValueError("temperature must be > 0")
    x = np.asarray(z, dtype=np.float64) / float(T)
    x = x - x.max(axis=-1, keepdims=True)
    e = np.exp(x)
    return e / e.sum(axis=-1, keepdims=True)


def inverse_cdf(weights, u):
    """Smallest v with C(v) > u * C(V-1), C = inclusive cumsum in ascending id.

    If rounding puts the threshold at or above the total, the last id with
    positive weight is returned. Works on float and Fraction arrays.
    """
    w = np.asarray(weights)
    c = np.cumsum(w)
    threshold = u * c[-1]
    v = int(np.searchsorted(c, threshold, side="right"))
    if v >= len(w):
        v = int(np.nonzero(w > 0)[0][-1])
    return v


def cdf_margin(weights, u, v):
    """Distance of the threshold u*Z to the nearer edge of token v's CDF interval, / Z."""
    w = np.asarray(weights, dtype=np.float64)
    c = np.cumsum(w)
    z = c[-1]
    t = u * z
    lo = c[v - 1] if v > 0 else 0.0
    return float(min(abs(t - lo), abs(c[v] - t)) / z)


def accept_threshold(p_d, q_d):
    """The u-threshold of the accept test: d is accepted iff u < min(1, p(d)/q(d)).

    q(d) = 0 cannot occur for a draft drawn from q; it is treated as accept.
    """
    if q_d == 0:
        return 1
    ratio = p_d / q_d
    return 1 if ratio >= 1 else ratio


def residual_weights(p, q):
    """Unnormalised residual max(p - q, 0), elementwise."""
    diff = np.asarray(p) - np.asarray(q)
    return np.where(diff > 0, diff, diff * 0)


# ---------------------------------------------------------------- draft sampler

def draft_sample(q_logits, T: float, seed: int, step: int, seq_offset: int = 0):
    """Linear sampler: d[b,j] ~ softmax(z_q[b,j] / T), uniform from stream 0.

    q_logits [B,k,V] (float); returns int32 [B,k].
    """
    q_logits = as_f64(q_logits)
    B, k, V = q_logits.shape
    idx = (np.arange(B, dtype=np.uint64)[:, None] + np.uint64(seq_offset)) * np.uint64(k) \
        + np.arange(k, dtype=np.uint64)[None, :]
    u = philox.uniforms(seed, step, philox.STREAM_DRAFT, idx)
    d = np.empty((B, k), dtype=np.int32)
    for b in range(B):
        q = softmax_t(q_logits[b], T)
        for j in range(k):
            d[b, j] = inverse_cdf(q[j], u[b, j])
    return d


# ---------------------------------------------------------------- verification

def verify_sequence(p_logits, q_logits, draft, T: float, seed: int, step: int, b_global: int):
    """Verify one sequence's block. p_logits [k_p,V], q_logits [k,V], draft [k].

    Returns a dict with accepted_len n, the emitted tokens, and diagnostics:
      u_accept[j], ratio[j] = p_j(d_j)/q_j(d_j) (inf if q = 0),
      draw ("residual", "residual_p", "bonus" or None), u_draw, draw_margin
      (distance of the draw's threshold to the nearest CDF edge of the chosen
      token, relative to the total weight).
    """
    p_logits, q_logits = as_f64(p_logits), as_f64(q_logits)
    k, V = q_logits.shape
    k_p = p_logits.shape[0]
    if k_p not in (k, k + 1):
        raise ValueError("k_p must be k or k+1")
    p = softmax_t(p_logits, T)
    q = softmax_t(q_logits, T)
    base = b_global * k
    u1 = philox.uniforms(seed, step, philox.STREAM_ACCEPT, np.arange(base, base + k))
    ratio = np.empty(k)
    n = k
    for j in range(k):
        d = int(draft[j])
        pd, qd = p[j, d], q[j, d]
        ratio[j] = pd / qd if qd > 0 else np.inf
        if n == k and not (u1[j] < accept_threshold(pd, qd)):
            n = j
    tokens = [int(t) for t in draft[:n]]
    out = dict(accepted_len=n, u_accept=u1, ratio=ratio, draw=None, u_draw=None,
               draw_margin=None, draw_token=None)
    if n < k:
        u2 = philox.uniforms(seed, step, philox.STREAM_RESIDUAL, base + n)
        w = residual_weights(p[n], q[n])
        kind = "residual"
        if not w.sum() > 0:
            w, kind = p[n], "residual_p"
        r = inverse_cdf(w, u2)
        out.update(draw=kind, u_draw=float(u2), draw_token=r, draw_margin=cdf_margin(w, u2, r))
        tokens.append(r)
    elif k_p == k + 1:
        u3 = philox.uniforms(seed, step, philox.STREAM_BONUS, base + k)
        w = p[k]
        r = inverse_cdf(w, u3)
        out.update(draw="bonus", u_draw=float(u3), draw_token=r, draw_margin=cdf_margin(w, u3, r))
        tokens.append(r)
    out["tokens"] = tokens
    return out


def psi_verify(p_logits, q_logits, draft, T: float, seed: int, step: int,
               seq_offset: int = 0, sequences=None):
    """Batch verification: p_logits [B,k_p,V], q_logits [B,k,V], draft [B,k].

    Returns accepted_len [B], out_tokens [B,k+1] (-1 padded), out_count [B]
    and the per-sequence diagnostics list. `sequences` restricts the work to
    a subset of b (the other rows stay -1 / 0).
    """
    p_logits = np.asarray(p_logits)
    q_logits = np.asarray(q_logits)
    B, k, V = q_logits.shape
    acc = np.zeros(B, np.int32)
    out_tokens = np.full((B, k + 1), -1, np.int32)
    count = np.zeros(B, np.int32)
    diags = [None] * B
    for b in (range(B) if sequences is None else sequences):
        r = verify_sequence(as_f64(p_logits[b]), as_f64(q_logits[b]),
                            draft[b], T, seed, step, b + seq_offset)
        acc[b] = r["accepted_len"]
        out_tokens[b, :len(r["tokens"])] = r["tokens"]
        count[b] = len(r["tokens"])
        diags[b] = r
    return dict(accepted_len=acc, out_tokens=out_tokens, out_count=count, diags=diags)
