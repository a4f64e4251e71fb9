"""Verification and the linear-sampler draft over a vocabulary split into G
contiguous shards (oracle; test infrastructure).

When the LM head's rows (the vocabulary) are split over G devices, each device
holds the logits of its own shard only. What the verification needs per
position is the softmax normaliser over the whole vocabulary and p(d), q(d) of
the drafted token (hyper.ai page, section "方法", the Psi-Spec paragraph:
rejection sampling against the AR distribution); the residual and bonus draws
need cumulative mass in vocabulary order. The steps, with the exchanges
between devices explicit:

  1. per shard and row: (m, s) = (max, sum of exp((z - m) / T)) over the
     shard, and the drafted token's logit when the shard holds it (else -inf);
  2. exchanged; merged in shard order into the row's (M, S) and z(d), from
     which p(d), q(d), acceptance and the first rejection n follow, the same
     on every device;
  3. per shard: the draw row's masses over the shard, Z_r = sum max(p - q, 0)
     (the residual at n) or the mass of p (the bonus; also the fallback when
     the residual mass is zero), exchanged;
  4. the shard whose cumulative range, in shard order, holds the threshold
     u Z draws the token inside its range; the others draw nothing.
The draft of the next block is the same two-round pattern on the draft rows:
per-shard (m, s), exchanged, then the shard holding u0 Z draws.

Only the order of floating-point sums differs from the unsharded oracle
(sampling.psi_verify, sampling.draft_sample); in exact arithmetic the results
are the same, which is what the tests pin. All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np

from . import philox
from .sampling import as_f64, inverse_cdf


def shard_bounds(V: int, G: int, align: int = 8):
    """G contiguous shards [v0, v1) covering [0, V), sizes rounded up to `align`
    ids (16-byte rows of bf16) except the last; shards past the end are empty."""
    per = -(-V // G)
    per = -(-per // align) * align
    return [(min(V, g * per), min(V, (g + 1) * per)) for g in range(G)]


def row_partials(z, ids, v0, T):
    """Per row of z [R, Vs] (one shard): (m, s) with s = sum exp((z - m) / T), and
    the logit of ids[row] (a global id) when v0 <= id < v0 + Vs, else -inf.
    Returns an [R, 3] array."""
    z = as_f64(z) / float(T)
    R, Vs = z.shape
    out = np.empty((R, 3))
    for i in range(R):
        m = z[i].max() if Vs else -np.inf
        out[i, 0] = m
        out[i, 1] = np.exp(z[i] - m).sum() if Vs else 0.0
        d = int(ids[i]) - v0 if ids is not None else -1
        out[i, 2] = z[i, d] if 0 <= d < Vs else -np.inf
    return out


def merge(parts):
    """Merge per-shard partials [G][R, 3] in shard order: (M, S, z_id) per row,
    M the max, S = sum_g s_g exp(m_g - M), z_id the one finite id logit."""
    parts = np.asarray(parts, dtype=np.float64)
    M = parts[:, :, 0].max(axis=0)
    S = np.zeros(parts.shape[1])
    for g in range(parts.shape[0]):
        S = S + np.where(parts[g, :, 1] > 0, parts[g, :, 1] * np.exp(parts[g, :, 0] - M), 0.0)
    return M, S, parts[:, :, 2].max(axis=0)


def _prob(z_id, M, S):
    return np.exp(z_id - M) / S if np.isfinite(z_id) else 0.0


def verify_decide(p_parts, q_parts, draft, k, k_p, seed, step, seq_offset):
    """Step 2 for all B sequences from the exchanged partials: p_parts [G][B k_p, 3]
    (rows b k_p + j), q_parts [G][B k, 3]. Returns per sequence (n, draw kind:
    "residual", "bonus" or None) and the merged stats."""
    Mp, Sp, zp = merge(p_parts)
    Mq, Sq, zq = merge(q_parts)
    B = len(draft)
    out = []
    for b in range(B):
        bg = b + seq_offset
        u1 = philox.uniforms(seed, step, philox.STREAM_ACCEPT, np.arange(bg * k, bg * k + k))
        n = k
        for j in range(k):
            pr, qr = b * k_p + j, b * k + j
            pd, qd = _prob(zp[pr], Mp[pr], Sp[pr]), _prob(zq[qr], Mq[qr], Sq[qr])
            if not (qd == 0 or u1[j] * qd < pd):
                n = j
                break
        kind = "residual" if n < k else ("bonus" if k_p == k + 1 else None)
        out.append((n, kind))
    return out, (Mp, Sp, Mq, Sq)


def draw_masses(p_shard, q_shard, decisions, stats, k, k_p, T):
    """Step 3 on one shard: per sequence (Z_r, P_r) = (sum max(p - q, 0), sum p) of its
    draw row over the shard (zeros when it draws nothing; the bonus has no q)."""
    Mp, Sp, Mq, Sq = stats
    p_shard, q_shard = as_f64(p_shard) / float(T), as_f64(q_shard) / float(T)
    masses = np.zeros((len(decisions), 2))
    for b, (n, kind) in enumerate(decisions):
        if kind is None:
            continue
        pr = b * k_p + n
        p = np.exp(p_shard[pr] - Mp[pr]) / Sp[pr]
        if kind == "residual":
            qr = b * k + n
            q = np.exp(q_shard[qr] - Mq[qr]) / Sq[qr]
            masses[b, 0] = np.maximum(p - q, 0.0).sum()
        masses[b, 1] = p.sum()
        if kind == "bonus":
            masses[b, 0] = masses[b, 1]
    return masses


def owner(masses_by_shard, u):
    """Step 4's choice: (shard, threshold inside it) for one draw. masses_by_shard [G];
    the last shard with positive mass whose prefix is <= u Z."""
    Z = float(np.sum(masses_by_shard))
    thr, pre, own, own_pre = u * Z, 0.0, -1, 0.0
    for g, w in enumerate(masses_by_shard):
        if w > 0 and pre <= thr:
            own, own_pre = g, pre
        pre += w
    return own, thr - own_pre, Z


def draw_in_shard(weights, t_local):
    """Smallest id of the shard whose inclusive cumulative weight exceeds t_local
    (the last id with positive weight if rounding leaves it beyond the total)."""
    w = np.asarray(weights, dtype=np.float64)
    c = np.cumsum(w)
    v = int(np.searchsorted(c, t_local, side="right"))
    if v >= len(w):
        v = int(np.nonzero(w > 0)[0][-1])
    return v


def vp_psi_verify(p_shards, q_shards, bounds, draft, T, seed, step, seq_offset=0):
    """The sharded verification: p_shards[g] [B, k_p, V_g], q_shards[g] [B, k, V_g]
    (shard g = ids [bounds[g][0], bounds[g][1])), draft [B, k] global ids. Returns
    accepted_len, out_tokens, out_count as sampling.psi_verify does."""
    G = len(bounds)
    B, k_p, _ = np.asarray(p_shards[0]).shape
    k = np.asarray(q_shards[0]).shape[1]
    draft = np.asarray(draft)
    p_rows = [as_f64(np.asarray(p).reshape(B * k_p, -1)) for p in p_shards]
    q_rows = [as_f64(np.asarray(q).reshape(B * k, -1)) for q in q_shards]
    ids_p = np.full(B * k_p, -1)
    for b in range(B):
        ids_p[b * k_p: b * k_p + k] = draft[b]
    ids_q = draft.reshape(-1)
    p_parts = [row_partials(p_rows[g], ids_p, bounds[g][0], T) for g in range(G)]   # round 1
    q_parts = [row_partials(q_rows[g], ids_q, bounds[g][0], T) for g in range(G)]
    decisions, stats = verify_decide(p_parts, q_parts, draft, k, k_p, seed, step, seq_offset)
    masses = np.stack([draw_masses(p_rows[g], q_rows[g], decisions, stats, k, k_p, T)
                       for g in range(G)])                                           # round 2
    Mp, Sp, Mq, Sq = stats
    acc = np.zeros(B, np.int32)
    out_tokens = np.full((B, k + 1), -1, np.int32)
    count = np.zeros(B, np.int32)
    for b, (n, kind) in enumerate(decisions):
        acc[b] = n
        out_tokens[b, :n] = draft[b, :n]
        count[b] = n
        if kind is None:
            continue
        bg = b + seq_offset
        if kind == "residual":
            u = philox.uniforms(seed, step, philox.STREAM_RESIDUAL, bg * k + n)
            col = 0 if masses[:, b, 0].sum() > 0 else 1        # zero residual: draw from p_n
        else:
            u = philox.uniforms(seed, step, philox.STREAM_BONUS, bg * k + k)
            col = 1
        g, t_local, _ = owner(masses[:, b, col], float(u))
        pr = b * k_p + n
        p = np.exp(p_rows[g][pr] / float(T) - Mp[pr]) / Sp[pr]
        if col == 0:
            qr = b * k + n
            w = np.maximum(p - np.exp(q_rows[g][qr] / float(T) - Mq[qr]) / Sq[qr], 0.0)
        else:
            w = p
        out_tokens[b, n] = bounds[g][0] + draw_in_shard(w, t_local)
        count[b] = n + 1
    return dict(accepted_len=acc, out_tokens=out_tokens, out_count=count)


def vp_draft_sample(q_shards, bounds, T, seed, step, seq_offset=0):
    """The sharded linear-sampler draft: q_shards[g] [B, k, V_g] -> d [B, k] global ids."""
    G = len(bounds)
    B, k, _ = np.asarray(q_shards[0]).shape
    rows = [as_f64(np.asarray(q).reshape(B * k, -1)) for q in q_shards]
    parts = np.stack([row_partials(rows[g], None, bounds[g][0], T) for g in range(G)])   # round 1
    M, _, _ = merge(parts)
    d = np.empty(B * k, np.int32)
    for i in range(B * k):
        b, j = divmod(i, k)
        u = float(philox.uniforms(seed, step, philox.STREAM_DRAFT, (b + seq_offset) * k + j))
        mass = np.where(parts[:, i, 1] > 0, parts[:, i, 1] * np.exp(parts[:, i, 0] - M[i]), 0.0)
        g, t_local, _ = owner(mass, u)
        w = np.exp(rows[g][i] / float(T) - M[i])
        d[i] = bounds[g][0] + draw_in_shard(w, t_local)
    return d.reshape(B, k)


def split(a, bounds):
    """Cut the last axis of `a` into the shards."""
    return [a[..., v0:v1] for v0, v1 in bounds]


__all__ = ["shard_bounds", "row_partials", "merge", "verify_decide", "draw_masses", "owner",
           "draw_in_shard", "vp_psi_verify", "vp_draft_sample", "split", "inverse_cdf"]
