"""The per-device steps of the vocabulary-sharded verification computed by the
fp64 oracle (oracle/vocab_parallel.py), on CPU tensors, in the layouts the
library's uno_vp_* kernels use: partials (m, s, z(d), 0) with m and z(d) in
logit units and s = sum exp((z - m) / T); draw positions (n < k residual,
k bonus, -1 none); masses (residual or bonus mass, p mass). Lets the
multi-process orchestration (sampling_gated_lora_b200.vocab_parallel) run on
CPU ranks with gloo collectives."""
import numpy as np
import torch

from oracle import philox
from oracle import vocab_parallel as VP


def _np(t):
    return t.detach().cpu().double().numpy()


class OracleOps:
    def partials(self, logits, draft, k, k_p, id_kind, v0, temperature, precise=False):
        z = _np(logits)
        rows = z.shape[0]
        ids = None
        if id_kind == 1:
            d = draft.numpy()
            ids = np.array([d[r // k_p, r % k_p] if r % k_p < k else -1 for r in range(rows)])
        elif id_kind == 2:
            ids = draft.numpy().reshape(-1)
        parts = VP.row_partials(z, ids, v0, temperature)          # in z / T units
        out = np.zeros((rows, 4))
        out[:, 0] = parts[:, 0] * temperature
        out[:, 1] = parts[:, 1]
        out[:, 2] = parts[:, 2] * temperature
        return torch.from_numpy(out)

    def decide(self, parts_p, parts_q, draft, k, k_p, V, temperature, seed, step, seq_offset,
               dev_status=None):
        T = temperature
        to_oracle = lambda a: [np.column_stack([g[:, 0] / T, g[:, 1], g[:, 2] / T]) for g in _np(a)]
        d = draft.numpy()
        decisions, (Mp, Sp, Mq, Sq) = VP.verify_decide(to_oracle(parts_p), to_oracle(parts_q), d, k,
                                                       k_p, seed, step, seq_offset)
        B = len(d)
        acc = np.zeros(B, np.int32)
        tok = np.full((B, k + 1), -1, np.int32)
        cnt = np.zeros(B, np.int32)
        draw = np.full(B, -1, np.int32)
        stats = np.zeros((B, 4))
        for b, (n, kind) in enumerate(decisions):
            acc[b] = n
            tok[b, :n] = d[b, :n]
            pos = -1 if kind is None else (n if kind == "residual" else k)
            draw[b] = pos
            cnt[b] = n + (pos >= 0)
            if pos >= 0:
                pr = b * k_p + pos
                stats[b, :2] = Mp[pr] * T, Sp[pr]
                if pos < k:
                    stats[b, 2:] = Mq[b * k + n] * T, Sq[b * k + n]
        t = torch.from_numpy
        return t(acc), t(tok), t(cnt), t(draw), t(stats)

    @staticmethod
    def _weights(p_row, q_row, st, residual, T):
        p = np.exp((p_row - st[0]) / T) / st[1]
        if not residual:
            return p, p
        q = np.exp((q_row - st[2]) / T) / st[3]
        return np.maximum(p - q, 0.0), p

    def masses(self, p_shard, q_shard, draw, stats, k, k_p, temperature):
        p, q, st = _np(p_shard), _np(q_shard), _np(stats)
        out = np.zeros((p.shape[0], 2))
        for b, pos in enumerate(draw.numpy()):
            if pos < 0:
                continue
            residual = pos < k
            w, pm = self._weights(p[b, pos], q[b, pos if residual else 0], st[b], residual,
                                  temperature)
            out[b] = w.sum(), pm.sum()
        return torch.from_numpy(out)

    def draw(self, p_shard, q_shard, draw, stats, masses_all, tok, k, k_p, v0, V, rank,
             temperature, seed, step, seq_offset):
        p, q, st, m = _np(p_shard), _np(q_shard), _np(stats), _np(masses_all)
        for b, pos in enumerate(draw.numpy()):
            if pos < 0:
                continue
            residual = pos < k
            use_res = residual and m[:, b, 0].sum() > 0
            stream = philox.STREAM_RESIDUAL if residual else philox.STREAM_BONUS
            u = float(philox.uniforms(seed, step, stream, (b + seq_offset) * k + pos))
            own, t_local, _ = VP.owner(m[:, b, 0] if use_res else m[:, b, 1], u)
            if own != rank:
                continue
            w, pm = self._weights(p[b, pos], q[b, pos if residual else 0], st[b], residual,
                                  temperature)
            tok[b, pos] = v0 + VP.draw_in_shard(w if use_res else pm, t_local)

    def draft_draw(self, q_shard, parts_all, k, v0, V, rank, temperature, seed, step, seq_offset,
                   dev_status=None):
        q, parts = _np(q_shard), _np(parts_all)
        B = q.shape[0]
        d = np.full((B, k), -1, np.int32)
        for i in range(B * k):
            b, j = divmod(i, k)
            M = parts[:, i, 0].max()
            mass = parts[:, i, 1] * np.exp((parts[:, i, 0] - M) / temperature)
            u = float(philox.uniforms(seed, step, philox.STREAM_DRAFT, (b + seq_offset) * k + j))
            own, t_local, _ = VP.owner(mass, u)
            if own == rank:
                d[b, j] = v0 + VP.draw_in_shard(np.exp((q[b, j] - M) / temperature), t_local)
        return torch.from_numpy(d)
