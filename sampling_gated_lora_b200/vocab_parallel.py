"""Verification and the linear-sampler draft with the vocabulary split over devices.

When the LM head's rows are split over G devices (one process per GPU), each
device holds the logits of one contiguous vocabulary shard. Verifying a block
against the AR distribution needs the normaliser over the whole vocabulary and
cumulative mass in vocabulary order (hyper.ai page, section "方法", the
Psi-Spec paragraph), so the step exchanges a few numbers per row between the
devices: two all-gathers and one all-reduce (max) for verification, one
all-gather and one all-reduce for the next block's draft. Every numeric step
runs in the library's kernels (the uno_vp_* entry points of include/uno.h);
this module only marshals arguments and issues the collectives between them.

`comm` is any object with rank, size, all_gather(t) -> [size, *t.shape] and
all_reduce_max(t) (in place); TorchComm wraps a torch.distributed group (NCCL
over NVLink on B200s). `ops` defaults to the library's kernels.
"""
from __future__ import annotations

from . import UNO_BF16, UNO_F32, _dev, _expect, _launch, _ptr, _torch, load


def shard_bounds(V: int, G: int, align: int = 8):
    """G contiguous shards [v0, v1) covering [0, V) in rank order, each a multiple of
    `align` ids (16-byte rows of bf16) except the one holding the end."""
    per = -(-V // G)
    per = -(-per // align) * align
    return [(min(V, g * per), min(V, (g + 1) * per)) for g in range(G)]


class TorchComm:
    """The exchanges over a torch.distributed process group."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.rank = dist.get_rank(group)
        self.size = dist.get_world_size(group)

    def all_gather(self, t):
        torch = _torch()
        t = t.contiguous()
        out = torch.empty((self.size * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                          device=t.device)
        self.dist.all_gather_into_tensor(out, t, group=self.group)   # rank order along dim 0
        return out.view((self.size,) + tuple(t.shape))

    def all_reduce_max(self, t):
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX, group=self.group)


def _dt(t):
    torch = _torch()
    return UNO_BF16 if t.dtype == torch.bfloat16 else UNO_F32


class NativeOps:
    """The per-device steps, run by the library's kernels on the tensors' device."""

    def partials(self, logits, draft, k, k_p, id_kind, v0, temperature, precise=False):
        torch = _torch()
        rows, Vs = logits.shape
        out = torch.empty((rows, 4), dtype=torch.float32, device=logits.device)
        dev = _dev(logits, draft, out)
        _launch(dev, None, load().uno_vp_partials, _dt(logits), rows, Vs, v0, _ptr(logits),
                _ptr(draft), k, k_p, id_kind, 1 if precise else 0, float(temperature), _ptr(out))
        return out

    def decide(self, parts_p, parts_q, draft, k, k_p, V, temperature, seed, step, seq_offset,
               dev_status=None):
        torch = _torch()
        G, B = parts_p.shape[0], draft.shape[0]
        i32 = dict(dtype=torch.int32, device=draft.device)
        acc, tok = torch.empty(B, **i32), torch.empty((B, k + 1), **i32)
        cnt, draw = torch.empty(B, **i32), torch.empty(B, **i32)
        stats = torch.empty((B, 4), dtype=torch.float32, device=draft.device)
        dev = _dev(parts_p, parts_q, draft, acc, tok, cnt, draw, stats, dev_status)
        _launch(dev, None, load().uno_vp_verify_decide, B, k, k_p, V, G, _ptr(parts_p),
                _ptr(parts_q), _ptr(draft), float(temperature), int(seed), int(step),
                int(seq_offset), _ptr(acc), _ptr(tok), _ptr(cnt), _ptr(draw), _ptr(stats),
                _ptr(dev_status))
        return acc, tok, cnt, draw, stats

    def masses(self, p_shard, q_shard, draw, stats, k, k_p, temperature):
        torch = _torch()
        B, _, Vs = p_shard.shape
        out = torch.empty((B, 2), dtype=torch.float64, device=p_shard.device)
        dev = _dev(p_shard, q_shard, draw, stats, out)
        _launch(dev, None, load().uno_vp_draw_masses, _dt(p_shard), B, k, k_p, Vs, _ptr(p_shard),
                _ptr(q_shard), _ptr(draw), _ptr(stats), float(temperature), _ptr(out))
        return out

    def draw(self, p_shard, q_shard, draw, stats, masses_all, tok, k, k_p, v0, V, rank,
             temperature, seed, step, seq_offset):
        B, _, Vs = p_shard.shape
        G = masses_all.shape[0]
        dev = _dev(p_shard, q_shard, draw, stats, masses_all, tok)
        _launch(dev, None, load().uno_vp_draw, _dt(p_shard), B, k, k_p, Vs, v0, V, G, rank,
                _ptr(p_shard), _ptr(q_shard), _ptr(draw), _ptr(stats), _ptr(masses_all),
                float(temperature), int(seed), int(step), int(seq_offset), _ptr(tok))

    def draft_draw(self, q_shard, parts_all, k, v0, V, rank, temperature, seed, step, seq_offset,
                   dev_status=None):
        torch = _torch()
        B, _, Vs = q_shard.shape
        G = parts_all.shape[0]
        d = torch.empty((B, k), dtype=torch.int32, device=q_shard.device)
        dev = _dev(q_shard, parts_all, d, dev_status)
        _launch(dev, None, load().uno_vp_draft_draw, _dt(q_shard), B, k, Vs, v0, V, G, rank,
                _ptr(q_shard), _ptr(parts_all), float(temperature), int(seed), int(step),
                int(seq_offset), _ptr(d), _ptr(dev_status))
        return d


def psi_verify_sharded(p_shard, q_shard, draft, V, temperature, seed, step, comm, seq_offset=0,
                       dev_status=None, ops=None):
    """uno_psi_verify with the vocabulary split over comm.size devices.

    p_shard [B, k_p, Vs], q_shard [B, k, Vs]: this device's shard (comm.rank of
    shard_bounds(V, comm.size)) of the AR and draft logits; draft [B, k] global
    ids. Returns (accepted_len, out_tokens, out_count), the same on every device.
    """
    torch = _torch()
    ops = NativeOps() if ops is None else ops
    B, k_p, Vs = p_shard.shape
    k = q_shard.shape[1]
    v0, v1 = shard_bounds(V, comm.size)[comm.rank]
    if v1 - v0 != Vs:
        raise ValueError(f"shard {comm.rank} holds ids [{v0}, {v1}), got {Vs} columns")
    _expect(q_shard, (B, k, Vs), (p_shard.dtype,), "q_shard")
    _expect(draft, (B, k), (torch.int32,), "draft")
    parts_p = ops.partials(p_shard.reshape(B * k_p, Vs), draft, k, k_p, 1, v0, temperature)
    parts_q = ops.partials(q_shard.reshape(B * k, Vs), draft, k, k_p, 2, v0, temperature)
    all_p, all_q = comm.all_gather(parts_p), comm.all_gather(parts_q)          # exchange 1
    acc, tok, cnt, draw, stats = ops.decide(all_p, all_q, draft, k, k_p, V, temperature, seed,
                                            step, seq_offset, dev_status)
    masses = ops.masses(p_shard, q_shard, draw, stats, k, k_p, temperature)
    all_m = comm.all_gather(masses)                                            # exchange 2
    ops.draw(p_shard, q_shard, draw, stats, all_m, tok, k, k_p, v0, V, comm.rank, temperature,
             seed, step, seq_offset)
    comm.all_reduce_max(tok)                                                   # the owner's token
    return acc, tok, cnt


def draft_sample_sharded(q_shard, V, temperature, seed, step, comm, seq_offset=0, dev_status=None,
                         ops=None):
    """uno_draft_sample with the vocabulary split over comm.size devices: q_shard
    [B, k, Vs] this device's shard of the draft logits. Returns d [B, k] global ids."""
    ops = NativeOps() if ops is None else ops
    B, k, Vs = q_shard.shape
    v0, v1 = shard_bounds(V, comm.size)[comm.rank]
    if v1 - v0 != Vs:
        raise ValueError(f"shard {comm.rank} holds ids [{v0}, {v1}), got {Vs} columns")
    parts = ops.partials(q_shard.reshape(B * k, Vs), None, k, k, 0, v0, temperature, precise=True)
    all_parts = comm.all_gather(parts)                                         # exchange
    d = ops.draft_draw(q_shard, all_parts, k, v0, V, comm.rank, temperature, seed, step,
                       seq_offset, dev_status)
    comm.all_reduce_max(d)
    return d


__all__ = ["shard_bounds", "TorchComm", "NativeOps", "psi_verify_sharded", "draft_sample_sharded"]
