"""Vocabulary-sharded verification and draft on the GPU (the uno_vp_* kernels
through sampling_gated_lora_b200.vocab_parallel) vs the fp64 oracle.

G shards are emulated on one GPU by G host threads, each launching its own
shard's kernels; the exchanges (all-gather, all-reduce max) are done on the
host between the kernel rounds, so no kernel ever waits on another. Every
thread must end with the tokens of the unsharded verification and draft,
except at logged near-ties."""
import threading

import numpy as np
import pytest

import workloads as W
from oracle import sampling as S
from gpu_util import api_T, compare_drafts, compare_verify, dev_tensor

pytestmark = pytest.mark.gpu


class _Shared:
    def __init__(self, G):
        self.G = G
        self.slots = [None] * G
        self.barrier = threading.Barrier(G)


class ThreadComm:
    """all_gather / all_reduce_max among G threads of one process (one GPU)."""

    def __init__(self, rank, shared):
        self.rank, self.size, self.sh = rank, shared.G, shared

    def _exchange(self, t):
        import torch
        self.sh.slots[self.rank] = t
        self.sh.barrier.wait()
        out = torch.stack(list(self.sh.slots))
        self.sh.barrier.wait()
        return out

    def all_gather(self, t):
        return self._exchange(t.contiguous())

    def all_reduce_max(self, t):
        t.copy_(self._exchange(t).max(dim=0).values)


def _run_sharded(G, fn):
    shared, results, errors = _Shared(G), [None] * G, []

    def body(rank):
        try:
            results[rank] = fn(rank, ThreadComm(rank, shared))
        except BaseException as e:   # noqa: BLE001 - reported below
            errors.append(e)
            shared.barrier.abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(G)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(120)
    assert not errors, errors
    return results


@pytest.mark.parametrize("G,V,k,k_p,T", [(2, 20000, 6, 7, 1.0), (3, 20000, 8, 8, 0.7),
                                         (4, 151936, 8, 9, 1.0), (8, 151936, 4, 5, 1.0)])
def test_sharded_verify_and_draft_match_the_oracle(G, V, k, k_p, T):
    import torch
    from sampling_gated_lora_b200 import vocab_parallel as VPD
    T = api_T(T)
    B = 16
    case = W.logits_case(B, k, V, k_p=k_p, ar_std=3.0, sigma=1.0, seed=G * 31 + k)
    d = S.draft_sample(case.q_logits, T, 5, 1, 3)
    P, Q = dev_tensor(case.p_logits, "bf16"), dev_tensor(case.q_logits, "bf16")
    D = dev_tensor(d, "i32")
    bounds = VPD.shard_bounds(V, G)

    def fn(rank, comm):
        v0, v1 = bounds[rank]
        ps, qs = P[..., v0:v1].contiguous(), Q[..., v0:v1].contiguous()
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        acc, tok, cnt = VPD.psi_verify_sharded(ps, qs, D, V, T, 11, 2, comm, seq_offset=3,
                                               dev_status=status)
        dn = VPD.draft_sample_sharded(qs, V, T, 12, 2, comm, seq_offset=3, dev_status=status)
        torch.cuda.synchronize()
        return acc.cpu().numpy(), tok.cpu().numpy(), cnt.cpu().numpy(), dn.cpu().numpy(), int(status.item())

    res = _run_sharded(G, fn)
    ora = S.psi_verify(case.p_logits, case.q_logits, d, T, 11, 2, 3)
    for acc, tok, cnt, dn, st in res:
        assert st == 0
        excused, bad = compare_verify((acc, tok, cnt), ora, k, range(B))
        assert not bad and len(excused) <= 1, (bad, excused)
        ex_d, bad_d = compare_drafts(dn, case.q_logits, T, 12, 2, 3)
        assert not bad_d and ex_d <= 1
    for r in res[1:]:                       # every device ends with the same tokens
        for a, b in zip(r[:4], res[0][:4]):
            np.testing.assert_array_equal(a, b)
