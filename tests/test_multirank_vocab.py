"""World-size-2 gloo test of the vocabulary-sharded verification and draft
(sampling_gated_lora_b200.vocab_parallel) on CPU ranks.

Each rank holds one vocabulary shard of the logits and runs the orchestration
with gloo collectives; the per-device steps come from the fp64 oracle in the
kernels' layouts (tests/vp_oracle_ops.py). The tokens every rank ends with
must equal the unsharded oracle's verification and draft of the whole
vocabulary."""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import workloads as W

B, K, V, WORLD = 6, 4, 1001, 2


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _case():
    c = W.logits_case(B, K, V, k_p=K + 1, ar_std=2.0, sigma=1.5, seed=17, dtype="f32", threads=1)
    return c.p_logits.astype(np.float64), c.q_logits.astype(np.float64)


def _worker(rank, world, port, out_dir):
    import datetime
    import torch
    import torch.distributed as dist
    from oracle import sampling as S
    from sampling_gated_lora_b200 import vocab_parallel as VPD
    from vp_oracle_ops import OracleOps
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        comm = VPD.TorchComm()
        v0, v1 = VPD.shard_bounds(V, world)[rank]
        p, q = _case()
        d = S.draft_sample(q, 1.0, 3, 1)
        P = torch.from_numpy(np.ascontiguousarray(p[..., v0:v1]))
        Q = torch.from_numpy(np.ascontiguousarray(q[..., v0:v1]))
        acc, tok, cnt = VPD.psi_verify_sharded(P, Q, torch.from_numpy(d), V, 1.0, 7, 2, comm,
                                               seq_offset=5, ops=OracleOps())
        dn = VPD.draft_sample_sharded(Q, V, 0.7, 9, 4, comm, seq_offset=5, ops=OracleOps())
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), acc=acc.numpy(), tok=tok.numpy(),
                 cnt=cnt.numpy(), dn=dn.numpy())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_vocabulary_shards_equal_unsharded(tmp_path):
    import sys
    from oracle import sampling as S
    here = os.path.dirname(os.path.abspath(__file__))
    if here not in sys.path:
        sys.path.insert(0, here)
    mp.start_processes(_worker, args=(WORLD, _free_port(), str(tmp_path)), nprocs=WORLD,
                       join=True, start_method="spawn")
    p, q = _case()
    d = S.draft_sample(q, 1.0, 3, 1)
    ref = S.psi_verify(p, q, d, 1.0, 7, 2, 5)
    ref_dn = S.draft_sample(q, 0.7, 9, 4, 5)
    assert np.any(ref["accepted_len"] < K)          # residual draws are exercised
    for r in range(WORLD):
        got = np.load(tmp_path / f"rank{r}.npz")
        np.testing.assert_array_equal(got["acc"], ref["accepted_len"])
        np.testing.assert_array_equal(got["tok"], ref["out_tokens"])
        np.testing.assert_array_equal(got["cnt"], ref["out_count"])
        np.testing.assert_array_equal(got["dn"], ref_dn)
