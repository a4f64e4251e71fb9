"""World-size-2 gloo tests of the multi-rank host logic (CPU only).

Under weak scaling each rank runs its own B sequences with global offset
rank * B; the per-sequence draws must then equal those of one batch of
2B sequences, and the bench combines ranks as max(time), sum(tokens).
"""
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, B, out_dir):
    import datetime
    import torch
    import torch.distributed as dist
    import bench
    from oracle import sampling as S
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        n, off = bench.shard(B, rank)
        case = W.logits_case(world * B, 4, 512, ar_std=2.0, sigma=1.0, seed=5, threads=1)
        p, q = case.p_logits[off:off + n], case.q_logits[off:off + n]
        d = S.draft_sample(q, 1.0, 9, 3, seq_offset=off)
        res = S.psi_verify(p, q, d, 1.0, 9, 3, seq_offset=off)
        toks = torch.from_numpy(res["out_tokens"].astype(np.int64))
        gathered = [torch.empty_like(toks) for _ in range(world)]
        dist.all_gather(gathered, toks)
        ms, tokens = bench.combine_over_ranks(10.0 + rank, int(res["out_count"].sum()), dist)
        if rank == 0:
            np.save(os.path.join(out_dir, "tokens.npy"), torch.cat(gathered).numpy())
            np.save(os.path.join(out_dir, "combined.npy"), np.array([ms, tokens]))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_shards_reproduce_one_batch(tmp_path):
    from oracle import sampling as S
    world, B = 2, 3
    mp.start_processes(_worker, args=(world, _free_port(), B, str(tmp_path)), nprocs=world,
                       join=True, start_method="spawn")
    got = np.load(tmp_path / "tokens.npy")
    case = W.logits_case(world * B, 4, 512, ar_std=2.0, sigma=1.0, seed=5, threads=1)
    d = S.draft_sample(case.q_logits, 1.0, 9, 3)
    ref = S.psi_verify(case.p_logits, case.q_logits, d, 1.0, 9, 3)
    np.testing.assert_array_equal(got, ref["out_tokens"])
    ms, tokens = np.load(tmp_path / "combined.npy")
    assert ms == 11.0                      # max over ranks
    assert tokens == ref["out_count"].sum()  # sum over ranks
