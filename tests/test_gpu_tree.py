"""Tree-sampler verification on the GPU vs the fp64 oracle (oracle/tree.py)."""
import numpy as np
import pytest

from oracle import tree as OT

pytestmark = pytest.mark.gpu


def _bf16(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16).cuda()


def _case(B, N, k, V, sigma, seed, T=1.0, zero_adapter=False):
    """Draft logits q [B,k,V]; candidates drawn by the oracle's sampler; AR logits of
    every trie node = q of the node's depth + noise (R = N*k + 1 rows, unused rows random)."""
    rng = np.random.default_rng(seed)
    q = rng.normal(0, 3.0, (B, k, V)).astype(np.float32)
    Q = _bf16(q)
    q_b = Q.float().cpu().numpy()
    cands = OT.tree_candidates(q_b, N, T, seed=seed + 1, step=2)
    R = N * k + 1
    p = rng.normal(0, 3.0, (B, R, V)).astype(np.float32)
    for b in range(B):
        _, parent, _, depth = OT.trie(cands[b])
        for n in range(len(parent)):
            d = min(int(depth[n]), k - 1)
            p[b, n] = q_b[b, d] + (0 if zero_adapter else rng.normal(0, sigma, V))
    P = _bf16(p)
    return P, Q, cands, P.float().cpu().numpy(), q_b


def _gpu(P, Q, cands, T, seed, step, bonus, seq_offset=0, status=None):
    import torch
    import sampling_gated_lora_b200 as U
    C = torch.from_numpy(np.ascontiguousarray(cands, np.int32)).cuda()
    acc, tok, cnt = U.tree_verify(P, Q, C, T, seed, step, seq_offset, bonus=bonus,
                                  dev_status=status)
    return acc.cpu().numpy(), tok.cpu().numpy(), cnt.cpu().numpy()


@pytest.mark.parametrize("bonus", [False, True])
def test_one_candidate_equals_linear_verification(bonus):
    import sampling_gated_lora_b200 as U
    B, k, V = 16, 8, 20000
    P, Q, cands, _, _ = _case(B, 1, k, V, sigma=1.0, seed=3)
    g = _gpu(P, Q, cands, 1.0, 9, 4, bonus)
    rows = P[:, :k + 1] if bonus else P[:, :k]
    import torch
    d = torch.from_numpy(np.ascontiguousarray(cands[:, 0, :], np.int32)).cuda()
    lin = U.psi_verify(rows.contiguous(), Q, d, 1.0, 9, 4)
    for x, y in zip(g, lin):
        np.testing.assert_array_equal(x, y.cpu().numpy())


@pytest.mark.parametrize("N,k,V,T,bonus", [(2, 4, 1000, 1.0, False), (4, 8, 1000, 0.7, True),
                                           (8, 4, 32000, 1.0, True), (3, 1, 5003, 1.0, False),
                                           (32, 2, 512, 1.0, True)])
def test_parity_with_oracle(N, k, V, T, bonus):
    T = float(np.float32(T))      # the C ABI's float32 temperature, given to the oracle too
    B = 12
    P, Q, cands, p_b, q_b = _case(B, N, k, V, sigma=1.5, seed=N * 7 + k, T=T)
    acc, tok, cnt = _gpu(P, Q, cands, T, 21, 5, bonus, seq_offset=2)
    excused = 0
    for b in range(B):
        n_nodes = len(OT.trie(cands[b])[1])          # the kernel reads rows [0, n_nodes) of R
        o = OT.tree_verify_sequence(p_b[b][:n_nodes], q_b[b], cands[b], T, 21, 5, b + 2,
                                    bonus=bonus)
        ref = np.full(k + 1, -1)
        ref[:len(o["tokens"])] = o["tokens"]
        same = acc[b] == o["accepted_len"] and (tok[b] == ref).all() and cnt[b] == len(o["tokens"])
        if not same:
            assert o["test_margin"] < 1e-4 or o["draw_margin"] < 1e-5, (b, o, acc[b], tok[b])
            excused += 1
    assert excused <= 1


def test_zero_adapter_accepts_every_block():
    B, N, k, V = 8, 4, 8, 4096
    P, Q, cands, _, _ = _case(B, N, k, V, sigma=0.0, seed=5, zero_adapter=True)
    acc, tok, cnt = _gpu(P, Q, cands, 1.0, 3, 1, bonus=False)
    assert (acc == k).all() and (cnt == k).all()


def test_bad_candidates_and_missing_rows_are_flagged():
    import torch
    import sampling_gated_lora_b200 as U
    B, N, k, V = 3, 4, 4, 1000
    P, Q, cands, _, _ = _case(B, N, k, V, sigma=1.0, seed=8)
    bad = cands.copy()
    bad[1, 2, 3] = V                       # out of range in sequence 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    acc, tok, cnt = _gpu(P, Q, bad, 1.0, 1, 1, False, status=status)
    assert acc[1] == -1 and cnt[1] == -1 and (tok[1] == -1).all()
    assert acc[0] >= 0 and acc[2] >= 0
    assert int(status.item()) & U.DEV_BAD_DRAFT
    # fewer node rows than the trie has nodes (distinct candidates: N*k + 1 nodes)
    distinct = np.arange(N * k, dtype=np.int32).reshape(1, N, k).repeat(B, 0)
    status.zero_()
    acc, tok, cnt = _gpu(P[:, :N * k].contiguous(), Q, distinct, 1.0, 1, 1, False, status=status)
    assert (acc == -1).all() and int(status.item()) & U.DEV_BAD_DRAFT


def test_empty_batch():
    import torch
    import sampling_gated_lora_b200 as U
    P = torch.zeros((0, 5, 64), dtype=torch.bfloat16, device="cuda")
    Q = torch.zeros((0, 2, 64), dtype=torch.bfloat16, device="cuda")
    C = torch.zeros((0, 2, 2), dtype=torch.int32, device="cuda")
    acc, tok, cnt = U.tree_verify(P, Q, C, 1.0, 0, 0)
    assert acc.shape == (0,) and tok.shape == (0, 3)


def test_first_token_follows_p_chi_square():
    """Lossless on the GPU: with k = 1 and N = 3 candidates drawn from q, the emitted
    token follows p of the root (10^6 samples: 1024 sequences x 977 steps)."""
    import torch
    from scipy import stats
    import sampling_gated_lora_b200 as U
    from oracle import sampling as S
    B, N, V = 1024, 3, 64
    rng = np.random.default_rng(12)
    p_row = rng.normal(0, 1.5, V).astype(np.float32)
    q_row = (p_row + rng.normal(0, 1.5, V)).astype(np.float32)
    P = _bf16(np.broadcast_to(p_row, (B, N + 1, V)))       # root row = p; leaf rows unused
    Q = _bf16(np.broadcast_to(q_row, (B, 1, V)))
    Qrep = Q.repeat_interleave(N, dim=0).contiguous()
    counts = np.zeros(V, np.int64)
    steps = 977
    for s in range(steps):
        C = U.draft_sample(Qrep, 1.0, 5, s).reshape(B, N, 1).contiguous()
        acc, tok, cnt = U.tree_verify(P, Q, C, 1.0, 6, s)
        counts += np.bincount(tok[:, 0].cpu().numpy(), minlength=V)
    probs = S.softmax_t(P[0, 0].float().cpu().numpy().astype(np.float64), 1.0)
    exp = probs * steps * B
    big = exp >= 5
    obs = np.append(counts[big], counts[~big].sum())
    ex = np.append(exp[big], exp[~big].sum())
    if ex[-1] < 5:
        obs, ex = obs[:-1], ex[:-1]
    ex = ex * obs.sum() / ex.sum()
    assert stats.chisquare(obs, ex).pvalue >= 1e-3
