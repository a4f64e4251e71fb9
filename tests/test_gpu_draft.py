"""Linear-sampler draft on the GPU vs the oracle, and chi-square checks of the
GPU's output distributions over 10^6 samples (the "lossless" property: the
emitted token follows p)."""
import numpy as np
import pytest
from scipy import stats

import workloads as W
from oracle import sampling as S
from gpu_util import TIE_CDF, api_T, dev_tensor

pytestmark = pytest.mark.gpu


def _gpu_draft(q, T, seed, step, seq_offset=0, dt="bf16"):
    import sampling_gated_lora_b200 as U
    Q = q if not isinstance(q, np.ndarray) else dev_tensor(q, dt)
    return U.draft_sample(Q, T, seed, step, seq_offset).cpu().numpy()


def _check_parity(q, T, seed, step, dt, seq_offset=0):
    T = api_T(T)
    g = _gpu_draft(q, T, seed, step, seq_offset, dt)
    o = S.draft_sample(q, T, seed, step, seq_offset)
    diff = np.argwhere(g != o)
    qf = S.as_f64(q)
    from oracle import philox
    for b, j in diff:
        idx = (b + seq_offset) * q.shape[1] + j
        u = philox.uniform_scalar(seed, step, 0, int(idx))
        w = S.softmax_t(qf[b, j], T)
        margin = S.cdf_margin(w, u, int(o[b, j]))
        assert margin < TIE_CDF, f"draft ({b},{j}): gpu {g[b, j]} oracle {o[b, j]} margin {margin}"
    assert len(diff) <= max(1, 1e-4 * g.size)
    return g


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_tiny_fp32(T):
    case = W.tiny_logits_case()
    _check_parity(case.q_logits, T, 0, 0, "f32")


@pytest.mark.parametrize("T", [1.0, 0.7])
@pytest.mark.parametrize("V", [50001, 151936, 2])
def test_bf16_parity(V, T):
    case = W.logits_case(8, 8, V, ar_std=3.0, sigma=1.0, seed=21)
    _check_parity(case.q_logits, T, 17, 4, "bf16", seq_offset=3)


@pytest.mark.parametrize("T", [1.0, 0.7])
def test_flat_rows_full_vocabulary(T):
    """1024 rows of N(0, 1) logits over V = 151936: near-flat rows whose tokens hold
    CDF intervals of ~1e-5 of the total, so a systematic error of the weights in the
    last digits of float precision shows up as differing draws."""
    import torch
    gen = torch.Generator().manual_seed(int(T * 100))
    q = W.from_torch_bf16(torch.randn((128, 8, 151936), generator=gen).to(torch.bfloat16))
    _check_parity(q, T, 23, 6, "bf16")


def test_masked_chunk_and_nan_rows_full_vocabulary():
    """V = 151936 bf16 rows (16-byte rows: the staged stats pass, 2048-id chunks): a row
    whose ids [10240, 12288) (one whole chunk) are -inf draws like the oracle and never
    inside the masked chunk; a row holding one NaN is flagged (draft -1, DEV_NAN) and its
    neighbours still match the oracle."""
    import torch
    import sampling_gated_lora_b200 as U
    gen = torch.Generator().manual_seed(44)
    q = W.from_torch_bf16((2.0 * torch.randn((4, 8, 151936), generator=gen)).to(torch.bfloat16))
    q[0, :, 10240:12288] = W.from_torch_bf16(torch.full((8, 2048), float("-inf")).to(torch.bfloat16))
    ok_rows = [0, 1, 3]
    g = _check_parity(q[ok_rows], 1.0, 29, 2, "bf16")
    assert not np.any((g[0] >= 10240) & (g[0] < 12288))
    q_nan = q.copy()
    q_nan[2, 5, 77777] = W.from_torch_bf16(torch.tensor([float("nan")]).to(torch.bfloat16))[0]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    d = U.draft_sample(dev_tensor(q_nan, "bf16"), 1.0, 29, 2, dev_status=status).cpu().numpy()
    assert d[2, 5] == -1 and int(status.item()) & U.DEV_NAN
    assert np.all(np.delete(d[2], 5) >= 0)
    # the other sequences draw exactly as in the same call without the NaN
    np.testing.assert_array_equal(d[ok_rows], _gpu_draft(q, 1.0, 29, 2)[ok_rows])


def _replicate(row_bits, n):
    import torch
    t = W.to_torch_bf16(row_bits, "cuda")
    return t.reshape(1, 1, -1).expand(n, 1, -1).contiguous()


def _chi2(counts, probs, n):
    """Chi-square with bins of expected count >= 5 and one pooled tail bin."""
    exp = probs * n
    big = exp >= 5
    obs = np.concatenate([counts[big], [counts[~big].sum()]])
    ex = np.concatenate([exp[big], [exp[~big].sum()]])
    if ex[-1] < 5:     # fold a tiny tail into the largest bin
        j = np.argmax(ex[:-1])
        obs[j] += obs[-1]
        ex[j] += ex[-1]
        obs, ex = obs[:-1], ex[:-1]
    ex = ex * obs.sum() / ex.sum()
    return stats.chisquare(obs, ex).pvalue


def _positions():
    """One peaked and one non-peaked position of the verify workload (sigma = 1, T = 1)."""
    p, q = W.logits_sequence(0, 16, 16, 151936, ar_std=3.0, sigma=1.0, seed=1234)
    peaked = int(np.argmax(W.bf16_to_f64(p).max(axis=1)))
    plain = int(np.argmin(W.bf16_to_f64(p).max(axis=1)))
    return p, q, [plain, peaked]


@pytest.mark.parametrize("which", [0, 1])
def test_draft_chi_square_million(which):
    """10^6 GPU draft samples of one position against softmax(q / T)."""
    p, q, pos = _positions()
    j = pos[which]
    Q = _replicate(q[j], 1024)
    V = q.shape[1]
    counts = np.zeros(V, np.int64)
    steps = 977
    for s in range(steps):
        d = _gpu_draft(Q, 1.0, 5, s)
        counts += np.bincount(d.ravel(), minlength=V)
    probs = S.softmax_t(W.bf16_to_f64(q[j]), 1.0)
    pv = _chi2(counts, probs, steps * 1024)
    assert pv >= 1e-3, pv


@pytest.mark.parametrize("which", [0, 1])
def test_verify_output_follows_p_chi_square_million(which):
    """Draft from q on the GPU, verify on the GPU: the emitted token ~ p (10^6 samples)."""
    import sampling_gated_lora_b200 as U
    p, q, pos = _positions()
    j = pos[which]
    P = _replicate(p[j], 1024)
    Q = _replicate(q[j], 1024)
    V = p.shape[1]
    counts = np.zeros(V, np.int64)
    steps = 977
    accepted = 0
    for s in range(steps):
        d = U.draft_sample(Q, 1.0, 7, s)
        acc, tok, cnt = U.psi_verify(P, Q, d, 1.0, 7, s)
        t0 = tok[:, 0].cpu().numpy()
        accepted += int(acc.sum())
        counts += np.bincount(t0, minlength=V)
    probs = S.softmax_t(W.bf16_to_f64(p[j]), 1.0)
    pv = _chi2(counts, probs, steps * 1024)
    assert pv >= 1e-3, pv
    assert 0 < accepted < steps * 1024


def test_joint_law_v8_k2():
    """V=8, k=2 on the GPU: the first two emitted tokens follow p_1 x p_2 (64 cells).

    When the step stops after one token, the second comes from the next step's
    first token, i.e. from p_2 (drawn on the host here).
    """
    import sampling_gated_lora_b200 as U
    rng = np.random.default_rng(5)
    pz = rng.standard_normal((2, 8)) * 1.5
    qz = pz + rng.standard_normal((2, 8)) * 1.0
    pb = W.bf16_round(pz)
    qb = W.bf16_round(qz)
    n = 4096
    P = W.to_torch_bf16(np.broadcast_to(pb, (n, 2, 8)).copy(), "cuda")
    Q = W.to_torch_bf16(np.broadcast_to(qb, (n, 2, 8)).copy(), "cuda")
    p = S.softmax_t(W.bf16_to_f64(pb), 1.0)
    counts = np.zeros((8, 8), np.int64)
    host = np.random.default_rng(6)
    for s in range(64):
        d = U.draft_sample(Q, 1.0, 11, s)
        acc, tok, cnt = U.psi_verify(P, Q, d, 1.0, 11, s)
        tok = tok.cpu().numpy()
        cnt = cnt.cpu().numpy()
        second = np.where(cnt >= 2, tok[:, 1], host.choice(8, size=n, p=p[1]))
        np.add.at(counts, (tok[:, 0], second), 1)
    probs = np.outer(p[0], p[1]).ravel()
    assert _chi2(counts.ravel(), probs, counts.sum()) >= 1e-3
