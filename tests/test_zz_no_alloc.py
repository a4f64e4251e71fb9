"""uno_psi_verify_noalloc (stats in the library's static device scratch, no
workspace argument) against uno_psi_verify with a caller workspace.

Both run the same kernels on the same inputs, so the integer outputs must be
identical; two calls in a row on one stream check that the shared scratch is
reused safely. Kept in the last-collected file so it runs alone and after
every other GPU test."""

import numpy as np
import pytest

import workloads as W
from oracle import sampling as S
from gpu_util import check_verify_outputs_valid, compare_verify, dev_tensor

pytestmark = pytest.mark.gpu

# (B, k, k_p, V, dtype, T, seed, step): a bf16 block with a bonus position and
# a fp32 case with ragged rows (V odd)
CASES = [(16, 8, 9, 20000, "bf16", 1.0, 21, 3),
         (6, 4, 5, 1001, "f32", 0.7, 22, 4)]


def _inputs(B, k, k_p, V, dt, T, seed, step):
    case = W.logits_case(B, k, V, k_p=k_p, ar_std=3.0, sigma=1.0, seed=seed, dtype=dt)
    d = S.draft_sample(case.q_logits, T, seed + 1, step)   # drafts ~ q, drawn on the CPU
    return dev_tensor(case.p_logits, dt), dev_tensor(case.q_logits, dt), dev_tensor(d, "i32"), d


def _host(outs):
    return tuple(o.cpu().numpy() for o in outs)


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    import torch
    import sampling_gated_lora_b200 as U
    ins = [_inputs(*c) for c in CASES]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    # the two static-scratch calls back to back on one stream, no sync between
    got = [U.psi_verify_noalloc(P, Q, D, c[5], c[6], c[7], dev_status=status)
           for (P, Q, D, _), c in zip(ins, CASES)]
    got = [_host(g) for g in got]
    want = [_host(U.psi_verify(P, Q, D, c[5], c[6], c[7]))
            for (P, Q, D, _), c in zip(ins, CASES)]
    assert int(status.item()) == 0
    for (B, k, k_p, V, *_), (_, _, _, d), g, w in zip(CASES, ins, got, want):
        check_verify_outputs_valid(*g, d, k, k_p, V)
        for a, b in zip(g, w):
            np.testing.assert_array_equal(a, b)
    # and once more on the first case: the scratch holds the second call's stats now
    (P, Q, D, _), c = ins[0], CASES[0]
    again = _host(U.psi_verify_noalloc(P, Q, D, c[5], c[6], c[7]))
    for a, b in zip(again, want[0]):
        np.testing.assert_array_equal(a, b)


def test_noalloc_more_logit_rows_than_a_grid_dimension_holds():
    """B (k_p + k) = 2048 * 33 = 67,584 logit rows, above 65,535 (the most one grid
    dimension other than x takes); V = 64 keeps the stats (8 bytes a row) inside the
    static scratch. The static-scratch call must match the workspace call exactly,
    and both the oracle on sampled sequences."""
    import sampling_gated_lora_b200 as U
    B, k, k_p, V, T, seed, step = 2048, 16, 17, 64, 1.0, 31, 2
    L = U.load()
    assert B * (k_p + k) > 65535
    assert L.uno_psi_verify_workspace(B, k, k_p, V) <= (2 << 20)
    case = W.logits_case(B, k, V, k_p=k_p, ar_std=2.0, sigma=1.0, peak_frac=0.0, seed=seed)
    d = S.draft_sample(case.q_logits, T, seed + 1, step)
    P, Q, D = dev_tensor(case.p_logits, "bf16"), dev_tensor(case.q_logits, "bf16"), dev_tensor(d, "i32")
    got = _host(U.psi_verify_noalloc(P, Q, D, T, seed, step))
    want = _host(U.psi_verify(P, Q, D, T, seed, step))
    for a, b in zip(got, want):
        np.testing.assert_array_equal(a, b)
    check_verify_outputs_valid(*got, d, k, k_p, V)
    sample = list(range(0, B, 97)) + [B - 1]
    ora = S.psi_verify(case.p_logits, case.q_logits, d, T, seed, step, sequences=sample)
    excused, bad = compare_verify(got, ora, k, sample)
    assert not bad and len(excused) <= 1


def test_noalloc_rejects_sizes_beyond_the_static_scratch():
    import sampling_gated_lora_b200 as U
    L = U.load()
    B, k, k_p, V = 8192, 16, 17, 151936          # 8192 * 33 rows > 262144
    assert L.uno_psi_verify_workspace(B, k, k_p, V) > (2 << 20)
    st = L.uno_psi_verify_noalloc(U.UNO_BF16, B, k, k_p, V, None, None, None, 1.0, 0, 0, 0,
                                  None, None, None, None, None)
    assert st == 2                               # UNO_ERR_UNSUPPORTED, nothing launched
    assert b"static scratch" in L.uno_last_error()
    # the largest size that fits is accepted by the size check (k_p = k: 2k rows per
    # sequence); the kernels' grids take any row count (one-dimensional)
    assert L.uno_psi_verify_workspace(8192, 16, 16, V) <= (2 << 20)
