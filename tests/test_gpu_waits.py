"""The bounded-wait give-up path, run on the GPU without a fault or a hang.

Every spin in the library's kernels has a time limit after which it reports
UNO_DEV_TIMEOUT and the kernel returns. uno_wait_selftest runs those wait
helpers on a condition nothing satisfies (a flag never raised, an mbarrier
phase with no arrival) with a 1 ms limit: each must give up promptly, set the
status bit, and leave the context usable."""
import time

import numpy as np
import pytest

import workloads as W
from oracle import sampling as S
from gpu_util import compare_verify, dev_tensor

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("which", [0, 1, 2])
def test_unsatisfied_wait_gives_up_and_reports(which):
    import torch
    import sampling_gated_lora_b200 as U
    U.device_status(clear=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    res = U.wait_selftest(which, limit_ns=1_000_000, dev_status=status)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert int(res.item()) == 0                      # gave up
    assert int(status.item()) & U.DEV_TIMEOUT
    assert U.device_status(clear=True) & U.DEV_TIMEOUT
    assert dt < 0.5, f"a 1 ms limit took {dt:.3f} s"


def test_satisfied_wait_reports_nothing_and_the_context_stays_usable():
    import torch
    import sampling_gated_lora_b200 as U
    U.wait_selftest(1, limit_ns=1_000_000)           # one give-up first
    U.device_status(clear=True)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = U.wait_selftest(3, limit_ns=1_000_000, dev_status=status)
    assert int(res.item()) == 1 and int(status.item()) == 0
    # a verification right after matches the oracle
    case = W.logits_case(8, 4, 4096, ar_std=3.0, sigma=1.0, seed=17)
    d = S.draft_sample(case.q_logits, 1.0, 5, 0)
    acc, tok, cnt = U.psi_verify(dev_tensor(case.p_logits, "bf16"), dev_tensor(case.q_logits, "bf16"),
                                 dev_tensor(d, "i32"), 1.0, 6, 0)
    ora = S.psi_verify(case.p_logits, case.q_logits, d, 1.0, 6, 0)
    excused, bad = compare_verify((acc.cpu().numpy(), tok.cpu().numpy(), cnt.cpu().numpy()), ora,
                                  4, range(8))
    assert not bad and len(excused) <= 1
    assert U.device_status(clear=True) == 0
