"""The step's glue kernels (RMSNorm, silu * up) vs the fp64 oracle, bf16 storage."""
import numpy as np
import pytest

import workloads as W
from oracle import stack as O
from gpu_util import dev_tensor, host_f64

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("M,D", [(1, 4096), (17, 4096), (300, 256), (5, 1000), (3, 13)])
def test_rmsnorm(M, D):
    import sampling_gated_lora_b200 as U
    x = W.bf16_round(np.random.default_rng(D).standard_normal((M, D)) * 3)
    y = host_f64(U.rmsnorm(dev_tensor(x, "bf16")))
    ref = O.rmsnorm(W.bf16_to_f64(x))
    # one bf16 rounding of a value computed in fp32: within 2^-8 relative
    np.testing.assert_allclose(y, ref, rtol=2.0 ** -8, atol=1e-30)


@pytest.mark.parametrize("n", [8, 12288 * 17, 1001])
def test_silu_mul(n):
    import sampling_gated_lora_b200 as U
    rng = np.random.default_rng(n)
    a = W.bf16_round(rng.standard_normal(n) * 4)
    b = W.bf16_round(rng.standard_normal(n))
    y = host_f64(U.silu_mul(dev_tensor(a, "bf16"), dev_tensor(b, "bf16")))
    ref = O.silu(W.bf16_to_f64(a)) * W.bf16_to_f64(b)
    np.testing.assert_allclose(y, ref, rtol=2.0 ** -8, atol=1e-30)
