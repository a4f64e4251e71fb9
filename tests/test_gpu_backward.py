"""Gated-LoRA adapter gradients on the GPU vs the fp64 oracle
(oracle.gated_linear.gated_linear_adapter_grads), element by element.

The gradients are bf16 sums over the gated rows, so their size grows with the
number of rows; the linear's tolerance is taken relative to the output's RMS:
rel-Frobenius <= 5e-3 and |err| <= 3e-2 RMS(ref) + 2^-8 |ref| elementwise
(the second term one bf16 rounding of the output)."""
import numpy as np
import pytest

import workloads as W
from oracle.gated_linear import gated_linear_adapter_grads
from gpu_util import MAX_ABS, REL_FROB, check_close, dev_tensor, host_f64

pytestmark = pytest.mark.gpu


def _run(M, K, N, r, gate, scale, seed, dy_std=1.0):
    import sampling_gated_lora_b200 as U
    case = W.gated_linear_case(M, K, N, r, gate, b_std=0.05, scale=scale, seed=seed)
    dy = W.bf16_round(np.random.default_rng(seed + 1).standard_normal((M, N)) * dy_std)
    t = lambda a: dev_tensor(a, "bf16")
    dA, dBl = U.gated_lora_adapter_grads(t(case.x), t(dy), t(case.A), t(case.Bl),
                                         dev_tensor(case.gate, "u8"), scale)
    f = W.bf16_to_f64
    ref = gated_linear_adapter_grads(f(case.x), f(case.A), f(case.Bl), case.gate, scale, f(dy))
    return (host_f64(dA), host_f64(dBl)), ref


def _check(got, ref, what):
    for g, r_, name in zip(got, ref, ("dA", "dBl")):
        rms = float(np.sqrt(np.mean(r_ * r_))) if r_.size else 0.0
        check_close(g, r_, REL_FROB, MAX_ABS * rms, what=f"{what} {name}", rel_elem=2.0 ** -8)


@pytest.mark.parametrize("which", ["up", "down"])
def test_mlp_concatenated_batch(which):
    """The training layout: M = 2048 (clean half gate 0, noisy half gate 1), rank 128."""
    K, N = (4096, 12288) if which == "up" else (12288, 4096)
    gate = np.concatenate([np.zeros(1024, np.uint8), np.ones(1024, np.uint8)])
    got, ref = _run(2048, K, N, 128, gate, 1.0, seed=3)
    _check(got, ref, f"mlp {which}")


@pytest.mark.parametrize("M,K,N,r,scale", [
    (1, 64, 128, 8, 1.0),
    (37, 72, 200, 16, 0.75),        # ragged M (padding columns), K and N off the tile grid
    (300, 520, 264, 24, 0.5),
    (1000, 1024, 1000, 128, 1.0),
])
def test_ragged_shapes(M, K, N, r, scale):
    gate = (np.random.default_rng(M).random(M) < 0.5).astype(np.uint8)
    got, ref = _run(M, K, N, r, gate, scale, seed=M + K)
    _check(got, ref, f"{M}x{K}x{N} r={r}")


def test_gate_zero_gives_zero_gradients_and_empty_batch():
    import torch
    import sampling_gated_lora_b200 as U
    got, ref = _run(96, 256, 384, 16, np.zeros(96, np.uint8), 1.0, seed=5)
    assert not np.any(got[0]) and not np.any(got[1])
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    dA, dBl = U.gated_lora_adapter_grads(x, torch.empty((0, 128), dtype=torch.bfloat16, device="cuda"),
                                         torch.ones((8, 64), dtype=torch.bfloat16, device="cuda"),
                                         torch.ones((128, 8), dtype=torch.bfloat16, device="cuda"),
                                         torch.empty((0,), dtype=torch.uint8, device="cuda"))
    assert not dA.any() and not dBl.any()
