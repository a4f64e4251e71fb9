"""Distillation losses and gradient on the GPU vs the fp64 oracle (oracle/distill.py)."""
import numpy as np
import pytest

from oracle import distill as OD

pytestmark = pytest.mark.gpu


def _rows(rows, V, seed, dt):
    import torch
    rng = np.random.default_rng(seed)
    zt = rng.normal(0, 3.0, (rows, V)).astype(np.float32)
    zs = (zt + rng.normal(0, 1.0, (rows, V))).astype(np.float32)
    tdt = torch.bfloat16 if dt == "bf16" else torch.float32
    Zt, Zs = (torch.from_numpy(a).to(tdt).cuda() for a in (zt, zs))
    return Zt, Zs, Zt.double().cpu().numpy(), Zs.double().cpu().numpy()


@pytest.mark.parametrize("rows,V,T,dt", [(64, 1000, 1.0, "bf16"), (16, 151936, 1.0, "bf16"),
                                         (32, 5003, 0.7, "f32"), (8, 2, 1.0, "f32")])
def test_parity_with_oracle(rows, V, T, dt):
    import sampling_gated_lora_b200 as U
    Zt, Zs, zt, zs = _rows(rows, V, rows + V, dt)
    alpha, beta = 0.7, 0.3
    losses, g = U.distill(Zt, Zs, alpha, beta, T)
    kl, tv = OD.distill_losses(zt, zs, T)
    got = losses.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(got[:, 0], kl, rtol=1e-3, atol=1e-6)
    np.testing.assert_allclose(got[:, 1], tv, rtol=1e-3, atol=1e-6)
    ref = OD.distill_grad(zt, zs, alpha, beta, T)
    err = np.abs(g.cpu().numpy().astype(np.float64) - ref).max()
    assert err <= 1e-4 * np.abs(ref).max() + 1e-10, err


def test_forward_only_and_equal_rows():
    import sampling_gated_lora_b200 as U
    Zt, Zs, _, _ = _rows(8, 4096, 1, "bf16")
    l1, g1 = U.distill(Zt, Zs, grad=False)
    l2, _ = U.distill(Zt, Zs)
    assert g1 is None
    np.testing.assert_array_equal(l1.cpu().numpy(), l2.cpu().numpy())
    l0, g0 = U.distill(Zt, Zt.clone())
    assert np.abs(l0.cpu().numpy()).max() < 1e-6 and np.abs(g0.cpu().numpy()).max() < 1e-9


def test_nan_row_is_flagged():
    import torch
    import sampling_gated_lora_b200 as U
    Zt, Zs, _, _ = _rows(4, 2048, 2, "bf16")
    Zt[2, 100] = float("nan")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    losses, g = U.distill(Zt, Zs, dev_status=status)
    l = losses.cpu().numpy()
    assert np.isnan(l[2]).all() and np.isfinite(l[[0, 1, 3]]).all()
    assert int(status.item()) & U.DEV_NAN


def test_empty():
    import torch
    import sampling_gated_lora_b200 as U
    Z = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    losses, g = U.distill(Z, Z)
    assert losses.shape == (0, 2) and g.shape == (0, 64)
