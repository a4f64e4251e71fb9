"""Gated-LoRA linear (oracle; test infrastructure).

Uno attaches a LoRA adapter theta_Delta to every AR weight matrix; the draft
path uses theta_AR + theta_Delta and the verify path theta_AR alone
(hyper.ai page, section "方法", the paragraph introducing theta_Delta). One
forward serves both paths through a per-row gate that switches the adapter
off on clean rows and on for noisy rows (same section, the gated-LoRA
paragraph; ainews page: "conditional LoRA").

    y = x W^T + s * g (.) ((x A^T) Bl^T)

W [N,K], A [r,K], Bl [N,r] (nn.Linear / PEFT layout), g in {0,1} per row,
scale s. Computed in fp64 from the exactly-widened inputs.
"""
from __future__ import annotations

import numpy as np


def gated_linear(x, W, A, Bl, gate, scale):
    """Return y [M,N] in float64."""
    x = np.asarray(x, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bl = np.asarray(Bl, dtype=np.float64)
    g = np.asarray(gate, dtype=np.float64).reshape(-1, 1)
    base = x @ W.T
    lora = (x @ A.T) @ Bl.T
    return base + float(scale) * g * lora


def gated_linear_adapter_grads(x, A, Bl, gate, scale, dy):
    """Gradients of sum(dy * y) w.r.t. the adapter (A, Bl), theta_AR frozen.

    The adapter is what the distillation stage trains while the AR weights stay
    fixed (hyper.ai page, section "方法", the training-order paragraph: the AR
    weights are frozen while the diffusion adapter is trained). With
    t = s g (.) (x A^T):
        dBl = dy^T t                      [N, r]
        dA  = (s g (.) (dy Bl))^T x       [r, K]
    Rows with gate 0 contribute nothing. Returns (dA, dBl) in float64.
    """
    x = np.asarray(x, dtype=np.float64)
    A = np.asarray(A, dtype=np.float64)
    Bl = np.asarray(Bl, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    sg = float(scale) * np.asarray(gate, dtype=np.float64).reshape(-1, 1)
    t = sg * (x @ A.T)
    dBl = dy.T @ t
    dA = (sg * (dy @ Bl)).T @ x
    return dA, dBl
