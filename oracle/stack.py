"""Synthetic decode step: gated-LoRA decoder stack + LM head + verify + draft (oracle; test infrastructure).

The pages give the model-side rule only: every AR matrix carries a LoRA
adapter, and one forward computes the verify path (adapter off) and the draft
path (adapter on) through a per-row gate (hyper.ai page, section "方法"; the
rank-128 adapters and the Qwen3-8B base in section "实验"). Attention and the
KV cache are not on the linear path, so the stand-in stack keeps only the
gated projections and the glue between them (a reading; the pages give no
layer equations):

    per layer:  n = rmsnorm(h);  q = L_q(n);  k = L_k(n);  v = L_v(n)  (k, v unused)
                h = h + L_o(q)
                n = rmsnorm(h);  h = h + L_down(silu(L_gate(n)) * L_up(n))
    then:       logits = L_head(rmsnorm(h))

with L(x) = x W^T + s g ((x A^T) Bl^T) and rmsnorm(x) = x / sqrt(mean(x^2) + 1e-6)
(no weight). Rows of one step: B(k+1) verify rows (gate 0, giving the k+1 AR
distributions p of the drafted block plus the bonus position, by the
factorisation's shift), then Bk mask rows (gate 1, giving the draft
distributions q for the next block).

Storage: the step stores every tensor passed between operations in bf16 (the
workload is a bf16 model). With `store="bf16"` the oracle rounds at those same
points and computes each operation in fp64; `store=None` keeps fp64 throughout.
Rounding to bf16 goes through torch's CPU conversion (round to nearest even).
"""
from __future__ import annotations

import numpy as np

from .gated_linear import gated_linear
from .sampling import as_f64, draft_sample, psi_verify

RMS_EPS = 1e-6


def round_bf16(x):
    """Round float64 values to the nearest bf16 (ties to even), returned as float64."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).to(torch.float64).numpy()


def rmsnorm(h, eps=RMS_EPS):
    h = np.asarray(h, dtype=np.float64)
    return h / np.sqrt(np.mean(h * h, axis=-1, keepdims=True) + eps)


def silu(x):
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


_widen = as_f64


def _lin(x, wab, gate, scale):
    W, A, Bl = (_widen(t) for t in wab)
    return gated_linear(x, W, A, Bl, gate, scale)


def layer_forward(h, lw, gate, scale, store="bf16"):
    """One stand-in decoder layer; lw maps name -> (W, A, Bl)."""
    rd = round_bf16 if store == "bf16" else (lambda a: a)
    n = rd(rmsnorm(h))
    q = rd(_lin(n, lw["q"], gate, scale))
    rd(_lin(n, lw["k"], gate, scale))          # computed by the step, not consumed
    rd(_lin(n, lw["v"], gate, scale))
    h = rd(h + rd(_lin(q, lw["o"], gate, scale)))
    n = rd(rmsnorm(h))
    g = rd(_lin(n, lw["gate"], gate, scale))
    u = rd(_lin(n, lw["up"], gate, scale))
    a = rd(silu(g) * u)
    h = rd(h + rd(_lin(a, lw["down"], gate, scale)))
    return h


def stack_logits(h_in, layers, head, gate, scale, store="bf16", n_layers=None):
    """Logits [M,V] of the stand-in stack (rounded to bf16 when store="bf16")."""
    rd = round_bf16 if store == "bf16" else (lambda a: a)
    h = _widen(h_in)
    for lw in layers[: (len(layers) if n_layers is None else n_layers)]:
        h = layer_forward(h, lw, gate, scale, store)
    return rd(_lin(rd(rmsnorm(h)), head, gate, scale))


def step_gate(B: int, k: int):
    return np.concatenate([np.zeros(B * (k + 1), np.uint8), np.ones(B * k, np.uint8)])


def psi_step(h_in, layers, head, B, k, q_prev_logits, d_prev, T, seed, step, scale,
             store="bf16"):
    """One linear-sampler decode step.

    Verifies the previous block (q_prev_logits [B,k,V], d_prev [B,k]) against
    this step's AR rows p [B,k+1,V] (bonus enabled), then drafts the next
    block from this step's mask rows. Returns (verify result, d_next, q_next
    logits, all logits).
    """
    gate = step_gate(B, k)
    logits = stack_logits(h_in, layers, head, gate, scale, store)
    V = logits.shape[1]
    p = logits[: B * (k + 1)].reshape(B, k + 1, V)
    q_next = logits[B * (k + 1):].reshape(B, k, V)
    ver = psi_verify(p, as_f64(q_prev_logits), d_prev, T, seed, step)
    d_next = draft_sample(q_next, T, seed, step)
    return ver, d_next, q_next, logits
