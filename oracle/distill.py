"""Diffusion-distillation losses over the vocabulary: forward and backward (oracle; test infrastructure).

What the pages fix (hyper.ai page, section "方法", the training objective and
the paragraph after it): the adapter is trained on one forward pass over the
concatenated clean and noisy sequences, gated so that the clean positions give
the teacher logits (theta_AR only) and the noisy positions the student logits
(theta_AR + theta_Delta); the objective is alpha * L_DCD + beta * L_TV, where
L_DCD is a block-wise Kullback-Leibler divergence between the student and
teacher distributions and L_TV a total-variation distance between them (which
raises the expected accepted length under rejection sampling).

Readings (the pages do not fix them):
  * direction: L_DCD = KL(teacher || student) = sum_v p (log p - log q), the
    usual distillation direction, with p = softmax(z_t / T) the teacher and
    q = softmax(z_s / T) the student;
  * pairing: student row i is matched with teacher row i (the same block
    position of the clean and the noisy copy);
  * L_TV = 1/2 sum_v |p - q| per row; both losses are averaged over rows;
  * gradients flow into the student logits only (the teacher is theta_AR,
    frozen while the adapter trains). Where p_v = q_v, |p - q| contributes
    the subgradient 0.
Gradients w.r.t. the student logits z_s (per row, before the 1/rows mean):
  d KL / d z_s = (q - p) / T
  d TV / d z_s[w] = q_w (s_w - sum_v s_v q_v) / (2 T),  s_v = sign(q_v - p_v).
All arithmetic is float64.
"""
from __future__ import annotations

import numpy as np

from .sampling import as_f64, softmax_t


def _log_softmax_t(z, T: float):
    x = as_f64(z) / float(T)
    x = x - x.max(axis=-1, keepdims=True)
    return x - np.log(np.exp(x).sum(axis=-1, keepdims=True))


def distill_losses(z_teacher, z_student, T: float = 1.0):
    """Per-row (KL(p || q), TV(p, q)) of teacher p and student q logits [rows, V]."""
    lp, lq = _log_softmax_t(z_teacher, T), _log_softmax_t(z_student, T)
    p, q = np.exp(lp), np.exp(lq)
    kl = np.where(p > 0, p * (lp - lq), 0.0).sum(axis=-1)
    tv = 0.5 * np.abs(p - q).sum(axis=-1)
    return kl, tv


def distill_objective(z_teacher, z_student, alpha: float, beta: float, T: float = 1.0):
    """alpha * mean KL + beta * mean TV over the rows."""
    kl, tv = distill_losses(z_teacher, z_student, T)
    return float(alpha * kl.mean() + beta * tv.mean())


def distill_grad(z_teacher, z_student, alpha: float, beta: float, T: float = 1.0):
    """Gradient of distill_objective w.r.t. the student logits, [rows, V]."""
    p = softmax_t(z_teacher, T)
    q = softmax_t(z_student, T)
    rows = p.shape[0]
    s = np.sign(q - p)
    g_kl = (q - p) / T
    g_tv = q * (s - (s * q).sum(axis=-1, keepdims=True)) / (2.0 * T)
    return (alpha * g_kl + beta * g_tv) / rows
