"""Pins for the oracle's synthetic decode stack (CPU only)."""
import math

import pytest

import numpy as np
from scipy import special

from oracle import stack as O
from oracle.sampling import draft_sample, psi_verify
import workloads as W


def test_rmsnorm_closed_form():
    h = np.random.default_rng(0).standard_normal((5, 64)) * 3
    n = O.rmsnorm(h)
    ms = np.mean(h * h, axis=1)
    np.testing.assert_allclose(np.mean(n * n, axis=1), ms / (ms + 1e-6), rtol=1e-12)
    np.testing.assert_allclose(O.rmsnorm(7.0 * h), n, rtol=1e-6)


def test_silu_matches_library():
    x = np.linspace(-30, 30, 1001)
    np.testing.assert_allclose(O.silu(x), x * special.expit(x), rtol=1e-13, atol=1e-300)


def test_bf16_rounding_two_implementations_agree():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-8, 8, 20000),
                        1.0 + np.arange(0, 2**-7, 2**-9),     # exact ties between bf16 values
                        -(3.0 + np.arange(0, 2**-5, 2**-8))])
    a = O.round_bf16(x)
    b = W.bf16_to_f64(W.bf16_round(x))
    np.testing.assert_array_equal(a, b)
    # ties to even: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 -> 1
    assert O.round_bf16(np.array([1.0 + 2**-8]))[0] == 1.0
    assert O.round_bf16(np.array([1.0 + 3 * 2**-8]))[0] == 1.0 + 2**-6


def _tiny_weights(shape, rng):
    lw = {}
    for name, K, N in shape.linears():
        lw[name] = (rng.standard_normal((N, K)) / math.sqrt(K), rng.standard_normal((shape.r, K)) / math.sqrt(K),
                    rng.standard_normal((N, shape.r)) * 0.3)
    return lw


def _py_lin(x, wab, g, s):
    Wt, A, Bl = wab
    t = [math.fsum(x[kk] * A[j][kk] for kk in range(len(x))) for j in range(len(A))]
    return [math.fsum(x[kk] * Wt[n][kk] for kk in range(len(x)))
            + s * g * math.fsum(t[j] * Bl[n][j] for j in range(len(t))) for n in range(len(Wt))]


def _py_rms(x):
    ms = math.fsum(v * v for v in x) / len(x)
    return [v / math.sqrt(ms + 1e-6) for v in x]


def test_layer_brute_force():
    """Row-by-row pure-Python evaluation of one layer vs the vectorised oracle."""
    shape = W.ModelShape(n_layers=1, hidden=6, q_out=6, kv_out=2, inter=10, vocab=9, r=2)
    rng = np.random.default_rng(2)
    lw = _tiny_weights(shape, rng)
    h = rng.standard_normal((3, 6))
    g = np.array([0, 1, 1], np.uint8)
    s = 0.8
    got = O.layer_forward(h, lw, g, s, store=None)
    py = {k: tuple(np.asarray(a).tolist() for a in v) for k, v in lw.items()}
    for m in range(3):
        x = h[m].tolist()
        n = _py_rms(x)
        q = _py_lin(n, py["q"], g[m], s)
        o = _py_lin(q, py["o"], g[m], s)
        x = [a + b for a, b in zip(x, o)]
        n = _py_rms(x)
        ga = _py_lin(n, py["gate"], g[m], s)
        up = _py_lin(n, py["up"], g[m], s)
        a = [gv / (1 + math.exp(-gv)) * uv for gv, uv in zip(ga, up)]
        dn = _py_lin(a, py["down"], g[m], s)
        x = [a_ + b_ for a_, b_ in zip(x, dn)]
        np.testing.assert_allclose(got[m], x, rtol=1e-12, atol=1e-12)


def test_step_zero_adapter_p_equals_q_and_full_accept():
    """Bl = 0: mask rows reproduce the drafted-token verify rows, so q == p and blocks pass."""
    shape = W.TINY_SHAPE
    layers, head = W.model_weights_np(shape, seed=3)
    zero = lambda wab: (wab[0], wab[1], np.zeros_like(wab[2]))
    layers = [{k: zero(v) for k, v in lw.items()} for lw in layers]
    head = zero(head)
    B, k = 2, 4
    h = W.step_hidden(B, k, shape.hidden, seed=4)
    logits = O.stack_logits(h, layers, head, O.step_gate(B, k), 1.0)
    V = shape.vocab
    p = logits[: B * (k + 1)].reshape(B, k + 1, V)
    q = logits[B * (k + 1):].reshape(B, k, V)
    np.testing.assert_array_equal(q, p[:, 1:])
    # verify this step's drafts against itself: everything accepted + bonus
    d = draft_sample(p[:, :k], 1.0, 5, 0)
    res = psi_verify(p, p[:, :k], d, 1.0, 5, 0)
    assert np.all(res["accepted_len"] == k) and np.all(res["out_count"] == k + 1)


def test_step_gate_changes_only_mask_rows():
    shape = W.TINY_SHAPE
    layers, head = W.model_weights_np(shape, seed=6)
    B, k = 2, 3
    h = W.step_hidden(B, k, shape.hidden, seed=7)
    g = O.step_gate(B, k)
    on = O.stack_logits(h, layers, head, g, 1.0, store=None)
    off = O.stack_logits(h, layers, head, np.zeros_like(g), 1.0, store=None)
    nv = B * (k + 1)
    np.testing.assert_array_equal(on[:nv], off[:nv])
    assert np.abs(on[nv:] - off[nv:]).max() > 1e-3


# ---------------------------------------------------------------- psi_step pins
#
# psi_step composes the stack, the row layout of a step, verification and the
# draft. The stack has no attention, so every row's logits depend on that row
# alone: evaluating the verify rows (gate 0) and the mask rows (gate 1) as two
# separate batches gives p and q_next independently of psi_step's row split.
# The pins below check psi_step against that, against the special case where
# the previous block's draft distributions equal this step's AR rows (every
# block accepted, then the bonus draw: k + 1 tokens), and show that planted
# wiring slips fail at least one of them.

def _pin_model(seed=11, b_scale=40.0):
    """Tiny model (float64) whose adapter moves the draft rows well away from the AR rows."""
    shape = W.TINY_SHAPE
    layers, head = W.model_weights_np(shape, seed=seed)
    f = lambda wab: (W.bf16_to_f64(wab[0]), W.bf16_to_f64(wab[1]), W.bf16_to_f64(wab[2]) * b_scale)
    return shape, [{k: f(v) for k, v in lw.items()} for lw in layers], f(head)


def _rows_apart(h, layers, head, B, k, scale):
    """(p [B,k+1,V], q [B,k,V]): the verify rows and the mask rows evaluated as separate batches."""
    nv = B * (k + 1)
    p = O.stack_logits(h[:nv], layers, head, np.zeros(nv, np.uint8), scale)
    q = O.stack_logits(h[nv:], layers, head, np.ones(B * k, np.uint8), scale)
    V = p.shape[1]
    return p.reshape(B, k + 1, V), q.reshape(B, k, V)


def _step_pin_failures(step_fn, B=3, k=4, T=1.0):
    """Names of the psi_step pins that `step_fn` (psi_step's signature) fails."""
    shape, layers, head = _pin_model()
    h = W.step_hidden(B, k, shape.hidden, seed=12)
    p, q = _rows_apart(h, layers, head, B, k, 1.0)
    fails = []
    # 1. a previous block drawn from other draft distributions: verification runs on
    #    this step's AR rows (all k + 1 per sequence, bonus enabled), the draft on its
    #    mask rows, with the step's seed and step index
    q_prev = W.bf16_to_f64(W.logits_case(B, k, shape.vocab, ar_std=2.0, sigma=0.0,
                                         peak_frac=0.0, seed=13).q_logits)
    d_prev = draft_sample(q_prev, T, 21, 4)
    ver, d_next, q_next, logits = step_fn(h, layers, head, B, k, q_prev, d_prev, T, 21, 5, 1.0)
    want = psi_verify(p, q_prev, d_prev, T, 21, 5)
    if not (np.array_equal(ver["accepted_len"], want["accepted_len"])
            and np.array_equal(ver["out_tokens"], want["out_tokens"])
            and np.array_equal(ver["out_count"], want["out_count"])):
        fails.append("verify on the AR rows")
    if not np.allclose(q_next, q, rtol=0, atol=1e-9):
        fails.append("q_next = mask rows")
    if not np.array_equal(d_next, draft_sample(q, T, 21, 5)):
        fails.append("draft from the mask rows")
    # 2. q_prev equal to this step's AR rows 0..k-1: every block is accepted and the
    #    bonus is drawn (k + 1 tokens), whatever the seed
    for seed in (0, 1, 2):
        d_same = draft_sample(p[:, :k], T, seed + 50, 3)
        ver, *_ = step_fn(h, layers, head, B, k, p[:, :k], d_same, T, seed, 3, 1.0)
        if not (np.all(ver["accepted_len"] == k) and np.all(ver["out_count"] == k + 1)
                and np.array_equal(ver["out_tokens"][:, :k], d_same)):
            fails.append(f"full acceptance + bonus (seed {seed})")
            break
    return fails


def test_psi_step_pins():
    assert _step_pin_failures(O.psi_step) == []
    # the pins do not depend on T
    assert _step_pin_failures(O.psi_step, B=2, k=3, T=0.7) == []


def _mutant(kind):
    """psi_step with one planted wiring slip."""
    def step(h_in, layers, head, B, k, q_prev_logits, d_prev, T, seed, step, scale):
        gate = O.step_gate(B, k)
        if kind == "gate_swapped":
            gate = 1 - gate
        logits = O.stack_logits(h_in, layers, head, gate, scale)
        V = logits.shape[1]
        nv = B * (k + 1)
        p = logits[:nv].reshape(B, k + 1, V)
        q_next = logits[nv:].reshape(B, k, V)
        if kind == "blocks_swapped":                     # mask rows taken as the AR rows
            q_next = logits[:B * k].reshape(B, k, V)
            p = logits[B * k:].reshape(B, k + 1, V)
        if kind == "no_bonus":                           # verify with k_p = k
            p = p[:, :k]
        if kind == "shifted":                            # AR rows 1..k instead of 0..k-1
            p = np.concatenate([p[:, 1:], p[:, -1:]], axis=1)
        ver = psi_verify(p, q_prev_logits, d_prev, T, seed, step)
        d_src = p[:, :k] if kind == "draft_from_p" else q_next
        d_next = draft_sample(d_src, T, seed, step + (1 if kind == "draft_step" else 0))
        return ver, d_next, q_next, logits
    return step


@pytest.mark.parametrize("kind", ["gate_swapped", "blocks_swapped", "no_bonus", "shifted",
                                  "draft_from_p", "draft_step"])
def test_psi_step_pins_catch_planted_slips(kind):
    assert _step_pin_failures(_mutant(kind)), f"planted slip {kind!r} passed every pin"
