"""Pins for the oracle's synthetic decode stack (CPU only)."""
import math

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
