"""The synthetic decode step at the benchmarked shapes, against the fp64 oracle.

Qwen3-8B projections (36 layers; q/k/v/o 4096 -> 4096/1024/1024/4096, gate/up
4096 -> 12288, down 12288 -> 4096), rank-128 adapters, the gated LM head
4096 -> 151936, k = 8, B in {1, 256} (M = B(2k+1) = 17 and 4352 rows). Random
weights from torch's seeded generator (the inputs; not produced by this
library).

Nothing compounds: every residual sub-block of every layer, and each of its
linears, is fed the GPU's own input to it (uno_psi_step_hidden runs the
step's own launches up to a sub-block and returns the hidden state and the
products of its linears). On sampled rows:
  q, k, v       = L(rmsnorm(h))                 linear bound (the benchmark spec)
  h + o(q)      from the GPU's q and h          linear bound + one bf16 rounding
  silu(gate)*up = from rmsnorm of the GPU's h   same (reading R15)
  h + down(act) from the GPU's act and h        same
  LM head       rows of rmsnorm(h_final): AR rows -> logits, mask rows -> q_next
and the emitted tokens of all B sequences and the next drafts against the
oracle's verification and draft run on the GPU's own bf16 logits.
"""
import numpy as np
import pytest

import workloads as W
from oracle import sampling as S
from oracle import stack as O
from gpu_util import MAX_ABS, REL_FROB, check_close, compare_drafts, compare_verify

pytestmark = pytest.mark.gpu

SHAPE = W.QWEN3_8B_SHAPE
K_BLOCK = 8
T = 1.0
SEED, STEP = 2027, 3
ROUND = 2.0 ** -8        # one bf16 rounding of a stored output, relative


def _bits(t):
    return W.from_torch_bf16(t)


def _f64(t):
    return W.bf16_to_f64(_bits(t))


def _take(t, rows):
    """Rows `rows` of a device tensor, widened to float64 on the host."""
    import torch
    return _f64(t[torch.from_numpy(rows).to(t.device)])


def _sample_rows(B, k):
    """Verify rows and mask rows of a few sequences (every row when B = 1)."""
    seqs = [0] if B == 1 else [0, B // 2 + 3, B - 1]
    rows = []
    for b in seqs:
        rows += list(range(b * (k + 1), (b + 1) * (k + 1)))                 # anchor + k drafted
        rows += list(range(B * (k + 1) + b * k, B * (k + 1) + (b + 1) * k))  # k mask rows
    return np.array(rows)


@pytest.fixture(scope="module")
def qwen3():
    import torch
    import sampling_gated_lora_b200 as U
    layers, head = W.model_weights_torch(SHAPE, "cuda", seed=0)
    m = U.Model(layers, head, SHAPE.hidden, SHAPE.q_out, SHAPE.kv_out, SHAPE.inter, SHAPE.vocab,
                SHAPE.r, SHAPE.scale)
    runs = {}
    for B in (1, 256):
        k, V = K_BLOCK, SHAPE.vocab
        h = W.to_torch_bf16(W.step_hidden(B, k, SHAPE.hidden, seed=40 + B), "cuda")
        _, q_prev = W.logits_case_torch(B, k, V, sigma=1.0, seed=50 + B)
        q_prev_bits = _bits(q_prev)
        d_prev = S.draft_sample(q_prev_bits, T, SEED + 1, STEP - 1)     # drafts ~ q, on the host
        i32 = dict(dtype=torch.int32, device="cuda")
        out = dict(q_next=torch.empty((B, k, V), dtype=torch.bfloat16, device="cuda"),
                   d_next=torch.empty((B, k), **i32), acc=torch.empty(B, **i32),
                   tok=torch.empty((B, k + 1), **i32), cnt=torch.empty(B, **i32),
                   logits=torch.empty((B * (k + 1), V), dtype=torch.bfloat16, device="cuda"),
                   status=torch.zeros(1, **i32))
        ws = torch.empty(m.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
        m.step(B, k, h, q_prev, torch.from_numpy(d_prev).cuda(), T, SEED, STEP, out["q_next"],
               out["d_next"], out["acc"], out["tok"], out["cnt"], ws, logits_out=out["logits"],
               dev_status=out["status"])
        torch.cuda.synchronize()
        runs[B] = dict(h=h, ws=ws, q_prev_bits=q_prev_bits, d_prev=d_prev, out=out,
                       rows=_sample_rows(B, k))
        del q_prev
    yield m, layers, head, runs
    m.close()
    del runs
    torch.cuda.empty_cache()


def _lin(x, wab, gate):
    return O._lin(x, wab, gate, SHAPE.scale)


def test_every_sub_block_and_linear_from_the_gpu_input(qwen3):
    m, layers, _, runs = qwen3
    k = K_BLOCK
    for li, lw_t in enumerate(layers):
        lw = {name: tuple(_f64(t) for t in wab) for name, wab in lw_t.items()}
        for B, run in runs.items():
            rows = run["rows"]
            g = O.step_gate(B, k)[rows]
            what = f"B={B} layer {li}"
            h_l = _take(m.hidden_state(B, k, run["h"], 2 * li, run["ws"]), rows)
            h_mid_t, mid = m.hidden_state(B, k, run["h"], 2 * li + 1, run["ws"], inter=True)
            h_next_t, nxt = m.hidden_state(B, k, run["h"], 2 * li + 2, run["ws"], inter=True)
            h_mid, h_next = _take(h_mid_t, rows), _take(h_next_t, rows)
            # projection sub-block: q, k, v from rmsnorm(h_l); h_mid = h_l + o(q)
            n1 = O.round_bf16(O.rmsnorm(h_l))
            for name in ("q", "k", "v"):
                check_close(_take(mid[name], rows), _lin(n1, lw[name], g), what=f"{what} {name}")
            q_gpu = _take(mid["q"], rows)
            check_close(h_mid, h_l + _lin(q_gpu, lw["o"], g), rel_elem=ROUND, what=f"{what} h+o(q)")
            # MLP sub-block: silu(gate) * up from rmsnorm(h_mid); h_next = h_mid + down(act)
            n2 = O.round_bf16(O.rmsnorm(h_mid))
            act_ref = O.silu(_lin(n2, lw["gate"], g)) * _lin(n2, lw["up"], g)
            act = _take(nxt["act"], rows)
            check_close(act, act_ref, rel_elem=ROUND, what=f"{what} silu(gate)*up")
            check_close(h_next, h_mid + _lin(act, lw["down"], g), rel_elem=ROUND,
                        what=f"{what} h+down(act)")
            # the projection products of the next call are this layer's too
            assert bool((nxt["q"] == mid["q"]).all())


def test_lm_head_rows_split_into_logits_and_q_next(qwen3):
    m, _, head_t, runs = qwen3
    k, V = K_BLOCK, SHAPE.vocab
    head = tuple(_bits(t) for t in head_t)          # bf16 bits; widened chunk by chunk
    for B, run in runs.items():
        rows = run["rows"]
        g = O.step_gate(B, k)[rows]
        h_final = _take(m.hidden_state(B, k, run["h"], 2 * SHAPE.n_layers, run["ws"]), rows)
        n_f = O.round_bf16(O.rmsnorm(h_final))
        nv = B * (k + 1)
        logits = _bits(run["out"]["logits"])
        q_next = _bits(run["out"]["q_next"]).reshape(B * k, V)
        got = W.bf16_to_f64(np.stack([logits[r] if r < nv else q_next[r - nv] for r in rows]))
        A, Bl = W.bf16_to_f64(head[1]), W.bf16_to_f64(head[2])
        ref = np.empty((len(rows), V))
        for v0 in range(0, V, 16384):
            v1 = min(V, v0 + 16384)
            ref[:, v0:v1] = O.gated_linear(n_f, W.bf16_to_f64(head[0][v0:v1]), A, Bl[v0:v1], g,
                                           SHAPE.scale)
        check_close(got, ref, REL_FROB, MAX_ABS, what=f"B={B} LM head")


def test_tokens_of_every_sequence_match_the_oracle_on_the_gpu_logits(qwen3):
    _, _, _, runs = qwen3
    k, V = K_BLOCK, SHAPE.vocab
    for B, run in runs.items():
        out = run["out"]
        assert int(out["status"].item()) == 0
        p = _bits(out["logits"]).reshape(B, k + 1, V)
        ora = S.psi_verify(p, run["q_prev_bits"], run["d_prev"], T, SEED, STEP)
        gpu = tuple(out[n].cpu().numpy() for n in ("acc", "tok", "cnt"))
        excused, bad = compare_verify(gpu, ora, k, range(B))
        assert not bad, f"B={B}: unexcused mismatches in sequences {bad}"
        assert len(excused) <= max(1, 1e-4 * B * k), excused
        assert np.all(gpu[2] == gpu[0] + 1)           # bonus enabled: a draw every step
        ex_d, bad_d = compare_drafts(out["d_next"].cpu().numpy(), _bits(out["q_next"]), T, SEED,
                                     STEP)
        assert not bad_d, f"B={B}: unexcused draft mismatches {bad_d}"
        assert ex_d <= max(1, 1e-4 * B * k)
        print(f"B={B}: mean accepted {gpu[0].mean():.3f}, excused {len(excused)} + {ex_d}")
