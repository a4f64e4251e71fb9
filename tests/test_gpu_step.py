"""One synthetic decode step (uno_psi_step) on a small model.

Logits of every row are compared with the fp64 oracle stack. The stack stores
bf16 between operations, so its logits carry bf16 rounding noise whose size
depends on where each side rounds; the bound is derived from the oracle itself:
the GPU's logits must lie within twice the distance between the oracle with
bf16 storage and the oracle in fp64 throughout (that distance, ~6e-3
relative on the small model, is the noise floor of the storage format). The
step's tokens are checked against the oracle's verification and draft run on
the step's own bf16 logits (decisions may differ only at logged near-ties).
The Qwen3-8B-shaped step is checked layer by layer in test_gpu_step_qwen3.py."""
import numpy as np
import pytest

import workloads as W
from oracle import sampling as S
from oracle import stack as O
from gpu_util import api_T, compare_drafts, compare_verify, dev_tensor, host_f64

pytestmark = pytest.mark.gpu


def _model(shape, seed):
    import sampling_gated_lora_b200 as U
    layers_np, head_np = W.model_weights_np(shape, seed=seed)
    tl = lambda wab: tuple(dev_tensor(a, "bf16") for a in wab)
    layers = [{k: tl(v) for k, v in lw.items()} for lw in layers_np]
    head = tl(head_np)
    m = U.Model(layers, head, shape.hidden, shape.q_out, shape.kv_out, shape.inter, shape.vocab,
                shape.r, shape.scale)
    return m, layers_np, head_np


def _buffers(B, k, V, dev="cuda"):
    import torch
    i32 = dict(dtype=torch.int32, device=dev)
    return dict(q_next=torch.empty((B, k, V), dtype=torch.bfloat16, device=dev),
                d_next=torch.empty((B, k), **i32), acc=torch.empty(B, **i32),
                tok=torch.empty((B, k + 1), **i32), cnt=torch.empty(B, **i32),
                logits=torch.empty((B * (k + 1), V), dtype=torch.bfloat16, device=dev),
                status=torch.zeros(1, **i32))


# One layer whose MLP is too wide for the fused decode kernel (2 * 9728 rows in
# 152 silu tiles > 148 SMs): at decode sizes the step folds the silu pair's
# down-projection into the RMSNorm launch.
WIDE_MLP_SHAPE = W.ModelShape(n_layers=1, hidden=256, q_out=256, kv_out=64, inter=9728,
                              vocab=1024, r=16)


@pytest.mark.parametrize("shape,B,k,T", [(W.TINY_SHAPE, 2, 4, 1.0), (W.TINY_SHAPE, 3, 8, 0.7),
                                         (W.TINY_SHAPE, 1, 1, 1.0), (W.TINY_SHAPE, 64, 8, 1.0),
                                         (WIDE_MLP_SHAPE, 1, 8, 1.0), (WIDE_MLP_SHAPE, 2, 4, 0.7)])
def test_tiny_step(shape, B, k, T):
    import torch
    import sampling_gated_lora_b200 as U
    T = api_T(T)
    m, layers_np, head_np = _model(shape, seed=1)
    V = shape.vocab
    h = W.step_hidden(B, k, shape.hidden, seed=2)
    qp = W.logits_case(B, k, V, ar_std=2.0, sigma=1.0, peak_frac=0.0, seed=3)
    q_prev = qp.q_logits
    d_prev = S.draft_sample(q_prev, T, 7, 4)             # drafted at the previous step
    buf = _buffers(B, k, V)
    ws = torch.empty(m.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
    Q_prev = dev_tensor(q_prev, "bf16")
    D_prev = dev_tensor(d_prev, "i32")
    m.step(B, k, dev_tensor(h, "bf16"), Q_prev, D_prev, T, 7, 5, buf["q_next"], buf["d_next"],
           buf["acc"], buf["tok"], buf["cnt"], ws, logits_out=buf["logits"],
           dev_status=buf["status"])
    torch.cuda.synchronize()
    assert int(buf["status"].item()) == 0
    # logits of every row vs the oracle stack
    gate = O.step_gate(B, k)
    ref = O.stack_logits(h, layers_np, head_np, gate, shape.scale, store="bf16")
    exact = O.stack_logits(h, layers_np, head_np, gate, shape.scale, store=None)
    got = np.concatenate([host_f64(buf["logits"]), host_f64(buf["q_next"]).reshape(B * k, V)])
    rel = lambda a, b: np.linalg.norm(a - b) / np.linalg.norm(b)
    floor = rel(ref, exact)
    assert rel(got, exact) <= 2 * floor, (rel(got, exact), floor)
    assert rel(got, ref) <= 2 * floor, (rel(got, ref), floor)
    assert np.abs(got - exact).max() <= 2 * np.abs(ref - exact).max() + 2.0 ** -7 * np.abs(exact).max()
    # tokens: the oracle's verification of the previous block against the step's own
    # (bf16) AR rows, and its draft from the step's mask rows, decide what is emitted
    p_gpu = host_f64(buf["logits"]).reshape(B, k + 1, V)
    ora = S.psi_verify(p_gpu, q_prev, d_prev, T, 7, 5)
    gpu = tuple(buf[n].cpu().numpy() for n in ("acc", "tok", "cnt"))
    excused, bad = compare_verify(gpu, ora, k, range(B))
    assert not bad and len(excused) <= 1, (bad, excused)
    excused, bad = compare_drafts(buf["d_next"].cpu().numpy(), host_f64(buf["q_next"]), T, 7, 5)
    assert not bad and excused <= 1, (bad, excused)
    m.close()


def test_zero_adapter_step_accepts_its_own_drafts():
    """Bl = 0 everywhere: q_next equals the drafted-token verify rows, so verifying the
    step's own drafts against its AR rows accepts every block."""
    import torch
    import sampling_gated_lora_b200 as U
    shape = W.TINY_SHAPE
    layers_np, head_np = W.model_weights_np(shape, seed=4)
    zero = lambda wab: (wab[0], wab[1], np.zeros_like(wab[2]))
    layers_np = [{k: zero(v) for k, v in lw.items()} for lw in layers_np]
    head_np = zero(head_np)
    tl = lambda wab: tuple(dev_tensor(a, "bf16") for a in wab)
    m = U.Model([{k: tl(v) for k, v in lw.items()} for lw in layers_np], tl(head_np), shape.hidden,
                shape.q_out, shape.kv_out, shape.inter, shape.vocab, shape.r)
    B, k, V = 4, 4, shape.vocab
    h = dev_tensor(W.step_hidden(B, k, shape.hidden, seed=5), "bf16")
    buf = _buffers(B, k, V)
    q0 = torch.zeros((B, k, V), dtype=torch.bfloat16, device="cuda")
    d0 = torch.zeros((B, k), dtype=torch.int32, device="cuda")
    ws = torch.empty(m.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
    m.step(B, k, h, q0, d0, 1.0, 3, 0, buf["q_next"], buf["d_next"], buf["acc"], buf["tok"],
           buf["cnt"], ws, logits_out=buf["logits"])
    p = buf["logits"].reshape(B, k + 1, V)
    np.testing.assert_array_equal(host_f64(p[:, 1:]), host_f64(buf["q_next"]))
    acc, tok, cnt = U.psi_verify(p[:, 1:].contiguous(), buf["q_next"], buf["d_next"], 1.0, 3, 1)
    assert np.all(acc.cpu().numpy() == k)
    m.close()


@pytest.mark.parametrize("B", [2, 40])
def test_launch_profile(B):
    """uno_model_profile / uno_model_last_profile: one entry per launch of the plan plus
    the verification and the draft, GEMM entries carrying the step's M, the entries adding
    up to the time between events around the whole step, and a step's results unchanged by
    profiling (same tokens and draft as an unprofiled step on the same inputs)."""
    import torch
    import sampling_gated_lora_b200 as U
    shape, k = W.TINY_SHAPE, 4
    m, _, _ = _model(shape, seed=6)
    V, M = shape.vocab, B * (2 * k + 1)
    h = dev_tensor(W.step_hidden(B, k, shape.hidden, seed=7), "bf16")
    gen = torch.Generator(device="cuda").manual_seed(8)
    q0 = (2.0 * torch.randn((B, k, V), generator=gen, device="cuda")).to(torch.bfloat16)
    d0 = dev_tensor(W.draft_ids(B, k, V, seed=9), "i32")
    ws = torch.empty(m.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
    outs = []
    for prof in (False, True):
        m.profile(prof)
        buf = _buffers(B, k, V)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        m.step(B, k, h, q0, d0, 1.0, 11, 2, buf["q_next"], buf["d_next"], buf["acc"], buf["tok"],
               buf["cnt"], ws)
        b.record()
        b.synchronize()
        outs.append((buf["tok"].cpu().numpy(), buf["cnt"].cpu().numpy(), buf["d_next"].cpu().numpy(),
                     a.elapsed_time(b)))
    prof = m.last_profile()
    assert len(prof) == m.kernel_count(B, k) - 2          # verify and draft: two kernels each
    kinds = [p[0] for p in prof]
    assert kinds[-2:] == ["verify", "draft"]
    assert kinds.count("rmsnorm") + kinds.count("rmsnorm_down") == 2 * shape.n_layers + 1
    for name, ms, dims in prof:
        assert ms >= 0.0
        if name.startswith("gemm"):
            assert dims[0] == M and dims[1] > 0 and dims[2] in (shape.hidden, shape.q_out, shape.inter)
    total = sum(p[1] for p in prof)
    assert 0.3 * outs[1][3] <= total <= 1.05 * outs[1][3], (total, outs[1][3])
    for x, y in zip(outs[0][:3], outs[1][:3]):
        np.testing.assert_array_equal(x, y)
    m.profile(False)
    m.close()
