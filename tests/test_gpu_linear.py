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
    """M = 2048: clean half gate 0, noisy half gate 1. Every row against the oracle; the
    clean rows also against the plain base product x W^T (they must not see the adapter),
    and the noisy rows must differ from it by the adapter's term."""
    case = W.mlp_case(which)
    y = _run(case)
    ref = _oracle(case)
    check_close(y, ref, what=f"mlp {which} all rows")
    f = lambda a: case_to_f64(a, case.dtype)
    clean = np.flatnonzero(case.gate == 0)
    noisy = np.flatnonzero(case.gate == 1)
    assert len(clean) == len(noisy) == 1024
    base_clean = f(case.x[clean]) @ f(case.W).T
    check_close(y[clean], base_clean, what=f"mlp {which} clean rows = base product")
    lora = ref[noisy] - f(case.x[noisy]) @ f(case.W).T          # the adapter's term
    moved = y[noisy] - f(case.x[noisy]) @ f(case.W).T
    check_close(moved, lora, rel=0.05, what=f"mlp {which} noisy rows carry the adapter")


@pytest.mark.parametrize("M,K,N,r,dt", [
    (1, 64, 128, 8, "bf16"),
    (3, 72, 200, 16, "bf16"),
    (17, 520, 264, 24, "bf16"),
    (40, 512, 640, 0, "bf16"),          # decode-size path without an adapter
    (24, 4096, 10240, 64, "bf16"),      # decode-size path: split tiles over two waves
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


@pytest.mark.parametrize("M,K,N,r", [
    (600, 8192, 8192, 8),     # 96 tiles of 129 K-blocks on 74 pairs
    (700, 8200, 8000, 24),    # ragged M, N and K (130 K-blocks)
])
def test_stream_k_tiles(M, K, N, r):
    """Deep tiles whose count would leave the last round of the CTA-pair kernel part-empty:
    the last tiles are shared out by K-blocks and two pairs add up each cut tile."""
    rng = np.random.default_rng(M + N)
    gate = (rng.random(M) < 0.5).astype(np.uint8)
    case = W.gated_linear_case(M, K, N, r, gate, b_std=0.05, scale=0.75, seed=5)
    check_close(_run(case), _oracle(case), what=f"stream-K {M}x{K}x{N} r={r}")


@pytest.mark.parametrize("r", [16, 0])
def test_stream_k_flags_cleared_by_the_call(r):
    """A workspace whose every word already reads "ready" (1), used by two calls in a row:
    each call clears its stream-K flags before the pairs use them (the down-projection
    does it when r > 0, a memset when r = 0), so both match the oracle."""
    import torch
    import sampling_gated_lora_b200 as U
    M, K, N = 600, 8192, 8192
    gate = (np.arange(M) % 3 == 0).astype(np.uint8)
    case = W.gated_linear_case(M, K, N, r, gate, b_std=0.05, seed=7)
    ref = _oracle(case)
    args = [dev_tensor(a, "bf16") for a in (case.x, case.W, case.A, case.Bl)]
    g = dev_tensor(case.gate, "u8")
    need = U.load().uno_gated_lora_linear_workspace(U.UNO_BF16, M, K, N, r)
    ws = torch.ones(need // 4, dtype=torch.int32, device="cuda").view(torch.uint8)
    for call in range(2):
        y = U.gated_lora_linear(*args, g, 1.0, workspace=ws)
        check_close(host_f64(y), ref, what=f"r={r} call {call}")


@pytest.mark.parametrize("G", [1, 2, 3])
def test_stale_workspace_grouped_calls(G):
    """Grouped calls on the CTA-pair kernel with every workspace byte at 0x7f (stale
    stream-K flags would never read "ready"), twice in a row: each call clears its flags
    before the pairs use them. 1 to 3 groups of the qkv shapes, 16 token blocks."""
    import torch
    import sampling_gated_lora_b200 as U
    M, K = 4000, 1024
    Ns = (4096, 1024, 1024)[:G]
    x, gate, cases = _group_case(M, K, Ns, 128, seed=40 + G)
    refs = [_oracle_group(x, gate, c) for c in cases]
    need = U.load().uno_gated_lora_linear_group_workspace(U.UNO_BF16, M, 128, G)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    for call in range(2):
        ys = _run_group(x, gate, cases, False, workspace=ws)
        for y, ref, c in zip(ys, refs, cases):
            check_close(y, ref, what=f"G={G} N={c.N} call {call}")


@pytest.mark.parametrize("G,M", [(1, 9), (3, 17), (1, 72)])
def test_decode_calls_reused_workspace_and_graph_replay(G, M):
    """Decode-size calls (the fused decode kernel): a workspace filled with 0x7f and one
    filled with zeros, each used by two calls in a row, and a CUDA graph of one call
    replayed three times. Every output matches the oracle, and the replays are
    bit-identical to the eager call."""
    import torch
    import sampling_gated_lora_b200 as U
    K = 4096
    Ns = (4096, 1024, 1024)[:G]
    x, gate, cases = _group_case(M, K, Ns, 128, seed=60 + G + M, b_std=0.05)
    refs = [_oracle_group(x, gate, c) for c in cases]
    need = U.load().uno_gated_lora_linear_group_workspace(U.UNO_BF16, M, 128, G)
    for fill in (0x7F, 0):
        ws = torch.full((need,), fill, dtype=torch.uint8, device="cuda")
        for call in range(2):
            ys = _run_group(x, gate, cases, False, workspace=ws)
            for y, ref, c in zip(ys, refs, cases):
                check_close(y, ref, what=f"G={G} M={M} N={c.N} fill={fill:#x} call {call}")
    t = lambda a: dev_tensor(a, "bf16")
    args = (t(x), [t(c.W) for c in cases], [t(c.A) for c in cases], [t(c.Bl) for c in cases],
            dev_tensor(gate, "u8"), 1.0)
    outs = [torch.empty((M, n), dtype=torch.bfloat16, device="cuda") for n in Ns]
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    U.gated_lora_linear_group(*args, ys=outs, workspace=ws)
    eager = [host_f64(o) for o in outs]
    stream = torch.cuda.Stream()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        U.gated_lora_linear_group(*args, ys=outs, workspace=ws,
                                  stream=torch.cuda.current_stream())
    for rep in range(3):
        for o in outs:
            o.fill_(0)
        graph.replay()
        torch.cuda.synchronize()
        for o, e, ref, c in zip(outs, eager, refs, cases):
            got = host_f64(o)
            np.testing.assert_array_equal(got, e)
            check_close(got, ref, what=f"G={G} M={M} N={c.N} graph replay {rep}")


def test_stream_k_without_workspace_scratch():
    """r = 0: with the workspace the size query asks for, the pair kernel cuts tiles; with
    none it runs whole tiles only. Both match the oracle."""
    import torch
    import sampling_gated_lora_b200 as U
    M, K, N = 600, 8192, 8192
    case = W.gated_linear_case(M, K, N, 0, np.zeros(M, np.uint8), seed=6)
    ref = _oracle(case)
    args = [dev_tensor(a, "bf16") for a in (case.x, case.W, case.A, case.Bl)]
    g = dev_tensor(case.gate, "u8")
    for ws in (None, torch.zeros(16, dtype=torch.uint8, device="cuda")):
        y = U.gated_lora_linear(*args, g, 1.0, workspace=ws)
        check_close(host_f64(y), ref, what=f"r=0 workspace={'full' if ws is None else 'none'}")


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


def _group_case(M, K, Ns, r, seed, b_std=0.01):
    rng = np.random.default_rng(seed)
    gate = (rng.random(M) < 0.5).astype(np.uint8)
    cases = [W.gated_linear_case(M, K, N, r, gate, b_std=b_std, seed=seed + i) for i, N in enumerate(Ns)]
    x = cases[0].x
    return x, gate, cases


def _run_group(x, gate, cases, silu_pair, workspace=None):
    import sampling_gated_lora_b200 as U
    t = lambda a: dev_tensor(a, "bf16")
    ys = U.gated_lora_linear_group(t(x), [t(c.W) for c in cases], [t(c.A) for c in cases],
                                   [t(c.Bl) for c in cases], dev_tensor(gate, "u8"), 1.0,
                                   silu_pair=silu_pair, workspace=workspace)
    return [host_f64(y) for y in ys]


def _oracle_group(x, gate, c, rows=None):
    f = W.bf16_to_f64
    xs = f(x) if rows is None else f(x[rows])
    g = gate if rows is None else gate[rows]
    return gated_linear(xs, f(c.W), f(c.A), f(c.Bl), g, 1.0)


@pytest.mark.parametrize("M", [9, 72, 576, 1088])
def test_grouped_qkv(M):
    """q, k, v of one layer in one launch (4096 -> 4096 / 1024 / 1024, r = 128)."""
    x, gate, cases = _group_case(M, 4096, (4096, 1024, 1024), 128, seed=M)
    ys = _run_group(x, gate, cases, False)
    rows = None if M <= 576 else np.arange(0, M, 7)
    for y, c in zip(ys, cases):
        ref = _oracle_group(x, gate, c, rows)
        check_close(y if rows is None else y[rows], ref, what=f"group N={c.N} M={M}")


@pytest.mark.parametrize("M,K,N,r", [(9, 4096, 12288, 128), (72, 4096, 1024, 128),
                                     (17, 264, 200, 24), (300, 1024, 520, 64),
                                     (600, 8192, 4096, 64),   # 96 deep tiles: stream-K
                                     (2048, 4096, 12288, 128)])
def test_silu_pair(M, K, N, r):
    """y = silu(gate(x)) * up(x) in one launch.

    The product reaches |y| >= 8, where one bf16 rounding of the output alone
    exceeds the single-linear max-abs bound: elements are held to
    3e-2 + 2^-8 |ref| (that bound plus one bf16 rounding of the product).
    """
    from oracle.stack import silu
    x, gate, cases = _group_case(M, K, (N, N), r, seed=N + M)
    y = _run_group(x, gate, cases, True)[0]
    rows = None if M <= 300 else np.concatenate([np.arange(0, M, 37), [M // 2 - 1, M // 2, M - 1]])
    ref = silu(_oracle_group(x, gate, cases[0], rows)) * _oracle_group(x, gate, cases[1], rows)
    check_close(y if rows is None else y[rows], ref, what=f"silu-pair M={M} K={K} N={N}",
                rel_elem=2.0 ** -8)
