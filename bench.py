#!/usr/bin/env python
"""Benchmark of the synthetic Psi-Spec linear decode step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--B 256] [--k 8] [--impl uno|reference]

One step = uno_psi_step on Qwen3-8B-shaped gated-LoRA projections (36 layers of
q/k/v/o/gate/up/down, rank 128, no attention) + the gated LM head
4096 -> 151936 + psi_verify (bonus enabled) + the linear-sampler draft, for B
sequences with block size k (M = B(2k+1) rows). Metric: verified tokens/s =
tokens emitted by verification / step time, summed over ranks (each rank runs
its own replica on its own B sequences: weak scaling, no collective on the
data path). Rank 0 prints one JSON line.

Timing: W untimed steps, then K steps between CUDA events on the launching
stream, bracketed by a barrier and device synchronisation; max over ranks.
Every step streams 15.1 GB of weights, far larger than the 126 MB L2.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "Ψ-Spec verified tokens/s at B=1..256; gated-LoRA/verify GB/s vs HBM peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--B", type=int, default=256)
    ap.add_argument("--k", type=int, default=8)
    ap.add_argument("--temperature", type=float, default=1.0)
    ap.add_argument("--impl", choices=["uno", "reference"], default="uno")
    ap.add_argument("--no-kernels", action="store_true", help="skip the per-config kernel lines")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--profile", choices=["gemm_up", "gemm_small", "step_up", "verify", "draft",
                                          "draft_full", "gemm_down", "backward"],
                    help="run a few launches of one kernel on a small case (for ncu) and exit")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured (MEASURED_PEAKS.json)"
    return dict(FALLBACK_PEAKS), "fallback"


def shard(B_per_rank, rank):
    """Sequences of one rank under weak scaling: (count, global offset of its first sequence)."""
    return B_per_rank, rank * B_per_rank


def combine_over_ranks(ms, tokens, dist=None, device="cpu"):
    """(max over ranks of the timed milliseconds, sum over ranks of the tokens)."""
    import torch
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(ms), int(tokens)
    mx = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    sm = torch.tensor([float(tokens)], dtype=torch.float64, device=device)
    dist.all_reduce(mx, op=dist.ReduceOp.MAX)
    dist.all_reduce(sm, op=dist.ReduceOp.SUM)
    return float(mx.item()), int(round(sm.item()))


def csrc_hash():
    import glob
    import hashlib
    srcs = sorted(glob.glob(os.path.join(ROOT, "sampling_gated_lora_b200", "csrc", "*")))
    return hashlib.sha256(b"".join(open(f, "rb").read() for f in srcs)).hexdigest()[:16]


def recorded_traffic(kernel):
    """DRAM bytes per launch of `kernel` from the committed ncu capture, or None when
    the kernel sources changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "roofline_traffic.json")
    if not os.path.exists(path):
        return None
    d = json.load(open(path))
    if d.get("kernel") != kernel or d.get("csrc_sha256_16") != csrc_hash():
        return None
    return d["traffic_bytes"]


def workload_config(B, k, T):
    return {"workload": f"psi_step Qwen3-8B-shaped: 36 layers q/k/v/o 4096->4096/1024/1024/4096, "
                        f"gate/up 4096->12288, down 12288->4096, LM head 4096->151936, rank 128, "
                        f"no attention; B={B}, k={k}, rows B(2k+1)={B * (2 * k + 1)}, T={T}",
            "B": B, "k": k, "rows": B * (2 * k + 1), "vocab": 151936, "rank": 128,
            "layers": 36, "temperature": T,
            "l2": "inputs larger than L2 (15.1 GB of weights streamed per step)"}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    def __init__(self, device_index):
        self.idx = device_index
        self.proc = None

    def __enter__(self):
        self.f = tempfile.NamedTemporaryFile("w+", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}",
                 "--query-gpu=clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        self.f.flush()
        rows = []
        for line in open(self.f.name):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 4:
                continue
            try:
                rows.append((float(parts[0]), float(parts[1]), float(parts[2]), int(parts[3], 16)))
            except ValueError:
                continue
        os.unlink(self.f.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        mask = 0
        for r in rows:
            mask |= r[3]
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows),
                "reasons": [n for b, n in REASONS.items() if mask & b and b != 0x1]}


# ---------------------------------------------------------------- oracle sample

HEAD_SLICE = 8   # the oracle's LM head is timed on 1/8 of the vocabulary rows and scaled x8


def expected_tokens(p, q, T, k):
    """Mean tokens one verification emits on these logits (bonus enabled), over the
    draft's and the sampler's randomness: with acceptance probabilities
    alpha_j = sum_v min(p_j(v), q_j(v)) (the closed form of one speculative test),
    E = sum_{n<k} (n+1) A_n (1 - alpha_n) + (k+1) A_k,  A_n = prod_{i<n} alpha_i."""
    from oracle import sampling as S
    P, Q = S.softmax_t(S.as_f64(p)[:k], T), S.softmax_t(S.as_f64(q), T)
    alpha = np.minimum(P, Q).sum(axis=1)
    e, run = 0.0, 1.0
    for n in range(k):
        e += (n + 1) * run * (1.0 - alpha[n])
        run *= alpha[n]
    return e + (k + 1) * run


def oracle_step_sample(k, layers_np, head_slice, T, seed=0):
    """One sequence (2k+1 rows) through the fp64 oracle, timed piecewise:
    `len(layers_np)` decoder layers (scaled to 36), the LM head on a 1/HEAD_SLICE
    vocabulary slice (scaled x HEAD_SLICE), then the draft sampler and verify
    over the full 151936-token vocabulary on seeded logits of the verify
    workload. Returns (seconds per full sequence-step, tokens emitted, expected
    tokens on these logits, wall seconds of the sample)."""
    import workloads as W
    from oracle import sampling as S
    from oracle import stack as O
    w0 = time.perf_counter()
    h = W.step_hidden(1, k, 4096, seed=seed)
    gate = O.step_gate(1, k)
    t0 = time.perf_counter()
    x = O.as_f64(h)
    for lw in layers_np:
        x = O.layer_forward(x, lw, gate, 1.0)
    t1 = time.perf_counter()
    O.round_bf16(O._lin(O.round_bf16(O.rmsnorm(x)), head_slice, gate, 1.0))
    t2 = time.perf_counter()
    p, q = W.logits_sequence(seed, k, k + 1, 151936, ar_std=3.0, sigma=1.0, peak_frac=0.05, seed=1234)
    t3 = time.perf_counter()
    d = S.draft_sample(q[None], T, seed, 0)
    res = S.psi_verify(p[None], q[None], d, T, seed, 1)
    t4 = time.perf_counter()
    per_layer = (t1 - t0) / max(1, len(layers_np))
    full = per_layer * 36 + (t2 - t1) * HEAD_SLICE + (t4 - t3)
    e = expected_tokens(p, q, T, k)
    return full, int(res["out_count"][0]), e, time.perf_counter() - w0


SAMPLE_TEXT = ("per sample: one sequence (2k+1 rows) through the fp64 NumPy oracle; 1 of 36 "
               "layers timed and scaled x36, the LM head on 1/8 of the vocabulary scaled x8, "
               "draft + verify over the full vocabulary timed in full")


def host_weights(layers, head, n_layers):
    """Copy n_layers layers and a 1/HEAD_SLICE row slice of the head (torch bf16, device) to host bits."""
    import workloads as W
    tl = lambda wab: tuple(W.from_torch_bf16(t) for t in wab)
    rows = head[0].shape[0] // HEAD_SLICE
    sl = (head[0][:rows], head[1], head[2][:rows])
    return [{k: tl(v) for k, v in lw.items()} for lw in layers[:n_layers]], tl(sl)


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ---------------------------------------------------------------- kernel lines

def kernel_lines(U, torch, pk, with_oracle=True):
    """Per-config kernel measurements (gated GEMM small M and M=2048, psi_verify).

    Gated linears are timed back to back, the way a decode step runs them: one
    CUDA graph of launches that cycle through weight sets whose total exceeds
    L2, so every launch reads its weights from HBM ("us"). The time of a
    single launch after an L2 flush is kept as "single_us".
    """
    import numpy as np
    import workloads as W
    out = {}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    if with_oracle:
        from oracle import distill as OD
        from oracle import gated_linear as OG
        from oracle import sampling as OS
        from oracle import tree as OT
    host = lambda t: t.float().cpu().numpy()   # bf16 values are exact in float32

    def oracle_line(line, fn, scale, sample):
        """The fp64 oracle on a bounded sample of a kernel line's work (host arrays copied
        before timing), scaled to the whole line: oracle_us beside the kernel's us."""
        if not with_oracle:
            return
        t0 = time.perf_counter()
        fn()
        line["oracle_us"] = round((time.perf_counter() - t0) * 1e6 * scale, 1)
        line["oracle_sample"] = sample
        line["oracle_cores"] = cpu_cores()

    def timed(fn, reps=20):
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3)
        return statistics.median(ts)

    def chained(calls, reps=5):
        """Median time per launch of the calls captured back to back in one graph."""
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for c in calls:
                c()
        g.replay()
        torch.cuda.synchronize()
        ts = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            g.replay()
            b.record()
            b.synchronize()
            ts.append(a.elapsed_time(b) * 1e3 / len(calls))
        del g
        return statistics.median(ts)

    dev = lambda shape, std: (torch.randn(shape, device="cuda") * std).to(torch.bfloat16)
    for B in (1, 8, 64):
        M, K, N, r = B * 9, 4096, 4096, 128
        sets = [(dev((N, K), K ** -0.5), dev((r, K), K ** -0.5), dev((N, r), 0.01)) for _ in range(10)]
        x = dev((M, K), 1)
        g = torch.from_numpy(W.decode_gate(B, 8)).cuda()
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(U.load().uno_gated_lora_linear_workspace(0, M, K, N, r), dtype=torch.uint8,
                         device="cuda")
        mk = lambda st: (lambda: U.gated_lora_linear(x, st[0], st[1], st[2], g, 1.0, y=y, workspace=ws))
        calls = [mk(sets[i % len(sets)]) for i in range(40)]
        calls[0]()
        single = timed(calls[0])
        us = chained(calls)
        Mg = int(g.sum())
        byts = 2 * (N * K + r * K + N * r + M * K + M * N)
        flops = 2 * M * K * N + 2 * Mg * r * (K + N)
        t_roof = max(byts / (pk["hbm_gbs"] * 1e9), flops / (pk["bf16_tflops"] * 1e12)) * 1e6
        line = out[f"gated_linear_4096x4096_M{M}"] = {
            "us": round(us, 2), "single_us": round(single, 2), "GBps": round(byts / us / 1e3, 1),
            "TFLOPs": round(flops / us / 1e6, 1), "roofline_us": round(t_roof, 2),
            "frac_of_roofline": round(t_roof / us, 3), "hbm_frac": round(byts / us / 1e3 / pk["hbm_gbs"], 3)}
        rs = min(M, 72)
        ho = [host(a) for a in (x[:rs], sets[0][0], sets[0][1], sets[0][2])] + [g[:rs].cpu().numpy()]
        oracle_line(line, lambda: OG.gated_linear(*ho, 1.0), M / rs, f"{rs} of {M} rows, scaled")
        del sets
    for name, K, N, M in (("up", 4096, 12288, 2048), ("down", 12288, 4096, 2048),
                          ("up", 4096, 12288, 4352)):
        r = 128
        sets = [(dev((N, K), K ** -0.5), dev((r, K), K ** -0.5), dev((N, r), 0.01)) for _ in range(3)]
        x = dev((M, K), 1)
        g = torch.cat([torch.zeros(M // 2, dtype=torch.uint8), torch.ones(M // 2, dtype=torch.uint8)]).cuda()
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        ws = torch.zeros(U.load().uno_gated_lora_linear_workspace(0, M, K, N, r), dtype=torch.uint8,
                         device="cuda")
        mk = lambda st: (lambda: U.gated_lora_linear(x, st[0], st[1], st[2], g, 1.0, y=y, workspace=ws))
        calls = [mk(sets[i % len(sets)]) for i in range(6)]
        calls[0]()
        single = timed(calls[0], reps=10)
        us = chained(calls)
        flops = 2 * M * K * N + 2 * (M // 2) * r * (K + N)
        line = out[f"gated_linear_mlp_{name}_M{M}"] = {
            "us": round(us, 2), "single_us": round(single, 2), "TFLOPs": round(flops / us / 1e6, 1),
            "tensor_frac": round(flops / us / 1e6 / pk["bf16_tflops"], 3)}
        rs = 64
        ho = [host(a) for a in (x[M - rs:], sets[0][0], sets[0][1], sets[0][2])] + [g[M - rs:].cpu().numpy()]
        oracle_line(line, lambda: OG.gated_linear(*ho, 1.0), M / rs, f"{rs} of {M} rows, scaled")
        del sets
    del x, y
    # adapter gradients (the training layout, MLP up shape): M = 2048 rows, 1024 of them
    # gated, 4096 -> 12288, r = 128. Algorithmic work counts the gated rows only (the
    # others contribute nothing): flops 2 Mg r (2K + 2N); bytes: the gated rows of x and
    # dy, A and Bl, and dA and dBl written.
    M, K, N, r = 2048, 4096, 12288, 128
    Mg = M // 2
    x, dy = dev((M, K), 1), dev((M, N), 1)
    A, Bl = dev((r, K), K ** -0.5), dev((N, r), 0.01)
    g = torch.cat([torch.zeros(M - Mg, dtype=torch.uint8), torch.ones(Mg, dtype=torch.uint8)]).cuda()
    dA = torch.empty((r, K), dtype=torch.bfloat16, device="cuda")
    dBl = torch.empty((N, r), dtype=torch.bfloat16, device="cuda")
    bws = torch.empty(U.load().uno_gated_lora_backward_workspace(M, K, N, r), dtype=torch.uint8,
                      device="cuda")
    f = lambda: U.gated_lora_adapter_grads(x, dy, A, Bl, g, 1.0, dA=dA, dBl=dBl, workspace=bws)
    f()
    us = timed(f, reps=10)
    flops = 2 * Mg * r * (2 * K + 2 * N)
    byts = 2 * (Mg * K + Mg * N + 2 * (r * K + N * r))
    t_roof = max(byts / (pk["hbm_gbs"] * 1e9), flops / (pk["bf16_tflops"] * 1e12)) * 1e6
    line = out["adapter_grads_mlp_up_M2048"] = {
        "us": round(us, 1), "TFLOPs": round(flops / us / 1e6, 1), "GBps": round(byts / us / 1e3, 1),
        "roofline_us": round(t_roof, 2), "frac_of_roofline": round(t_roof / us, 3)}
    rs = 64
    ho = [host(x[M - rs:]), host(A), host(Bl), g[M - rs:].cpu().numpy()]
    hdy = host(dy[M - rs:])
    oracle_line(line, lambda: OG.gated_linear_adapter_grads(*ho, 1.0, hdy), M / rs,
                f"{rs} of {M} rows (gated), scaled")
    del x, dy, A, Bl, bws
    # psi_verify at B=256, k=16, V=151936 (sigma 1.0 and 0.25, T = 1)
    B, k, V = 256, 16, 151936
    for sigma in (1.0, 0.25):
        p, q = W.logits_case_torch(B, k, V, sigma=sigma, seed=1234)
        d = U.draft_sample(q, 1.0, 99, 0)
        ws = torch.empty(U.load().uno_psi_verify_workspace(B, k, k, V), dtype=torch.uint8, device="cuda")
        outs = [torch.empty(B, dtype=torch.int32, device="cuda"),
                torch.empty((B, k + 1), dtype=torch.int32, device="cuda"),
                torch.empty(B, dtype=torch.int32, device="cuda")]
        f = lambda: U.psi_verify(p, q, d, 1.0, 1234, 0, accepted_len=outs[0], out_tokens=outs[1],
                                 out_count=outs[2], workspace=ws)
        f()
        us = timed(f, reps=10)
        byts = 2 * B * k * V * 2
        line = out[f"psi_verify_B256_k16_sigma{sigma}"] = {
            "us": round(us, 1), "GBps": round(byts / us / 1e3, 1),
            "hbm_frac": round(byts / us / 1e3 / pk["hbm_gbs"], 3),
            "mean_accepted": round(float(outs[0].float().mean()), 3)}
        hp, hq, hd = host(p[:2]), host(q[:2]), d[:2].cpu().numpy()
        oracle_line(line, lambda: OS.psi_verify(hp, hq, hd, 1.0, 1234, 0), B / 2,
                    f"2 of {B} sequences, scaled")
        del p, q
    # linear-sampler draft of the step at B=256, k=8: 2048 rows of V=151936 bf16 logits.
    # Algorithmic bytes: one read of every logit (the draw re-reads one vocab chunk a row).
    Bd, kd = 256, 8
    _, qd = W.logits_case_torch(Bd, kd, V, sigma=1.0, seed=4321)
    dws = torch.empty(U.load().uno_draft_sample_workspace(Bd, kd, V), dtype=torch.uint8,
                      device="cuda")
    dout = torch.empty((Bd, kd), dtype=torch.int32, device="cuda")
    f = lambda: U.draft_sample(qd, 1.0, 99, 0, draft=dout, workspace=dws)
    f()
    us = timed(f, reps=10)
    byts = Bd * kd * V * 2
    line = out[f"draft_sample_B{Bd}_k{kd}"] = {
        "us": round(us, 1), "GBps": round(byts / us / 1e3, 1),
        "hbm_frac": round(byts / us / 1e3 / pk["hbm_gbs"], 3)}
    hq = host(qd[:2])
    oracle_line(line, lambda: OS.draft_sample(hq, 1.0, 99, 0), Bd / 2, f"2 of {Bd} sequences, scaled")
    del qd
    # tree_verify at low batch: B=8 sequences, N=4 candidate blocks of k=8, V=151936.
    # Candidates: the linear sampler on q repeated N times per sequence (Philox index
    # (b N + i) k + j, the tree sampler's); AR row of each trie node = the draft row of
    # its depth + N(0, 1) noise. Algorithmic bytes: one read of every node row and q row.
    B, N, k, V = 8, 4, 8, 151936
    _, q = W.logits_case_torch(B, k, V, sigma=1.0, seed=77)
    cands = U.draft_sample(q.repeat_interleave(N, dim=0), 1.0, 5, 0).reshape(B, N, k).contiguous()
    c_host = cands.cpu().numpy()
    R = N * k + 1
    depth_idx = torch.zeros((B, R), dtype=torch.long)
    nodes = 0
    nodes_0 = 0
    for b in range(B):
        ids = {(): 0}
        for i in range(N):
            for j in range(k):
                pre = tuple(c_host[b, i, :j + 1])
                if pre not in ids:
                    ids[pre] = len(ids)
                    depth_idx[b, ids[pre]] = min(j + 1, k - 1)
        nodes += len(ids)
        nodes_0 = nodes_0 or len(ids)
    gen = torch.Generator(device="cuda").manual_seed(78)
    qf = q.float()
    p_nodes = (torch.gather(qf, 1, depth_idx.cuda()[:, :, None].expand(B, R, V))
               + torch.randn((B, R, V), device="cuda", generator=gen)).to(torch.bfloat16)
    ws = torch.empty(U.load().uno_tree_verify_workspace(B, N, k, R, V), dtype=torch.uint8,
                     device="cuda")
    touts = [torch.empty(B, dtype=torch.int32, device="cuda"),
             torch.empty((B, k + 1), dtype=torch.int32, device="cuda"),
             torch.empty(B, dtype=torch.int32, device="cuda")]
    f = lambda: U.tree_verify(p_nodes, q, cands, 1.0, 1234, 0, bonus=True, accepted_len=touts[0],
                              out_tokens=touts[1], out_count=touts[2], workspace=ws)
    f()
    us = timed(f, reps=10)
    byts = (nodes + B * k) * V * 2
    line = out[f"tree_verify_B{B}_N{N}_k{k}"] = {
        "us": round(us, 1), "GBps": round(byts / us / 1e3, 1),
        "hbm_frac": round(byts / us / 1e3 / pk["hbm_gbs"], 3), "trie_nodes": nodes,
        "mean_accepted": round(float(touts[0].float().mean()), 3)}
    hp, hq = host(p_nodes[0, :nodes_0]), host(q[0])
    oracle_line(line, lambda: OT.tree_verify_sequence(hp, hq, c_host[0], 1.0, 1234, 0, 0, bonus=True),
                B, f"1 of {B} sequences, scaled")
    del p_nodes, q
    # distillation losses + gradient on the MLP batch layout: 1024 clean (teacher) rows
    # against 1024 noisy (student) rows, V=151936, bf16 logits, fp32 gradient.
    # Algorithmic bytes: one read of both logit rows and one write of the gradient.
    rows, V = 1024, 151936
    gen = torch.Generator(device="cuda").manual_seed(91)
    zt = (torch.randn((rows, V), device="cuda", generator=gen) * 3).to(torch.bfloat16)
    zs = (zt.float() + torch.randn((rows, V), device="cuda", generator=gen)).to(torch.bfloat16)
    dl = torch.empty((rows, 2), dtype=torch.float32, device="cuda")
    dg = torch.empty((rows, V), dtype=torch.float32, device="cuda")
    f = lambda: U.distill(zt, zs, 1.0, 1.0, 1.0, losses=dl, grad_out=dg)
    f()
    us = timed(f, reps=10)
    byts = rows * V * (2 + 2 + 4)
    line = out[f"distill_rows{rows}_V{V}"] = {
        "us": round(us, 1), "GBps": round(byts / us / 1e3, 1),
        "hbm_frac": round(byts / us / 1e3 / pk["hbm_gbs"], 3)}
    ht, hs = host(zt[:8]), host(zs[:8])
    oracle_line(line, lambda: (OD.distill_losses(ht, hs, 1.0), OD.distill_grad(ht, hs, 1.0, 1.0, 1.0)),
                rows / 8, f"8 of {rows} row pairs, scaled")
    del zt, zs, dg
    torch.cuda.empty_cache()
    return out


# ---------------------------------------------------------------- main arms

def run_uno(args):
    import numpy as np
    import torch
    import torch.distributed as dist

    import sampling_gated_lora_b200 as U
    import workloads as W

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    U.load()
    pk, pk_src = peaks()
    shape = W.QWEN3_8B_SHAPE
    B, k, T = args.B, args.k, args.temperature
    V = shape.vocab
    layers, head = W.model_weights_torch(shape, "cuda", seed=0)
    model = U.Model(layers, head, shape.hidden, shape.q_out, shape.kv_out, shape.inter, V, shape.r,
                    shape.scale)
    M = B * (2 * k + 1)
    h_host = torch.from_numpy(W.step_hidden(B, k, shape.hidden, seed=rank).view(np.int16)).view(
        torch.bfloat16).pin_memory()
    h = h_host.cuda()
    i32 = dict(dtype=torch.int32, device="cuda")
    qb = [torch.zeros((B, k, V), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    db = [torch.zeros((B, k), **i32) for _ in range(2)]
    n_total = args.warmup + args.steps
    acc = torch.empty((n_total, B), **i32)
    tok = torch.empty((n_total, B, k + 1), **i32)
    cnt = torch.empty((n_total, B), **i32)
    status = torch.zeros(1, **i32)
    ws = torch.empty(model.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
    B, seq_off = shard(B, rank)

    def step(t):   # outputs of step t in row t % n_total (steps past the timed ones reuse rows)
        i = t % n_total
        model.step(B, k, h, qb[t % 2], db[t % 2], T, 2026, t, qb[(t + 1) % 2], db[(t + 1) % 2],
                   acc[i], tok[i], cnt[i], ws, dev_status=status, seq_offset=seq_off)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for t in range(args.warmup):
        step(t)
    barrier()
    dev_idx = os.environ.get("CUDA_VISIBLE_DEVICES", str(local)).split(",")[local]
    with ClockSampler(dev_idx) as clk:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for t in range(args.warmup, n_total):
            step(t)
        e1.record()
        e1.synchronize()
        barrier()
    clocks = clk.summary()
    ms = e0.elapsed_time(e1)
    tokens = int(cnt[args.warmup:].sum())
    st = int(status.item())
    ms_max, tokens_all = combine_over_ranks(ms, tokens, dist if world > 1 else None, "cuda")
    value = tokens_all / (ms_max / 1e3)

    # e2e: the public API with host buffers; H2D of the step's hidden states and
    # D2H of its results inside the timed region, every step.
    acc_h = torch.empty((args.steps, B), dtype=torch.int32).pin_memory()
    tok_h = torch.empty((args.steps, B, k + 1), dtype=torch.int32).pin_memory()
    cnt_h = torch.empty((args.steps, B), dtype=torch.int32).pin_memory()
    # the copy of step i + 1's hidden states runs on a second stream while step i
    # computes (two device buffers, events order the reuse), the way a serving
    # loop pipelines them; every copy and read-back still lies inside the region
    hbuf = [h, torch.empty_like(h)]
    copy_stream = torch.cuda.Stream()
    comp = torch.cuda.current_stream()
    copied = [torch.cuda.Event() for _ in range(2)]
    freed = [torch.cuda.Event() for _ in range(2)]
    barrier()
    e2, e3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2.record()
    with torch.cuda.stream(copy_stream):
        copy_stream.wait_event(e2)
        hbuf[0].copy_(h_host, non_blocking=True)
        copied[0].record(copy_stream)
    for i in range(args.steps):
        t = n_total + i
        j = i % 2
        if i + 1 < args.steps:   # next step's input into the other buffer
            with torch.cuda.stream(copy_stream):
                if i >= 1:
                    copy_stream.wait_event(freed[1 - j])
                hbuf[1 - j].copy_(h_host, non_blocking=True)
                copied[1 - j].record(copy_stream)
        comp.wait_event(copied[j])
        model.step(B, k, hbuf[j], qb[t % 2], db[t % 2], T, 2026, t, qb[(t + 1) % 2],
                   db[(t + 1) % 2], acc[i], tok[i], cnt[i], ws, dev_status=status,
                   seq_offset=seq_off)
        freed[j].record(comp)
        acc_h[i].copy_(acc[i], non_blocking=True)
        tok_h[i].copy_(tok[i], non_blocking=True)
        cnt_h[i].copy_(cnt[i], non_blocking=True)
    e3.record()
    e3.synchronize()
    e2e_ms = e2.elapsed_time(e3)
    e2e_tokens = int(cnt_h.sum())
    e2e_ms_max, e2e_tok_all = combine_over_ranks(e2e_ms, e2e_tokens, dist if world > 1 else None,
                                                  "cuda")
    # the e2e steps draw other tokens than the timed steps (other step indices), so their
    # tokens/s also moves with the accepted counts; ms_per_step shows the copies' cost
    e2e = {"value": round(e2e_tok_all / (e2e_ms_max / 1e3), 1), "unit": "tokens/s",
           "ms_per_step": round(e2e_ms_max / args.steps, 3),
           "h2d_bytes_per_step": h_host.numel() * 2,
           "d2h_bytes_per_step": (acc_h[0].numel() + tok_h[0].numel() + cnt_h[0].numel()) * 4,
           "copies": "H2D of each step's inputs on a second stream, overlapped with the "
                     "previous step; D2H of its results after it, all inside the timed region"}

    # dominant kernel: the launch of the step with the largest share of its time,
    # timed inside the step (CUDA events after every launch of a few extra steps)
    roof = None
    if rank == 0:
        roof = step_roofline(model, step, n_total + args.steps, shape, B, k, pk, pk_src)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_max / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded random-init weights and hidden states; no attention)",
        "config": workload_config(B, k, T), "clocks": clocks,
        "gpu_launches": model.kernel_count(B, k) * args.steps, "e2e": e2e, "roofline": roof,
        "mean_accepted": round(float(acc[args.warmup:n_total].float().mean()), 3),
        "device_status": st,
    }
    if world == 1 and rank == 0 and not args.no_kernels:
        # kernel lines and the B sweep (N = 1 only)
        sweep = {}
        for Bs in (1, 32, 128):
            sweep[f"B{Bs}"] = sweep_point(U, torch, W, model, Bs, k, T, V, shape)
        result["sweep_tokens_per_s"] = sweep
        del ws, qb, db
        torch.cuda.empty_cache()
        result["kernels"] = kernel_lines(U, torch, pk, with_oracle=not args.no_cpu)
    if rank == 0 and world == 1 and not args.no_cpu:
        # the oracle's time per sequence-step, over several sampled sequences, converted
        # with this run's measured tokens per sequence-step (a single sample's 1..k+1
        # tokens would otherwise dominate the ratio)
        lw_np, head_np = host_weights(layers, head, 1)
        n_samples = 6
        secs = sum(oracle_step_sample(k, lw_np, head_np, T, seed=i)[0] for i in range(n_samples))
        seq_steps_per_s = n_samples / secs
        tok_per_seq_step = tokens_all / (args.steps * B * world)
        result["cpu_baseline"] = {
            "value": round(seq_steps_per_s * tok_per_seq_step, 4), "unit": "tokens/s",
            "cores": cpu_cores(), "kind": "oracle",
            "sequence_steps_per_s": round(seq_steps_per_s, 5),
            "tokens_per_sequence_step": round(tok_per_seq_step, 3),
            "sample": f"{n_samples} sequence-steps; " + SAMPLE_TEXT + "; tokens per "
                      "sequence-step taken from this run's device-timed steps"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    model.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# (N, K) of the step's linears -> (name, groups, output width)
def linear_names(shape):
    return {(shape.q_out + 2 * shape.kv_out, shape.hidden): ("qkv", 3, shape.q_out + 2 * shape.kv_out),
            (shape.hidden, shape.q_out): ("o", 1, shape.hidden),
            (2 * shape.inter, shape.hidden): ("gate/up silu pair", 2, shape.inter),
            (shape.hidden, shape.inter): ("down", 1, shape.hidden),
            (shape.vocab, shape.hidden): ("LM head", 1, shape.vocab)}


def launch_work(shape, B, k, kind, dims):
    """Algorithmic flops and bytes of one GEMM launch of the step: x W^T over all M rows,
    the adapter (x A^T, t Bl^T) over the B k gated rows; bytes = W, A, Bl, x, y once (y
    also read when the launch adds into it), t not counted (it stays on chip or in L2)."""
    M, N, K, mode = dims
    name, G, n_out = linear_names(shape).get((N, K), ("?", 1, N))
    r, Mg = shape.r, B * k
    flops = 2 * M * N * K + 2 * Mg * r * (G * K + N)
    byts = 2 * (N * K + G * r * K + N * r + M * K + M * n_out * (2 if mode == 1 else 1))
    return name, flops, byts


def step_roofline(model, step, t0, shape, B, k, pk, pk_src, n_prof=3):
    """Roofline line of the step's dominant launch: per (kind, shape) group of launches
    the summed in-step time over n_prof profiled steps; the largest group's average launch
    time against its algorithmic work."""
    groups = {}
    model.profile(True)
    for i in range(n_prof):
        step(t0 + i)
        for kind, ms, dims in model.last_profile():
            g = groups.setdefault((kind, dims), [0.0, 0])
            g[0] += ms
            g[1] += 1
    model.profile(False)
    total = sum(v[0] for v in groups.values())
    (kind, dims), (ms_sum, n) = max(groups.items(), key=lambda kv: kv[1][0])
    us = ms_sum / n * 1e3
    name, flops, byts = launch_work(shape, B, k, kind, dims)
    tensor_bound = flops / (pk["bf16_tflops"] * 1e12) > byts / (pk["hbm_gbs"] * 1e9)
    # timed inside a long step: the sustained peak (the burst one for context)
    if tensor_bound:
        ach = flops / us / 1e6
        roof = {"bound": "tensor", "achieved": round(ach, 1), "peak": pk["bf16_tflops_sustained"],
                "unit": "TFLOP/s", "frac": round(ach / pk["bf16_tflops_sustained"], 3),
                "traffic": None, "peak_burst": pk["bf16_tflops"],
                "frac_burst": round(ach / pk["bf16_tflops"], 3)}
    else:
        ach = byts / us / 1e3
        roof = {"bound": "hbm", "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(ach / pk["hbm_gbs"], 3), "traffic": None}
    M, N, K, _ = dims
    kname = f"{kind} {name} {K}->{N} M={M}, in the step"
    roof["traffic"] = recorded_traffic(kname)
    roof.update({"kernel": kname, "us_per_launch": round(us, 2), "launches_per_step": n // n_prof,
                 "share_of_step": round(ms_sum / total, 3),
                 "timing": f"CUDA events after every launch of {n_prof} extra steps",
                 "peak_source": pk_src + (" sustained" if tensor_bound else ""),
                 "algorithmic_flops": flops, "algorithmic_bytes": byts})
    return roof


def sweep_point(U, torch, W, model, B, k, T, V, shape):
    import numpy as np
    i32 = dict(dtype=torch.int32, device="cuda")
    h = W.to_torch_bf16(W.step_hidden(B, k, shape.hidden, seed=7), "cuda")
    qb = [torch.zeros((B, k, V), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    db = [torch.zeros((B, k), **i32) for _ in range(2)]
    acc, tok, cnt = torch.empty(B, **i32), torch.empty((B, k + 1), **i32), torch.empty((8, B), **i32)
    ws = torch.empty(model.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
    step = lambda t, c: model.step(B, k, h, qb[t % 2], db[t % 2], T, 5, t, qb[(t + 1) % 2],
                                   db[(t + 1) % 2], acc, tok, c, ws)
    for t in range(3):
        step(t, cnt[0])
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(8):
        step(3 + i, cnt[i])
    b.record()
    b.synchronize()
    ms = a.elapsed_time(b)
    return {"tokens_per_s": round(int(cnt.sum()) / (ms / 1e3), 1), "ms_per_step": round(ms / 8, 3)}


def run_reference(args):
    """The fp64 CPU oracle as the reference arm, on bounded samples of the same workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import numpy as np
    import torch
    import workloads as W
    shape = W.QWEN3_8B_SHAPE
    # one layer of weights and the head, drawn by torch's seeded CPU generator
    gen = torch.Generator().manual_seed(0)
    mk = lambda n, k_, std: W.from_torch_bf16((torch.randn((n, k_), generator=gen) * std).to(torch.bfloat16))
    lw = {}
    for name, K, N in shape.linears():
        lw[name] = (mk(N, K, K ** -0.5), mk(shape.r, K, K ** -0.5), mk(N, shape.r, 0.01))
    rows = shape.vocab // HEAD_SLICE
    head = (mk(rows, shape.hidden, shape.hidden ** -0.5), mk(shape.r, shape.hidden, shape.hidden ** -0.5),
            mk(rows, shape.r, 0.01))
    for t in range(args.warmup):
        oracle_step_sample(args.k, [lw], head, args.temperature, seed=t)
    secs, exp_tok, wall = 0.0, 0.0, 0.0
    for t in range(args.steps):
        s, _, e, w = oracle_step_sample(args.k, [lw], head, args.temperature, seed=100 + t)
        secs += s
        exp_tok += e
        wall += w
    # one step = one sampled sequence-step; tokens per sequence-step = the exact mean of
    # the verification on each sample's logits (not the one draw it made)
    seq_steps_per_s = args.steps / secs
    tok_per_seq_step = exp_tok / args.steps
    value = seq_steps_per_s * tok_per_seq_step
    sample = (SAMPLE_TEXT + "; tokens per sequence-step = the expected emitted count on "
              "each sample's logits, from its acceptance probabilities")
    print(json.dumps({
        "metric": METRIC, "value": round(value, 4), "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(wall / args.steps * 1e3, 1),
        "extrapolated_s_per_sequence_step": round(secs / args.steps, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(args.B, args.k, args.temperature),
        "impl": "reference",
        "cpu_baseline": {"value": round(value, 4), "unit": "tokens/s", "cores": cpu_cores(),
                         "kind": "oracle", "sequence_steps_per_s": round(seq_steps_per_s, 5),
                         "tokens_per_sequence_step": round(tok_per_seq_step, 3),
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0}}), flush=True)


def run_profile(args):
    """A few launches of one hot kernel on a small case, for an ncu capture.

    gemm_up:    gated linear 4096 -> 12288, M = B(2k+1) rows (the step's MLP shape)
    step_up:    two steps of a 1-layer Qwen3-8B-shaped model at B (M = B(2k+1)); with
                M > 3840 each step runs 5 CTA-pair launches (qkv, o, the gate/up silu
                pair computing t itself, down, LM head): launch 7 is the second
                step's silu pair
    gemm_small: gated linear 4096 -> 4096, M = 9 (split-K cluster path)
    verify:     psi_verify B=32, k=16, V=151936 (311 MB of logits)
    draft:      draft sampler B=32, k=8, V=151936
    draft_full: draft sampler at B (default 256), k=8, V=151936 (622 MB of logits at B=256)
    gemm_down:  gated linear 12288 -> 4096, M = 2048, half the rows gated (the MLP-down
                kernel line)
    backward:   adapter gradients, MLP-up shape 4096 -> 12288, r = 128, M = 2048, half the
                rows gated (the adapter-gradient kernel line)
    """
    import torch
    import sampling_gated_lora_b200 as U
    import workloads as W
    torch.cuda.set_device(0)
    dev = lambda shape, std: (torch.randn(shape, device="cuda") * std).to(torch.bfloat16)
    if args.profile == "step_up":
        shape = dataclasses.replace(W.QWEN3_8B_SHAPE, n_layers=1)
        layers, head = W.model_weights_torch(shape, "cuda", seed=0)
        m = U.Model(layers, head, shape.hidden, shape.q_out, shape.kv_out, shape.inter,
                    shape.vocab, shape.r, shape.scale)
        B, k, V = args.B, args.k, shape.vocab
        i32 = dict(dtype=torch.int32, device="cuda")
        h = W.to_torch_bf16(W.step_hidden(B, k, shape.hidden, seed=7), "cuda")
        qb = [torch.zeros((B, k, V), dtype=torch.bfloat16, device="cuda") for _ in range(2)]
        db = [torch.zeros((B, k), **i32) for _ in range(2)]
        acc, tok, cnt = torch.empty(B, **i32), torch.empty((B, k + 1), **i32), torch.empty(B, **i32)
        ws = torch.empty(m.workspace_bytes(B, k), dtype=torch.uint8, device="cuda")
        for t in range(2):
            m.step(B, k, h, qb[t % 2], db[t % 2], 1.0, 5, t, qb[(t + 1) % 2], db[(t + 1) % 2], acc,
                   tok, cnt, ws)
        torch.cuda.synchronize()
        print(json.dumps({"profile": args.profile, "status": U.device_status(),
                          "launches_per_step": m.kernel_count(B, k)}))
        m.close()
        return
    if args.profile == "gemm_down":
        M, K, N, r = 2048, 12288, 4096, 128
        x, Wt, A, Bl = dev((M, K), 1), dev((N, K), K ** -0.5), dev((r, K), K ** -0.5), dev((N, r), 0.01)
        g = (torch.arange(M, device="cuda") >= M // 2).to(torch.uint8)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        f = lambda: U.gated_lora_linear(x, Wt, A, Bl, g, 1.0, y=y)
    elif args.profile == "backward":
        M, K, N, r = 2048, 4096, 12288, 128
        x, dy = dev((M, K), 1), dev((M, N), 1)
        A, Bl = dev((r, K), K ** -0.5), dev((N, r), 0.01)
        g = (torch.arange(M, device="cuda") >= M // 2).to(torch.uint8)
        f = lambda: U.gated_lora_adapter_grads(x, dy, A, Bl, g, 1.0)
    elif args.profile in ("gemm_up", "gemm_small"):
        M, K, N = ((args.B * (2 * args.k + 1), 4096, 12288) if args.profile == "gemm_up"
                   else (9, 4096, 4096))
        r = 128
        x, Wt, A, Bl = dev((M, K), 1), dev((N, K), K ** -0.5), dev((r, K), K ** -0.5), dev((N, r), 0.01)
        g = (torch.arange(M, device="cuda") % 2).to(torch.uint8)
        y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        f = lambda: U.gated_lora_linear(x, Wt, A, Bl, g, 1.0, y=y)
    elif args.profile == "verify":
        p, q = W.logits_case_torch(32, 16, 151936, sigma=1.0, seed=1234)
        d = U.draft_sample(q, 1.0, 99, 0)
        f = lambda: U.psi_verify(p, q, d, 1.0, 1234, 0)
    else:
        _, q = W.logits_case_torch(args.B if args.profile == "draft_full" else 32, 8, 151936,
                                   sigma=1.0, seed=1234)
        f = lambda: U.draft_sample(q, 1.0, 99, 0)
    for _ in range(4):
        f()
    torch.cuda.synchronize()
    print(json.dumps({"profile": args.profile, "status": U.device_status()}))


def main():
    args = parse()
    if args.profile:
        run_profile(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_uno(args)


if __name__ == "__main__":
    main()
