"""Helpers for the GPU parity tests: device transfer, tolerances, verify comparison.

The oracle sees only seeded inputs (from `workloads`, or drawn by the oracle
itself); it never consumes a value produced by the CUDA path.
"""
import numpy as np

import workloads as W

# Gated-linear tolerances (bf16 inputs, fp32 accumulation, bf16 output; the
# tf32 path of the fp32 case meets the same bounds).
REL_FROB = 5e-3
MAX_ABS = 3e-2
# Verify: a decision may differ only where the fp64 oracle is within these of a
# tie: |u - p/q| < TIE_U at the accept test, or the draw threshold within
# TIE_CDF (relative to the total weight) of a CDF edge.
TIE_U = 1e-4
TIE_CDF = 1e-5
EXCUSED_CAP = 1e-4   # excused positions / all positions, at full size


def api_T(T):
    """The temperature as the library receives it: the C ABI takes an IEEE float32,
    so the oracle is given that same value (0.7 becomes 0.699999988...)."""
    return float(np.float32(T))


def torch_mod():
    import torch
    return torch


def dev_tensor(a, dtype):
    """Host array -> CUDA tensor. dtype "bf16" takes uint16 bit patterns."""
    torch = torch_mod()
    if dtype == "bf16":
        return W.to_torch_bf16(a, "cuda")
    if dtype == "f32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    if dtype == "u8":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()
    if dtype == "i32":
        return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
    raise ValueError(dtype)


def host_f64(t):
    torch = torch_mod()
    if t.dtype == torch.bfloat16:
        return W.bf16_to_f64(W.from_torch_bf16(t))
    return t.detach().cpu().double().numpy()


def case_to_f64(a, dtype):
    return W.bf16_to_f64(a) if dtype == "bf16" else np.asarray(a, dtype=np.float64)


def check_close(y, ref, rel=REL_FROB, max_abs=MAX_ABS, what="", rel_elem=0.0):
    """rel-Frobenius <= rel and |y - ref| <= max_abs + rel_elem |ref| elementwise."""
    err = y - ref
    rf = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-30)
    excess = (np.abs(err) - rel_elem * np.abs(ref)).max() if err.size else 0.0
    assert rf <= rel and excess <= max_abs, f"{what}: rel-Frobenius {rf:.3e}, max-abs excess {excess:.3e}"
    return rf, excess


def compare_verify(gpu, ora, k, sequences):
    """Compare GPU verify outputs with the oracle's on the given sequences.

    gpu: (accepted_len, out_tokens, out_count) numpy arrays; ora: oracle
    psi_verify result. Returns (excused, unexcused) lists of sequence ids.
    """
    acc_g, tok_g, cnt_g = gpu
    excused, bad = [], []
    for b in sequences:
        d = ora["diags"][b]
        n_o, n_g = int(ora["accepted_len"][b]), int(acc_g[b])
        same = (n_o == n_g and int(ora["out_count"][b]) == int(cnt_g[b])
                and np.array_equal(ora["out_tokens"][b], tok_g[b]))
        if same:
            continue
        if n_o != n_g:
            j = min(n_o, n_g)
            ok = j < k and np.isfinite(d["ratio"][j]) and abs(d["u_accept"][j] - d["ratio"][j]) < TIE_U
        else:
            ok = (d["draw_margin"] is not None and d["draw_margin"] < TIE_CDF
                  and np.array_equal(ora["out_tokens"][b][:n_o], tok_g[b][:n_o]))
        (excused if ok else bad).append(b)
    return excused, bad


def check_verify_outputs_valid(acc, tok, cnt, draft, k, k_p, V):
    """Properties every verify output has, at any size."""
    B = acc.shape[0]
    assert np.all((acc >= 0) & (acc <= k))
    has_draw = (acc < k) | (k_p == k + 1)
    np.testing.assert_array_equal(cnt, acc + has_draw.astype(np.int32))
    for b in range(B):
        n, c = int(acc[b]), int(cnt[b])
        np.testing.assert_array_equal(tok[b, :n], draft[b, :n])
        assert np.all(tok[b, c:] == -1)
        assert np.all((tok[b, :c] >= 0) & (tok[b, :c] < V))


def compare_drafts(gpu, q_logits, T, seed, step, seq_offset=0):
    """GPU drafts [B,k] against the oracle's draft sampler on the same logits.

    A differing draw is excused only where the oracle's threshold u * Z lies within
    TIE_CDF (relative to Z) of an edge of its token's CDF interval. Returns
    (number excused, list of unexcused (b, j)).
    """
    from oracle import philox
    from oracle import sampling as S
    q = S.as_f64(q_logits)
    o = S.draft_sample(q, T, seed, step, seq_offset)
    bad, excused = [], 0
    for b, j in np.argwhere(np.asarray(gpu) != o):
        idx = (int(b) + seq_offset) * q.shape[1] + int(j)
        u = philox.uniform_scalar(seed, step, philox.STREAM_DRAFT, idx)
        margin = S.cdf_margin(S.softmax_t(q[b, j], T), u, int(o[b, j]))
        if margin < TIE_CDF:
            excused += 1
        else:
            bad.append((int(b), int(j)))
    return excused, bad
