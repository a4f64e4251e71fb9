"""Seeded synthetic inputs shared by the CPU oracle, the CUDA-path tests and the bench.

This module draws random numbers and rounds them to the storage dtype. It holds
none of the method's arithmetic (no softmax, no sampling, no projection): the
oracle and the CUDA path both consume what it returns.

Distributions follow the Qwen3-8B-shaped workloads of the Psi-Spec linear
decode step (rank-128 LoRA adapters on every AR matrix: hyper.ai page, section
"实验"). Notation: "var 1/K" means a normal with variance 1/K; a decimal or an
integer means a standard deviation.

bf16 tensors are returned as uint16 bit patterns (numpy has no bf16 dtype);
`to_torch_bf16` views them as torch.bfloat16 without changing a bit.
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np

# Qwen3-8B projection shapes (hidden 4096, 8 KV heads of 128 -> 1024,
# intermediate 12288, vocab 151936), 36 decoder layers.
QWEN3_8B = dict(n_layers=36, hidden=4096, q_out=4096, kv_out=1024,
                inter=12288, vocab=151936)


# ---------------------------------------------------------------- bf16 bits

def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float32/float64 values to bf16 (round to nearest, ties to even).

    Returns the uint16 bit patterns. NaN stays NaN.
    """
    f = np.ascontiguousarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    out = rounded.astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float32 (exact)."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns to float64 (exact)."""
    return bf16_to_f32(bits).astype(np.float64)


def to_torch_bf16(bits: np.ndarray, device="cpu"):
    """View uint16 bf16 bits as a torch.bfloat16 tensor (bit-exact)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def from_torch_bf16(t) -> np.ndarray:
    """Inverse of `to_torch_bf16`: the uint16 bit patterns of a bf16 tensor."""
    import torch
    assert t.dtype == torch.bfloat16
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _rng(*key: int) -> np.random.Generator:
    return np.random.default_rng([int(v) for v in key])


def _normal(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    return rng.standard_normal(shape, dtype=np.float32) * np.float32(std)


# ---------------------------------------------------------------- linears

@dataclasses.dataclass
class GatedLinearCase:
    """One gated-LoRA linear problem: y = x W^T + s g (x A^T) Bl^T.

    dtype "bf16": arrays hold uint16 bf16 bits. dtype "f32": float32 arrays.
    Layouts are row-major: x [M,K], W [N,K], A [r,K], Bl [N,r], gate [M] uint8.
    """
    dtype: str
    x: np.ndarray
    W: np.ndarray
    A: np.ndarray
    Bl: np.ndarray
    gate: np.ndarray
    scale: float

    @property
    def M(self): return self.x.shape[0]

    @property
    def K(self): return self.x.shape[1]

    @property
    def N(self): return self.W.shape[0]

    @property
    def r(self): return self.A.shape[0]


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_round(x)
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    raise ValueError(dtype)


def gated_linear_case(M: int, K: int, N: int, r: int, gate: np.ndarray, *,
                      dtype="bf16", w_std=None, a_std=None, b_std=0.01,
                      x_std=1.0, scale=1.0, seed=0) -> GatedLinearCase:
    """Random gated-LoRA linear with the default weight law W, A ~ var 1/K."""
    rng = _rng(seed, M, K, N, r)
    w_std = (1.0 / np.sqrt(K)) if w_std is None else w_std
    a_std = (1.0 / np.sqrt(K)) if a_std is None else a_std
    gate = np.ascontiguousarray(gate, dtype=np.uint8)
    assert gate.shape == (M,)
    return GatedLinearCase(
        dtype=dtype,
        x=_store(_normal(rng, (M, K), x_std), dtype),
        W=_store(_normal(rng, (N, K), w_std), dtype),
        A=_store(_normal(rng, (r, K), a_std), dtype),
        Bl=_store(_normal(rng, (N, r), b_std), dtype),
        gate=gate, scale=float(scale))


def decode_gate(B: int, k: int) -> np.ndarray:
    """Per sequence [anchor row, gate 0] + [k draft rows, gate 1]: M = B(k+1)."""
    g = np.ones((B, k + 1), dtype=np.uint8)
    g[:, 0] = 0
    return g.reshape(-1)


def step_gate(B: int, k: int) -> np.ndarray:
    """Rows of one decode step: B(k+1) verify rows (gate 0) then B k mask rows (gate 1)."""
    return np.concatenate([np.zeros(B * (k + 1), np.uint8), np.ones(B * k, np.uint8)])


def tiny_linear_case(seed=0) -> GatedLinearCase:
    """Tiny oracle case: B=2, k=4, 256 -> 256, r=8, fp32.

    W ~ var 1/256, A and Bl ~ std 0.02, x ~ N(0,1); rows laid out as one decode
    step (2k+1 rows per sequence, gate 0 on the k+1 verify rows, 1 on the k
    mask rows), so M = 18.
    """
    B, k = 2, 4
    return gated_linear_case(B * (2 * k + 1), 256, 256, 8, step_gate(B, k), dtype="f32",
                             w_std=1 / 16, a_std=0.02, b_std=0.02, seed=seed)


def small_m_case(B: int, k=8, seed=0) -> GatedLinearCase:
    """4096 -> 4096 attention projection, r=128, bf16, M = B(k+1)."""
    return gated_linear_case(B * (k + 1), 4096, 4096, 128, decode_gate(B, k), seed=seed)


def mlp_case(which: str, B=64, k=16, seed=0) -> GatedLinearCase:
    """Concatenated clean+noisy batch M = 2Bk: gate 0 on the clean half, 1 on the noisy half.

    which = "up" (4096 -> 12288) or "down" (12288 -> 4096).
    """
    M = 2 * B * k
    g = np.concatenate([np.zeros(M // 2, np.uint8), np.ones(M // 2, np.uint8)])
    K, N = (4096, 12288) if which == "up" else (12288, 4096)
    return gated_linear_case(M, K, N, 128, g, seed=seed)


# ---------------------------------------------------------------- logits

@dataclasses.dataclass
class LogitsCase:
    """AR logits p [B,k_p,V] and draft logits q [B,k,V] (uint16 bf16 bits or float32)."""
    dtype: str
    p_logits: np.ndarray
    q_logits: np.ndarray

    @property
    def B(self): return self.p_logits.shape[0]

    @property
    def k(self): return self.q_logits.shape[1]

    @property
    def k_p(self): return self.p_logits.shape[1]

    @property
    def V(self): return self.p_logits.shape[2]


def logits_sequence(b: int, k: int, k_p: int, V: int, *, ar_std: float, sigma: float,
                    peak_frac=0.0, peak_add=12.0, seed=0, dtype="bf16"):
    """Logits of sequence b alone (so any sequence can be regenerated by itself).

    AR logits ~ N(0, ar_std); each position is peaked with probability
    peak_frac (one uniform token gets +peak_add); draft = AR + N(0, sigma).
    """
    rng = _rng(seed, b, k, k_p, V)
    ar = _normal(rng, (k_p, V), ar_std)
    if peak_frac > 0:
        peaked = rng.random(k_p) < peak_frac
        tok = rng.integers(0, V, size=k_p)
        rows = np.nonzero(peaked)[0]
        ar[rows, tok[rows]] += np.float32(peak_add)
    q = ar[:k] + _normal(rng, (k, V), sigma)
    return _store(ar, dtype), _store(q, dtype)


def logits_case(B: int, k: int, V: int, *, k_p=None, ar_std=3.0, sigma=1.0,
                peak_frac=0.05, peak_add=12.0, seed=1234, dtype="bf16",
                threads=8) -> LogitsCase:
    """Psi-Spec verify inputs; sequences are generated independently (threads)."""
    k_p = k if k_p is None else k_p
    sd = np.uint16 if dtype == "bf16" else np.float32
    p = np.empty((B, k_p, V), sd)
    q = np.empty((B, k, V), sd)

    def one(b):
        p[b], q[b] = logits_sequence(b, k, k_p, V, ar_std=ar_std, sigma=sigma,
                                     peak_frac=peak_frac, peak_add=peak_add,
                                     seed=seed, dtype=dtype)

    if threads > 1 and B > 1:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, range(B)))
    else:
        for b in range(B):
            one(b)
    return LogitsCase(dtype, p, q)


def tiny_logits_case(seed=0) -> LogitsCase:
    """Tiny oracle case: B=2, k=4, V=1024, fp32; AR ~ N(0,2), draft = AR + N(0,0.5)."""
    return logits_case(2, 4, 1024, ar_std=2.0, sigma=0.5, peak_frac=0.0,
                       seed=seed, dtype="f32", threads=1)


def verify_config_case(sigma: float, B=256, k=16, V=151936, seed=1234) -> LogitsCase:
    """Full verify workload: B=256, k=16, V=151936, AR ~ N(0,3), 5% peaked (+12)."""
    return logits_case(B, k, V, ar_std=3.0, sigma=sigma, peak_frac=0.05, seed=seed)


# ---------------------------------------------------------------- e2e model

@dataclasses.dataclass
class ModelShape:
    n_layers: int
    hidden: int
    q_out: int
    kv_out: int
    inter: int
    vocab: int
    r: int
    scale: float = 1.0

    def linears(self):
        """(name, K, N) of every gated linear in one layer, in the fixed order."""
        h, qo, kv, it = self.hidden, self.q_out, self.kv_out, self.inter
        return [("q", h, qo), ("k", h, kv), ("v", h, kv), ("o", qo, h),
                ("gate", h, it), ("up", h, it), ("down", it, h)]


QWEN3_8B_SHAPE = ModelShape(r=128, **QWEN3_8B)
TINY_SHAPE = ModelShape(n_layers=2, hidden=256, q_out=256, kv_out=64, inter=512,
                        vocab=1024, r=16)


def model_weights_np(shape: ModelShape, seed=0):
    """Per-layer dict of {name: (W, A, Bl)} bf16 bits plus ("lm_head", (W, A, Bl)).

    W ~ var 1/K, A ~ var 1/K, Bl ~ std 0.01 (host generation; small shapes only).
    """
    layers = []
    for li in range(shape.n_layers):
        d = {}
        for ni, (name, K, N) in enumerate(shape.linears()):
            rng = _rng(seed, li, ni)
            d[name] = (bf16_round(_normal(rng, (N, K), 1 / np.sqrt(K))),
                       bf16_round(_normal(rng, (shape.r, K), 1 / np.sqrt(K))),
                       bf16_round(_normal(rng, (N, shape.r), 0.01)))
        layers.append(d)
    rng = _rng(seed, shape.n_layers, 99)
    K, N = shape.hidden, shape.vocab
    head = (bf16_round(_normal(rng, (N, K), 1 / np.sqrt(K))),
            bf16_round(_normal(rng, (shape.r, K), 1 / np.sqrt(K))),
            bf16_round(_normal(rng, (N, shape.r), 0.01)))
    return layers, head


def model_weights_torch(shape: ModelShape, device, seed=0):
    """Same weight law generated by torch's seeded generator on `device` (fast at full size).

    Returns (layers, head) with torch bf16 tensors; not bit-identical to
    `model_weights_np` (a different generator), but seeded and reproducible.
    """
    import torch
    gen = torch.Generator(device=device)
    layers = []

    def normal(shape_, std, key):
        gen.manual_seed(int(seed) * 1_000_003 + key)
        t = torch.randn(shape_, generator=gen, device=device, dtype=torch.float32)
        return (t * std).to(torch.bfloat16)

    key = 0
    for li in range(shape.n_layers):
        d = {}
        for name, K, N in shape.linears():
            d[name] = (normal((N, K), 1 / np.sqrt(K), key), normal((shape.r, K), 1 / np.sqrt(K), key + 1),
                       normal((N, shape.r), 0.01, key + 2))
            key += 3
        layers.append(d)
    K, N = shape.hidden, shape.vocab
    head = (normal((N, K), 1 / np.sqrt(K), key), normal((shape.r, K), 1 / np.sqrt(K), key + 1),
            normal((N, shape.r), 0.01, key + 2))
    return layers, head


def step_hidden(B: int, k: int, hidden: int, seed=0) -> np.ndarray:
    """Input hidden states of one step, [B(k+1) + Bk, hidden] bf16 bits.

    Rows: B(k+1) verify rows (sequence-major: anchor then k drafted tokens),
    then Bk mask rows. The k mask rows of a sequence take the same vectors as
    its k drafted-token rows, so p and q differ only through the adapter; the
    anchor row has its own vector.
    """
    rng = _rng(seed, B, k, hidden)
    verify = _normal(rng, (B, k + 1, hidden), 1.0)
    mask = verify[:, 1:, :]
    h = np.concatenate([verify.reshape(-1, hidden), mask.reshape(-1, hidden)], axis=0)
    return bf16_round(h)


def draft_ids(B: int, k: int, V: int, seed=0) -> np.ndarray:
    """Uniform draft token ids [B,k] int32 (for shape-only uses, e.g. the first step)."""
    return _rng(seed, B, k, V).integers(0, V, size=(B, k), dtype=np.int32)


def logits_case_torch(B: int, k: int, V: int, *, k_p=None, ar_std=3.0, sigma=1.0,
                      peak_frac=0.05, peak_add=12.0, seed=1234, device="cuda", chunk=32):
    """Same recipe as `logits_case`, drawn by torch's seeded generator on `device`.

    For full-size workloads (B=256, k=16, V=151936 is 1.24e9 normals), where
    host generation takes minutes. Returns bf16 tensors (p [B,k_p,V], q [B,k,V]);
    tests copy the rows they check back to the host.
    """
    import torch
    k_p = k if k_p is None else k_p
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed) * 7919 + int(round(sigma * 1000)))
    p = torch.empty((B, k_p, V), dtype=torch.bfloat16, device=device)
    q = torch.empty((B, k, V), dtype=torch.bfloat16, device=device)
    for b0 in range(0, B, chunk):
        nb = min(chunk, B - b0)
        ar = torch.randn((nb, k_p, V), generator=gen, device=device) * ar_std
        if peak_frac > 0:
            peaked = torch.rand((nb, k_p), generator=gen, device=device) < peak_frac
            tok = torch.randint(0, V, (nb, k_p), generator=gen, device=device)
            bump = torch.zeros((nb, k_p, V), device=device)
            bump.scatter_(2, tok.unsqueeze(-1), (peaked.float() * peak_add).unsqueeze(-1))
            ar += bump
        noise = torch.randn((nb, k, V), generator=gen, device=device) * sigma
        p[b0:b0 + nb] = ar.to(torch.bfloat16)
        q[b0:b0 + nb] = (ar[:, :k] + noise).to(torch.bfloat16)
    return p, q
