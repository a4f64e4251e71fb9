"""Python binding of libuno.so — the sm_100a Psi-Spec linear decode step.

Argument marshalling only: every operation runs in the library's CUDA kernels
(include/uno.h). PyTorch supplies device memory and streams. There is no CPU
fallback: if libuno.so is missing or cannot load, every call raises.

Functions mirror the C ABI:
    gated_lora_linear  y = x W^T + s g (x A^T) Bl^T
    psi_verify         accept u q(d) < p(d), longest prefix, residual / bonus draw
    draft_sample       linear-sampler draft from softmax(q / T)
    philox_uniforms    the generator's words and uniforms, for bit-exact checks
    rmsnorm, silu_mul  the step's glue operations
    Model              synthetic decoder stack + LM head; Model.step = uno_psi_step
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libuno.so")

UNO_BF16, UNO_F32 = 0, 1
DEV_BAD_DRAFT, DEV_NAN, DEV_TIMEOUT = 1, 2, 4
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "UNSUPPORTED", 3: "CUDA", 4: "TIMEOUT",
                5: "DEVICE_FLAG", 6: "WORKSPACE"}

EXPORTS = [
    "uno_last_error", "uno_version", "uno_device_status",
    "uno_gated_lora_linear_workspace", "uno_gated_lora_linear",
    "uno_gated_lora_linear_group_workspace", "uno_gated_lora_linear_group",
    "uno_gated_lora_backward_workspace", "uno_gated_lora_backward",
    "uno_psi_verify_workspace", "uno_psi_verify", "uno_psi_verify_noalloc",
    "uno_draft_sample_workspace", "uno_draft_sample", "uno_distill",
    "uno_tree_verify_workspace", "uno_tree_verify",
    "uno_philox_uniforms",
    "uno_model_create", "uno_model_destroy", "uno_psi_step_workspace", "uno_psi_step",
    "uno_psi_step_hidden", "uno_psi_step_kernel_count", "uno_model_profile",
    "uno_model_last_profile",
    "uno_rmsnorm", "uno_silu_mul", "uno_wait_selftest",
    "uno_vp_partials", "uno_vp_verify_decide", "uno_vp_draw_masses", "uno_vp_draw",
    "uno_vp_draft_draw",
]


class UnoError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


_lib = None


def load():
    """Load libuno.so (raises if it is missing or broken)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m sampling_gated_lora_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u32, u64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64,
                                       ctypes.c_uint32, ctypes.c_uint64, ctypes.c_float,
                                       ctypes.c_size_t)
    sig = {
        "uno_last_error": (ctypes.c_char_p, []),
        "uno_version": (ctypes.c_char_p, []),
        "uno_device_status": (i32, [vp, i32, vp]),
        "uno_gated_lora_linear_workspace": (sz, [i32, i64, i64, i64, i32]),
        "uno_gated_lora_linear": (i32, [i32, i64, i64, i64, i32, vp, vp, vp, vp, vp, f32, vp, vp,
                                        sz, vp]),
        "uno_gated_lora_linear_group_workspace": (sz, [i32, i64, i32, i32]),
        "uno_gated_lora_linear_group": (i32, [i32, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp, f32,
                                              i32, vp, vp, sz, vp]),
        "uno_gated_lora_backward_workspace": (sz, [i64, i64, i64, i32]),
        "uno_gated_lora_backward": (i32, [i32, i64, i64, i64, i32, vp, vp, vp, vp, vp, f32, vp,
                                          vp, vp, sz, vp]),
        "uno_psi_verify_workspace": (sz, [i32, i32, i32, i32]),
        "uno_psi_verify": (i32, [i32, i32, i32, i32, i32, vp, vp, vp, f32, u64, u64, u64, vp, vp,
                                 vp, vp, vp, sz, vp]),
        "uno_psi_verify_noalloc": (i32, [i32, i32, i32, i32, i32, vp, vp, vp, f32, u64, u64, u64,
                                         vp, vp, vp, vp, vp]),
        "uno_draft_sample_workspace": (sz, [i32, i32, i32]),
        "uno_tree_verify_workspace": (sz, [i32, i32, i32, i32, i32]),
        "uno_tree_verify": (i32, [i32, i32, i32, i32, i32, i32, vp, vp, vp, i32, f32, u64, u64, u64,
                                  vp, vp, vp, vp, vp, sz, vp]),
        "uno_distill": (i32, [i32, i32, i32, vp, vp, f32, f32, f32, vp, vp, vp, vp]),
        "uno_draft_sample": (i32, [i32, i32, i32, i32, vp, f32, u64, u64, u64, vp, vp, vp, sz, vp]),
        "uno_philox_uniforms": (i32, [u64, u64, u32, u32, i64, vp, vp, vp]),
        "uno_model_create": (i32, [vp, i32, i32, i32, i32, i32, i32, i32, f32, vp]),
        "uno_model_destroy": (None, [vp]),
        "uno_psi_step_workspace": (sz, [vp, i32, i32]),
        "uno_psi_step": (i32, [vp, i32, i32, vp, vp, vp, f32, u64, u64, u64, vp, vp, vp, vp, vp,
                               vp, vp, vp, sz, vp]),
        "uno_psi_step_hidden": (i32, [vp, i32, i32, vp, i32, vp, vp, vp, vp, vp, vp, sz, vp]),
        "uno_psi_step_kernel_count": (i32, [vp, i32, i32]),
        "uno_model_profile": (i32, [vp, i32]),
        "uno_model_last_profile": (i32, [vp, i32, vp, vp, vp, vp]),
        "uno_rmsnorm": (i32, [i64, i64, vp, vp, f32, vp]),
        "uno_silu_mul": (i32, [i64, vp, vp, vp, vp]),
        "uno_wait_selftest": (i32, [i32, u64, vp, vp, vp]),
        "uno_vp_partials": (i32, [i32, i32, i32, i32, vp, vp, i32, i32, i32, i32, f32, vp, vp]),
        "uno_vp_verify_decide": (i32, [i32, i32, i32, i32, i32, vp, vp, vp, f32, u64, u64, u64,
                                       vp, vp, vp, vp, vp, vp, vp]),
        "uno_vp_draw_masses": (i32, [i32, i32, i32, i32, i32, vp, vp, vp, vp, f32, vp, vp]),
        "uno_vp_draw": (i32, [i32, i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, f32,
                              u64, u64, u64, vp, vp]),
        "uno_vp_draft_draw": (i32, [i32, i32, i32, i32, i32, i32, i32, i32, vp, vp, f32, u64, u64,
                                    u64, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def version() -> str:
    return load().uno_version().decode()


def _check(st: int):
    if st != 0:
        raise UnoError(st, load().uno_last_error().decode())


# ---------------------------------------------------------------- marshalling helpers

def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream, device=None):
    """cudaStream_t of `stream` (default: the current stream of `device`); an
    explicit stream must belong to `device`."""
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    elif device is not None and stream.device != device:
        raise ValueError(f"stream is on {stream.device}, the tensors on {device}")
    return ctypes.c_void_p(stream.cuda_stream)


def _launch(device, stream, cfn, *args):
    """Call library function `cfn(*args, stream)` with `device` current, so the
    library's device queries and launches address the device that holds the
    tensors; raise on a non-OK status."""
    torch = _torch()
    with torch.cuda.device(device):
        _check(cfn(*args, _stream(stream, device)))


def _dtype(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return UNO_BF16
    if t.dtype == torch.float32:
        return UNO_F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _dev(*ts):
    """Check that the tensors are contiguous and all on one CUDA device; return it."""
    device = None
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")
            if device is None:
                device = t.device
            elif t.device != device:
                raise ValueError(f"tensors on {device} and {t.device}: one device per call")
    return device


def _expect(t, shape, dtypes, name, optional=False):
    """Check that tensor `t` has `shape` (None entries match any size) and one of
    `dtypes` before any pointer reaches the library: the C ABI takes sizes from
    a few arguments only, so a smaller buffer elsewhere would be read past its end."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if t.dim() != len(shape) or any(d is not None and t.shape[i] != d for i, d in enumerate(shape)):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {tuple(dtypes)}")


def _floats():
    torch = _torch()
    return (torch.bfloat16, torch.float32)


def _workspace(nbytes, device, workspace):
    torch = _torch()
    if nbytes == 0:
        return None, 0
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
    return workspace, workspace.numel() * workspace.element_size()


# ---------------------------------------------------------------- operations

def gated_lora_linear(x, W, A, Bl, gate, scale=1.0, y=None, workspace=None, stream=None):
    """y [M,N] = x W^T + scale * gate (x A^T) Bl^T (bf16 or f32 tensors, uint8 gate)."""
    torch = _torch()
    _expect(x, (None, None), _floats(), "x")
    M, K = x.shape
    _expect(W, (None, K), (x.dtype,), "W")
    N = W.shape[0]
    r = A.shape[0] if A is not None else 0
    _expect(A, (r, K), (x.dtype,), "A", optional=r == 0)
    _expect(Bl, (N, r), (x.dtype,), "Bl", optional=r == 0)
    _expect(gate, (M,), (torch.uint8,), "gate", optional=r == 0)
    _expect(y, (M, N), (x.dtype,), "y", optional=True)
    L = load()
    if y is None:
        y = torch.empty((M, N), dtype=x.dtype, device=x.device)
    dev = _dev(x, W, A, Bl, gate, y, workspace)
    dt = _dtype(x)
    need = L.uno_gated_lora_linear_workspace(dt, M, K, N, r)
    ws, wsb = _workspace(need, dev, workspace)
    _launch(dev, stream, L.uno_gated_lora_linear, dt, M, K, N, r, _ptr(x), _ptr(W), _ptr(A),
            _ptr(Bl), _ptr(gate), float(scale), _ptr(y), _ptr(ws), wsb)
    return y


def gated_lora_linear_group(x, Ws, As, Bls, gate, scale=1.0, silu_pair=False, ys=None,
                            workspace=None, stream=None):
    """Up to three gated linears on one input x; silu_pair: y = silu(lin_0(x)) * lin_1(x).

    Returns the list of outputs ([y] in silu-pair mode).
    """
    torch = _torch()
    _expect(x, (None, None), _floats(), "x")
    M, K = x.shape
    G = len(Ws)
    if not 1 <= G <= 3:
        raise ValueError(f"1 to 3 linears per call, got {G}")
    r = As[0].shape[0] if As else 0
    if r > 0 and (len(As) != G or len(Bls) != G):
        raise ValueError("As and Bls need one entry per linear")
    Ns = []
    for i, w in enumerate(Ws):
        _expect(w, (None, K), (x.dtype,), f"Ws[{i}]")
        Ns.append(w.shape[0])
        if r > 0:
            _expect(As[i], (r, K), (x.dtype,), f"As[{i}]")
            _expect(Bls[i], (Ns[i], r), (x.dtype,), f"Bls[{i}]")
    _expect(gate, (M,), (torch.uint8,), "gate", optional=r == 0)
    if ys is not None:
        outs = Ns[:1] if silu_pair else Ns
        if len(ys) != len(outs):
            raise ValueError(f"ys needs {len(outs)} outputs")
        for i, (yt, n) in enumerate(zip(ys, outs)):
            _expect(yt, (M, n), (x.dtype,), f"ys[{i}]")
    L = load()
    if ys is None:
        ys = [torch.empty((M, n), dtype=x.dtype, device=x.device) for n in (Ns[:1] if silu_pair else Ns)]
    dev = _dev(x, gate, *Ws, *As, *Bls, *ys, workspace)
    dt = _dtype(x)
    need = L.uno_gated_lora_linear_group_workspace(dt, M, r, G)
    ws, wsb = _workspace(need, dev, workspace)
    arr = lambda ts: (ctypes.c_void_p * G)(*[t.data_ptr() for t in ts])
    yarr = (ctypes.c_void_p * G)(*[ys[min(i, len(ys) - 1)].data_ptr() for i in range(G)])
    Narr = (ctypes.c_int64 * G)(*Ns)
    _launch(dev, stream, L.uno_gated_lora_linear_group, dt, M, K, r, G, Narr, _ptr(x), arr(Ws),
            arr(As), arr(Bls), _ptr(gate), float(scale), 1 if silu_pair else 0, yarr, _ptr(ws),
            wsb)
    return ys


def gated_lora_adapter_grads(x, dy, A, Bl, gate, scale=1.0, dA=None, dBl=None, workspace=None,
                             stream=None):
    """(dA [r,K], dBl [N,r]) of sum(dy * y) for y = gated_lora_linear(x, W, A, Bl, gate, scale),
    the AR weight W frozen (bf16 tensors, uint8 gate)."""
    torch = _torch()
    bf16 = (torch.bfloat16,)
    _expect(x, (None, None), bf16, "x")
    M, K = x.shape
    _expect(A, (None, K), bf16, "A")
    r = A.shape[0]
    _expect(Bl, (None, r), bf16, "Bl")
    N = Bl.shape[0]
    _expect(dy, (M, N), bf16, "dy")
    _expect(gate, (M,), (torch.uint8,), "gate")
    _expect(dA, (r, K), bf16, "dA", optional=True)
    _expect(dBl, (N, r), bf16, "dBl", optional=True)
    L = load()
    dA = torch.empty((r, K), dtype=torch.bfloat16, device=x.device) if dA is None else dA
    dBl = torch.empty((N, r), dtype=torch.bfloat16, device=x.device) if dBl is None else dBl
    dev = _dev(x, dy, A, Bl, gate, dA, dBl, workspace)
    ws, wsb = _workspace(L.uno_gated_lora_backward_workspace(M, K, N, r), dev, workspace)
    _launch(dev, stream, L.uno_gated_lora_backward, UNO_BF16, M, K, N, r, _ptr(x), _ptr(dy),
            _ptr(A), _ptr(Bl), _ptr(gate), float(scale), _ptr(dA), _ptr(dBl), _ptr(ws), wsb)
    return dA, dBl


def _verify_shapes(p_logits, q_logits, draft, accepted_len, out_tokens, out_count, dev_status):
    torch = _torch()
    _expect(p_logits, (None, None, None), _floats(), "p_logits")
    B, k_p, V = p_logits.shape
    _expect(q_logits, (B, None, V), (p_logits.dtype,), "q_logits")
    k = q_logits.shape[1]
    _expect(draft, (B, k), (torch.int32,), "draft")
    _expect(accepted_len, (B,), (torch.int32,), "accepted_len", optional=True)
    _expect(out_tokens, (B, k + 1), (torch.int32,), "out_tokens", optional=True)
    _expect(out_count, (B,), (torch.int32,), "out_count", optional=True)
    _expect(dev_status, (1,), (torch.int32,), "dev_status", optional=True)
    return B, k, k_p, V


def psi_verify(p_logits, q_logits, draft, temperature, seed, step, seq_offset=0,
               accepted_len=None, out_tokens=None, out_count=None, dev_status=None,
               workspace=None, stream=None):
    """Verify one block per sequence; returns (accepted_len [B], out_tokens [B,k+1], out_count [B])."""
    torch = _torch()
    B, k, k_p, V = _verify_shapes(p_logits, q_logits, draft, accepted_len, out_tokens, out_count,
                                  dev_status)
    L = load()
    dev = p_logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    accepted_len = torch.empty(B, **i32) if accepted_len is None else accepted_len
    out_tokens = torch.empty((B, k + 1), **i32) if out_tokens is None else out_tokens
    out_count = torch.empty(B, **i32) if out_count is None else out_count
    _dev(p_logits, q_logits, draft, accepted_len, out_tokens, out_count, dev_status, workspace)
    need = L.uno_psi_verify_workspace(B, k, k_p, V)
    ws, wsb = _workspace(need, dev, workspace)
    _launch(dev, stream, L.uno_psi_verify, _dtype(p_logits), B, k, k_p, V, _ptr(p_logits),
            _ptr(q_logits), _ptr(draft), float(temperature), int(seed), int(step),
            int(seq_offset), _ptr(accepted_len), _ptr(out_tokens), _ptr(out_count),
            _ptr(dev_status), _ptr(ws), wsb)
    return accepted_len, out_tokens, out_count


def psi_verify_noalloc(p_logits, q_logits, draft, temperature, seed, step, seq_offset=0,
                       accepted_len=None, out_tokens=None, out_count=None, dev_status=None,
                       stream=None):
    """psi_verify with the library's static stats scratch (no workspace argument)."""
    torch = _torch()
    B, k, k_p, V = _verify_shapes(p_logits, q_logits, draft, accepted_len, out_tokens, out_count,
                                  dev_status)
    L = load()
    dev = p_logits.device
    i32 = dict(dtype=torch.int32, device=dev)
    accepted_len = torch.empty(B, **i32) if accepted_len is None else accepted_len
    out_tokens = torch.empty((B, k + 1), **i32) if out_tokens is None else out_tokens
    out_count = torch.empty(B, **i32) if out_count is None else out_count
    _dev(p_logits, q_logits, draft, accepted_len, out_tokens, out_count, dev_status)
    _launch(dev, stream, L.uno_psi_verify_noalloc, _dtype(p_logits), B, k, k_p, V,
            _ptr(p_logits), _ptr(q_logits), _ptr(draft), float(temperature), int(seed),
            int(step), int(seq_offset), _ptr(accepted_len), _ptr(out_tokens), _ptr(out_count),
            _ptr(dev_status))
    return accepted_len, out_tokens, out_count


def tree_verify(p_nodes, q_logits, cands, temperature, seed, step, seq_offset=0, bonus=False,
                accepted_len=None, out_tokens=None, out_count=None, dev_status=None,
                workspace=None, stream=None):
    """Tree-sampler verification; returns (accepted_len [B], out_tokens [B,k+1], out_count [B]).

    p_nodes [B,R,V]: AR logits of every trie node of each sequence's candidates
    (numbered in order of first visit, candidates walked in index order);
    q_logits [B,k,V]; cands [B,N,k] int32.
    """
    torch = _torch()
    _expect(p_nodes, (None, None, None), _floats(), "p_nodes")
    B, R, V = p_nodes.shape
    _expect(q_logits, (B, None, V), (p_nodes.dtype,), "q_logits")
    k = q_logits.shape[1]
    _expect(cands, (B, None, k), (torch.int32,), "cands")
    N = cands.shape[1]
    _expect(accepted_len, (B,), (torch.int32,), "accepted_len", optional=True)
    _expect(out_tokens, (B, k + 1), (torch.int32,), "out_tokens", optional=True)
    _expect(out_count, (B,), (torch.int32,), "out_count", optional=True)
    _expect(dev_status, (1,), (torch.int32,), "dev_status", optional=True)
    L = load()
    dev = p_nodes.device
    i32 = dict(dtype=torch.int32, device=dev)
    accepted_len = torch.empty(B, **i32) if accepted_len is None else accepted_len
    out_tokens = torch.empty((B, k + 1), **i32) if out_tokens is None else out_tokens
    out_count = torch.empty(B, **i32) if out_count is None else out_count
    _dev(p_nodes, q_logits, cands, accepted_len, out_tokens, out_count, dev_status)
    need = L.uno_tree_verify_workspace(B, N, k, R, V)
    ws, wsb = _workspace(need, dev, workspace)
    _check(L.uno_tree_verify(_dtype(p_nodes), B, N, k, R, V, _ptr(p_nodes), _ptr(q_logits),
                             _ptr(cands), 1 if bonus else 0, float(temperature), int(seed),
                             int(step), int(seq_offset), _ptr(accepted_len), _ptr(out_tokens),
                             _ptr(out_count), _ptr(dev_status), _ptr(ws), wsb, _stream(stream)))
    return accepted_len, out_tokens, out_count


def distill(z_teacher, z_student, alpha=1.0, beta=1.0, temperature=1.0, grad=True, losses=None,
            grad_out=None, dev_status=None, stream=None):
    """Per-row (KL(p||q), TV(p,q)) [rows,2] and, if `grad`, d(alpha mean KL + beta mean TV)/d z_student.

    Returns (losses, grad or None).
    """
    torch = _torch()
    _expect(z_teacher, (None, None), _floats(), "z_teacher")
    rows, V = z_teacher.shape
    _expect(z_student, (rows, V), (z_teacher.dtype,), "z_student")
    _expect(losses, (rows, 2), (torch.float32,), "losses", optional=True)
    _expect(grad_out, (rows, V), (torch.float32,), "grad_out", optional=True)
    _expect(dev_status, (1,), (torch.int32,), "dev_status", optional=True)
    L = load()
    dev = z_teacher.device
    losses = torch.empty((rows, 2), dtype=torch.float32, device=dev) if losses is None else losses
    if grad and grad_out is None:
        grad_out = torch.empty((rows, V), dtype=torch.float32, device=dev)
    g = grad_out if grad else None
    _dev(z_teacher, z_student, losses, g, dev_status)
    _check(L.uno_distill(_dtype(z_teacher), rows, V, _ptr(z_teacher), _ptr(z_student),
                         float(alpha), float(beta), float(temperature), _ptr(losses), _ptr(g),
                         _ptr(dev_status), _stream(stream)))
    return losses, g


def draft_sample(q_logits, temperature, seed, step, seq_offset=0, draft=None, dev_status=None,
                 workspace=None, stream=None):
    """Linear-sampler draft: draft [B,k] int32 from softmax(q_logits / T)."""
    torch = _torch()
    _expect(q_logits, (None, None, None), _floats(), "q_logits")
    B, k, V = q_logits.shape
    _expect(draft, (B, k), (torch.int32,), "draft", optional=True)
    _expect(dev_status, (1,), (torch.int32,), "dev_status", optional=True)
    L = load()
    draft = torch.empty((B, k), dtype=torch.int32, device=q_logits.device) if draft is None else draft
    dev = _dev(q_logits, draft, dev_status, workspace)
    ws, wsb = _workspace(L.uno_draft_sample_workspace(B, k, V), dev, workspace)
    _launch(dev, stream, L.uno_draft_sample, _dtype(q_logits), B, k, V, _ptr(q_logits),
            float(temperature), int(seed), int(step), int(seq_offset), _ptr(draft),
            _ptr(dev_status), _ptr(ws), wsb)
    return draft


def philox_uniforms(seed, step, stream_id, index0, n, device="cuda", stream=None):
    """(words uint32 as int64 tensor, u float32) of Philox word 0 at indices index0..index0+n-1."""
    torch = _torch()
    L = load()
    words = torch.empty(n, dtype=torch.int32, device=device)
    u = torch.empty(n, dtype=torch.float32, device=device)
    _launch(words.device, stream, L.uno_philox_uniforms, int(seed), int(step), int(stream_id),
            int(index0), int(n), _ptr(words), _ptr(u))
    return words.to(torch.int64) & 0xFFFFFFFF, u


def rmsnorm(x, eps=1e-6, y=None, stream=None):
    torch = _torch()
    _expect(x, (None, None), (torch.bfloat16,), "x")
    _expect(y, tuple(x.shape), (torch.bfloat16,), "y", optional=True)
    L = load()
    y = torch.empty_like(x) if y is None else y
    dev = _dev(x, y)
    M, D = x.shape
    _launch(dev, stream, L.uno_rmsnorm, M, D, _ptr(x), _ptr(y), float(eps))
    return y


def silu_mul(a, b, y=None, stream=None):
    torch = _torch()
    _expect(a, tuple(a.shape), (torch.bfloat16,), "a")
    _expect(b, tuple(a.shape), (torch.bfloat16,), "b")
    _expect(y, tuple(a.shape), (torch.bfloat16,), "y", optional=True)
    L = load()
    y = torch.empty_like(a) if y is None else y
    dev = _dev(a, b, y)
    _launch(dev, stream, L.uno_silu_mul, a.numel(), _ptr(a), _ptr(b), _ptr(y))
    return y


def wait_selftest(which, limit_ns=1_000_000, dev_status=None, device="cuda", stream=None):
    """uno_wait_selftest: one bounded wait (0 flag, 1 mbarrier, 2 cluster-scope mbarrier,
    3 control) on a condition nothing satisfies; returns the device result word
    (1 satisfied, 0 gave up)."""
    torch = _torch()
    L = load()
    result = torch.full((1,), -1, dtype=torch.int32, device=device)
    dev = _dev(result, dev_status)
    _launch(dev, stream, L.uno_wait_selftest, int(which), int(limit_ns), _ptr(result),
            _ptr(dev_status))
    return result


def device_status(clear=True, stream=None, device=None) -> int:
    """The library-wide device status bits (UNO_DEV_*) of `device` (default: the
    current device), optionally cleared."""
    torch = _torch()
    L = load()
    v = ctypes.c_int32(0)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _launch(dev, stream, L.uno_device_status, ctypes.byref(v), 1 if clear else 0)
    return v.value


LINEAR_NAMES = ("q", "k", "v", "o", "gate", "up", "down")


class Model:
    """Handle over caller-owned bf16 weights of the synthetic decoder stack.

    layers: list of dicts name -> (W, A, Bl) for the names in LINEAR_NAMES;
    head: (W, A, Bl) of the LM head. The tensors must stay alive with the model.
    """

    def __init__(self, layers, head, hidden, q_out, kv_out, inter, vocab, r, scale=1.0):
        torch = _torch()
        # (out, in) of every linear, in LINEAR_NAMES order
        dims = {"q": (q_out, hidden), "k": (kv_out, hidden), "v": (kv_out, hidden),
                "o": (hidden, q_out), "gate": (inter, hidden), "up": (inter, hidden),
                "down": (hidden, inter)}
        bf16 = (torch.bfloat16,)

        def check(parts, n_out, n_in, name):
            if len(parts) != 3:
                raise ValueError(f"{name}: expected (W, A, Bl)")
            _expect(parts[0], (n_out, n_in), bf16, f"{name} W")
            _expect(parts[1], (r, n_in), bf16, f"{name} A", optional=r == 0)
            _expect(parts[2], (n_out, r), bf16, f"{name} Bl", optional=r == 0)

        for li, lw in enumerate(layers):
            for name in LINEAR_NAMES:
                check(lw[name], *dims[name], f"layer {li} {name}")
        check(head, vocab, hidden, "head")
        L = load()
        self._keep = (layers, head)
        ptrs = []
        tensors = [t for parts in [lw[name] for lw in layers for name in LINEAR_NAMES] + [head]
                   for t in parts]
        self.device = _dev(*tensors)
        for t in tensors:
            ptrs.append(None if t is None else t.data_ptr())
        arr = (ctypes.c_void_p * len(ptrs))(*ptrs)
        h = ctypes.c_void_p()
        _check(L.uno_model_create(ctypes.byref(h), len(layers), hidden, q_out, kv_out, inter,
                                  vocab, r, float(scale), arr))
        self._h = h
        self.n_layers, self.hidden, self.vocab, self.r = len(layers), hidden, vocab, r
        self.q_out, self.kv_out, self.inter = q_out, kv_out, inter

    def close(self):
        if getattr(self, "_h", None) is not None and self._h.value:
            load().uno_model_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def workspace_bytes(self, B, k):
        return load().uno_psi_step_workspace(self._h, B, k)

    def kernel_count(self, B, k):
        """Kernel launches issued by one step for (B, k) (0 before the first such step)."""
        return load().uno_psi_step_kernel_count(self._h, B, k)

    PROFILE_KINDS = {0: "gemm_one_cta", 1: "gemm_pair", 2: "gemm_pair_computes_t",
                     3: "gemm_decode", 10: "rmsnorm", 11: "rmsnorm_down", 12: "row_sumsq", 20: "verify",
                     21: "draft"}

    def profile(self, enable=True):
        """uno_model_profile: time every launch of the following steps with CUDA events."""
        _check(load().uno_model_profile(self._h, 1 if enable else 0))

    def last_profile(self):
        """uno_model_last_profile: [(kind name, ms, (M, N, K, mode))] of the last profiled step,
        in launch order (waits for that step)."""
        L = load()
        n = ctypes.c_int32(0)
        _check(L.uno_model_last_profile(self._h, 0, None, None, None, ctypes.byref(n)))
        cap = n.value
        if cap == 0:
            return []
        ms = (ctypes.c_float * cap)()
        kind = (ctypes.c_int32 * cap)()
        dims = (ctypes.c_int64 * (4 * cap))()
        _check(L.uno_model_last_profile(self._h, cap, ms, kind, dims, ctypes.byref(n)))
        return [(self.PROFILE_KINDS.get(kind[i], str(kind[i])), float(ms[i]),
                 tuple(int(d) for d in dims[4 * i: 4 * i + 4])) for i in range(n.value)]

    def hidden_state(self, B, k, h_in, n_blocks, workspace, h_out=None, inter=False, stream=None):
        """uno_psi_step_hidden: the step's hidden state after its first n_blocks residual
        sub-blocks (two per layer). With inter=True also returns the products of the last
        sub-blocks run: dict q, k, v (n_blocks >= 1) and act = silu(gate) * up (n_blocks >= 2)."""
        torch = _torch()
        bf16 = (torch.bfloat16,)
        M = B * (2 * k + 1)
        _expect(h_in, (M, self.hidden), bf16, "h_in")
        _expect(h_out, (M, self.hidden), bf16, "h_out", optional=True)
        if workspace is None:
            raise ValueError("workspace is required (Model.workspace_bytes(B, k) bytes)")
        h_out = torch.empty_like(h_in) if h_out is None else h_out
        mk = lambda n: torch.empty((M, n), dtype=torch.bfloat16, device=h_in.device)
        outs = {}
        if inter and n_blocks >= 1:
            outs.update(q=mk(self.q_out), k=mk(self.kv_out), v=mk(self.kv_out))
        if inter and n_blocks >= 2:
            outs["act"] = mk(self.inter)
        dev = _dev(h_in, h_out, workspace, *outs.values())
        if dev != self.device:
            raise ValueError(f"buffers on {dev}, the model's weights on {self.device}")
        wsb = workspace.numel() * workspace.element_size()
        _launch(dev, stream, load().uno_psi_step_hidden, self._h, B, k, _ptr(h_in), int(n_blocks),
                _ptr(h_out), _ptr(outs.get("q")), _ptr(outs.get("k")), _ptr(outs.get("v")),
                _ptr(outs.get("act")), _ptr(workspace), wsb)
        return (h_out, outs) if inter else h_out

    def step(self, B, k, h_in, q_prev, d_prev, temperature, seed, step, q_next, d_next,
             accepted_len, out_tokens, out_count, workspace, logits_out=None, dev_status=None,
             seq_offset=0, stream=None):
        """uno_psi_step on caller-provided device buffers (see include/uno.h)."""
        torch = _torch()
        bf16, i32 = (torch.bfloat16,), (torch.int32,)
        V = self.vocab
        _expect(h_in, (B * (2 * k + 1), self.hidden), bf16, "h_in")
        _expect(q_prev, (B, k, V), bf16, "q_prev")
        _expect(q_next, (B, k, V), bf16, "q_next")
        _expect(d_prev, (B, k), i32, "d_prev")
        _expect(d_next, (B, k), i32, "d_next")
        _expect(accepted_len, (B,), i32, "accepted_len")
        _expect(out_tokens, (B, k + 1), i32, "out_tokens")
        _expect(out_count, (B,), i32, "out_count")
        _expect(logits_out, (B * (k + 1), V), bf16, "logits_out", optional=True)
        _expect(dev_status, (1,), i32, "dev_status", optional=True)
        if workspace is None:
            raise ValueError("workspace is required (Model.workspace_bytes(B, k) bytes)")
        dev = _dev(h_in, q_prev, d_prev, q_next, d_next, accepted_len, out_tokens, out_count,
                   workspace, logits_out, dev_status)
        if dev != self.device:
            raise ValueError(f"step buffers on {dev}, the model's weights on {self.device}")
        wsb = workspace.numel() * workspace.element_size()
        _launch(dev, stream, load().uno_psi_step, self._h, B, k, _ptr(h_in), _ptr(q_prev),
                _ptr(d_prev), float(temperature), int(seed), int(step), int(seq_offset),
                _ptr(q_next), _ptr(d_next), _ptr(logits_out), _ptr(accepted_len),
                _ptr(out_tokens), _ptr(out_count), _ptr(dev_status), _ptr(workspace), wsb)
