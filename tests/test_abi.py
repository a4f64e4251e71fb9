"""The C-ABI library loads, exports every symbol of include/uno.h, and rejects
bad arguments on the host (no GPU needed: these calls return before any CUDA work)."""
import ctypes
import os
import re

import pytest

import sampling_gated_lora_b200 as U

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "uno.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(uno_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_what_binding_uses():
    assert set(_declared()) == set(U.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = U.load()
    for name in _declared():
        assert hasattr(lib, name), name
    assert "sm_100a" in U.version()


def _status(st):
    return st, U.load().uno_last_error().decode()


def test_linear_rejects_bad_arguments():
    L = U.load()
    null = None
    # K not a multiple of 8 (bf16 rows must be 16-byte multiples)
    st, msg = _status(L.uno_gated_lora_linear(U.UNO_BF16, 4, 12, 16, 8, null, null, null, null, null,
                                              1.0, null, null, 0, null))
    assert st == 2 and "multiples" in msg
    st, _ = _status(L.uno_gated_lora_linear(U.UNO_BF16, -1, 16, 16, 8, null, null, null, null, null,
                                            1.0, null, null, 0, null))
    assert st == 1
    st, msg = _status(L.uno_gated_lora_linear(U.UNO_BF16, 4, 16, 16, 264, null, null, null, null, null,
                                              1.0, null, null, 0, null))
    assert st == 2 and "rank" in msg
    st, _ = _status(L.uno_gated_lora_linear(7, 4, 16, 16, 8, null, null, null, null, null,
                                            1.0, null, null, 0, null))
    assert st == 1
    # M = 0 is a valid empty call that launches nothing
    assert L.uno_gated_lora_linear(U.UNO_BF16, 0, 16, 16, 8, null, null, null, null, null,
                                   1.0, null, null, 0, null) == 0
    # NULL inputs with M > 0
    st, _ = _status(L.uno_gated_lora_linear(U.UNO_BF16, 4, 16, 16, 8, null, null, null, null, null,
                                            1.0, null, null, 0, null))
    assert st == 1
    # misaligned pointers
    fake = ctypes.c_void_p(0x1008)
    st, msg = _status(L.uno_gated_lora_linear(U.UNO_BF16, 4, 16, 16, 8, fake, fake, fake, fake, fake,
                                              1.0, fake, fake, 1 << 20, null))
    assert st == 1 and "aligned" in msg
    # workspace too small
    ok = ctypes.c_void_p(0x10000)
    st, _ = _status(L.uno_gated_lora_linear(U.UNO_BF16, 4, 16, 16, 8, ok, ok, ok, ok, ok,
                                            1.0, ok, ok, 1, null))
    assert st == 6
    assert L.uno_gated_lora_linear_workspace(U.UNO_BF16, 9, 4096, 4096, 128) >= 9 * 128 * 2


def test_verify_rejects_bad_arguments():
    L = U.load()
    null = None
    ok = ctypes.c_void_p(0x10000)
    args = lambda dt, B, k, kp, V, T: L.uno_psi_verify(dt, B, k, kp, V, ok, ok, ok, T, 0, 0, 0, ok,
                                                     ok, ok, null, ok, 1 << 30, null)
    assert _status(args(U.UNO_BF16, 2, 4, 4, 1024, 0.0))[0] == 1        # T <= 0
    assert _status(args(U.UNO_BF16, 2, 4, 4, 1024, -1.0))[0] == 1
    assert _status(args(U.UNO_BF16, 2, 33, 33, 1024, 1.0))[0] == 2      # k > 32
    assert _status(args(U.UNO_BF16, 2, 0, 0, 1024, 1.0))[0] == 2        # k < 1
    assert _status(args(U.UNO_BF16, 2, 4, 6, 1024, 1.0))[0] == 1        # k_p not k or k+1
    assert _status(args(U.UNO_BF16, 2, 4, 4, 1, 1.0))[0] == 2           # V < 2
    assert _status(args(U.UNO_BF16, 2, 4, 4, 300000, 1.0))[0] == 2      # V too large
    assert _status(args(U.UNO_BF16, -1, 4, 4, 1024, 1.0))[0] == 1
    assert args(U.UNO_BF16, 0, 4, 4, 1024, 1.0) == 0                    # empty batch
    st = L.uno_psi_verify(U.UNO_BF16, 2, 4, 4, 1024, null, ok, ok, 1.0, 0, 0, 0, ok, ok, ok, null,
                          ok, 1 << 30, null)
    assert st == 1
    st = L.uno_psi_verify(U.UNO_BF16, 2, 4, 4, 1024, ok, ok, ok, 1.0, 0, 0, 0, ok, ok, ok, null,
                          ok, 0, null)
    assert st == 6
    assert L.uno_psi_verify_workspace(256, 16, 16, 151936) > 0
    assert L.uno_psi_verify_workspace(2, 4, 7, 1024) == 0


def test_draft_and_misc_reject_bad_arguments():
    L = U.load()
    null = None
    ok = ctypes.c_void_p(0x10000)
    assert L.uno_draft_sample(U.UNO_BF16, 2, 4, 1024, ok, 0.0, 0, 0, 0, ok, null, null, 0, null) == 1
    assert L.uno_draft_sample(U.UNO_BF16, 2, 4, 1024, null, 1.0, 0, 0, 0, ok, null, null, 0, null) == 1
    # the draft's stats pass needs its workspace: (rows, vocab chunks of <= 8192 ids) pairs
    need = L.uno_draft_sample_workspace(2, 4, 151936)
    assert need >= 2 * 4 * 19 * 8
    assert L.uno_draft_sample(U.UNO_BF16, 2, 4, 151936, ok, 1.0, 0, 0, 0, ok, null, null, 0,
                              null) == 6
    assert L.uno_draft_sample(U.UNO_BF16, 2, 4, 151936, ok, 1.0, 0, 0, 0, ok, null, ok,
                              need - 1, null) == 6
    assert L.uno_philox_uniforms(0, 0, 0, 0xFFFFFFFF, 2, ok, ok, null) == 1
    assert L.uno_philox_uniforms(0, 0, 0, 0, -1, ok, ok, null) == 1
    assert L.uno_rmsnorm(-1, 8, ok, ok, 1e-6, null) == 1
    assert L.uno_silu_mul(-1, ok, ok, ok, null) == 1
    assert L.uno_device_status(null, 0, null) == 1
    assert L.uno_wait_selftest(4, 1000000, ok, null, null) == 1           # which in [0, 3]
    assert L.uno_wait_selftest(0, 10, ok, null, null) == 1                # limit >= 1 us
    assert L.uno_wait_selftest(0, 10 ** 9, ok, null, null) == 1           # limit <= 100 ms
    assert L.uno_wait_selftest(0, 1000000, null, null, null) == 1


def test_adapter_backward_rejects_bad_arguments():
    L = U.load()
    ok = ctypes.c_void_p(0x10000)
    null = None
    call = lambda dt=U.UNO_BF16, M=64, K=64, N=128, r=8, x=ok, dA=ok, ws=1 << 30: L.uno_gated_lora_backward(
        dt, M, K, N, r, x, ok, ok, ok, ok, 1.0, dA, ok, ok, ws, null)
    assert call(dt=U.UNO_F32) == 2                # bf16 only
    assert call(K=60) == 2 and call(r=0) == 1     # 16-byte rows; an adapter is needed
    assert call(x=null) == 1 and call(dA=null) == 1
    assert call(dA=ctypes.c_void_p(0x10008)) == 1
    assert call(ws=16) == 6
    need = L.uno_gated_lora_backward_workspace(2048, 4096, 12288, 128)
    # x^T and dy^T at 2048 padded rows, Bl^T and the two rank-r products
    assert need >= 2 * 2048 * (4096 + 12288) + 2 * 128 * 12288 + 2 * 2 * 128 * 2048


def test_model_create_validates():
    L = U.load()
    h = ctypes.c_void_p()
    assert L.uno_model_create(ctypes.byref(h), 1, 12, 16, 16, 16, 16, 8, 1.0, None) == 2
    assert L.uno_model_create(ctypes.byref(h), 1, 16, 16, 16, 16, 16, 8, 1.0, None) == 1
    ptrs = (ctypes.c_void_p * 24)(*([0x10000] * 24))
    ptrs[5] = 0x10008    # misaligned
    assert L.uno_model_create(ctypes.byref(h), 1, 16, 16, 16, 16, 16, 8, 1.0, ptrs) == 1
    ptrs[5] = 0x10000
    assert L.uno_model_create(ctypes.byref(h), 1, 16, 16, 16, 16, 16, 8, 1.0, ptrs) == 0
    assert h.value
    assert L.uno_psi_step_workspace(h, 2, 4) > 0
    st = L.uno_psi_step(h, 2, 4, None, None, None, 1.0, 0, 0, 0, None, None, None, None, None,
                        None, None, None, 0, None)
    assert st == 1
    assert L.uno_psi_step_kernel_count(h, 2, 4) == 0      # no plan before a first step
    ok = ctypes.c_void_p(0x10000)
    ws = 1 << 30
    hid = lambda B=2, k=4, n=1, hi=ok, ho=ok, q=None, act=None, wsb=ws: L.uno_psi_step_hidden(
        h, B, k, hi, n, ho, q, None, None, act, ok, wsb, None)
    assert hid(n=-1) == 1 and hid(n=3) == 1                 # 0 <= n_blocks <= 2 per layer
    assert hid(n=0, q=ok) == 1 and hid(n=1, act=ok) == 1    # outputs of sub-blocks not run
    assert hid(B=0) == 1 and hid(k=33) == 1
    assert hid(hi=None) == 1 and hid(ho=ctypes.c_void_p(0x10008)) == 1
    assert hid(wsb=16) == 6
    L.uno_model_destroy(h)


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(U, "_lib", None)
    monkeypatch.setattr(U, "LIB_PATH", "/nonexistent/libuno.so")
    with pytest.raises(RuntimeError, match="missing"):
        U.load()


def test_workspace_sizes_hold_the_stream_k_scratch():
    """bf16 batches of more than 256 rows (the CTA-pair kernel) add the stream-K scratch:
    one fp32 256 x 256 partial tile per pair of SMs and 32 bytes of flags per pair
    (148 SMs assumed without a GPU); f32 and smaller batches do not."""
    L = U.load()
    pairs = 148 // 2
    part, flags = pairs * 256 * 256 * 4, pairs * 32
    ws = lambda dt, M, r: L.uno_gated_lora_linear_workspace(dt, M, 4096, 4096, r)
    t_bytes = 300 * 128 * 2
    assert ws(U.UNO_BF16, 256, 128) == 256 * 128 * 2
    assert ws(U.UNO_BF16, 300, 128) >= t_bytes + part + flags
    assert ws(U.UNO_BF16, 300, 0) >= part + flags            # r = 0: the scratch alone
    assert ws(U.UNO_F32, 300, 128) == 300 * 128 * 4
    g = L.uno_gated_lora_linear_group_workspace
    assert g(U.UNO_BF16, 300, 128, 3) >= 3 * t_bytes + part + flags
    assert g(U.UNO_BF16, 200, 128, 3) == 200 * 3 * 128 * 2
    # the step: one partial-sum region and a flag block per main GEMM (4 a layer + head)
    h = ctypes.c_void_p()
    ptrs = (ctypes.c_void_p * 24)(*([0x10000] * 24))
    assert L.uno_model_create(ctypes.byref(h), 1, 16, 16, 16, 16, 16, 8, 1.0, ptrs) == 0
    small, big = L.uno_psi_step_workspace(h, 8, 8), L.uno_psi_step_workspace(h, 16, 8)
    L.uno_model_destroy(h)
    # 136 rows (no scratch) vs 272 rows: every other buffer only grows with the rows
    assert big - small >= part + 5 * flags


def test_tree_verify_rejects_bad_arguments():
    L = U.load()
    ok = ctypes.c_void_p(0x10000)
    null = None

    def call(B=2, N=2, k=4, R=9, V=1024, T=1.0, ws_bytes=1 << 30, off=0):
        st = L.uno_tree_verify(U.UNO_BF16, B, N, k, R, V, ok, ok, ok, 0, T, 0, 0, off, ok, ok, ok,
                               null, ok, ws_bytes, null)
        return st, L.uno_last_error().decode()

    assert call(N=0)[0] == 2 and call(N=33)[0] == 2
    assert call(R=0)[0] == 1 and call(R=10)[0] == 1           # R <= N*k + 1
    assert call(k=33)[0] == 2 and call(T=0.0)[0] == 1
    # more logit rows than one grid dimension other than x holds pass the size checks
    # (the stats grid is one-dimensional) and stop at the workspace check
    assert call(B=4000, N=32, k=16, R=400, ws_bytes=1)[0] == 6
    assert call(off=1 << 32)[0] == 2                          # Philox index range
    assert call(ws_bytes=1)[0] == 6
    assert call(B=0)[0] == 0
    assert L.uno_tree_verify_workspace(2, 2, 4, 9, 1024) > 0
    assert L.uno_tree_verify_workspace(2, 0, 4, 9, 1024) == 0


def test_distill_rejects_bad_arguments():
    L = U.load()
    ok = ctypes.c_void_p(0x10000)
    call = lambda rows=4, V=64, T=1.0, zt=ok, loss=ok: L.uno_distill(
        U.UNO_BF16, rows, V, zt, ok, 1.0, 1.0, T, loss, None, None, None)
    assert call(rows=-1) == 1 and call(V=1) == 2 and call(V=196609) == 2
    assert call(T=0.0) == 1 and call(zt=None) == 1 and call(loss=None) == 1
    assert call(zt=ctypes.c_void_p(0x10008)) == 1
    assert call(rows=0) == 0
