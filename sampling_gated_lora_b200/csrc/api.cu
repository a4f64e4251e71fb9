// C ABI of the library (include/uno.h): argument validation, error reporting,
// the model handle and the orchestration of one synthetic decode step.
#include <cstdarg>
#include <cstdlib>
#include <cstdio>
#include <algorithm>
#include <cstring>
#include <memory>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "internal.h"

namespace uno {

namespace {
thread_local char g_err[512] = "no error";

constexpr size_t kAlign = 256;
size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t dt_size(uno_dtype dt) { return dt == UNO_F32 ? 4 : 2; }

bool valid_dtype(uno_dtype dt) { return dt == UNO_BF16 || dt == UNO_F32; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
}  // namespace

uno_status set_error(uno_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return st;
}

bool pdl_enabled() {
  static const bool on = [] {
    const char* v = getenv("UNO_PDL");
    return !(v && v[0] == '0');
  }();
  return on;
}

uno_status cuda_error(cudaError_t e, const char* what) {
  return set_error(UNO_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

// ---------------------------------------------------------------- gated linear

namespace {

struct LinearLayout {
  size_t t_off, sk_part_off, sk_flag_off, total;
  bool sk;
};

// Workspace of a gated linear: t (used when the down-projection runs as its
// own launch), then, for batches the CTA-pair kernel takes (bf16, M > 256),
// its stream-K partial sums and flags.
LinearLayout linear_layout(uno_dtype dt, int64_t M, int32_t r, int32_t G = 1) {
  LinearLayout l{};
  l.t_off = 0;
  size_t off = align_up(static_cast<size_t>(M) * static_cast<size_t>(r) * G * dt_size(dt));
  l.sk = dt == UNO_BF16 && M > 256;
  if (l.sk) {
    l.sk_part_off = off;
    off += align_up(pair_sk_part_bytes());
    l.sk_flag_off = off;
    off += align_up(pair_sk_flag_bytes());
  }
  l.total = off;
  return l;
}

// Points a problem at the stream-K scratch of a linear's workspace (when it has one).
void attach_sk(GemmProblem* pm, const LinearLayout& L, void* workspace) {
  if (!L.sk || !workspace) return;
  pm->sk_part = reinterpret_cast<float*>(static_cast<char*>(workspace) + L.sk_part_off);
  pm->sk_flag = reinterpret_cast<int32_t*>(static_cast<char*>(workspace) + L.sk_flag_off);
  pm->sk_slots = pair_sk_slots();
}

// Prepares the down-projection launched right before `main`; it clears the
// stream-K flags of `main` once it has waited for its own predecessor.
uno_status prepare_down(GemmProblem d, const GemmLaunch& main, GemmLaunch* out) {
  if (main.sk_flag) {
    d.zero_flags = main.sk_flag;
    d.zero_words = static_cast<int>(main.sk_flag_bytes / sizeof(int32_t));
  }
  return gemm_prepare(d, out);
}

// Runs the down-projection (if any) and the main launch of a gated linear.
// The main launch's stream-K flags are cleared by the down-projection (see
// prepare_down); without one, by a memset first. (Single calls leave
// GemmProblem::t_ready unset: back to back, a separate down-projection that
// overlaps the previous call's tail measured faster than a GEMM that
// computes t itself behind a memset.)
uno_status run_linear(const GemmLaunch* down, const GemmLaunch& main, cudaStream_t st) {
  if (main.sk_flag && !down) {
    const cudaError_t e = cudaMemsetAsync(main.sk_flag, 0, main.sk_flag_bytes, st);
    if (e != cudaSuccess) return cuda_error(e, "clearing the stream-K flags");
  }
  uno_status s;
  if (down && (s = gemm_run(*down, st)) != UNO_OK) return s;
  return gemm_run(main, st);
}

uno_status check_linear(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r) {
  if (!valid_dtype(dt)) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", dt);
  if (M < 0 || K < 1 || N < 1 || r < 0)
    return set_error(UNO_ERR_INVALID_ARG, "bad sizes M=%lld K=%lld N=%lld r=%d",
                     static_cast<long long>(M), static_cast<long long>(K),
                     static_cast<long long>(N), r);
  const int64_t q = dt == UNO_F32 ? 4 : 8;
  if (K % q || N % q || r % q)
    return set_error(UNO_ERR_UNSUPPORTED,
                     "K, N and r must be multiples of %lld (16-byte rows): K=%lld N=%lld r=%d",
                     static_cast<long long>(q), static_cast<long long>(K),
                     static_cast<long long>(N), r);
  if (r > 256) return set_error(UNO_ERR_UNSUPPORTED, "rank r=%d > 256", r);
  if (M > (1ll << 30) || N > (1ll << 30) || K > (1ll << 30))
    return set_error(UNO_ERR_UNSUPPORTED, "sizes above 2^30");
  return UNO_OK;
}

// The rank-r down-projections t_g = scale * gate * (x A_g^T) of up to three
// linears that share x, written side by side into t [M, G r].
GemmProblem down_problem(uno_dtype dt, int64_t M, int64_t K, int32_t r, const void* x,
                         const void* const* A, int G, const uint8_t* gate, int64_t gate_row0,
                         float scale, void* t) {
  GemmProblem d{};
  d.dt = dt;
  d.M = M;
  d.K = K;
  d.r = 0;
  d.x = x;
  d.ngroups = G;
  const size_t esz = dt_size(dt);
  for (int i = 0; i < G; ++i)
    d.g[i] = GemmGroup{A[i], nullptr, r, static_cast<char*>(t) + i * r * esz,
                       static_cast<int64_t>(G) * r, 0};
  d.mode = kEpiRowScale;
  d.M0 = M;
  d.gate = gate;
  d.gate_row0 = gate_row0;
  d.scale = scale;
  return d;
}

}  // namespace

}  // namespace uno

using namespace uno;

extern "C" {

const char* uno_last_error(void) { return g_err; }

const char* uno_version(void) { return "uno-psispec-b200 0.1 (sm_100a)"; }

uno_status uno_device_status(int32_t* bits_out, int32_t clear, void* stream) {
  if (!bits_out) return set_error(UNO_ERR_INVALID_ARG, "bits_out is NULL");
  cudaStream_t s = as_stream(stream);
  int32_t v = 0;
  cudaError_t e = cudaMemcpyFromSymbolAsync(&v, g_device_status, sizeof(v), 0,
                                            cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_error(e, "reading the device status word");
  if (clear) {
    const int32_t zero = 0;
    e = cudaMemcpyToSymbolAsync(g_device_status, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_error(e, "clearing the device status word");
  }
  *bits_out = v;
  return UNO_OK;
}

size_t uno_gated_lora_linear_workspace(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r) {
  (void)K;
  (void)N;
  if (M < 0 || r < 0) return 0;
  return linear_layout(dt, M, r).total;
}

uno_status uno_gated_lora_linear(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r,
                                 const void* x, const void* W, const void* A, const void* Bl,
                                 const uint8_t* gate, float scale, void* y, void* workspace,
                                 size_t ws_bytes, void* stream) {
  uno_status s = check_linear(dt, M, K, N, r);
  if (s != UNO_OK) return s;
  if (M == 0) return UNO_OK;
  if (!x || !W || !y) return set_error(UNO_ERR_INVALID_ARG, "x, W and y must be non-NULL");
  if (r > 0 && (!A || !Bl || !gate))
    return set_error(UNO_ERR_INVALID_ARG, "A, Bl and gate must be non-NULL when r > 0");
  if (!aligned16(x) || !aligned16(W) || !aligned16(y) || (r > 0 && (!aligned16(A) || !aligned16(Bl))))
    return set_error(UNO_ERR_INVALID_ARG, "x, W, A, Bl and y must be 16-byte aligned");
  const LinearLayout L = linear_layout(dt, M, r);
  if (r > 0 && (!workspace || ws_bytes < L.total || !aligned16(workspace)))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", L.total,
                     ws_bytes);
  const bool use_ws = workspace && ws_bytes >= L.total && aligned16(workspace);
  void* t_buf = r > 0 ? static_cast<char*>(workspace) + L.t_off : nullptr;
  GemmLaunch down{}, main{};
  GemmProblem pm{};
  pm.dt = dt;
  pm.M = M;
  pm.K = K;
  pm.r = r;
  pm.x = x;
  pm.t = t_buf;
  pm.ldt = r;
  pm.ngroups = 1;
  pm.g[0] = GemmGroup{W, Bl, N, y, N, 0};
  pm.A[0] = A;
  pm.mode = kEpiStore;
  pm.M0 = M;
  pm.gate = gate;
  pm.scale = scale;
  if (use_ws) attach_sk(&pm, L, workspace);
  const bool fused = r > 0 && gemm_dec_suits(pm);
  pm.x_ready = r > 0 && !fused;
  if ((s = gemm_prepare(pm, &main)) != UNO_OK) return s;
  if (r > 0 && !fused) {
    const void* As[1] = {A};
    if ((s = prepare_down(down_problem(dt, M, K, r, x, As, 1, gate, 0, scale, t_buf), main,
                          &down)) != UNO_OK)
      return s;
  }
  return run_linear(r > 0 && !fused ? &down : nullptr, main, as_stream(stream));
}

size_t uno_gated_lora_linear_group_workspace(uno_dtype dt, int64_t M, int32_t r, int32_t G) {
  if (M < 0 || r < 0 || G < 1 || G > kMaxGroups) return 0;
  return linear_layout(dt, M, r, G).total;
}

uno_status uno_gated_lora_linear_group(uno_dtype dt, int64_t M, int64_t K, int32_t r, int32_t G,
                                       const int64_t* N, const void* x, const void* const* W,
                                       const void* const* A, const void* const* Bl,
                                       const uint8_t* gate, float scale, int32_t mode,
                                       void* const* y, void* workspace, size_t ws_bytes,
                                       void* stream) {
  if (G < 1 || G > kMaxGroups) return set_error(UNO_ERR_INVALID_ARG, "G=%d outside [1, 3]", G);
  if (!N || !W || !y || (r > 0 && (!A || !Bl)))
    return set_error(UNO_ERR_INVALID_ARG, "NULL array argument");
  if (mode != 0 && mode != 1) return set_error(UNO_ERR_INVALID_ARG, "mode must be 0 or 1");
  if (mode == 1 && (G != 2 || N[0] != N[1] || dt != UNO_BF16))
    return set_error(UNO_ERR_INVALID_ARG, "mode 1 needs G = 2, N[0] = N[1] and bf16");
  uno_status s;
  for (int i = 0; i < G; ++i)
    if ((s = check_linear(dt, M, K, N[i], r)) != UNO_OK) return s;
  if (M == 0) return UNO_OK;
  if (!x || !aligned16(x)) return set_error(UNO_ERR_INVALID_ARG, "x must be non-NULL and 16-byte aligned");
  if (r > 0 && !gate) return set_error(UNO_ERR_INVALID_ARG, "gate must be non-NULL when r > 0");
  for (int i = 0; i < G; ++i) {
    if (!W[i] || !aligned16(W[i]) || (r > 0 && (!A[i] || !Bl[i] || !aligned16(A[i]) || !aligned16(Bl[i]))))
      return set_error(UNO_ERR_INVALID_ARG, "group %d: NULL or unaligned weight", i);
    if ((mode == 0 || i == 0) && (!y[i] || !aligned16(y[i])))
      return set_error(UNO_ERR_INVALID_ARG, "group %d: NULL or unaligned output", i);
  }
  const LinearLayout L = linear_layout(dt, M, r, G);
  const size_t need = L.total;
  if (r > 0 && (!workspace || ws_bytes < need || !aligned16(workspace)))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", need, ws_bytes);
  const bool use_ws = workspace && ws_bytes >= need && aligned16(workspace);
  GemmLaunch down{}, main{};
  GemmProblem pm{};
  void* t_buf = r > 0 ? workspace : nullptr;
  pm.dt = dt;
  pm.M = M;
  pm.K = K;
  pm.r = r;
  pm.x = x;
  pm.t = t_buf;
  pm.ldt = static_cast<int64_t>(G) * r;
  pm.ngroups = G;
  for (int i = 0; i < G; ++i)
    pm.g[i] = GemmGroup{W[i], r > 0 ? Bl[i] : nullptr, N[i], mode == 1 ? y[0] : y[i],
                        mode == 1 ? N[0] : N[i], static_cast<int64_t>(i) * r};
  for (int i = 0; i < G; ++i) pm.A[i] = r > 0 ? A[i] : nullptr;
  pm.mode = mode == 1 ? kEpiSiluPair : kEpiStore;
  pm.M0 = M;
  pm.gate = gate;
  pm.scale = scale;
  if (use_ws) attach_sk(&pm, L, workspace);
  const bool fused = r > 0 && gemm_dec_suits(pm);
  pm.x_ready = r > 0 && !fused;
  if ((s = gemm_prepare(pm, &main)) != UNO_OK) return s;
  if (r > 0 && !fused &&
      (s = prepare_down(down_problem(dt, M, K, r, x, A, G, gate, 0, scale, t_buf), main, &down)) !=
          UNO_OK)
    return s;
  return run_linear(r > 0 && !fused ? &down : nullptr, main, as_stream(stream));
}

size_t uno_gated_lora_backward_workspace(int64_t M, int64_t K, int64_t N, int32_t r) {
  if (M < 0 || K < 1 || N < 1 || r < 1) return 0;
  return align_up(adapter_backward_workspace(M, K, N, r));
}

uno_status uno_gated_lora_backward(uno_dtype dt, int64_t M, int64_t K, int64_t N, int32_t r,
                                   const void* x, const void* dy, const void* A, const void* Bl,
                                   const uint8_t* gate, float scale, void* dA, void* dBl,
                                   void* workspace, size_t ws_bytes, void* stream) {
  if (dt != UNO_BF16) return set_error(UNO_ERR_UNSUPPORTED, "the adapter backward takes bf16 only");
  uno_status s = check_linear(dt, M, K, N, r);
  if (s != UNO_OK) return s;
  if (r < 8) return set_error(UNO_ERR_INVALID_ARG, "rank r=%d: the backward needs an adapter", r);
  if (M > (1ll << 24)) return set_error(UNO_ERR_UNSUPPORTED, "M above 2^24 rows");
  if (!dA || !dBl || !A || !Bl) return set_error(UNO_ERR_INVALID_ARG, "NULL adapter or gradient pointer");
  if (!aligned16(dA) || !aligned16(dBl) || !aligned16(A) || !aligned16(Bl))
    return set_error(UNO_ERR_INVALID_ARG, "A, Bl, dA and dBl must be 16-byte aligned");
  cudaStream_t st = as_stream(stream);
  if (M == 0) {   // no rows: both gradients are zero
    cudaError_t e = cudaMemsetAsync(dA, 0, static_cast<size_t>(r) * K * 2, st);
    if (e == cudaSuccess) e = cudaMemsetAsync(dBl, 0, static_cast<size_t>(N) * r * 2, st);
    return e == cudaSuccess ? UNO_OK : cuda_error(e, "clearing the gradients");
  }
  if (!x || !dy || !gate) return set_error(UNO_ERR_INVALID_ARG, "x, dy and gate must be non-NULL");
  if (!aligned16(x) || !aligned16(dy)) return set_error(UNO_ERR_INVALID_ARG, "x and dy must be 16-byte aligned");
  const size_t need = uno_gated_lora_backward_workspace(M, K, N, r);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", need, ws_bytes);
  return adapter_backward_launch(M, K, N, r, x, dy, A, Bl, gate, scale, dA, dBl, workspace, st);
}

// ---------------------------------------------------------------- sampler

size_t uno_psi_verify_workspace(int32_t B, int32_t k, int32_t k_p, int32_t V) {
  if (B < 0 || k < 1 || V < 1 || (k_p != k && k_p != k + 1)) return 0;
  return align_up(verify_workspace(B, k, k_p, V));
}

static uno_status check_sampler(uno_dtype dt, int32_t B, int32_t k, int32_t V, float T) {
  if (!valid_dtype(dt)) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", dt);
  if (B < 0) return set_error(UNO_ERR_INVALID_ARG, "B=%d < 0", B);
  if (k < 1 || k > 32) return set_error(UNO_ERR_UNSUPPORTED, "block size k=%d outside [1, 32]", k);
  if (V < 2 || V > 196608) return set_error(UNO_ERR_UNSUPPORTED, "vocabulary V=%d outside [2, 196608]", V);
  if (!(T > 0.f) || !(T < 1e30f)) return set_error(UNO_ERR_INVALID_ARG, "temperature must be > 0 (got %g)", T);
  return UNO_OK;
}

uno_status uno_psi_verify(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t V,
                          const void* p_logits, const void* q_logits, const int32_t* draft,
                          float temperature, uint64_t seed, uint64_t step, uint64_t seq_offset,
                          int32_t* accepted_len, int32_t* out_tokens, int32_t* out_count,
                          int32_t* dev_status, void* workspace, size_t ws_bytes, void* stream) {
  uno_status s = check_sampler(dt, B, k, V, temperature);
  if (s != UNO_OK) return s;
  if (k_p != k && k_p != k + 1) return set_error(UNO_ERR_INVALID_ARG, "k_p=%d must be k or k+1", k_p);
  if (B == 0) return UNO_OK;
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k + 1) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * (k + 1) must be <= 2^32");
  if (!p_logits || !q_logits || !draft || !accepted_len || !out_tokens || !out_count)
    return set_error(UNO_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(p_logits) || !aligned16(q_logits))
    return set_error(UNO_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  const size_t need = uno_psi_verify_workspace(B, k, k_p, V);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", need, ws_bytes);
  VerifyArgs a{};
  a.dt = dt;
  a.B = B;
  a.k = k;
  a.k_p = k_p;
  a.V = V;
  a.p_logits = p_logits;
  a.q_logits = q_logits;
  a.draft = draft;
  a.temperature = temperature;
  a.seed = seed;
  a.step = step;
  a.seq_offset = seq_offset;
  a.accepted_len = accepted_len;
  a.out_tokens = out_tokens;
  a.out_count = out_count;
  a.dev_status = dev_status;
  return verify_launch(a, workspace, as_stream(stream));
}

size_t uno_tree_verify_workspace(int32_t B, int32_t N, int32_t k, int32_t R, int32_t V) {
  if (B < 0 || N < 1 || N > 32 || k < 1 || k > 32 || R < 1 || V < 1) return 0;
  return align_up(tree_verify_workspace(B, k, R, V));
}

uno_status uno_tree_verify(uno_dtype dt, int32_t B, int32_t N, int32_t k, int32_t R, int32_t V,
                           const void* p_logits, const void* q_logits, const int32_t* cands,
                           int32_t bonus, float temperature, uint64_t seed, uint64_t step,
                           uint64_t seq_offset, int32_t* accepted_len, int32_t* out_tokens,
                           int32_t* out_count, int32_t* dev_status, void* workspace,
                           size_t ws_bytes, void* stream) {
  uno_status s = check_sampler(dt, B, k, V, temperature);
  if (s != UNO_OK) return s;
  if (N < 1 || N > 32) return set_error(UNO_ERR_UNSUPPORTED, "candidates N=%d outside [1, 32]", N);
  if (R < 1 || static_cast<int64_t>(R) > static_cast<int64_t>(N) * k + 1)
    return set_error(UNO_ERR_INVALID_ARG, "node rows R=%d outside [1, N*k+1]", R);
  if (B == 0) return UNO_OK;
  if (static_cast<int64_t>(B) * (R + k) > (1ll << 30))
    return set_error(UNO_ERR_UNSUPPORTED, "B * (R + k) = %lld logit rows > 2^30",
                     static_cast<long long>(B) * (R + k));
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k + 1) *
          static_cast<uint64_t>(N) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * (k + 1) * N must be <= 2^32");
  if (!p_logits || !q_logits || !cands || !accepted_len || !out_tokens || !out_count)
    return set_error(UNO_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(p_logits) || !aligned16(q_logits))
    return set_error(UNO_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  const size_t need = uno_tree_verify_workspace(B, N, k, R, V);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", need, ws_bytes);
  TreeVerifyArgs a{};
  a.dt = dt;
  a.B = B;
  a.N = N;
  a.k = k;
  a.R = R;
  a.V = V;
  a.bonus = bonus ? 1 : 0;
  a.p_logits = p_logits;
  a.q_logits = q_logits;
  a.cands = cands;
  a.temperature = temperature;
  a.seed = seed;
  a.step = step;
  a.seq_offset = seq_offset;
  a.accepted_len = accepted_len;
  a.out_tokens = out_tokens;
  a.out_count = out_count;
  a.dev_status = dev_status;
  return tree_verify_launch(a, workspace, as_stream(stream));
}

uno_status uno_distill(uno_dtype dt, int32_t rows, int32_t V, const void* z_teacher,
                       const void* z_student, float alpha, float beta, float temperature,
                       float* losses, float* grad, int32_t* dev_status, void* stream) {
  if (!valid_dtype(dt)) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", dt);
  if (rows < 0) return set_error(UNO_ERR_INVALID_ARG, "rows=%d < 0", rows);
  if (V < 2 || V > 196608) return set_error(UNO_ERR_UNSUPPORTED, "vocabulary V=%d outside [2, 196608]", V);
  if (!(temperature > 0.f) || !(temperature < 1e30f))
    return set_error(UNO_ERR_INVALID_ARG, "temperature must be > 0 (got %g)", temperature);
  if (rows == 0) return UNO_OK;
  if (!z_teacher || !z_student || !losses)
    return set_error(UNO_ERR_INVALID_ARG, "NULL logits or losses pointer");
  if (!aligned16(z_teacher) || !aligned16(z_student))
    return set_error(UNO_ERR_INVALID_ARG, "logits must be 16-byte aligned");
  DistillArgs a{};
  a.dt = dt;
  a.rows = rows;
  a.V = V;
  a.z_teacher = z_teacher;
  a.z_student = z_student;
  a.alpha = alpha;
  a.beta = beta;
  a.temperature = temperature;
  a.losses = losses;
  a.grad = grad;
  a.dev_status = dev_status;
  return distill_launch(a, as_stream(stream));
}

// ---------------------------------------------------------------- vocabulary shards

namespace {
uno_status check_vp(uno_dtype dt, int32_t B, int32_t k, int32_t Vs, int32_t v0, int32_t V,
                    int32_t G, int32_t rank, float T) {
  uno_status s = check_sampler(dt, B, k, V, T);
  if (s != UNO_OK) return s;
  if (G < 1 || G > 64) return set_error(UNO_ERR_UNSUPPORTED, "shards G=%d outside [1, 64]", G);
  if (rank < 0 || rank >= G) return set_error(UNO_ERR_INVALID_ARG, "rank=%d outside [0, G)", rank);
  if (Vs < 1 || v0 < 0 || static_cast<int64_t>(v0) + Vs > V)
    return set_error(UNO_ERR_INVALID_ARG, "shard [v0, v0 + Vs) = [%d, %d) outside [0, V=%d)", v0,
                     v0 + Vs, V);
  return UNO_OK;
}
}  // namespace

uno_status uno_vp_partials(uno_dtype dt, int32_t rows, int32_t Vs, int32_t v0, const void* logits,
                           const int32_t* draft, int32_t k, int32_t k_p, int32_t id_kind,
                           int32_t precise, float temperature, float* out, void* stream) {
  if (!valid_dtype(dt)) return set_error(UNO_ERR_INVALID_ARG, "unknown dtype %d", dt);
  if (rows < 0 || Vs < 1 || v0 < 0) return set_error(UNO_ERR_INVALID_ARG, "bad sizes");
  if (id_kind < 0 || id_kind > 2) return set_error(UNO_ERR_INVALID_ARG, "id_kind=%d outside [0, 2]", id_kind);
  if (id_kind != 0 && (k < 1 || k > 32 || (id_kind == 1 && k_p != k && k_p != k + 1)))
    return set_error(UNO_ERR_INVALID_ARG, "k=%d, k_p=%d", k, k_p);
  if (id_kind == 1 && rows % k_p) return set_error(UNO_ERR_INVALID_ARG, "rows not a multiple of k_p");
  if (!(temperature > 0.f) || !(temperature < 1e30f))
    return set_error(UNO_ERR_INVALID_ARG, "temperature must be > 0 (got %g)", temperature);
  if (rows == 0) return UNO_OK;
  if (!logits || !out || (id_kind != 0 && !draft))
    return set_error(UNO_ERR_INVALID_ARG, "NULL logits, draft or out");
  if (!aligned16(logits) || !aligned16(out))
    return set_error(UNO_ERR_INVALID_ARG, "logits and out must be 16-byte aligned");
  return vp_partials_launch(dt, rows, Vs, v0, logits, draft, k, k_p, id_kind, precise != 0,
                            temperature, out, as_stream(stream));
}

uno_status uno_vp_verify_decide(int32_t B, int32_t k, int32_t k_p, int32_t V, int32_t G,
                                const float* parts_p, const float* parts_q, const int32_t* draft,
                                float temperature, uint64_t seed, uint64_t step,
                                uint64_t seq_offset, int32_t* accepted_len, int32_t* out_tokens,
                                int32_t* out_count, int32_t* draw, float* draw_stats,
                                int32_t* dev_status, void* stream) {
  uno_status s = check_vp(UNO_BF16, B, k, 1, 0, V, G, 0, temperature);
  if (s != UNO_OK) return s;
  if (k_p != k && k_p != k + 1) return set_error(UNO_ERR_INVALID_ARG, "k_p=%d must be k or k+1", k_p);
  if (B == 0) return UNO_OK;
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k + 1) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * (k + 1) must be <= 2^32");
  if (!parts_p || !parts_q || !draft || !accepted_len || !out_tokens || !out_count || !draw ||
      !draw_stats)
    return set_error(UNO_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(parts_p) || !aligned16(parts_q) || !aligned16(draw_stats))
    return set_error(UNO_ERR_INVALID_ARG, "partials and draw_stats must be 16-byte aligned");
  VpArgs a{};
  a.B = B;
  a.k = k;
  a.k_p = k_p;
  a.V = V;
  a.G = G;
  a.temperature = temperature;
  a.seed = seed;
  a.step = step;
  a.seq_offset = seq_offset;
  a.draft = draft;
  a.parts_p = parts_p;
  a.parts_q = parts_q;
  a.accepted_len = accepted_len;
  a.out_tokens = out_tokens;
  a.out_count = out_count;
  a.draw = draw;
  a.draw_stats = draw_stats;
  a.dev_status = dev_status;
  return vp_decide_launch(a, as_stream(stream));
}

uno_status uno_vp_draw_masses(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t Vs,
                              const void* p_shard, const void* q_shard, const int32_t* draw,
                              const float* draw_stats, float temperature, double* masses,
                              void* stream) {
  uno_status s = check_vp(dt, B, k, Vs, 0, Vs, 1, 0, temperature);
  if (s != UNO_OK) return s;
  if (k_p != k && k_p != k + 1) return set_error(UNO_ERR_INVALID_ARG, "k_p=%d must be k or k+1", k_p);
  if (B == 0) return UNO_OK;
  if (!p_shard || !q_shard || !draw || !draw_stats || !masses)
    return set_error(UNO_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(draw_stats) || !aligned16(masses))
    return set_error(UNO_ERR_INVALID_ARG, "draw_stats and masses must be 16-byte aligned");
  VpArgs a{};
  a.dt = dt;
  a.B = B;
  a.k = k;
  a.k_p = k_p;
  a.Vs = Vs;
  a.temperature = temperature;
  a.p = p_shard;
  a.q = q_shard;
  a.draw = const_cast<int32_t*>(draw);
  a.draw_stats = const_cast<float*>(draw_stats);
  a.masses = masses;
  return vp_masses_launch(a, as_stream(stream));
}

uno_status uno_vp_draw(uno_dtype dt, int32_t B, int32_t k, int32_t k_p, int32_t Vs, int32_t v0,
                       int32_t V, int32_t G, int32_t rank, const void* p_shard,
                       const void* q_shard, const int32_t* draw, const float* draw_stats,
                       const double* masses_all, float temperature, uint64_t seed, uint64_t step,
                       uint64_t seq_offset, int32_t* out_tokens, void* stream) {
  uno_status s = check_vp(dt, B, k, Vs, v0, V, G, rank, temperature);
  if (s != UNO_OK) return s;
  if (k_p != k && k_p != k + 1) return set_error(UNO_ERR_INVALID_ARG, "k_p=%d must be k or k+1", k_p);
  if (B == 0) return UNO_OK;
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k + 1) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * (k + 1) must be <= 2^32");
  if (!p_shard || !q_shard || !draw || !draw_stats || !masses_all || !out_tokens)
    return set_error(UNO_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(draw_stats) || !aligned16(masses_all))
    return set_error(UNO_ERR_INVALID_ARG, "draw_stats and masses must be 16-byte aligned");
  VpArgs a{};
  a.dt = dt;
  a.B = B;
  a.k = k;
  a.k_p = k_p;
  a.Vs = Vs;
  a.v0 = v0;
  a.V = V;
  a.G = G;
  a.rank = rank;
  a.temperature = temperature;
  a.seed = seed;
  a.step = step;
  a.seq_offset = seq_offset;
  a.p = p_shard;
  a.q = q_shard;
  a.draw = const_cast<int32_t*>(draw);
  a.draw_stats = const_cast<float*>(draw_stats);
  a.masses = const_cast<double*>(masses_all);
  a.out_tokens = out_tokens;
  return vp_draw_launch(a, as_stream(stream));
}

uno_status uno_vp_draft_draw(uno_dtype dt, int32_t B, int32_t k, int32_t Vs, int32_t v0, int32_t V,
                             int32_t G, int32_t rank, const void* q_shard, const float* parts_all,
                             float temperature, uint64_t seed, uint64_t step, uint64_t seq_offset,
                             int32_t* draft, int32_t* dev_status, void* stream) {
  uno_status s = check_vp(dt, B, k, Vs, v0, V, G, rank, temperature);
  if (s != UNO_OK) return s;
  if (B == 0) return UNO_OK;
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * k must be <= 2^32");
  if (!q_shard || !parts_all || !draft) return set_error(UNO_ERR_INVALID_ARG, "NULL pointer");
  if (!aligned16(parts_all)) return set_error(UNO_ERR_INVALID_ARG, "partials must be 16-byte aligned");
  VpArgs a{};
  a.dt = dt;
  a.B = B;
  a.k = k;
  a.Vs = Vs;
  a.v0 = v0;
  a.V = V;
  a.G = G;
  a.rank = rank;
  a.temperature = temperature;
  a.seed = seed;
  a.step = step;
  a.seq_offset = seq_offset;
  a.q = q_shard;
  a.parts_q = parts_all;
  a.draft_out = draft;
  a.dev_status = dev_status;
  return vp_draft_draw_launch(a, as_stream(stream));
}

size_t uno_draft_sample_workspace(int32_t B, int32_t k, int32_t V) {
  if (B < 0 || k < 1 || V < 1) return 0;
  return align_up(draft_workspace(B, k, V));
}

uno_status uno_draft_sample(uno_dtype dt, int32_t B, int32_t k, int32_t V, const void* q_logits,
                            float temperature, uint64_t seed, uint64_t step, uint64_t seq_offset,
                            int32_t* draft, int32_t* dev_status, void* workspace, size_t ws_bytes,
                            void* stream) {
  uno_status s = check_sampler(dt, B, k, V, temperature);
  if (s != UNO_OK) return s;
  if (B == 0) return UNO_OK;
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * k must be <= 2^32");
  if (static_cast<int64_t>(B) * k > (1ll << 30)) return set_error(UNO_ERR_UNSUPPORTED, "B * k > 2^30");
  if (!q_logits || !draft) return set_error(UNO_ERR_INVALID_ARG, "NULL q_logits or draft");
  const size_t need = uno_draft_sample_workspace(B, k, V);
  if (!workspace || ws_bytes < need || !aligned16(workspace))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", need, ws_bytes);
  DraftArgs a{};
  a.dt = dt;
  a.B = B;
  a.k = k;
  a.V = V;
  a.q_logits = q_logits;
  a.temperature = temperature;
  a.seed = seed;
  a.step = step;
  a.seq_offset = seq_offset;
  a.draft = draft;
  a.dev_status = dev_status;
  return draft_launch(a, workspace, as_stream(stream));
}

uno_status uno_philox_uniforms(uint64_t seed, uint64_t step, uint32_t stream_id, uint32_t index0,
                               int64_t n, uint32_t* words, float* u, void* stream) {
  if (n < 0) return set_error(UNO_ERR_INVALID_ARG, "n < 0");
  if (static_cast<uint64_t>(index0) + static_cast<uint64_t>(n) > (1ull << 32))
    return set_error(UNO_ERR_INVALID_ARG, "index0 + n > 2^32");
  return philox_launch(seed, step, stream_id, index0, n, words, u, as_stream(stream));
}

uno_status uno_wait_selftest(int32_t which, uint64_t limit_ns, int32_t* result,
                             int32_t* dev_status, void* stream) {
  if (which < 0 || which > 3) return set_error(UNO_ERR_INVALID_ARG, "which=%d outside [0, 3]", which);
  if (limit_ns < 1000 || limit_ns > 100000000ull)
    return set_error(UNO_ERR_INVALID_ARG, "limit_ns=%llu outside [1e3, 1e8]",
                     static_cast<unsigned long long>(limit_ns));
  if (!result) return set_error(UNO_ERR_INVALID_ARG, "result is NULL");
  return wait_selftest_launch(which, limit_ns, result, dev_status, as_stream(stream));
}

uno_status uno_rmsnorm(int64_t M, int64_t D, const void* x, void* y, float eps, void* stream) {
  if (M < 0 || D < 1) return set_error(UNO_ERR_INVALID_ARG, "bad sizes");
  if (M > 0 && (!x || !y)) return set_error(UNO_ERR_INVALID_ARG, "NULL pointer");
  if (M > 0 && (!aligned16(x) || !aligned16(y))) return set_error(UNO_ERR_INVALID_ARG, "unaligned pointer");
  if (M > 0x7fffffffll || D > (1ll << 30)) return set_error(UNO_ERR_UNSUPPORTED, "sizes too large");
  return rmsnorm_launch(M, D, x, y, eps, as_stream(stream));
}

uno_status uno_silu_mul(int64_t n, const void* a, const void* b, void* y, void* stream) {
  if (n < 0) return set_error(UNO_ERR_INVALID_ARG, "n < 0");
  if (n > 0 && (!a || !b || !y)) return set_error(UNO_ERR_INVALID_ARG, "NULL pointer");
  if (n > 0 && (!aligned16(a) || !aligned16(b) || !aligned16(y)))
    return set_error(UNO_ERR_INVALID_ARG, "unaligned pointer");
  return silu_mul_launch(n, a, b, y, as_stream(stream));
}

}  // extern "C"

// ---------------------------------------------------------------- model + step

namespace uno {
namespace {

constexpr int kLinPerLayer = 7;   // q, k, v, o, gate, up, down
enum { kQ = 0, kK, kV, kO, kGate, kUp, kDown };

struct StepLayout {
  size_t h, n, q, k, v, act, t, logits, vstat, dstat, sk_part, sk_flag, sk_flag_bytes, flag_block,
      ss, ss_block, total;
};

// One operation of a step plan.
struct StepOp {
  int kind;            // 0 GEMM, 1 rmsnorm, 2 rmsnorm + LoRA down-projection, 3 row sums of squares
  GemmLaunch gemm;
  const void* x;
  void* y;
  NormDownArgs nd;
  int64_t dims[4];     // M, total N, K, epilogue mode (GEMMs; what uno_model_last_profile reports)
};

// Launch kinds of uno_model_last_profile.
enum ProfKind : int32_t {
  kProfGemmOne = 0,      // one-CTA tcgen05 GEMM (down-projections, mid-size batches)
  kProfGemmPair = 1,     // CTA-pair GEMM
  kProfGemmPairT = 2,    // CTA-pair GEMM that computes t itself
  kProfGemmDecode = 3,   // fused decode-size GEMM
  kProfNorm = 10,        // RMSNorm
  kProfNormDown = 11,    // RMSNorm + LoRA down-projection
  kProfSumSq = 12,       // rows' sums of squares (the first folded RMSNorm)
  kProfVerify = 20,      // row stats + verify finalize
  kProfDraft = 21,       // draft stats + draft draw
};

int32_t prof_kind(const StepOp& op) {
  if (op.kind == 1) return kProfNorm;
  if (op.kind == 2) return kProfNormDown;
  if (op.kind == 3) return kProfSumSq;
  if (op.gemm.kind == 1) return op.gemm.computes_t ? kProfGemmPairT : kProfGemmPair;
  return op.gemm.kind == 2 ? kProfGemmDecode : kProfGemmOne;
}

void set_dims(StepOp* op, const GemmProblem& pb) {
  int64_t n = 0;
  for (int i = 0; i < pb.ngroups; ++i) n += pb.g[i].N;
  op->dims[0] = pb.M;
  op->dims[1] = n;
  op->dims[2] = pb.K;
  op->dims[3] = pb.mode;
}

// Decode-size batches fold the LoRA down-projection of an input that an
// RMSNorm produces into that RMSNorm's launch (one launch instead of two).
constexpr int64_t kNormDownMaxRows = 32;

// From this many rows every main GEMM of a step is a CTA-pair launch, and the
// step folds its RMSNorms into the GEMMs around them (GemmProblem::in_ss):
// the residual-add launches write their rows' sums of squares, the next
// launch scales its output rows. No RMSNorm launch and no normalised copy.
constexpr int64_t kFoldNormMinRows = 512;
constexpr float kNormEps = 1e-6f;

}  // namespace
}  // namespace uno

struct uno_model {
  int32_t n_layers, hidden, q_out, kv_out, inter, vocab, r;
  float scale;
  std::vector<const void*> w;   // 21 * n_layers + 3

  // The launches of one (B, k, buffers) combination, in step order.
  struct Plan {
    int32_t B, k;
    const void* ws;
    const void* q_next;       // NULL: the decoder layers only (no LM head)
    const void* logits_out;
    std::vector<uno::StepOp> ops;
    std::vector<size_t> block_end;   // ops.size() after each residual sub-block
  };
  std::mutex mu;
  std::vector<std::unique_ptr<Plan>> plans;   // most recently used last

  // Launch timing (uno_model_profile): an event after each launch of a step.
  bool profiling = false;
  int prof_device = -1;
  std::vector<cudaEvent_t> events;
  std::vector<int32_t> prof_kinds;
  std::vector<int64_t> prof_dims;
  size_t prof_n = 0;   // events recorded by the last profiled step (launches + 1)

  ~uno_model() {
    if (events.empty()) return;
    int cur = -1;
    cudaGetDevice(&cur);
    if (prof_device >= 0) cudaSetDevice(prof_device);
    for (cudaEvent_t e : events) cudaEventDestroy(e);
    if (cur >= 0) cudaSetDevice(cur);
  }

  const void* wp(int layer, int i, int part) const {
    return w[static_cast<size_t>(layer * uno::kLinPerLayer + i) * 3 + part];
  }
  const void* head(int part) const {
    return w[static_cast<size_t>(n_layers) * uno::kLinPerLayer * 3 + part];
  }
};

namespace uno {
namespace {

StepLayout step_layout(const uno_model* m, int32_t B, int32_t k) {
  const size_t M = static_cast<size_t>(B) * (2 * k + 1);
  const size_t Mv = static_cast<size_t>(B) * (k + 1);
  StepLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes);
    return o;
  };
  L.h = take(M * m->hidden * 2);
  L.n = take(M * m->hidden * 2);
  L.q = take(M * m->q_out * 2);
  L.k = take(M * m->kv_out * 2);
  L.v = take(M * m->kv_out * 2);
  L.act = take(M * m->inter * 2);
  L.t = take(M * 3 * static_cast<size_t>(m->r) * 2);
  L.logits = take(Mv * static_cast<size_t>(m->vocab) * 2);
  L.vstat = take(verify_workspace(B, k, k + 1, m->vocab));
  L.dstat = take(draft_workspace(B, k, m->vocab));
  // stream-K scratch of the CTA-pair GEMMs (M > 256): partial sums shared by
  // the step's launches, one block of stream-K flags and t counters per
  // launch (4 per layer + head), all cleared at the start of a step
  if (M > 256) {
    L.sk_part = take(pair_sk_part_bytes());
    L.flag_block = align_up(pair_sk_flag_bytes()) + align_up(pair_t_ready_bytes(M));
    L.sk_flag_bytes = (static_cast<size_t>(m->n_layers) * 4 + 1) * L.flag_block;
    L.sk_flag = take(L.sk_flag_bytes);
  }
  // folded RMSNorm: per residual stream state (2 per layer + the input) the
  // rows' sums of squares in 256-column partials
  if (static_cast<int64_t>(M) >= kFoldNormMinRows) {
    L.ss_block = align_up(M * ((static_cast<size_t>(m->hidden) + 255) / 256) * sizeof(float));
    L.ss = take((static_cast<size_t>(m->n_layers) * 2 + 1) * L.ss_block);
  }
  L.total = off;
  return L;
}

// Plan of one step: per layer
//   rmsnorm(h) -> n; down(n; A_q, A_k, A_v) -> t; gemm(n, t; q, k, v)
//   down(q; A_o) -> t; gemm(q, t; o) += h
//   rmsnorm(h) -> n; down(n; A_gate, A_up) -> t; gemm(n, t; silu(gate) * up) -> act
//   down(act; A_down) -> t; gemm(act, t; down) += h
// then rmsnorm(h) -> n, the LM head's down-projection and GEMM (AR rows ->
// logits, mask rows -> q_next). Rows >= B(k+1) carry the adapter (gate 1).
uno_status build_plan(uno_model* m, int32_t B, int32_t k, void* ws, void* q_next,
                      void* logits_out, uno_model::Plan* P) {
  const StepLayout L = step_layout(m, B, k);
  char* base = static_cast<char*>(ws);
  const int64_t M = static_cast<int64_t>(B) * (2 * k + 1);
  const int64_t Mv = static_cast<int64_t>(B) * (k + 1);
  const int32_t r = m->r;
  P->B = B;
  P->k = k;
  P->ws = ws;
  P->q_next = q_next;
  P->logits_out = logits_out;
  P->ops.clear();
  P->block_end.clear();
  void* t = base + L.t;
  int main_launches = 0;   // stream-K flag block of the next main GEMM
  auto norm = [&](const void* x, void* y) {
    StepOp op{};
    op.kind = 1;
    op.x = x;
    op.y = y;
    P->ops.push_back(op);
  };
  auto gemm = [&](const GemmProblem& pb) -> uno_status {
    StepOp op{};
    op.kind = 0;
    set_dims(&op, pb);
    const uno_status s = gemm_prepare(pb, &op.gemm);
    if (s == UNO_OK) P->ops.push_back(op);
    return s;
  };
  // gated linear(s) on input x (width K): down-projections then the main GEMM
  // (or the main GEMM alone, when it computes t itself or is the fused
  // decode kernel). t_ready: the preceding launch wrote t as well as x.
  const bool fold_norm = L.ss_block != 0;
  auto ss_at = [&](int i) { return reinterpret_cast<float*>(base + L.ss + static_cast<size_t>(i) * L.ss_block); };
  const int ss_cols = (m->hidden + 255) / 256;
  // in_ss / out_ss: the folded RMSNorm's sums of squares read / written (or NULL)
  auto linear = [&](const void* x, int64_t K, int G, const int* which, int layer, void* const* y,
                    const int64_t* ldy, int mode, void* y1, int64_t M0, bool t_ready = false,
                    const float* in_ss = nullptr, float* out_ss = nullptr) -> uno_status {
    uno_status s;
    const void* As[kMaxGroups] = {nullptr, nullptr, nullptr};
    for (int i = 0; i < G; ++i)
      As[i] = layer >= 0 ? m->wp(layer, which[i], 1) : m->head(1);
    GemmProblem pm{};
    pm.dt = UNO_BF16;
    pm.M = M;
    pm.K = K;
    pm.r = r;
    pm.x = x;
    pm.t = t;
    pm.ldt = static_cast<int64_t>(G) * r;
    pm.ngroups = G;
    for (int i = 0; i < G; ++i) {
      const void* W = layer >= 0 ? m->wp(layer, which[i], 0) : m->head(0);
      const void* Bl = layer >= 0 ? m->wp(layer, which[i], 2) : m->head(2);
      const int64_t N = layer >= 0 ? 0 : m->vocab;
      pm.g[i] = GemmGroup{W, Bl, N, y[i], ldy[i], static_cast<int64_t>(i) * r};
    }
    for (int i = 0; i < G && layer >= 0; ++i) {
      switch (which[i]) {
        case kQ: pm.g[i].N = m->q_out; break;
        case kK:
        case kV: pm.g[i].N = m->kv_out; break;
        case kGate:
        case kUp: pm.g[i].N = m->inter; break;
        default: pm.g[i].N = m->hidden; break;
      }
    }
    pm.mode = mode;
    pm.y1 = y1;
    pm.M0 = M0;
    pm.gate = nullptr;
    pm.gate_row0 = Mv;
    pm.scale = m->scale;
    for (int i = 0; i < G; ++i) pm.A[i] = r > 0 ? As[i] : nullptr;
    pm.in_ss = in_ss;
    pm.in_ss_cols = in_ss ? ss_cols : 0;
    pm.out_ss = out_ss;
    pm.norm_dim = m->hidden;
    pm.norm_eps = kNormEps;
    pm.x_ready = r > 0 && !gemm_dec_suits(pm) && !t_ready;
    if (L.sk_flag_bytes) {
      char* blk = base + L.sk_flag + static_cast<size_t>(main_launches) * L.flag_block;
      pm.sk_part = reinterpret_cast<float*>(base + L.sk_part);
      pm.sk_flag = reinterpret_cast<int32_t*>(blk);
      pm.sk_slots = pair_sk_slots();
      if (pm.x_ready) pm.t_ready = reinterpret_cast<int32_t*>(blk + align_up(pair_sk_flag_bytes()));
      ++main_launches;
    }
    StepOp op{};
    op.kind = 0;
    set_dims(&op, pm);
    if ((s = gemm_prepare(pm, &op.gemm)) != UNO_OK) return s;
    if (pm.x_ready && !op.gemm.computes_t &&
        (s = gemm(down_problem(UNO_BF16, M, K, r, x, As, G, nullptr, Mv, m->scale, t))) != UNO_OK)
      return s;
    P->ops.push_back(op);
    return UNO_OK;
  };
  uno_status s;
  if (fold_norm) {   // the input's sums of squares (the later ones come from the residual adds)
    StepOp op{};
    op.kind = 3;
    op.x = base + L.h;
    op.y = ss_at(0);
    P->ops.push_back(op);
  }
  for (int l = 0; l < m->n_layers; ++l) {
    if (!fold_norm) norm(base + L.h, base + L.n);
    {
      const int which[3] = {kQ, kK, kV};
      void* y[3] = {base + L.q, base + L.k, base + L.v};
      const int64_t ld[3] = {m->q_out, m->kv_out, m->kv_out};
      if ((s = linear(fold_norm ? base + L.h : base + L.n, m->hidden, 3, which, l, y, ld, kEpiStore,
                      nullptr, M, false, fold_norm ? ss_at(2 * l) : nullptr)) != UNO_OK)
        return s;
    }
    {
      const int which[1] = {kO};
      void* y[1] = {base + L.h};
      const int64_t ld[1] = {m->hidden};
      if ((s = linear(base + L.q, m->q_out, 1, which, l, y, ld, kEpiAdd, nullptr, M, false, nullptr,
                      fold_norm ? ss_at(2 * l + 1) : nullptr)) != UNO_OK)
        return s;
    }
    P->block_end.push_back(P->ops.size());
    {
      const int which[2] = {kGate, kUp};
      void* y[2] = {base + L.act, base + L.act};
      const int64_t ld[2] = {m->inter, m->inter};
      // the silu pair never fits the fused decode kernel (2 * inter rows > one wave): at
      // decode sizes its down-projection rides in the RMSNorm launch
      GemmProblem probe{};   // would the silu pair take the fused decode kernel?
      probe.dt = UNO_BF16;
      probe.M = M;
      probe.K = m->hidden;
      probe.r = r;
      probe.ngroups = 2;
      probe.mode = kEpiSiluPair;
      probe.A[0] = m->wp(l, kGate, 1);
      probe.A[1] = m->wp(l, kUp, 1);
      probe.g[0].N = probe.g[1].N = m->inter;
      const bool fold = !fold_norm && r > 0 && M <= kNormDownMaxRows && m->hidden % 8 == 0 &&
                        !gemm_dec_suits(probe);
      if (fold) {
        StepOp op{};
        op.kind = 2;
        op.nd.x = base + L.h;
        op.nd.y = base + L.n;
        op.nd.D = m->hidden;
        op.nd.eps = 1e-6f;
        op.nd.A[0] = m->wp(l, kGate, 1);
        op.nd.A[1] = m->wp(l, kUp, 1);
        op.nd.A[2] = op.nd.A[1];
        op.nd.G = 2;
        op.nd.r = r;
        op.nd.t = t;
        op.nd.ldt = 2 * r;
        op.nd.scale = m->scale;
        op.nd.gate_row0 = Mv;
        P->ops.push_back(op);
      } else if (!fold_norm) {
        norm(base + L.h, base + L.n);
      }
      if ((s = linear(fold_norm ? base + L.h : base + L.n, m->hidden, 2, which, l, y, ld,
                      kEpiSiluPair, nullptr, M, fold, fold_norm ? ss_at(2 * l + 1) : nullptr)) != UNO_OK)
        return s;
    }
    {
      const int which[1] = {kDown};
      void* y[1] = {base + L.h};
      const int64_t ld[1] = {m->hidden};
      if ((s = linear(base + L.act, m->inter, 1, which, l, y, ld, kEpiAdd, nullptr, M, false,
                      nullptr, fold_norm ? ss_at(2 * l + 2) : nullptr)) != UNO_OK)
        return s;
    }
    P->block_end.push_back(P->ops.size());
  }
  if (!q_next) return UNO_OK;   // decoder layers only
  if (!fold_norm) norm(base + L.h, base + L.n);
  void* p_dst = logits_out ? logits_out : base + L.logits;
  const int which[1] = {0};
  void* y[1] = {p_dst};
  const int64_t ld[1] = {m->vocab};
  return linear(fold_norm ? base + L.h : base + L.n, m->hidden, 1, which, -1, y, ld, kEpiStore,
                q_next, Mv, false, fold_norm ? ss_at(2 * m->n_layers) : nullptr);
}

uno_model::Plan* find_plan(uno_model* m, int32_t B, int32_t k, void* ws, void* q_next,
                           void* logits_out, uno_status* st) {
  for (size_t i = 0; i < m->plans.size(); ++i) {
    uno_model::Plan* p = m->plans[i].get();
    if (p->B == B && p->k == k && p->ws == ws && p->q_next == q_next &&
        p->logits_out == logits_out) {
      if (i + 1 != m->plans.size()) {
        std::unique_ptr<uno_model::Plan> keep = std::move(m->plans[i]);
        m->plans.erase(m->plans.begin() + static_cast<long>(i));
        m->plans.push_back(std::move(keep));
      }
      *st = UNO_OK;
      return m->plans.back().get();
    }
  }
  std::unique_ptr<uno_model::Plan> p(new uno_model::Plan());
  *st = build_plan(m, B, k, ws, q_next, logits_out, p.get());
  if (*st != UNO_OK) return nullptr;
  if (m->plans.size() >= 4) m->plans.erase(m->plans.begin());
  m->plans.push_back(std::move(p));
  return m->plans.back().get();
}

}  // namespace
}  // namespace uno

extern "C" {

uno_status uno_model_create(uno_model** out, int32_t n_layers, int32_t hidden, int32_t q_out,
                            int32_t kv_out, int32_t inter, int32_t vocab, int32_t r, float scale,
                            const void* const* weights) {
  if (!out) return set_error(UNO_ERR_INVALID_ARG, "out is NULL");
  *out = nullptr;
  if (n_layers < 0 || hidden < 8 || q_out < 8 || kv_out < 8 || inter < 8 || vocab < 2 || r < 0)
    return set_error(UNO_ERR_INVALID_ARG, "bad model sizes");
  if (hidden % 8 || q_out % 8 || kv_out % 8 || inter % 8 || vocab % 8 || r % 8)
    return set_error(UNO_ERR_UNSUPPORTED, "model sizes must be multiples of 8");
  if (r > 256) return set_error(UNO_ERR_UNSUPPORTED, "rank r=%d > 256", r);
  if (vocab > 196608) return set_error(UNO_ERR_UNSUPPORTED, "vocab=%d > 196608", vocab);
  if (!weights) return set_error(UNO_ERR_INVALID_ARG, "weights is NULL");
  const size_t nw = static_cast<size_t>(n_layers) * kLinPerLayer * 3 + 3;
  for (size_t i = 0; i < nw; ++i) {
    const bool lora_part = (i % 3) != 0;
    if ((!weights[i] && !(lora_part && r == 0)) || (weights[i] && !aligned16(weights[i])))
      return set_error(UNO_ERR_INVALID_ARG, "weight pointer %zu is NULL or unaligned", i);
  }
  uno_model* m = new uno_model();
  m->n_layers = n_layers;
  m->hidden = hidden;
  m->q_out = q_out;
  m->kv_out = kv_out;
  m->inter = inter;
  m->vocab = vocab;
  m->r = r;
  m->scale = scale;
  m->w.assign(weights, weights + nw);
  *out = m;
  return UNO_OK;
}

void uno_model_destroy(uno_model* m) { delete m; }

size_t uno_psi_step_workspace(const uno_model* m, int32_t B, int32_t k) {
  if (!m || B < 1 || k < 1 || k > 32) return 0;
  return step_layout(m, B, k).total;
}

int32_t uno_psi_step_kernel_count(const uno_model* m, int32_t B, int32_t k) {
  if (!m || B < 1 || k < 1) return 0;
  // per layer: 2 rmsnorm + 4 GEMM launches, each with a separate
  // down-projection launch unless the GEMM computes t itself; then rmsnorm +
  // LM head; verify (2 kernels) + draft (2)
  std::lock_guard<std::mutex> lock(const_cast<uno_model*>(m)->mu);
  for (const auto& p : m->plans)
    if (p->B == B && p->k == k && p->q_next) return static_cast<int32_t>(p->ops.size()) + 4;
  return 0;
}

uno_status uno_psi_step(uno_model* m, int32_t B, int32_t k, const void* h_in, const void* q_prev,
                        const int32_t* d_prev, float temperature, uint64_t seed, uint64_t step,
                        uint64_t seq_offset, void* q_next, int32_t* d_next, void* logits_out,
                        int32_t* accepted_len, int32_t* out_tokens, int32_t* out_count,
                        int32_t* dev_status, void* workspace, size_t ws_bytes, void* stream) {
  if (!m) return set_error(UNO_ERR_INVALID_ARG, "model is NULL");
  uno_status s = check_sampler(UNO_BF16, B, k, m->vocab, temperature);
  if (s != UNO_OK) return s;
  if (B < 1) return set_error(UNO_ERR_INVALID_ARG, "B must be >= 1");
  if ((seq_offset + static_cast<uint64_t>(B)) * static_cast<uint64_t>(k + 1) > (1ull << 32))
    return set_error(UNO_ERR_UNSUPPORTED, "(seq_offset + B) * (k + 1) must be <= 2^32");
  if (static_cast<int64_t>(B) * (2 * k + 1) > (1ll << 30))
    return set_error(UNO_ERR_UNSUPPORTED, "too many rows");
  if (!h_in || !q_prev || !d_prev || !q_next || !d_next || !accepted_len || !out_tokens ||
      !out_count)
    return set_error(UNO_ERR_INVALID_ARG, "NULL input or output pointer");
  if (!aligned16(h_in) || !aligned16(q_prev) || !aligned16(q_next) ||
      (logits_out && !aligned16(logits_out)))
    return set_error(UNO_ERR_INVALID_ARG, "h_in, q_prev, q_next and logits_out must be 16-byte aligned");
  if (q_prev == q_next) return set_error(UNO_ERR_INVALID_ARG, "q_next must not alias q_prev");
  const StepLayout L = step_layout(m, B, k);
  if (!workspace || ws_bytes < L.total || !aligned16(workspace))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", L.total, ws_bytes);

  std::lock_guard<std::mutex> lock(m->mu);
  uno_model::Plan* P = find_plan(m, B, k, workspace, q_next, logits_out, &s);
  if (!P) return s;
  cudaStream_t st = as_stream(stream);
  char* base = static_cast<char*>(workspace);
  const int64_t M = static_cast<int64_t>(B) * (2 * k + 1);
  cudaError_t e = cudaMemcpyAsync(base + L.h, h_in, static_cast<size_t>(M) * m->hidden * 2,
                                  cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return cuda_error(e, "copying h_in");
  if (L.sk_flag_bytes && (e = cudaMemsetAsync(base + L.sk_flag, 0, L.sk_flag_bytes, st)) != cudaSuccess)
    return cuda_error(e, "clearing the stream-K flags");
  // launch timing: event 0 before the first launch, event i + 1 after launch i
  const size_t n_ev = P->ops.size() + 3;
  const bool prof = m->profiling;
  if (prof) {
    int dev = 0;
    cudaGetDevice(&dev);
    if (m->prof_device >= 0 && m->prof_device != dev)
      return set_error(UNO_ERR_INVALID_ARG, "profiling on device %d, step on device %d",
                       m->prof_device, dev);
    m->prof_device = dev;
    while (m->events.size() < n_ev) {
      cudaEvent_t ev;
      if ((e = cudaEventCreate(&ev)) != cudaSuccess) return cuda_error(e, "creating a timing event");
      m->events.push_back(ev);
    }
    m->prof_kinds.clear();
    m->prof_dims.clear();
    m->prof_n = 0;
    if ((e = cudaEventRecord(m->events[0], st)) != cudaSuccess) return cuda_error(e, "recording an event");
  }
  auto mark = [&](int32_t kind, const int64_t* dims) -> uno_status {
    if (!prof) return UNO_OK;
    m->prof_kinds.push_back(kind);
    for (int i = 0; i < 4; ++i) m->prof_dims.push_back(dims ? dims[i] : 0);
    const cudaError_t er = cudaEventRecord(m->events[m->prof_kinds.size()], st);
    if (er != cudaSuccess) return cuda_error(er, "recording an event");
    m->prof_n = m->prof_kinds.size() + 1;
    return UNO_OK;
  };
  for (const StepOp& op : P->ops) {
    s = op.kind == 0 ? gemm_run(op.gemm, st)
        : op.kind == 1 ? rmsnorm_launch(M, m->hidden, op.x, op.y, kNormEps, st)
        : op.kind == 2 ? norm_down_launch(op.nd, M, st)
                       : row_sumsq_launch(M, m->hidden, op.x, static_cast<float*>(op.y), st);
    if (s != UNO_OK) return s;
    if ((s = mark(prof_kind(op), op.kind == 0 ? op.dims : nullptr)) != UNO_OK) return s;
  }

  VerifyArgs va{};
  va.dt = UNO_BF16;
  va.B = B;
  va.k = k;
  va.k_p = k + 1;
  va.V = m->vocab;
  va.p_logits = logits_out ? logits_out : static_cast<const void*>(base + L.logits);
  va.q_logits = q_prev;
  va.draft = d_prev;
  va.temperature = temperature;
  va.seed = seed;
  va.step = step;
  va.seq_offset = seq_offset;
  va.accepted_len = accepted_len;
  va.out_tokens = out_tokens;
  va.out_count = out_count;
  va.dev_status = dev_status;
  if ((s = verify_launch(va, base + L.vstat, st)) != UNO_OK) return s;
  if ((s = mark(kProfVerify, nullptr)) != UNO_OK) return s;

  DraftArgs da{};
  da.dt = UNO_BF16;
  da.B = B;
  da.k = k;
  da.V = m->vocab;
  da.q_logits = q_next;
  da.temperature = temperature;
  da.seed = seed;
  da.step = step;
  da.seq_offset = seq_offset;
  da.draft = d_next;
  da.dev_status = dev_status;
  if ((s = draft_launch(da, base + L.dstat, st)) != UNO_OK) return s;
  return mark(kProfDraft, nullptr);
}

uno_status uno_model_profile(uno_model* m, int32_t enable) {
  if (!m) return set_error(UNO_ERR_INVALID_ARG, "model is NULL");
  std::lock_guard<std::mutex> lock(m->mu);
  m->profiling = enable != 0;
  m->prof_n = 0;
  return UNO_OK;
}

uno_status uno_model_last_profile(uno_model* m, int32_t cap, float* ms, int32_t* kind,
                                  int64_t* dims, int32_t* n_out) {
  if (!m || !n_out) return set_error(UNO_ERR_INVALID_ARG, "model or n_out is NULL");
  std::lock_guard<std::mutex> lock(m->mu);
  const int32_t n = m->prof_n > 0 ? static_cast<int32_t>(m->prof_n - 1) : 0;
  *n_out = n;
  if (n == 0 || !ms) return UNO_OK;   // ms == NULL: the count only
  if (cap < n || !kind) return set_error(UNO_ERR_INVALID_ARG, "cap=%d below the %d entries", cap, n);
  int cur = -1;
  cudaGetDevice(&cur);
  if (m->prof_device >= 0 && (cur != m->prof_device))
    return set_error(UNO_ERR_INVALID_ARG, "read the profile on device %d", m->prof_device);
  cudaError_t e = cudaEventSynchronize(m->events[static_cast<size_t>(n)]);
  if (e != cudaSuccess) return cuda_error(e, "waiting for the profiled step");
  for (int32_t i = 0; i < n; ++i) {
    if ((e = cudaEventElapsedTime(&ms[i], m->events[static_cast<size_t>(i)],
                                  m->events[static_cast<size_t>(i) + 1])) != cudaSuccess)
      return cuda_error(e, "reading a timing event");
    kind[i] = m->prof_kinds[static_cast<size_t>(i)];
    if (dims)
      for (int j = 0; j < 4; ++j) dims[4 * i + j] = m->prof_dims[static_cast<size_t>(4 * i + j)];
  }
  return UNO_OK;
}

uno_status uno_psi_step_hidden(uno_model* m, int32_t B, int32_t k, const void* h_in,
                               int32_t n_blocks, void* h_out, void* q_out, void* k_out,
                               void* v_out, void* act_out, void* workspace, size_t ws_bytes,
                               void* stream) {
  if (!m) return set_error(UNO_ERR_INVALID_ARG, "model is NULL");
  if (B < 1 || k < 1 || k > 32)
    return set_error(UNO_ERR_INVALID_ARG, "B=%d must be >= 1 and k=%d in [1, 32]", B, k);
  if (n_blocks < 0 || n_blocks > 2 * m->n_layers)
    return set_error(UNO_ERR_INVALID_ARG, "n_blocks=%d outside [0, %d]", n_blocks,
                     2 * m->n_layers);
  if ((q_out || k_out || v_out) && n_blocks < 1)
    return set_error(UNO_ERR_INVALID_ARG, "q/k/v outputs need n_blocks >= 1");
  if (act_out && n_blocks < 2) return set_error(UNO_ERR_INVALID_ARG, "act_out needs n_blocks >= 2");
  if (static_cast<int64_t>(B) * (2 * k + 1) > (1ll << 30))
    return set_error(UNO_ERR_UNSUPPORTED, "too many rows");
  if (!h_in || !h_out) return set_error(UNO_ERR_INVALID_ARG, "NULL h_in or h_out");
  if (!aligned16(h_in) || !aligned16(h_out))
    return set_error(UNO_ERR_INVALID_ARG, "h_in and h_out must be 16-byte aligned");
  const StepLayout L = step_layout(m, B, k);
  if (!workspace || ws_bytes < L.total || !aligned16(workspace))
    return set_error(UNO_ERR_WORKSPACE, "workspace must hold %zu bytes (got %zu)", L.total, ws_bytes);
  std::lock_guard<std::mutex> lock(m->mu);
  uno_status s;
  uno_model::Plan* P = find_plan(m, B, k, workspace, nullptr, nullptr, &s);
  if (!P) return s;
  cudaStream_t st = as_stream(stream);
  char* base = static_cast<char*>(workspace);
  const size_t M = static_cast<size_t>(B) * (2 * k + 1);
  cudaError_t e = cudaMemcpyAsync(base + L.h, h_in, M * m->hidden * 2, cudaMemcpyDeviceToDevice, st);
  if (e != cudaSuccess) return cuda_error(e, "copying h_in");
  if (L.sk_flag_bytes && (e = cudaMemsetAsync(base + L.sk_flag, 0, L.sk_flag_bytes, st)) != cudaSuccess)
    return cuda_error(e, "clearing the stream-K flags");
  const size_t n_ops = n_blocks > 0 ? P->block_end[static_cast<size_t>(n_blocks) - 1] : 0;
  for (size_t i = 0; i < n_ops; ++i) {
    const StepOp& op = P->ops[i];
    s = op.kind == 0 ? gemm_run(op.gemm, st)
        : op.kind == 1 ? rmsnorm_launch(static_cast<int64_t>(M), m->hidden, op.x, op.y, kNormEps, st)
        : op.kind == 2 ? norm_down_launch(op.nd, static_cast<int64_t>(M), st)
                       : row_sumsq_launch(static_cast<int64_t>(M), m->hidden, op.x,
                                          static_cast<float*>(op.y), st);
    if (s != UNO_OK) return s;
  }
  // the step's buffers still hold the last sub-blocks' products
  const struct { void* dst; size_t off, width; } outs[] = {
      {h_out, L.h, static_cast<size_t>(m->hidden)}, {q_out, L.q, static_cast<size_t>(m->q_out)},
      {k_out, L.k, static_cast<size_t>(m->kv_out)}, {v_out, L.v, static_cast<size_t>(m->kv_out)},
      {act_out, L.act, static_cast<size_t>(m->inter)}};
  for (const auto& o : outs) {
    if (!o.dst) continue;
    e = cudaMemcpyAsync(o.dst, base + o.off, M * o.width * 2, cudaMemcpyDeviceToDevice, st);
    if (e != cudaSuccess) return cuda_error(e, "copying a hidden-state output");
  }
  return UNO_OK;
}

}  // extern "C"
