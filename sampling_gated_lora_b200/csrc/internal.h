// Host-side declarations shared by the C-ABI layer and the kernel files.
#pragma once

#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/uno.h"

namespace uno {

// ---------------------------------------------------------------- errors
uno_status set_error(uno_status st, const char* fmt, ...);
uno_status cuda_error(cudaError_t e, const char* what);

// ---------------------------------------------------------------- gated GEMM

enum EpilogueMode : int {
  kEpiStore = 0,     // y = acc
  kEpiAdd = 1,       // y = y + acc (in place: the residual add)
  kEpiRowScale = 2,  // y = scale * gate[m] * acc   (the gated LoRA down-projection)
  kEpiSiluPair = 3,  // groups 0 (gate) and 1 (up): y0 = silu(acc_gate) * acc_up
};

constexpr int kMaxGroups = 3;

// One output group of a GEMM launch: its weights, adapter and output.
struct GemmGroup {
  const void* W;          // [N, K]
  const void* Bl;         // [N, r]  (unused when r == 0)
  int64_t N;
  void* y;                // [M, ldy], features [0, N)
  int64_t ldy;
  int64_t t_col;          // first column of this group's rank-r block in t
};

// One launch of the gated-LoRA GEMM over up to kMaxGroups linears that share
// the input x (and its LoRA activations t):
//   y_g[m, n] = epi( sum_k x[m,k] W_g[n,k] + sum_j t[m, t_col_g + j] Bl_g[n,j] )
// Group 0 rows m >= M0 are written to y1 (row m - M0) instead of y_0.
struct GemmProblem {
  uno_dtype dt;
  const void* A[kMaxGroups];   // adapters' A [r, K]: lets a decode-size launch fuse the down-projection
  int64_t M, K;
  int32_t r;              // LoRA rank per group (0: no LoRA term)
  const void* x;          // [M, K]
  const void* t;          // [M, ldt] rank-r activations, already gated and scaled
  int64_t ldt;
  int ngroups;
  GemmGroup g[kMaxGroups];
  int mode;
  void* y1;
  int64_t M0;
  const uint8_t* gate;    // kEpiRowScale; NULL: gate[m] = (m >= gate_row0)
  int64_t gate_row0;
  float scale;            // kEpiRowScale
  // The launch right before this one is the down-projection that writes t and
  // only triggers its dependents once the writer of x has finished: x may be
  // read at once, and only t must wait (so the two launches overlap).
  bool x_ready;
  // Stream-K scratch of the CTA-pair kernel (NULL: whole tiles only). The
  // partial sums may be shared by launches of one stream; the flags are this
  // launch's own and must be zero when it starts (see pair_sk_bytes).
  float* sk_part;
  int32_t* sk_flag;
  int sk_slots;           // pairs the scratch serves
  // Words this launch sets to zero once it has waited for its predecessor: a
  // down-projection clears the stream-K flags of the GEMM launched behind it.
  int32_t* zero_flags;
  int zero_words;
  // RMSNorm folded into the GEMMs around it (CTA-pair kernel only). in_ss:
  // x is an unnormalised residual stream whose rows' sums of squares come as
  // in_ss_cols partials per row ([M, in_ss_cols] floats, added in order); every
  // output row is scaled by 1 / sqrt(sum / norm_dim + norm_eps), which equals
  // the GEMM of the normalised rows (the adapter term included, t being
  // computed from the same unnormalised x). out_ss (kEpiAdd): the launch
  // writes, per row and 256-column feature tile, the sum of squares of the
  // bf16 values it stores ([M, feature tiles] floats).
  const float* in_ss;
  int in_ss_cols;
  float* out_ss;
  int64_t norm_dim;
  float norm_eps;
  // Non-NULL: the CTA-pair kernel may compute t = scale * gate * (x A_g^T)
  // itself (A[] and t above; r <= 128, 16 or more 256-row blocks, see
  // gemm_pair_prepare), counting the finished parts of each 256-row block
  // here: ceil(M / 256) words that are zero when the launch starts.
  // GemmLaunch::computes_t tells the caller whether it does.
  int32_t* t_ready;
};

// All tensor maps of one launch (passed to the kernel as one parameter).
// a[] (the adapters' A matrices) is used by the kernels that compute t themselves.
struct TensorMaps {
  CUtensorMap x, t, w[kMaxGroups], b[kMaxGroups], a[kMaxGroups];
};

constexpr size_t kLaunchParamBytes = 320;

// Cached launch of a GemmProblem (tensor maps + grid); valid while the
// pointers of the problem stay the same.
struct GemmLaunch {
  TensorMaps tm;
  alignas(8) unsigned char params[kLaunchParamBytes];
  int kind;               // 0: one-CTA kernel, 1: persistent CTA-pair kernel
  int swap;
  int grid_x, grid_y, splits;
  int smem_bytes;
  int dtype;
  int32_t* sk_flag;       // stream-K flags this launch reads: zero them before it runs (or NULL)
  size_t sk_flag_bytes;
  int32_t* t_ready;       // the t counters (computes_t): zero them before it runs
  size_t t_ready_bytes;
  bool computes_t;        // the launch writes t itself: no separate down-projection
};

uno_status gemm_prepare(const GemmProblem& pb, GemmLaunch* out);
uno_status gemm_run(const GemmLaunch& l, cudaStream_t stream);
// Row-major [rows, inner] tensor map: box = 128 bytes of K x box_rows rows, 128-byte swizzle.
uno_status make_map(CUtensorMap* tm, uno_dtype dt, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride_elems, uint32_t box_rows);
// The persistent CTA-pair kernel (bf16, 256x256 tiles): whether it takes the
// problem, its preparation and its launch.
bool gemm_pair_suits(const GemmProblem& pb);
// Stream-K scratch of the CTA-pair kernel on this device: the fp32 partial
// tiles (one per pair) and one launch's flags (eight words per pair).
size_t pair_sk_part_bytes();
size_t pair_sk_flag_bytes();
int pair_sk_slots();
// The t counters of a CTA-pair launch over M rows (GemmProblem::t_ready).
size_t pair_t_ready_bytes(int64_t M);
uno_status gemm_pair_prepare(const GemmProblem& pb, GemmLaunch* out);
uno_status gemm_pair_run(const GemmLaunch& l, cudaStream_t stream);
// The fused decode kernel (bf16, M <= 256, r <= 128): computes t = scale * gate
// * (x A^T) in the same launch, so no separate down-projection is needed.
bool gemm_dec_suits(const GemmProblem& pb);
uno_status gemm_dec_prepare(const GemmProblem& pb, GemmLaunch* out);
uno_status gemm_dec_run(const GemmLaunch& l, cudaStream_t stream);

// ---------------------------------------------------------------- sampler

struct VerifyArgs {
  uno_dtype dt;
  int32_t B, k, k_p, V;
  const void* p_logits;
  const void* q_logits;
  const int32_t* draft;
  float temperature;
  uint64_t seed, step, seq_offset;
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* out_count;
  int32_t* dev_status;
};
struct DistillArgs {
  uno_dtype dt;
  int32_t rows, V;
  const void* z_teacher;   // [rows, V]
  const void* z_student;   // [rows, V]
  float alpha, beta, temperature;
  float* losses;           // [rows, 2]
  float* grad;             // [rows, V] or NULL
  int32_t* dev_status;
};
uno_status distill_launch(const DistillArgs& a, cudaStream_t s);

size_t verify_workspace(int32_t B, int32_t k, int32_t k_p, int32_t V);
uno_status verify_launch(const VerifyArgs& a, void* ws, cudaStream_t s);

struct TreeVerifyArgs {
  uno_dtype dt;
  int32_t B, N, k, R, V, bonus;
  const void* p_logits;   // [B, R, V]: AR logits of the trie nodes
  const void* q_logits;   // [B, k, V]
  const int32_t* cands;   // [B, N, k]
  float temperature;
  uint64_t seed, step, seq_offset;
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* out_count;
  int32_t* dev_status;
};
size_t tree_verify_workspace(int32_t B, int32_t k, int32_t R, int32_t V);
uno_status tree_verify_launch(const TreeVerifyArgs& a, void* ws, cudaStream_t s);

struct DraftArgs {
  uno_dtype dt;
  int32_t B, k, V;
  const void* q_logits;
  float temperature;
  uint64_t seed, step, seq_offset;
  int32_t* draft;
  int32_t* dev_status;
};
size_t draft_workspace(int32_t B, int32_t k, int32_t V);
uno_status draft_launch(const DraftArgs& a, void* ws, cudaStream_t s);

uno_status philox_launch(uint64_t seed, uint64_t step, uint32_t stream_id, uint32_t index0,
                         int64_t n, uint32_t* words, float* u, cudaStream_t s);

// ---------------------------------------------------------------- glue
// Per row m and 256-column tile c of x [M, D] bf16: out[m * ceil(D / 256) + c]
// = sum of the squares of the tile's values (fp32), the layout a residual-add
// GEMM writes with GemmProblem::out_ss.
uno_status row_sumsq_launch(int64_t M, int64_t D, const void* x, float* out, cudaStream_t s);
uno_status rmsnorm_launch(int64_t M, int64_t D, const void* x, void* y, float eps,
                          cudaStream_t s);
uno_status silu_mul_launch(int64_t n, const void* a, const void* b, void* y, cudaStream_t s);

// RMSNorm of x into y plus the gated LoRA down-projection of y for G adapters
// into t (see rmsnorm_down_kernel); D % 8 == 0.
struct NormDownArgs {   // bf16 tensors
  const void* x;
  void* y;
  int D;
  float eps;
  const void* A[3];
  int G, r;
  void* t;
  int ldt;
  float scale;
  int64_t gate_row0;
};
uno_status norm_down_launch(const NormDownArgs& a, int64_t M, cudaStream_t s);

// Vocabulary-shard verification and draft (psi_verify.cu): the arguments of
// the uno_vp_* entry points of one device's shard [v0, v0 + Vs).
struct VpArgs {
  uno_dtype dt;
  int32_t B, k, k_p, Vs, v0, V, G, rank;
  float temperature;
  uint64_t seed, step, seq_offset;
  const void* p;            // this shard's AR logits [B, k_p, Vs]
  const void* q;            // this shard's draft logits [B, k, Vs]
  const int32_t* draft;     // [B, k] global ids
  const float* parts_p;     // [G, B k_p, 4]
  const float* parts_q;     // [G, B k, 4]
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* out_count;
  int32_t* draw;            // [B]
  float* draw_stats;        // [B, 4]
  double* masses;           // [B, 2] (this shard) or [G, B, 2] (all shards)
  int32_t* draft_out;       // [B k]
  int32_t* dev_status;
};
uno_status vp_partials_launch(uno_dtype dt, int rows, int Vs, int v0, const void* z,
                              const int32_t* draft, int k, int k_p, int id_kind, bool precise,
                              float temperature, float* out, cudaStream_t s);
uno_status vp_decide_launch(const VpArgs& a, cudaStream_t s);
uno_status vp_masses_launch(const VpArgs& a, cudaStream_t s);
uno_status vp_draw_launch(const VpArgs& a, cudaStream_t s);
uno_status vp_draft_draw_launch(const VpArgs& a, cudaStream_t s);

// Gradients of the gated-LoRA adapter (backward.cu): dA [r,K], dBl [N,r] bf16.
size_t adapter_backward_workspace(int64_t M, int64_t K, int64_t N, int32_t r);
uno_status adapter_backward_launch(int64_t M, int64_t K, int64_t N, int32_t r, const void* x,
                                   const void* dy, const void* A, const void* Bl,
                                   const uint8_t* gate, float scale, void* dA, void* dBl,
                                   void* ws, cudaStream_t s);

// The bounded-wait self-test (waits.cu).
uno_status wait_selftest_launch(int32_t which, uint64_t limit_ns, int32_t* result,
                                int32_t* status, cudaStream_t s);

int device_sm_count();

// Launch attributes shared by every kernel launch: programmatic stream
// serialisation (unless UNO_PDL=0 in the environment) and, when cluster_x *
// cluster_y * cluster_z > 1, the cluster shape. Returns the attribute count.
bool pdl_enabled();
inline int launch_attrs(cudaLaunchAttribute (&attr)[2], unsigned cluster_x = 1,
                        unsigned cluster_y = 1, unsigned cluster_z = 1) {
  int n = 0;
  if (cluster_x * cluster_y * cluster_z > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = cluster_y;
    attr[n].val.clusterDim.z = cluster_z;
    ++n;
  }
  if (pdl_enabled()) {
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
  }
  return n;
}

// Launch a kernel on `s` with the library's launch attributes (see launch_attrs).
template <typename... KArgs, typename... Args>
cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                          cudaStream_t s, unsigned cluster_x, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, cluster_x, 1, 1);
  cfg.attrs = attr;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace uno
