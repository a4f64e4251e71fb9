// Gradients of the gated-LoRA adapter with the AR weights frozen (bf16).
//
// The adapter theta_Delta is what the distillation stage trains while the AR
// weights stay fixed (hyper.ai page, section "方法", the training-order
// paragraph). For y = x W^T + s g (.) (x A^T) Bl^T and an output gradient dy:
//   t_u = x A^T              [M, r]      u = dy Bl            [M, r]
//   dBl = sum_m s g_m dy[m,:]^T t_u[m,:]  = (s g (.) dy)^T t_u       [N, r]
//   dA  = sum_m s g_m u[m,:]^T x[m,:]     = u^T (s g (.) x)          [r, K]
// All four products are dense contractions and run on the tensor-core GEMM
// kernels of this library, which take K-major operands (the contracted index
// contiguous). Contractions over the M rows need M contiguous, so x and dy
// are transposed once, with the row factor s g_m folded into the copy, and
// Bl once to put N contiguous:
//   xs^T  = (s g (.) x)^T  [K, Mp]   dys^T = (s g (.) dy)^T  [N, Mp]   Bl^T [r, N]
//   t_u^T = A   . x^T   as y = X W^T with X = A     [r, K],  W = x     [M, K]
//   u^T   = Bl^T . dy^T  as y = X W^T with X = Bl^T [r, N],  W = dy    [M, N]
//   dBl   = dys^T . t_u  as y = X W^T with X = dys^T [N, Mp], W = t_u^T [r, Mp]
//   dA    = u^T . xs     as y = X W^T with X = u^T  [r, Mp], W = xs^T  [K, Mp]
// Mp = M rounded up to 64; the padding columns are zero so the contractions
// over Mp equal those over M. t_u^T and u^T are rounded to bf16 (they are
// tensor-core operands), as t is in the forward pass.
#include <algorithm>

#include "common.cuh"
#include "internal.h"

namespace uno {

namespace {

constexpr int kTile = 64;

// out[c, r] = f(r) in[r, c] for r < R, c < C (out row stride ld_out >= R);
// out[c, r] = 0 for R <= r < ld_out, and rows with f(r) = 0 are not read. f(r) = scale * gate(r) when gated
// (gate[r], or r >= gate_row0 without a gate vector), else 1. One 64 x 64
// tile per CTA of 256 threads, staged in shared memory so that both the
// reads and the writes are row-contiguous.
__global__ void __launch_bounds__(256)
    transpose_scale_kernel(const __nv_bfloat16* __restrict__ in, int R, int C, int ld_in,
                           __nv_bfloat16* __restrict__ out, int ld_out, int gated,
                           const uint8_t* __restrict__ gate, int gate_row0, float scale) {
  __shared__ float tile[kTile][kTile + 1];
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const int c0 = blockIdx.x * kTile, r0 = blockIdx.y * kTile;
#pragma unroll
  for (int i = 0; i < kTile / 8; ++i) {
    const int rl = ty + 8 * i, r = r0 + rl;
    float f = 1.f;
    if (gated && r < R) f = scale * (gate ? static_cast<float>(gate[r]) : (r >= gate_row0 ? 1.f : 0.f));
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int cl = 2 * tx + h, c = c0 + cl;
      float v = 0.f;
      if (r < R && c < C && f != 0.f) v = f * __bfloat162float(in[static_cast<size_t>(r) * ld_in + c]);
      tile[rl][cl] = v;
    }
  }
  cta_sync();
#pragma unroll
  for (int i = 0; i < kTile / 8; ++i) {
    const int cl = ty + 8 * i, c = c0 + cl;
    if (c >= C) continue;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rl = 2 * tx + h, r = r0 + rl;
      if (r < ld_out) out[static_cast<size_t>(c) * ld_out + r] = __float2bfloat16_rn(tile[rl][cl]);
    }
  }
}

uno_status transpose_launch(const void* in, int64_t R, int64_t C, int64_t ld_in, void* out,
                            int64_t ld_out, bool gated, const uint8_t* gate, int64_t gate_row0,
                            float scale, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((C + kTile - 1) / kTile),
                  static_cast<unsigned>((ld_out + kTile - 1) / kTile));
  const cudaError_t e = launch_kernel(
      transpose_scale_kernel, grid, dim3(256), 0, s, 1, static_cast<const __nv_bfloat16*>(in),
      static_cast<int>(R), static_cast<int>(C), static_cast<int>(ld_in),
      static_cast<__nv_bfloat16*>(out), static_cast<int>(ld_out), gated ? 1 : 0, gate,
      static_cast<int>(gate_row0), scale);
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "transpose launch");
}

size_t align256(size_t v) { return (v + 255) / 256 * 256; }

struct BackwardLayout {
  size_t xT, dyT, blT, tT, uT, total;
  int64_t Mp;
};

BackwardLayout backward_layout(int64_t M, int64_t K, int64_t N, int32_t r) {
  BackwardLayout L{};
  L.Mp = (M + kTile - 1) / kTile * kTile;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align256(bytes);
    return o;
  };
  L.xT = take(static_cast<size_t>(K) * L.Mp * 2);
  L.dyT = take(static_cast<size_t>(N) * L.Mp * 2);
  L.blT = take(static_cast<size_t>(r) * N * 2);
  L.tT = take(static_cast<size_t>(r) * L.Mp * 2);
  L.uT = take(static_cast<size_t>(r) * L.Mp * 2);
  L.total = off;
  return L;
}

// y [rows, ldy] (n columns) = X [rows, K] . W [n, K]^T, bf16, plain store.
uno_status plain_gemm(int64_t rows, int64_t K, int64_t n, const void* X, const void* Wt, void* y,
                      int64_t ldy, cudaStream_t s) {
  GemmProblem pm{};
  pm.dt = UNO_BF16;
  pm.M = rows;
  pm.K = K;
  pm.r = 0;
  pm.x = X;
  pm.ngroups = 1;
  pm.g[0] = GemmGroup{Wt, nullptr, n, y, ldy, 0};
  pm.mode = kEpiStore;
  pm.M0 = rows;
  pm.scale = 1.f;
  GemmLaunch l{};
  uno_status st = gemm_prepare(pm, &l);
  if (st != UNO_OK) return st;
  return gemm_run(l, s);
}

}  // namespace

size_t adapter_backward_workspace(int64_t M, int64_t K, int64_t N, int32_t r) {
  return backward_layout(M, K, N, r).total;
}

uno_status adapter_backward_launch(int64_t M, int64_t K, int64_t N, int32_t r, const void* x,
                                   const void* dy, const void* A, const void* Bl,
                                   const uint8_t* gate, float scale, void* dA, void* dBl,
                                   void* ws, cudaStream_t s) {
  const BackwardLayout L = backward_layout(M, K, N, r);
  char* base = static_cast<char*>(ws);
  void* xT = base + L.xT;
  void* dyT = base + L.dyT;
  void* blT = base + L.blT;
  void* tT = base + L.tT;
  void* uT = base + L.uT;
  uno_status st;
  // t_u^T and u^T are written on columns [0, M) only: their padding must read zero
  cudaError_t e = cudaMemsetAsync(tT, 0, L.uT + static_cast<size_t>(r) * L.Mp * 2 - L.tT, s);
  if (e != cudaSuccess) return cuda_error(e, "clearing the backward workspace");
  if ((st = transpose_launch(x, M, K, K, xT, L.Mp, true, gate, M, scale, s)) != UNO_OK) return st;
  if ((st = transpose_launch(dy, M, N, N, dyT, L.Mp, true, gate, M, scale, s)) != UNO_OK) return st;
  if ((st = transpose_launch(Bl, N, r, r, blT, N, false, nullptr, 0, 1.f, s)) != UNO_OK) return st;
  if ((st = plain_gemm(r, K, M, A, x, tT, L.Mp, s)) != UNO_OK) return st;        // t_u^T
  if ((st = plain_gemm(r, N, M, blT, dy, uT, L.Mp, s)) != UNO_OK) return st;     // u^T
  if ((st = plain_gemm(N, L.Mp, r, dyT, tT, dBl, r, s)) != UNO_OK) return st;    // dBl
  return plain_gemm(r, L.Mp, K, uT, xT, dA, K, s);                              // dA
}

}  // namespace uno
