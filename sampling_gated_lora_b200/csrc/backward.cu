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

// One transpose of a launch: out[c, r] = f(r) in[r, c] for r < R, c < C (out
// row stride ld_out >= R, a multiple of 8); out[c, r] = 0 for R <= r < ld_out.
// f(r) = scale * gate(r) when gated (gate[r], or r >= gate_row0 without a gate
// vector), else 1; rows with f(r) = 0 are not read. C, ld_in and ld_out are
// multiples of 8 and the bases 16-byte aligned (16-byte vectors throughout).
struct TransposeJob {
  const __nv_bfloat16* in;
  __nv_bfloat16* out;
  int R, C, ld_in, ld_out, gated;
  int tiles_c, tile0;   // 64 x 64 tiles: tiles_c across C; first tile of the job in the grid
};
struct TransposeArgs {
  TransposeJob job[3];
  int njobs;
  const uint8_t* gate;
  int gate_row0;
  float scale;
};

// One 64 x 64 tile per CTA of 256 threads: each thread reads two 16-byte
// vectors (rows t/8 and t/8 + 32, columns 8 (t%8) ..), scales them in float
// into a padded shared tile, and writes two 16-byte vectors of the transposed
// tile (output rows t/8 and t/8 + 32). With 65 floats a row, both the row
// writes and the column reads of a warp touch 32 different banks.
__global__ void __launch_bounds__(256)
    transpose_scale_kernel(const __grid_constant__ TransposeArgs a) {
  __shared__ float tile[kTile][kTile + 1];
  if (threadIdx.x == 0) pdl_trigger();
  int j = 0;
#pragma unroll
  for (int i = 1; i < 3; ++i)
    if (i < a.njobs && static_cast<int>(blockIdx.x) >= a.job[i].tile0) j = i;
  const TransposeJob& J = a.job[j];
  const int t = static_cast<int>(blockIdx.x) - J.tile0;
  const int c0 = (t % J.tiles_c) * kTile, r0 = (t / J.tiles_c) * kTile;
  const int v = threadIdx.x & 7, rr = threadIdx.x >> 3;
  pdl_wait();
  // row factors first, then all four loads in flight at once
  float f[2];
  uint4 w[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = r0 + rr + 32 * h;
    f[h] = 0.f;
    if (r < J.R)
      f[h] = J.gated ? a.scale * (a.gate ? static_cast<float>(a.gate[r]) : (r >= a.gate_row0 ? 1.f : 0.f))
                     : 1.f;
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = r0 + rr + 32 * h, c = c0 + 8 * v;
    w[h] = make_uint4(0u, 0u, 0u, 0u);
    if (f[h] != 0.f && c < J.C)
      w[h] = __ldg(reinterpret_cast<const uint4*>(J.in + static_cast<size_t>(r) * J.ld_in + c));
  }
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint32_t ws[4] = {w[h].x, w[h].y, w[h].z, w[h].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      tile[rr + 32 * h][8 * v + 2 * q] = f[h] * bf16_lo(ws[q]);
      tile[rr + 32 * h][8 * v + 2 * q + 1] = f[h] * bf16_hi(ws[q]);
    }
  }
  cta_sync();
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int c = c0 + rr + 32 * h, r = r0 + 8 * v;
    if (c >= J.C || r >= J.ld_out) continue;
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const __nv_bfloat162 p = __floats2bfloat162_rn(tile[8 * v + 2 * q][rr + 32 * h],
                                                     tile[8 * v + 2 * q + 1][rr + 32 * h]);
      o[q] = *reinterpret_cast<const uint32_t*>(&p);
    }
    *reinterpret_cast<uint4*>(J.out + static_cast<size_t>(c) * J.ld_out + r) =
        make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// Adds a job (in [R, C] -> out [C, ld_out]) to a transpose launch.
void add_job(TransposeArgs* a, const void* in, int64_t R, int64_t C, int64_t ld_in, void* out,
             int64_t ld_out, bool gated) {
  TransposeJob& J = a->job[a->njobs];
  J.in = static_cast<const __nv_bfloat16*>(in);
  J.out = static_cast<__nv_bfloat16*>(out);
  J.R = static_cast<int>(R);
  J.C = static_cast<int>(C);
  J.ld_in = static_cast<int>(ld_in);
  J.ld_out = static_cast<int>(ld_out);
  J.gated = gated ? 1 : 0;
  J.tiles_c = static_cast<int>((C + kTile - 1) / kTile);
  J.tile0 = a->njobs == 0 ? 0 : a->job[a->njobs - 1].tile0 +
                                    a->job[a->njobs - 1].tiles_c *
                                        ((a->job[a->njobs - 1].ld_out + kTile - 1) / kTile);
  ++a->njobs;
}

uno_status transpose_launch(const TransposeArgs& a, cudaStream_t s) {
  const TransposeJob& L = a.job[a.njobs - 1];
  const unsigned tiles = static_cast<unsigned>(L.tile0 + L.tiles_c * ((L.ld_out + kTile - 1) / kTile));
  const cudaError_t e = launch_kernel(transpose_scale_kernel, dim3(tiles), dim3(256), 0, s, 1, a);
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
  // one launch transposes x and dy (gated, scaled) and Bl
  TransposeArgs ta{};
  ta.gate = gate;
  ta.gate_row0 = static_cast<int>(M);
  ta.scale = scale;
  add_job(&ta, x, M, K, K, xT, L.Mp, true);
  add_job(&ta, dy, M, N, N, dyT, L.Mp, true);
  add_job(&ta, Bl, N, r, r, blT, N, false);
  if ((st = transpose_launch(ta, s)) != UNO_OK) return st;
  if ((st = plain_gemm(r, K, M, A, x, tT, L.Mp, s)) != UNO_OK) return st;        // t_u^T
  if ((st = plain_gemm(r, N, M, blT, dy, uT, L.Mp, s)) != UNO_OK) return st;     // u^T
  if ((st = plain_gemm(N, L.Mp, r, dyT, tT, dBl, r, s)) != UNO_OK) return st;    // dBl
  return plain_gemm(r, L.Mp, K, uT, xT, dA, K, s);                              // dA
}

}  // namespace uno
