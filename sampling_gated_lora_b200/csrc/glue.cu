// Glue between the gated projections of the synthetic decode step (bf16,
// HBM-bound): RMSNorm without weight and silu(gate) * up.
#include "common.cuh"
#include "internal.h"

namespace uno {

namespace {

constexpr int kNormThreads = 256;

// One CTA per row: y = x / sqrt(mean(x^2) + eps), fp32 arithmetic.
__global__ void __launch_bounds__(kNormThreads)
    rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ y, int D,
                   float eps) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const size_t row = blockIdx.x;
  const __nv_bfloat16* xr = x + row * D;
  __nv_bfloat16* yr = y + row * D;
  const bool vec = (D % 8) == 0;
  float ss = 0.f;
  if (vec) {
    for (int i = threadIdx.x; i < D / 8; i += kNormThreads) {
      const uint4 w = reinterpret_cast<const uint4*>(xr)[i];
      const uint32_t a[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float lo = bf16_lo(a[e]), hi = bf16_hi(a[e]);
        ss += lo * lo + hi * hi;
      }
    }
  } else {
    for (int i = threadIdx.x; i < D; i += kNormThreads) {
      const float v = __bfloat162float(xr[i]);
      ss += v * v;
    }
  }
  ss = warp_sum(ss);
  __shared__ float red[kNormThreads / 32];
  __shared__ float s_inv;
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kNormThreads / 32; ++w) t += red[w];
    s_inv = 1.0f / sqrtf(t / static_cast<float>(D) + eps);
  }
  __syncthreads();
  const float inv = s_inv;
  if (vec) {
    for (int i = threadIdx.x; i < D / 8; i += kNormThreads) {
      const uint4 w = reinterpret_cast<const uint4*>(xr)[i];
      const uint32_t a[4] = {w.x, w.y, w.z, w.w};
      uint32_t o[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(bf16_lo(a[e]) * inv, bf16_hi(a[e]) * inv);
        o[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      reinterpret_cast<uint4*>(yr)[i] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    for (int i = threadIdx.x; i < D; i += kNormThreads)
      yr[i] = __float2bfloat16_rn(__bfloat162float(xr[i]) * inv);
  }
}

// RMSNorm of row blockIdx.x, with rmsnorm_kernel's arithmetic, and the gated
// LoRA down-projection of the normalised (bf16-rounded) row for 32 rows of the
// adapters' concatenated A (rows [32 blockIdx.y, +32)):
//   t[m, j] = bf16(scale * g_m * sum_k y[m, k] A[j, k]),  g_m = (m >= gate_row0)
// (the gated LoRA of hyper.ai page, section "方法"). Block y = 0 writes the
// normalised row. For decode-size batches, where it replaces a separate
// down-projection launch. D must be a multiple of 8.
constexpr int kNdRows = 32;

__global__ void __launch_bounds__(kNormThreads)
    rmsnorm_down_kernel(const NormDownArgs a) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const size_t row = blockIdx.x;
  const int D = a.D;
  const int nv = D / 8;
  const __nv_bfloat16* xr = static_cast<const __nv_bfloat16*>(a.x) + row * D;
  float ss = 0.f;
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    const uint4 w = reinterpret_cast<const uint4*>(xr)[i];
    const uint32_t q[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float lo = bf16_lo(q[e]), hi = bf16_hi(q[e]);
      ss += lo * lo + hi * hi;
    }
  }
  ss = warp_sum(ss);
  __shared__ float red[kNormThreads / 32];
  __shared__ float s_inv;
  __shared__ float s_dot[kNormThreads / 32][kNdRows];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  cta_sync();
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < kNormThreads / 32; ++w) t += red[w];
    s_inv = 1.0f / sqrtf(t / static_cast<float>(D) + a.eps);
  }
  cta_sync();
  const float inv = s_inv;
  const int j0 = blockIdx.y * kNdRows;
  const int rows_a = a.G * a.r;
  const __nv_bfloat16* arow[kNdRows];
#pragma unroll
  for (int jj = 0; jj < kNdRows; ++jj) {
    const int j = min(j0 + jj, rows_a - 1);   // rows past the end repeat the last; not stored
    arow[jj] = static_cast<const __nv_bfloat16*>(a.A[j / a.r == 0 ? 0 : (j / a.r == 1 ? 1 : 2)]) +
               static_cast<size_t>(j % a.r) * D;
  }
  float acc[kNdRows];
#pragma unroll
  for (int jj = 0; jj < kNdRows; ++jj) acc[jj] = 0.f;
  __nv_bfloat16* yr = static_cast<__nv_bfloat16*>(a.y) + row * D;
  for (int i = threadIdx.x; i < nv; i += kNormThreads) {
    const uint4 w = reinterpret_cast<const uint4*>(xr)[i];
    const uint32_t q[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[4];
    float n[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = __floats2bfloat162_rn(bf16_lo(q[e]) * inv, bf16_hi(q[e]) * inv);
      o[e] = *reinterpret_cast<uint32_t*>(&h);
      n[2 * e] = bf16_lo(o[e]);
      n[2 * e + 1] = bf16_hi(o[e]);
    }
    if (blockIdx.y == 0) reinterpret_cast<uint4*>(yr)[i] = make_uint4(o[0], o[1], o[2], o[3]);
#pragma unroll
    for (int jj = 0; jj < kNdRows; ++jj) {
      const uint4 b = __ldg(reinterpret_cast<const uint4*>(arow[jj]) + i);
      acc[jj] += n[0] * bf16_lo(b.x) + n[1] * bf16_hi(b.x) + n[2] * bf16_lo(b.y) +
                 n[3] * bf16_hi(b.y) + n[4] * bf16_lo(b.z) + n[5] * bf16_hi(b.z) +
                 n[6] * bf16_lo(b.w) + n[7] * bf16_hi(b.w);
    }
  }
#pragma unroll
  for (int jj = 0; jj < kNdRows; ++jj) {
    const float v = warp_sum(acc[jj]);
    if ((threadIdx.x & 31) == 0) s_dot[threadIdx.x >> 5][jj] = v;
  }
  cta_sync();
  if (threadIdx.x < kNdRows && j0 + static_cast<int>(threadIdx.x) < rows_a) {
    float t = 0.f;
    for (int w = 0; w < kNormThreads / 32; ++w) t += s_dot[w][threadIdx.x];
    const float g = static_cast<int64_t>(row) >= a.gate_row0 ? 1.f : 0.f;
    static_cast<__nv_bfloat16*>(a.t)[row * a.ldt + j0 + threadIdx.x] =
        __float2bfloat16_rn(a.scale * g * t);
  }
}

__device__ __forceinline__ float silu_mul(float a, float b) { return a / (1.0f + expf(-a)) * b; }

__global__ void silu_mul_kernel(const __nv_bfloat16* __restrict__ a,
                                const __nv_bfloat16* __restrict__ b,
                                __nv_bfloat16* __restrict__ y, int64_t n) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int64_t nv = n / 8;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < nv;
       i += stride) {
    const uint4 wa = reinterpret_cast<const uint4*>(a)[i];
    const uint4 wb = reinterpret_cast<const uint4*>(b)[i];
    const uint32_t xa[4] = {wa.x, wa.y, wa.z, wa.w}, xb[4] = {wb.x, wb.y, wb.z, wb.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      __nv_bfloat162 h = __floats2bfloat162_rn(silu_mul(bf16_lo(xa[e]), bf16_lo(xb[e])),
                                               silu_mul(bf16_hi(xa[e]), bf16_hi(xb[e])));
      o[e] = *reinterpret_cast<uint32_t*>(&h);
    }
    reinterpret_cast<uint4*>(y)[i] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  for (int64_t i = nv * 8 + blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += stride)
    y[i] = __float2bfloat16_rn(silu_mul(__bfloat162float(a[i]), __bfloat162float(b[i])));
}

}  // namespace

// One warp per (row, 256-column tile): the sum of the squares of the tile's
// bf16 values, fp32, in the layout of a residual-add GEMM's out_ss (so the
// first GEMM of a step with folded RMSNorm reads its input's scales the same
// way as every later one).
__global__ void __launch_bounds__(kNormThreads)
    row_sumsq_kernel(const __nv_bfloat16* __restrict__ x, int64_t M, int D, int cols,
                     float* __restrict__ out) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (kNormThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= M * cols) return;
  const int64_t m = w / cols;
  const int c = static_cast<int>(w - m * cols);
  const __nv_bfloat16* xr = x + m * D;
  float ss = 0.f;
  for (int i = c * 256 + lane; i < min(D, c * 256 + 256); i += 32) {
    const float v = __bfloat162float(xr[i]);
    ss += v * v;
  }
  ss = warp_sum(ss);
  if (lane == 0) out[w] = ss;
}

uno_status row_sumsq_launch(int64_t M, int64_t D, const void* x, float* out, cudaStream_t s) {
  if (M == 0) return UNO_OK;
  const int cols = static_cast<int>((D + 255) / 256);
  const int64_t warps = M * cols;
  const cudaError_t e = launch_kernel(
      row_sumsq_kernel, dim3(static_cast<unsigned>((warps + kNormThreads / 32 - 1) / (kNormThreads / 32))),
      dim3(kNormThreads), 0, s, 1, static_cast<const __nv_bfloat16*>(x), M, static_cast<int>(D), cols, out);
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "row sum-of-squares launch");
}

uno_status rmsnorm_launch(int64_t M, int64_t D, const void* x, void* y, float eps,
                          cudaStream_t s) {
  if (M == 0) return UNO_OK;
  const cudaError_t e = launch_kernel(
      rmsnorm_kernel, dim3(static_cast<unsigned>(M)), dim3(kNormThreads), 0, s, 1,
      static_cast<const __nv_bfloat16*>(x), static_cast<__nv_bfloat16*>(y), static_cast<int>(D), eps);
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "rmsnorm launch");
}

uno_status norm_down_launch(const NormDownArgs& a, int64_t M, cudaStream_t s) {
  if (M == 0) return UNO_OK;
  const unsigned blocks_y = static_cast<unsigned>((a.G * a.r + kNdRows - 1) / kNdRows);
  const cudaError_t e = launch_kernel(rmsnorm_down_kernel, dim3(static_cast<unsigned>(M), blocks_y),
                                     dim3(kNormThreads), 0, s, 1, a);
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "rmsnorm_down launch");
}

uno_status silu_mul_launch(int64_t n, const void* a, const void* b, void* y, cudaStream_t s) {
  if (n == 0) return UNO_OK;
  const int threads = 256;
  const int64_t want = (n / 8 + threads - 1) / threads + 1;
  const int blocks = static_cast<int>(std::min<int64_t>(want, 16 * device_sm_count()));
  const cudaError_t e = launch_kernel(silu_mul_kernel, dim3(blocks), dim3(threads), 0, s, 1,
                                      static_cast<const __nv_bfloat16*>(a),
                                      static_cast<const __nv_bfloat16*>(b),
                                      static_cast<__nv_bfloat16*>(y), n);
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "silu_mul launch");
}

}  // namespace uno
