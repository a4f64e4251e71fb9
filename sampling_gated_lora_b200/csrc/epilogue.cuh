// Epilogue of the gated GEMM kernels: output groups, row gate, residual add,
// row split, silu(gate) * up, and vectorised stores of fp32 accumulators.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace uno {

struct GroupArgs {
  void* y;
  long long ldy;
  int N;          // features of the group
  int tile0;      // first flattened feature tile of the group
  int t_col;      // first column of the group's rank-r block in t
  int b_rows;     // rows of Bl (a row coordinate at or past it reads zeros)
};

// What a kernel needs to know about the problem besides its tensor maps.
struct GemmArgs {
  int M;
  int mode;
  int ngroups;
  int nkb_main;   // K-blocks of x W^T
  int nkb_r;      // K-blocks of one group's rank-r block
  int M0;
  int gate_row0;
  float scale;
  void* y1;
  const uint8_t* gate;
  int32_t* status;
  int x_ready;    // x complete at launch: wait for the predecessor only before reading t
  // folded RMSNorm (see GemmProblem): input row scales from in_ss, and the
  // output rows' sums of squares to out_ss
  const float* in_ss;
  float* out_ss;
  int in_ss_cols, out_ss_cols;   // partials per row: of the input, of this launch (its feature tiles)
  float norm_inv_d, norm_eps;
  GroupArgs g[kMaxGroups];
};

// 1 / sqrt(mean square + eps) of input row m from its in_ss partials, added
// in order (so every launch and every tile of the row gets the same scale).
__device__ __forceinline__ float in_row_scale(const GemmArgs& a, int m) {
  if (!a.in_ss || m >= a.M) return 1.0f;
  const float* p = a.in_ss + static_cast<size_t>(m) * a.in_ss_cols;
  float ss = 0.f;
  for (int c = 0; c < a.in_ss_cols; ++c) ss += p[c];
  return rsqrtf(ss * a.norm_inv_d + a.norm_eps);
}

// Host: the device-side description of a problem; `tile_n` is the number of
// output features per feature tile (silu-pair tiles count output features).
inline GemmArgs make_gemm_args(const GemmProblem& pb, int tile_n, int row_bytes) {
  GemmArgs a{};
  const int64_t kb = row_bytes / (pb.dt == UNO_F32 ? 4 : 2);
  a.M = static_cast<int>(pb.M);
  a.mode = pb.mode;
  a.ngroups = pb.ngroups;
  a.nkb_main = static_cast<int>((pb.K + kb - 1) / kb);
  a.nkb_r = pb.r > 0 ? static_cast<int>((pb.r + kb - 1) / kb) : 0;
  a.M0 = static_cast<int>(pb.M0 < pb.M ? pb.M0 : pb.M);
  a.gate_row0 = static_cast<int>(pb.gate_row0 < pb.M ? pb.gate_row0 : pb.M);
  a.scale = pb.scale;
  a.y1 = pb.y1;
  a.gate = pb.gate;
  a.status = nullptr;
  a.x_ready = pb.x_ready ? 1 : 0;
  a.in_ss = pb.in_ss;
  a.out_ss = pb.out_ss;
  a.in_ss_cols = pb.in_ss_cols;
  a.norm_inv_d = pb.norm_dim > 0 ? 1.0f / static_cast<float>(pb.norm_dim) : 0.f;
  a.norm_eps = pb.norm_eps;
  int tiles = 0;
  for (int i = 0; i < pb.ngroups; ++i) {
    a.g[i].y = pb.g[i].y;
    a.g[i].ldy = pb.g[i].ldy;
    a.g[i].N = static_cast<int>(pb.g[i].N);
    a.g[i].tile0 = tiles;
    a.g[i].t_col = static_cast<int>(pb.g[i].t_col);
    a.g[i].b_rows = static_cast<int>(pb.g[i].N);
    if (pb.mode != kEpiSiluPair || i == 0) tiles += static_cast<int>((pb.g[i].N + tile_n - 1) / tile_n);
  }
  if (pb.mode == kEpiSiluPair) a.g[1].tile0 = tiles;   // the up group shares group 0's tiles
  a.out_ss_cols = static_cast<int>((pb.g[0].N + tile_n - 1) / tile_n);
  return a;
}

inline int feature_tiles(const GemmArgs& a, int tile_n) {
  return a.mode == kEpiSiluPair ? (a.g[0].N + tile_n - 1) / tile_n
                                : a.g[a.ngroups - 1].tile0 + (a.g[a.ngroups - 1].N + tile_n - 1) / tile_n;
}

// Group of flattened feature tile ft.
__device__ __forceinline__ int group_of(const GemmArgs& a, int ft) {
  int g = 0;
#pragma unroll
  for (int i = 1; i < kMaxGroups; ++i)
    if (i < a.ngroups && a.mode != kEpiSiluPair && ft >= a.g[i].tile0) g = i;
  return g;
}

// Adapter gate of token row m: the gate vector, or (m >= gate_row0) without one.
__device__ __forceinline__ float row_gate(const GemmArgs& a, int m) {
  return a.gate ? static_cast<float>(a.gate[m]) : (m >= a.gate_row0 ? 1.0f : 0.0f);
}

template <typename T>
__device__ __forceinline__ T* out_ptr(const GemmArgs& a, int g, int m, int n) {
  const GroupArgs& G = a.g[g];
  if (g == 0 && m >= a.M0) return static_cast<T*>(a.y1) + static_cast<long long>(m - a.M0) * G.ldy + n;
  return static_cast<T*>(G.y) + static_cast<long long>(m) * G.ldy + n;
}

__device__ __forceinline__ float silu_f(float g) { return g / (1.0f + __expf(-g)); }

// Apply the epilogue to one value of (group g, token m, feature n) and store it.
template <typename T>
__device__ __forceinline__ void epi_store1(const GemmArgs& a, int g, int m, int n, float v) {
  if (m >= a.M || n >= a.g[g].N) return;
  T* dst = out_ptr<T>(a, g, m, n);
  if (a.mode == kEpiRowScale) v *= a.scale * row_gate(a, m);
  if (a.mode == kEpiAdd) v += to_f32<T>(*dst);
  *dst = from_f32<T>(v);
}

// 4 consecutive features n..n+3 (n % 4 == 0, N % 4 == 0) of token row m.
template <typename T>
__device__ __forceinline__ void epi_store4(const GemmArgs& a, int g, int m, int n, float4 v) {
  if (m >= a.M || n >= a.g[g].N) return;
  T* dst = out_ptr<T>(a, g, m, n);
  if (a.mode == kEpiRowScale) {
    const float rs = a.scale * row_gate(a, m);
    v.x *= rs; v.y *= rs; v.z *= rs; v.w *= rs;
  }
  if constexpr (std::is_same<T, float>::value) {
    float4* d = reinterpret_cast<float4*>(dst);
    if (a.mode == kEpiAdd) {
      const float4 o = *d;
      v.x += o.x; v.y += o.y; v.z += o.z; v.w += o.w;
    }
    *d = v;
  } else {
    uint2* d = reinterpret_cast<uint2*>(dst);
    if (a.mode == kEpiAdd) {
      const uint2 o = *d;
      v.x += bf16_lo(o.x); v.y += bf16_hi(o.x); v.z += bf16_lo(o.y); v.w += bf16_hi(o.y);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
    *d = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
  }
}

// 16 consecutive features n0..n0+15 of token row m (n0 % 16 == 0): two
// 16-byte stores for bf16, four for f32; element by element at a ragged end.
// sq (optional, bf16 only): adds the squares of the values stored.
template <typename T>
__device__ __forceinline__ void epi_store16(const GemmArgs& a, int g, int m, int n0,
                                            const float (&v)[16], float* sq = nullptr) {
  if (m >= a.M) return;
  if (n0 + 16 > a.g[g].N) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      epi_store1<T>(a, g, m, n0 + j, v[j]);
      if (sq && n0 + j < a.g[g].N) {
        const float s = to_f32<T>(*out_ptr<T>(a, g, m, n0 + j));
        *sq += s * s;
      }
    }
    return;
  }
  T* dst = out_ptr<T>(a, g, m, n0);
  float w[16];
  const float rs = a.mode == kEpiRowScale ? a.scale * row_gate(a, m) : 1.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = v[j] * rs;
  if constexpr (std::is_same<T, float>::value) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4 o = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      if (a.mode == kEpiAdd) {
        const float4 old = d4[q];
        o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
      }
      d4[q] = o;
    }
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      if (a.mode == kEpiAdd) {
        const uint4 old = d4[q];
        const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          w[8 * q + 2 * e] += bf16_lo(ow[e]);
          w[8 * q + 2 * e + 1] += bf16_hi(ow[e]);
        }
      }
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(w[8 * q + 2 * e], w[8 * q + 2 * e + 1]);
        pk[e] = *reinterpret_cast<uint32_t*>(&h);
        if (sq) {
          const float lo = bf16_lo(pk[e]), hi = bf16_hi(pk[e]);
          *sq += lo * lo + hi * hi;
        }
      }
      d4[q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}

}  // namespace uno
