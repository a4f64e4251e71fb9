// Epilogue of the gated GEMM kernels: row gate, residual add, row split and
// vectorised stores of fp32 accumulators to bf16 / f32 outputs.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace uno {

// What the epilogue does with an accumulator element of (token m, feature n).
struct EpiArgs {
  int M, N;
  int mode;               // EpilogueMode
  int M0;                 // rows m >= M0 go to y1 (row m - M0)
  long long ldy;
  void* y;
  void* y1;
  const uint8_t* gate;    // kEpiRowScale; NULL: gate = (m >= gate_row0)
  int gate_row0;
  float scale;
};

inline EpiArgs epi_args(const GemmProblem& pb) {
  EpiArgs e{};
  e.M = static_cast<int>(pb.M);
  e.N = static_cast<int>(pb.N);
  e.mode = pb.mode;
  e.M0 = static_cast<int>(pb.M0 < pb.M ? pb.M0 : pb.M);
  e.ldy = pb.ldy;
  e.y = pb.y;
  e.y1 = pb.y1;
  e.gate = pb.gate;
  e.gate_row0 = static_cast<int>(pb.gate_row0 < pb.M ? pb.gate_row0 : pb.M);
  e.scale = pb.scale;
  return e;
}

// Adapter gate of token row m: the gate vector, or (m >= gate_row0) without one.
__device__ __forceinline__ float row_gate(const EpiArgs& p, int m) {
  return p.gate ? static_cast<float>(p.gate[m]) : (m >= p.gate_row0 ? 1.0f : 0.0f);
}

// Store one output element (accumulator row i, column j of this tile).
template <typename T, bool kSwap>
__device__ __forceinline__ void epi_store1(const EpiArgs& p, int p_row0, int q_row0, int i,
                                           int j, float acc) {
  const int m = kSwap ? q_row0 + j : p_row0 + i;
  const int n = kSwap ? p_row0 + i : q_row0 + j;
  if (m >= p.M || n >= p.N) return;
  T* base = static_cast<T*>(m < p.M0 ? p.y : p.y1);
  const long long row = m < p.M0 ? m : m - p.M0;
  T* dst = base + row * p.ldy + n;
  float v = acc;
  if (p.mode == kEpiRowScale) v *= p.scale * row_gate(p, m);
  if (p.mode == kEpiAdd) v += to_f32<T>(*dst);
  *dst = from_f32<T>(v);
}

// 4 consecutive features n..n+3 of token row m (n a multiple of 4, N % 4 == 0).
template <typename T>
__device__ __forceinline__ void epi_store4(const EpiArgs& p, int m, int n, float4 a) {
  T* base = static_cast<T*>(m < p.M0 ? p.y : p.y1);
  const long long row = m < p.M0 ? m : m - p.M0;
  T* dst = base + row * p.ldy + n;
  if (p.mode == kEpiRowScale) {
    const float rs = p.scale * row_gate(p, m);
    a.x *= rs; a.y *= rs; a.z *= rs; a.w *= rs;
  }
  if constexpr (std::is_same<T, float>::value) {
    float4* d = reinterpret_cast<float4*>(dst);
    if (p.mode == kEpiAdd) {
      const float4 o = *d;
      a.x += o.x; a.y += o.y; a.z += o.z; a.w += o.w;
    }
    *d = a;
  } else {
    uint2* d = reinterpret_cast<uint2*>(dst);
    if (p.mode == kEpiAdd) {
      const uint2 o = *d;
      a.x += bf16_lo(o.x); a.y += bf16_hi(o.x); a.z += bf16_lo(o.y); a.w += bf16_hi(o.y);
    }
    __nv_bfloat162 lo = __floats2bfloat162_rn(a.x, a.y), hi = __floats2bfloat162_rn(a.z, a.w);
    *d = make_uint2(*reinterpret_cast<uint32_t*>(&lo), *reinterpret_cast<uint32_t*>(&hi));
  }
}

// 16 consecutive features of one token row (non-swapped layout), vectorised.
template <typename T>
__device__ __forceinline__ void epi_store16_row(const EpiArgs& p, int m, int n0,
                                                const float (&v)[16]) {
  T* base = static_cast<T*>(m < p.M0 ? p.y : p.y1);
  const long long row = m < p.M0 ? m : m - p.M0;
  T* dst = base + row * p.ldy + n0;
  float w[16];
  const float rs = (p.mode == kEpiRowScale) ? p.scale * row_gate(p, m) : 1.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) w[j] = v[j] * rs;
  if constexpr (std::is_same<T, float>::value) {
    float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4 o = make_float4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
      if (p.mode == kEpiAdd) {
        const float4 old = d4[q];
        o.x += old.x; o.y += old.y; o.z += old.z; o.w += old.w;
      }
      d4[q] = o;
    }
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      float a[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) a[e] = w[8 * q + e];
      if (p.mode == kEpiAdd) {
        const uint4 old = d4[q];
        const uint32_t ow[4] = {old.x, old.y, old.z, old.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          a[2 * e] += bf16_lo(ow[e]);
          a[2 * e + 1] += bf16_hi(ow[e]);
        }
      }
      uint32_t pk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        __nv_bfloat162 h = __floats2bfloat162_rn(a[2 * e], a[2 * e + 1]);
        pk[e] = *reinterpret_cast<uint32_t*>(&h);
      }
      d4[q] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
    }
  }
}


}  // namespace uno
