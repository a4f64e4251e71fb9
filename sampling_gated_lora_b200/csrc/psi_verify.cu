// Psi-Spec verification and the linear-sampler draft (sm_100a).
//
// Method (hyper.ai page, section "方法", the Psi-Spec paragraph; ainews page):
// the draft path proposes a block from its per-position marginals q_j; the
// block is checked against the AR distributions p_j by rejection sampling and
// the longest accepted prefix is kept; the result follows p exactly.
//
// Kernels
//   row_stats_kernel     for every logit row (p rows, then q rows) and vocab
//                        chunk: the chunk max m and s = sum exp((z - m) / T).
//                        Streams the logits once with 16-byte loads; this is
//                        where the HBM time goes.
//   verify_finalize      one thread-block cluster per sequence: merge the
//                        chunk stats, test u1 q(d) < p(d) per position (lane
//                        j of warp 0), ballot -> first rejection n, then the
//                        residual (or bonus) inverse-CDF draw split over the
//                        cluster's CTAs (chunk totals exchanged through
//                        distributed shared memory).
//   draft_draw_kernel    after draft_stats_kernel has streamed the q rows once:
//                        one CTA per (sequence, position) finds the vocab
//                        chunk holding the draw from the chunk totals and
//                        reads only that chunk again for the inverse-CDF draw.
// Uniforms: Philox4x32-10 word 0 at counter (index, step lo, step hi,
// stream), key (seed lo, seed hi); u = (x >> 8) 2^-24. The counter depends on
// (sequence, position, stream) only, never on the launch shape.
#include <algorithm>
#include <cfloat>
#include <cmath>
#include <mutex>
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace uno {

__device__ int32_t g_device_status = 0;

namespace {

constexpr int kStatThreads = 256;
constexpr int kDrawThreads = 256;

// The softmax weights are 2^((z - max) c) with c = log2(e) / T.
// Verification takes c as one float: its rounding (up to 6e-8 relative)
// scales a weight by 2^(-(max - z) err), far below what the accept test
// resolves. The draft sampler, whose draws on near-flat 151936-way rows must
// land in token intervals ~1e-5 of the total wide, holds c as an unevaluated
// sum hi + lo of two floats and forms the exponent with one fused multiply-add
// (z - max is exact for bf16 logits). hi is taken strictly below c, so lo > 0
// and an infinite d gives an infinite exponent of its own sign.
struct TScale {
  float hi, lo;
};
__device__ __forceinline__ float operator*(float d, TScale c) { return fmaf(d, c.hi, d * c.lo); }
TScale make_tscale(float temperature) {
  const double cd = 1.4426950408889634073599 / static_cast<double>(temperature);
  TScale t;
  t.hi = static_cast<float>(cd);
  if (static_cast<double>(t.hi) >= cd) t.hi = std::nextafter(t.hi, 0.f);
  t.lo = static_cast<float>(cd - static_cast<double>(t.hi));
  return t;
}
float make_scale(float temperature) {
  return static_cast<float>(1.4426950408889634073599 / static_cast<double>(temperature));
}

template <typename T>
struct Vec;   // 16-byte vector of logits (global-memory loads through the read-only path)
template <>
struct Vec<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(p));
    v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
    v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
  }
};
template <>
struct Vec<float> {
  static constexpr int n = 4;
  __device__ static void load(const float* p, float (&v)[4]) {
    const float4 w = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = w.x; v[1] = w.y; v[2] = w.z; v[3] = w.w;
  }
};

// Online (max, sum of exp2((z - max) * c)) of one thread.
struct OnlineStat {
  float m = -INFINITY;
  float s = 0.f;
  template <typename C>
  __device__ __forceinline__ void add(const float* v, int n, C c) {
    float mx = v[0];
    for (int e = 1; e < n; ++e) mx = fmaxf(mx, v[e]);
    if (mx > m) {
      s *= fast_exp2((m - mx) * c);
      m = mx;
    }
    for (int e = 0; e < n; ++e) s += fast_exp2((v[e] - m) * c);
  }
};

// Merge (m1, s1) with (m2, s2); s is relative to m, exp base 2 with scale c.
template <typename C>
__device__ __forceinline__ void merge_stat(float& m, float& s, float m2, float s2, C c) {
  if (isnan(s2) || isnan(s)) {   // keep a NaN seen anywhere
    s = NAN;
    m = fmaxf(m, m2);
    return;
  }
  if (m2 == -INFINITY) return;
  if (m == -INFINITY) {
    m = m2;
    s = s2;
    return;
  }
  const float mx = fmaxf(m, m2);
  s = s * fast_exp2((m - mx) * c) + s2 * fast_exp2((m2 - mx) * c);
  m = mx;
}

// (max, sum of 2^((z - max) c)) of ids [lo, hi) of row z over the CTA
// (kStatThreads threads, every one calls): 16-byte loads, four in flight per
// thread, each thread an online stat, then shuffle and shared-memory merges.
// The result is valid in thread 0. A NaN anywhere makes s NaN.
template <typename T, typename C>
__device__ __forceinline__ float2 block_row_stat(const T* z, int lo, int hi, C c) {
  constexpr int kN = Vec<T>::n;
  OnlineStat st;
  // aligned body [a0, a1) in whole 16-byte vectors; scalar head and tail
  int a0 = lo;
  while (a0 < hi && (reinterpret_cast<uintptr_t>(z + a0) & 15u)) ++a0;
  const int nvec = (hi - a0) / kN;
  const int a1 = a0 + nvec * kN;
  for (int v = lo + threadIdx.x; v < a0; v += kStatThreads) {
    float x = to_f32<T>(z[v]);
    st.add(&x, 1, c);
  }
  constexpr int kUnroll = 4;
  int i = threadIdx.x;
  for (; i + (kUnroll - 1) * kStatThreads < nvec; i += kUnroll * kStatThreads) {
    float v[kUnroll][kN];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) Vec<T>::load(z + a0 + (i + u * kStatThreads) * kN, v[u]);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) st.add(v[u], kN, c);
  }
  for (; i < nvec; i += kStatThreads) {
    float v[kN];
    Vec<T>::load(z + a0 + i * kN, v);
    st.add(v, kN, c);
  }
  for (int v = a1 + threadIdx.x; v < hi; v += kStatThreads) {
    float x = to_f32<T>(z[v]);
    st.add(&x, 1, c);
  }
  float m = st.m, s = st.s;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
    const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
    merge_stat(m, s, m2, s2, c);
  }
  __shared__ float sm[kStatThreads / 32], ss[kStatThreads / 32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (lane == 0) {
    sm[warp] = m;
    ss[warp] = s;
  }
  cta_sync();
  float M = sm[0], S = ss[0];
  if (threadIdx.x == 0)
    for (int w = 1; w < kStatThreads / 32; ++w) merge_stat(M, S, sm[w], ss[w], c);
  return make_float2(M, S);
}

// Grid: rows * chunks blocks, one per (row, vocab chunk), chunk fastest (a
// one-dimensional grid, so the row count is not held to gridDim.y's 65535).
// Row r < rows_p reads p_logits row r, else q_logits row r - rows_p. Writes
// stats[r * chunks + chunk] = (m, s).
template <typename T>
__global__ void __launch_bounds__(kStatThreads)
    row_stats_kernel(const T* __restrict__ p_logits, const T* __restrict__ q_logits, int rows_p,
                     int V, int chunks, int chunk_len, float c, float2* __restrict__ stats) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int row = static_cast<int>(blockIdx.x / static_cast<unsigned>(chunks));
  const int chunk = static_cast<int>(blockIdx.x - static_cast<unsigned>(row) * chunks);
  const T* z = row < rows_p ? p_logits + static_cast<size_t>(row) * V
                            : q_logits + static_cast<size_t>(row - rows_p) * V;
  const int lo = chunk * chunk_len;
  const float2 st = block_row_stat<T>(z, lo, min(V, lo + chunk_len), c);
  if (threadIdx.x == 0) stats[blockIdx.x] = st;
}

// Statistics of one vocab chunk for the draft (see draft_stats_kernel).
struct DraftStat {
  float m;    // chunk max (NaN: a NaN logit in the chunk)
  float pad;
  double s;   // sum of 2^((z - m) c) over the chunk
};

// The draft's stats pass: warp w of the grid (8 per CTA) takes (row w / nsub,
// chunk w % nsub) of kSubLen ids and holds the whole chunk in registers (all
// 16-byte loads of a lane in flight at once). Two passes over the registers,
// no online rescaling: the chunk max by shuffles, then the weights
// 2^((z - m) c) summed per vector in float and across vectors and lanes in
// double. Shuffles only, no block barrier.
constexpr int kSubLen = 2048;   // ids per chunk (multiple of 8)

template <typename T>
__global__ void __launch_bounds__(kStatThreads)
    draft_stats_kernel(const T* __restrict__ z_all, int rows, int V, int nsub, TScale c,
                       DraftStat* __restrict__ stats) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (kStatThreads / 32) + (threadIdx.x >> 5);
  if (w >= static_cast<int64_t>(rows) * nsub) return;
  const int row = static_cast<int>(w / nsub);
  const int sc = static_cast<int>(w - static_cast<int64_t>(row) * nsub);
  const T* z = z_all + static_cast<size_t>(row) * V;
  const int lo = sc * kSubLen;
  const int hi = min(V, lo + kSubLen);
  constexpr int kN = Vec<T>::n;
  constexpr int kPerLane = kSubLen / kN / 32;   // vectors per lane
  float v[kPerLane][kN];
  const bool whole = hi - lo == kSubLen && (reinterpret_cast<uintptr_t>(z + lo) & 15u) == 0;
  if (whole) {
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) Vec<T>::load(z + lo + (lane + u * 32) * kN, v[u]);
  } else {   // a ragged last chunk or unaligned rows: element loads, -inf past the end
#pragma unroll
    for (int u = 0; u < kPerLane; ++u)
#pragma unroll
      for (int q = 0; q < kN; ++q) {
        const int e = lo + (lane + u * 32) * kN + q;
        v[u][q] = e < hi ? to_f32<T>(z[e]) : -INFINITY;
      }
  }
  float m = -INFINITY;
  bool nan = false;
#pragma unroll
  for (int u = 0; u < kPerLane; ++u)
#pragma unroll
    for (int q = 0; q < kN; ++q) {
      nan |= isnan(v[u][q]);
      m = fmaxf(m, v[u][q]);
    }
  m = warp_max(m);
  nan = __any_sync(0xffffffffu, nan);
  double acc = 0.0;
  if (m != -INFINITY) {
#pragma unroll
    for (int u = 0; u < kPerLane; ++u) {
      float part = 0.f;
#pragma unroll
      for (int q = 0; q < kN; ++q) part += fast_exp2((v[u][q] - m) * c);
      acc += static_cast<double>(part);
    }
  }
  acc = warp_sum(acc);
  if (lane == 0) {
    DraftStat st;
    st.m = nan ? NAN : m;
    st.pad = 0.f;
    st.s = acc;
    stats[w] = st;
  }
}

// The same statistics, with the chunks staged in shared memory by bulk
// copies (rows whose byte length is a multiple of 16 and a 16-byte aligned
// base): a persistent grid of one CTA per SM, each of its kStagedWarps warps
// walking the chunks w, w + W, ... (W = all warps of the grid) with a private
// ring of kDraftSlots slots. Lane 0 keeps the ring's next copies in flight
// (an mbarrier per slot), so an SM has kStagedWarps * kDraftSlots chunks of
// loads outstanding while its warps compute. A warp reads its slot twice
// (the max, then the sums), one 16-byte vector per lane at a time, so a
// thread holds a few registers and many warps fit beside the copies. A slot
// is refilled only after the warp has read it (an async-proxy fence orders
// the reads before the copy). Waits are bounded: on a timeout the warp
// records UNO_DEV_TIMEOUT, waits (bounded) for its copies still in flight
// and stops.
constexpr int kStagedWarps = 24;
constexpr int kStagedThreads = kStagedWarps * 32;
constexpr int kDraftSlots = 2;
constexpr uint32_t kDraftSlotBytes = kSubLen * 2;   // one bf16 chunk (4 KB)

__device__ __forceinline__ void unpack8(const uint4 w, float (&v)[8]) {
  v[0] = bf16_lo(w.x); v[1] = bf16_hi(w.x); v[2] = bf16_lo(w.y); v[3] = bf16_hi(w.y);
  v[4] = bf16_lo(w.z); v[5] = bf16_hi(w.z); v[6] = bf16_lo(w.w); v[7] = bf16_hi(w.w);
}

// Two bf16 maxima per instruction; a NaN operand gives NaN (so the chunk max
// also tells whether the chunk holds a NaN).
__device__ __forceinline__ uint32_t bmax2_nan(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.NaN.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Two floats in one 64-bit register (element 0 in the low half) and the
// packed fp32 arithmetic of sm_100 on them: one instruction per two elements,
// each with the rounding of its scalar counterpart.
using f32x2 = unsigned long long;
__device__ __forceinline__ f32x2 f2_make(float a, float b) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void f2_split(f32x2 v, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(v));
}
__device__ __forceinline__ f32x2 f2_sub(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_fma(f32x2 a, f32x2 b, f32x2 c) {
  f32x2 d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
// The two elements of a bf16x2 word as floats.
__device__ __forceinline__ f32x2 f2_from_bf16x2(uint32_t w) { return f2_make(bf16_lo(w), bf16_hi(w)); }

__global__ void __launch_bounds__(kStagedThreads, 1)
    draft_stats_staged_kernel(const __nv_bfloat16* __restrict__ z_all, int rows, int V, int nsub,
                              TScale c, DraftStat* __restrict__ stats, int32_t* status) {
  extern __shared__ __align__(128) uint8_t dsmem[];
  __shared__ __align__(8) uint64_t bars[kStagedWarps][kDraftSlots];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint8_t* ring = dsmem + static_cast<size_t>(warp) * kDraftSlots * kDraftSlotBytes;
  const int64_t units = static_cast<int64_t>(rows) * nsub;
  const int64_t W = static_cast<int64_t>(gridDim.x) * kStagedWarps;
  const int64_t w0 = static_cast<int64_t>(blockIdx.x) * kStagedWarps + warp;
  if (lane == 0) {
    for (int q = 0; q < kDraftSlots; ++q) mbar_init(smem_u32(&bars[warp][q]), 1);
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  // unit u -> (row, chunk, ids) and its copy into slot q
  auto issue = [&](int64_t u, int q) {
    const int row = static_cast<int>(u / nsub);
    const int sc = static_cast<int>(u - static_cast<int64_t>(row) * nsub);
    const int lo = sc * kSubLen;
    const int len = min(V, lo + kSubLen) - lo;
    const uint32_t bytes = static_cast<uint32_t>(len) * 2u;
    const uint32_t bar = smem_u32(&bars[warp][q]);
    mbar_arrive_expect_tx(bar, bytes);
    bulk_load(smem_u32(ring + static_cast<size_t>(q) * kDraftSlotBytes),
              z_all + static_cast<size_t>(row) * V + lo, bytes, bar);
  };
  if (lane == 0)
    for (int q = 0; q < kDraftSlots; ++q)
      if (w0 + q * W < units) issue(w0 + q * W, q);
  constexpr int kPerLane = kSubLen / 8 / 32;   // 16-byte vectors per lane
  int it = 0;
  bool ok = true;
  for (int64_t u = w0; u < units; u += W, ++it) {
    const int q = it % kDraftSlots;
    const uint32_t phase = static_cast<uint32_t>(it / kDraftSlots) & 1u;
    ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&bars[warp][q]), phase));
    if (!ok) break;
    const int row = static_cast<int>(u / nsub);
    const int sc = static_cast<int>(u - static_cast<int64_t>(row) * nsub);
    const int len = min(V, sc * kSubLen + kSubLen) - sc * kSubLen;
    const __nv_bfloat16* slot =
        reinterpret_cast<const __nv_bfloat16*>(ring + static_cast<size_t>(q) * kDraftSlotBytes);
    // 16-byte vector k of this lane from the slot (shared-memory loads), -inf past the chunk
    auto vec = [&](int k, float (&v)[8]) {
      const int e = (lane + k * 32) * 8;
      if (e + 8 <= len) {
        unpack8(*reinterpret_cast<const uint4*>(slot + e), v);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) v[j] = e + j < len ? to_f32<__nv_bfloat16>(slot[e + j]) : -INFINITY;
      }
    };
    // the chunk max, two bf16 per instruction (a NaN makes it NaN); rows are
    // whole 16-byte vectors, so a vector lies wholly inside or past the chunk
    uint32_t m2 = 0xFF80FF80u;   // (-inf, -inf)
#pragma unroll
    for (int k = 0; k < kPerLane; ++k) {
      const int e = (lane + k * 32) * 8;
      if (e + 8 <= len) {
        const uint4 w = *reinterpret_cast<const uint4*>(slot + e);
        m2 = bmax2_nan(m2, bmax2_nan(bmax2_nan(w.x, w.y), bmax2_nan(w.z, w.w)));
      } else if (e < len) {
        float v[8];
        vec(k, v);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t b = __float_as_uint(v[j]) >> 16;
          m2 = bmax2_nan(m2, b | (b << 16));
        }
      }
    }
    const float mlo = bf16_lo(m2), mhi = bf16_hi(m2);
    bool nan = isnan(mlo) || isnan(mhi);
    float m = fmaxf(mlo, mhi);
    m = warp_max(m);
    nan = __any_sync(0xffffffffu, nan);
    // sum of 2^((z - m) c): the difference, the float-pair scale and the sum of
    // each 16-byte vector two elements per instruction, across vectors in double
    double acc = 0.0;
    if (m != -INFINITY && !nan) {
      const f32x2 mm = f2_make(m, m), chi = f2_make(c.hi, c.hi), clo = f2_make(c.lo, c.lo);
#pragma unroll
      for (int k = 0; k < kPerLane; ++k) {
        const int e = (lane + k * 32) * 8;
        if (e + 8 <= len) {
          const uint4 w = *reinterpret_cast<const uint4*>(slot + e);
          const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
          f32x2 part = f2_make(0.f, 0.f);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const f32x2 d = f2_sub(f2_from_bf16x2(ws[j]), mm);
            float x0, x1;
            f2_split(f2_fma(d, chi, f2_mul(d, clo)), x0, x1);
            part = f2_add(part, f2_make(fast_exp2(x0), fast_exp2(x1)));
          }
          float p0, p1;
          f2_split(part, p0, p1);
          acc += static_cast<double>(p0 + p1);
        } else if (e < len) {
          float v[8];
          vec(k, v);
          float part = 0.f;
#pragma unroll
          for (int j = 0; j < 8; ++j) part += fast_exp2((v[j] - m) * c);
          acc += static_cast<double>(part);
        }
      }
    }
    // every lane has read the slot: it may be refilled
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0 && u + static_cast<int64_t>(kDraftSlots) * W < units)
      issue(u + static_cast<int64_t>(kDraftSlots) * W, q);
    acc = warp_sum(acc);
    if (lane == 0) {
      DraftStat st;
      st.m = nan ? NAN : m;
      st.pad = 0.f;
      st.s = acc;
      stats[u] = st;
    }
  }
  if (!ok) {
    // the copies this warp still has in flight land before it leaves
    if (lane == 0) {
      raise_status(status, kDevTimeout);
      int k = it;
      for (int64_t u = w0 + static_cast<int64_t>(it) * W; u < units && k < it + kDraftSlots;
           u += W, ++k)
        (void)mbar_wait(smem_u32(&bars[warp][k % kDraftSlots]),
                        static_cast<uint32_t>(k / kDraftSlots) & 1u);
    }
    __syncwarp();
  }
}

// Merge the chunk stats of one row.
__device__ __forceinline__ float2 row_stat(const float2* stats, int row, int chunks, float c) {
  float m = -INFINITY, s = 0.f;
  bool nan = false;
  for (int i = 0; i < chunks; ++i) {
    const float2 v = stats[static_cast<size_t>(row) * chunks + i];
    nan |= isnan(v.y);
    merge_stat(m, s, v.x, v.y, c);
  }
  return make_float2(m, nan ? NAN : s);
}

// ------------------------------------------------------------------ cluster inverse-CDF draw

// Shared state of one draw (per CTA).
struct DrawSmem {
  double prefix[kDrawThreads + 1];   // exclusive prefix of the per-thread segment sums
  double warp_tot[kDrawThreads / 32];
  double chunk_total;
  int owner[kDrawThreads / 32];
  int token;
};

// Block-wide exclusive scan of one double per thread (kDrawThreads threads).
// Writes sh.prefix[t] and sh.prefix[kDrawThreads] = sh.chunk_total = the total.
__device__ __forceinline__ void block_scan(DrawSmem& sh, double v) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  double incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const double n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  double excl = __shfl_up_sync(0xffffffffu, incl, 1);
  if (lane == 0) excl = 0.0;
  if (lane == 31) sh.warp_tot[warp] = incl;
  cta_sync();
  if (warp == 0) {
    double w = lane < kDrawThreads / 32 ? sh.warp_tot[lane] : 0.0;
#pragma unroll
    for (int o = 1; o < kDrawThreads / 32; o <<= 1) {
      const double n = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += n;
    }
    if (lane < kDrawThreads / 32) sh.warp_tot[lane] = w;   // inclusive over warps
  }
  cta_sync();
  const double base = warp ? sh.warp_tot[warp - 1] : 0.0;
  sh.prefix[t] = base + excl;
  if (t == 0) {
    sh.prefix[kDrawThreads] = sh.warp_tot[kDrawThreads / 32 - 1];
    sh.chunk_total = sh.warp_tot[kDrawThreads / 32 - 1];
  }
  cta_sync();
}

// Largest index t in [0, kDrawThreads) with `ok` true, over the block (-1 if none).
__device__ __forceinline__ int block_max_index(DrawSmem& sh, bool ok) {
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int w = __reduce_max_sync(0xffffffffu, ok ? t : -1);
  if (lane == 0) sh.owner[warp] = w;
  cta_sync();
  int best = -1;
#pragma unroll
  for (int i = 0; i < kDrawThreads / 32; ++i) best = max(best, sh.owner[i]);
  cta_sync();
  return best;
}

// Inverse-CDF draw over the cluster. This CTA holds `len` weights w(i) of
// vocab ids [lo, lo + len), computed on demand by `wfn` (deterministic: the
// same call returns the same bits). Thread t owns the contiguous segment
// [t*seg, (t+1)*seg) of the chunk. The draw picks the smallest id whose
// inclusive cumulative weight exceeds u * Z (Z = cluster total): the owning
// CTA is the last one with prefix <= u*Z and positive mass, the owning
// segment likewise, and the segment is scanned in ascending id. These rules
// pick exactly one owner even when rounding makes prefixes of nested sums
// disagree in the last bit. Returns the drawn id in the owning CTA, -1
// elsewhere; *zero_total reports Z == 0. Every thread of every CTA of the
// cluster must call it. No CTA reads another's shared memory after the last
// cluster barrier inside, so callers may exit right after.
template <typename WFn>
__device__ int cluster_draw(DrawSmem& sh, const WFn& wfn, int lo, int len, double u,
                            bool* zero_total) {
  const int t = threadIdx.x;
  const int seg = (len + kDrawThreads - 1) / kDrawThreads;
  const int s0 = min(len, t * seg), s1 = min(len, s0 + seg);
  double my = 0.0;
  for (int i = s0; i < s1; ++i) my += static_cast<double>(wfn(i));
  block_scan(sh, my);
  if (t == 0) sh.token = -1;
  cluster_sync();
  // every CTA reads the chunk totals in rank order -> identical prefixes
  const uint32_t nrank = cluster_nctarank();
  const uint32_t myrank = cluster_ctarank();
  const uint32_t tot_addr = smem_u32(&sh.chunk_total);
  // (unrolled to the largest cluster with constant indices: registers, not stack)
  double Z = 0.0, thr_prefix[8], tots[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    thr_prefix[r] = Z;
    tots[r] = 0.0;
    if (r < static_cast<int>(nrank)) {
      tots[r] = ld_cluster_f64(map_shared_rank(tot_addr, static_cast<uint32_t>(r)));
      Z += tots[r];
    }
  }
  cluster_sync();   // totals read everywhere before anyone reuses the slot or exits
  if (!(Z > 0.0)) {
    *zero_total = true;
    return -1;
  }
  *zero_total = false;
  const double thr = u * Z;
  int owner_rank = -1;
  double my_prefix = 0.0;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r < static_cast<int>(nrank) && tots[r] > 0.0 && thr_prefix[r] <= thr) owner_rank = r;
    if (r == static_cast<int>(myrank)) my_prefix = thr_prefix[r];
  }
  if (owner_rank != static_cast<int>(myrank)) return -1;   // uniform over this CTA
  const double tl = thr - my_prefix;
  const int own = block_max_index(sh, my > 0.0 && sh.prefix[t] <= tl);
  if (t == own) {
    const double tt = tl - sh.prefix[t];
    double run = 0.0;
    int pick = -1, last_nz = -1;
    for (int i = s0; i < s1; ++i) {
      const float w = wfn(i);
      if (w > 0.f) last_nz = i;
      run += static_cast<double>(w);
      if (run > tt) {
        pick = i;
        break;
      }
    }
    sh.token = lo + (pick >= 0 ? pick : last_nz);
  }
  cta_sync();
  return sh.token;
}

// The same draw with the weights read 8 ids at a time straight from global
// memory instead of a staged chunk: w8(i, w) fills w[0..7] with the weights
// of ids lo + i .. lo + i + 7 (0 past len, i a multiple of 8). Thread
// segments are whole multiples of 8 ids, so every read is one 16-byte vector;
// the owning segment is read a second time (from L2) for the walk. Same
// rules, same call protocol as cluster_draw.
template <typename W8>
__device__ int cluster_draw8(DrawSmem& sh, const W8& w8, int lo, int len, double u,
                             bool* zero_total) {
  const int t = threadIdx.x;
  const int seg = (((len + kDrawThreads - 1) / kDrawThreads) + 7) & ~7;
  const int s0 = min(len, t * seg), s1 = min(len, s0 + seg);
  double my = 0.0;
  for (int i = s0; i < s1; i += 8) {
    float w[8];
    w8(i, w);
#pragma unroll
    for (int j = 0; j < 8; ++j) my += static_cast<double>(w[j]);
  }
  block_scan(sh, my);
  if (t == 0) sh.token = -1;
  cluster_sync();
  const uint32_t nrank = cluster_nctarank();
  const uint32_t myrank = cluster_ctarank();
  const uint32_t tot_addr = smem_u32(&sh.chunk_total);
  double Z = 0.0, thr_prefix[8], tots[8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    thr_prefix[r] = Z;
    tots[r] = 0.0;
    if (r < static_cast<int>(nrank)) {
      tots[r] = ld_cluster_f64(map_shared_rank(tot_addr, static_cast<uint32_t>(r)));
      Z += tots[r];
    }
  }
  cluster_sync();   // totals read everywhere before anyone reuses the slot or exits
  if (!(Z > 0.0)) {
    *zero_total = true;
    return -1;
  }
  *zero_total = false;
  const double thr = u * Z;
  int owner_rank = -1;
  double my_prefix = 0.0;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r < static_cast<int>(nrank) && tots[r] > 0.0 && thr_prefix[r] <= thr) owner_rank = r;
    if (r == static_cast<int>(myrank)) my_prefix = thr_prefix[r];
  }
  if (owner_rank != static_cast<int>(myrank)) return -1;   // uniform over this CTA
  const double tl = thr - my_prefix;
  const int own = block_max_index(sh, my > 0.0 && sh.prefix[t] <= tl);
  if (t == own) {
    const double tt = tl - sh.prefix[t];
    double run = 0.0;
    int pick = -1, last_nz = -1;
    for (int i = s0; i < s1 && pick < 0; i += 8) {
      float w[8];
      w8(i, w);
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (pick >= 0 || i + j >= s1) continue;
        if (w[j] > 0.f) last_nz = i + j;
        run += static_cast<double>(w[j]);
        if (run > tt) pick = i + j;
      }
    }
    sh.token = lo + (pick >= 0 ? pick : last_nz);
  }
  cta_sync();
  return sh.token;
}

// Eight bf16 logits of ids i .. i + 7 of a row chunk z (16-byte aligned at
// every multiple of 8), -inf past len.
__device__ __forceinline__ void load8_bf16(const __nv_bfloat16* z, int i, int len, float (&v)[8]) {
  if (i + 8 <= len) {
    Vec<__nv_bfloat16>::load(z + i, v);
  } else {
#pragma unroll
    for (int j = 0; j < 8; ++j) v[j] = i + j < len ? __bfloat162float(z[i + j]) : -INFINITY;
  }
}

// Vocab range of CTA `rank` among `n`: chunks are multiples of 8 ids.
__device__ __forceinline__ void chunk_range(int V, int n, int rank, int* lo, int* len) {
  int per = (V + n - 1) / n;
  per = (per + 7) & ~7;
  const int a = min(V, rank * per);
  *lo = a;
  *len = min(V, a + per) - a;
}

// Stage `len` logits into shared memory: 16-byte streaming loads, four in
// flight per thread, when the source is 16-byte aligned; scalar otherwise.
template <typename T>
__device__ __forceinline__ void load_chunk(T* dst, const T* src, int len) {
  constexpr int kN = 16 / static_cast<int>(sizeof(T));
  if ((reinterpret_cast<uintptr_t>(src) & 15u) == 0) {
    const int nv = len / kN;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    int i = threadIdx.x;
    const int step = blockDim.x;
    for (; i + 3 * step < nv; i += 4 * step) {
      const uint4 a = __ldcs(s4 + i), b = __ldcs(s4 + i + step);
      const uint4 c = __ldcs(s4 + i + 2 * step), d = __ldcs(s4 + i + 3 * step);
      d4[i] = a;
      d4[i + step] = b;
      d4[i + 2 * step] = c;
      d4[i + 3 * step] = d;
    }
    for (; i < nv; i += step) d4[i] = __ldcs(s4 + i);
    for (int j = nv * kN + threadIdx.x; j < len; j += step) dst[j] = src[j];
  } else {
    for (int j = threadIdx.x; j < len; j += blockDim.x) dst[j] = src[j];
  }
}

// Stage `len` logits of s0 (and of s1 when it is not NULL) into d0 (d1) with
// all of their bytes in flight at once: bulk copies completing on the
// mbarrier `bar` when the sources are 16-byte aligned and len * sizeof(T) is
// a multiple of 16, the threads' loads otherwise. `bar` has been initialised
// (count 1) before a block barrier; `phase` is its next phase, and the phase
// after is returned. The wait is bounded: on a timeout the status word gets
// UNO_DEV_TIMEOUT and thread 0 waits for the copies once more before the CTA
// goes on. Every thread calls it; it ends with a block barrier.
template <typename T>
__device__ uint32_t stage_chunks(T* d0, const T* s0, T* d1, const T* s1, int len, uint64_t* bar,
                                 uint32_t phase, int32_t* status) {
  const uint32_t bytes = static_cast<uint32_t>(len) * sizeof(T);
  const uintptr_t addr = reinterpret_cast<uintptr_t>(s0) | (s1 ? reinterpret_cast<uintptr_t>(s1) : 0);
  if ((addr & 15u) != 0 || bytes % 16 != 0 || bytes == 0) {
    load_chunk(d0, s0, len);
    if (s1) load_chunk(d1, s1, len);
    cta_sync();
    return phase;
  }
  cta_sync();   // earlier reads of d0 / d1 (generic proxy) are done
  if (threadIdx.x == 0) {
    fence_proxy_async_smem();   // and ordered before the copies' writes
    mbar_arrive_expect_tx(smem_u32(bar), (s1 ? 2u : 1u) * bytes);
    bulk_load(smem_u32(d0), s0, bytes, smem_u32(bar));
    if (s1) bulk_load(smem_u32(d1), s1, bytes, smem_u32(bar));
  }
  if (!mbar_wait(smem_u32(bar), phase) && threadIdx.x == 0) {
    raise_status(status, kDevTimeout);
    (void)mbar_wait(smem_u32(bar), phase);
  }
  cta_sync();
  return phase ^ 1u;
}

struct FinalizeParams {
  int B, k, k_p, V, chunks;
  float c;   // log2(e) / T
  uint64_t seed, step, seq_offset;
  const int32_t* draft;
  const float2* stats;
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* out_count;
  int32_t* status;
  int chunk_elems;   // per-CTA smem capacity in elements (per row)
  int direct;        // bf16 rows, 16-byte aligned: the draw reads them in place (no staging)
};

// One cluster per sequence; blockDim = kDrawThreads. Four CTAs per SM (64
// registers a thread: one 4-byte spill) when the draw reads its rows in
// place: psi_verify B=256, k=16 470 us against 484 at three CTAs per SM.
template <typename T>
__global__ void __launch_bounds__(kDrawThreads, 4)
    verify_finalize_kernel(const T* __restrict__ p_logits, const T* __restrict__ q_logits,
                           const FinalizeParams a) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ DrawSmem sh;
  __shared__ int s_n, s_bad, s_nan;
  __shared__ float s_stat[4];   // Mp, Sp, Mq, Sq of the drawing row(s)
  __shared__ __align__(8) uint64_t s_bar;   // the staged rows' bulk copies

  if (threadIdx.x == 0) {
    pdl_trigger();
    mbar_init(smem_u32(&s_bar), 1);
    fence_mbar_init();
  }
  pdl_wait();
  const uint32_t nrank = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int b = blockIdx.x / nrank;
  const int k = a.k, V = a.V;
  const uint64_t bg = a.seq_offset + static_cast<uint64_t>(b);
  const int rows_p = a.B * a.k_p;

  if (threadIdx.x < 32) {
    const int j = threadIdx.x;
    bool acc = true, bad = false, nan = false;
    if (j < k) {
      const int d = a.draft[b * k + j];
      bad = d < 0 || d >= V;
      const int prow = b * a.k_p + j, qrow = rows_p + b * k + j;
      const float2 sp = row_stat(a.stats, prow, a.chunks, a.c);
      const float2 sq = row_stat(a.stats, qrow, a.chunks, a.c);
      nan = isnan(sp.y) || isnan(sq.y);
      if (!bad && !nan) {
        const float zp = to_f32<T>(p_logits[static_cast<size_t>(prow) * V + d]);
        const float zq = to_f32<T>(q_logits[static_cast<size_t>(b * k + j) * V + d]);
        const float pd = fast_exp2((zp - sp.x) * a.c) / sp.y;
        const float qd = fast_exp2((zq - sq.x) * a.c) / sq.y;
        const uint32_t idx = static_cast<uint32_t>(bg * static_cast<uint64_t>(k) + j);
        const float u1 = uniform24(philox_word0(a.seed, a.step, kStreamAccept, idx));
        acc = (qd == 0.f) || (u1 * qd < pd);
      }
    }
    const uint32_t in_k = k >= 32 ? 0xffffffffu : ((1u << k) - 1u);
    const uint32_t rej = __ballot_sync(0xffffffffu, !acc) & in_k;
    const uint32_t badm = __ballot_sync(0xffffffffu, bad) & in_k;
    const uint32_t nanm = __ballot_sync(0xffffffffu, nan) & in_k;
    if (j == 0) {
      s_n = rej ? __ffs(rej) - 1 : k;
      s_bad = badm != 0;
      s_nan = nanm != 0;
    }
  }
  cta_sync();
  const int n = s_n;
  int32_t* tok = a.out_tokens + static_cast<size_t>(b) * (k + 1);
  if (s_bad || s_nan) {
    if (rank == 0) {
      if (threadIdx.x == 0) {
        a.accepted_len[b] = -1;
        a.out_count[b] = -1;
        raise_status(a.status, (s_bad ? kDevBadDraft : 0) | (s_nan ? kDevNaN : 0));
      }
      for (int i = threadIdx.x; i <= k; i += blockDim.x) tok[i] = -1;
    }
    return;   // uniform over the cluster: every CTA saw the same flags
  }
  const bool residual = n < k;
  const bool bonus = !residual && a.k_p == k + 1;
  const bool draw = residual || bonus;
  if (rank == 0) {
    if (threadIdx.x == 0) {
      a.accepted_len[b] = n;
      a.out_count[b] = n + (draw ? 1 : 0);
    }
    for (int i = threadIdx.x; i <= k; i += blockDim.x) {
      if (i < n) tok[i] = a.draft[b * k + i];
      else if (i > n || !draw) tok[i] = -1;
    }
  }
  if (!draw) return;

  // Rows of the draw: residual at position n (p row and q row), or the bonus p row k.
  const int prow = b * a.k_p + (residual ? n : k);
  const int qrow_local = b * k + n;   // q row index within q_logits
  if (threadIdx.x == 0) {
    const float2 sp = row_stat(a.stats, prow, a.chunks, a.c);
    s_stat[0] = sp.x;
    s_stat[1] = sp.y;
    if (residual) {
      const float2 sq = row_stat(a.stats, rows_p + qrow_local, a.chunks, a.c);
      s_stat[2] = sq.x;
      s_stat[3] = sq.y;
    }
  }
  int lo, len;
  chunk_range(V, static_cast<int>(nrank), static_cast<int>(rank), &lo, &len);
  T* zp = reinterpret_cast<T*>(dyn);
  T* zq = zp + a.chunk_elems;
  if (!a.direct) {
    stage_chunks(zp, p_logits + static_cast<size_t>(prow) * V + lo, zq,
                 residual ? q_logits + static_cast<size_t>(qrow_local) * V + lo : nullptr, len,
                 &s_bar, 0u, a.status);
  } else {
    cta_sync();   // s_stat is set
  }
  const float Mp = s_stat[0], inv_sp = 1.f / s_stat[1];
  const float Mq = s_stat[2], inv_sq = residual ? 1.f / s_stat[3] : 0.f;
  const float c = a.c;
  const uint32_t idx = static_cast<uint32_t>(bg * static_cast<uint64_t>(k) + (residual ? n : k));
  const double u = static_cast<double>(uniform24(
      philox_word0(a.seed, a.step, residual ? kStreamResidual : kStreamBonus, idx)));

  bool zero = false;
  int token;
  if constexpr (std::is_same<T, __nv_bfloat16>::value) {
    if (a.direct) {   // the draw rows read in place, 16-byte vectors
      const __nv_bfloat16* gp = p_logits + static_cast<size_t>(prow) * V + lo;
      const __nv_bfloat16* gq = q_logits + static_cast<size_t>(qrow_local) * V + lo;
      auto w8_p = [&](int i, float (&w)[8]) {
        float zv[8];
        load8_bf16(gp, i, len, zv);
#pragma unroll
        for (int j = 0; j < 8; ++j) w[j] = fast_exp2((zv[j] - Mp) * c);
      };
      if (residual) {
        auto w8_res = [&](int i, float (&w)[8]) {
          float zv[8], zw[8];
          load8_bf16(gp, i, len, zv);
          load8_bf16(gq, i, len, zw);
#pragma unroll
          for (int j = 0; j < 8; ++j)
            w[j] = fmaxf(fast_exp2((zv[j] - Mp) * c) * inv_sp - fast_exp2((zw[j] - Mq) * c) * inv_sq, 0.f);
        };
        token = cluster_draw8(sh, w8_res, lo, len, u, &zero);
      } else {
        token = cluster_draw8(sh, w8_p, lo, len, u, &zero);
      }
      if (zero) token = cluster_draw8(sh, w8_p, lo, len, u, &zero);
      if (token >= 0 && threadIdx.x == 0) tok[n] = token;
      return;
    }
  }
  if (residual) {
    auto w_res = [&](int i) {
      const float p = fast_exp2((to_f32<T>(zp[i]) - Mp) * c) * inv_sp;
      const float q = fast_exp2((to_f32<T>(zq[i]) - Mq) * c) * inv_sq;
      return fmaxf(p - q, 0.f);
    };
    token = cluster_draw(sh, w_res, lo, len, u, &zero);
  } else {
    auto w_p = [&](int i) { return fast_exp2((to_f32<T>(zp[i]) - Mp) * c); };
    token = cluster_draw(sh, w_p, lo, len, u, &zero);
  }
  if (zero) {   // residual mass 0 (only through rounding): draw from p_n
    auto w_p = [&](int i) { return fast_exp2((to_f32<T>(zp[i]) - Mp) * c); };
    token = cluster_draw(sh, w_p, lo, len, u, &zero);
  }
  if (token >= 0 && threadIdx.x == 0) tok[n] = token;
}

// ------------------------------------------------------------------ tree sampler
//
// Several drafted blocks per sequence, verified as a prefix tree (hyper.ai
// page, section "方法", the tree sampler; lossless as for the linear sampler).
// The candidates form a trie, numbered in order of first visit when they are
// walked from the root in index order (node 0 = root). At a node of depth j
// the live candidates (prefix = the accepted path) are tested in index order:
// candidate i with token x is accepted iff u * q_j(x) < r_i(x), where r_1 = p
// of the node and r_{i+1} = max(r_i - q_j, 0) / Z_i after each rejection
// (Z_i its mass; the target stays when Z_i = 0). On acceptance the walk moves
// to the child x with every candidate that has token x there; if all are
// rejected, a token is drawn from the last residual. With one candidate this
// is exactly the linear verification above.

constexpr int kTreeMaxN = 32;   // candidate blocks per sequence
constexpr int kTreeMaxK = 32;   // block length

struct TreeParams {
  int B, N, k, R, V, chunks, bonus;
  float c;   // log2(e) / T
  uint64_t seed, step, seq_offset;
  const int32_t* cands;   // [B, N, k]
  const float2* stats;    // chunk stats of node rows b*R + n, then q rows B*R + b*k + j
  int32_t* accepted_len;
  int32_t* out_tokens;
  int32_t* out_count;
  int32_t* status;
  int chunk_elems;
};

// Sum of one double per thread over the block and then over the cluster, the
// CTAs' sums added in rank order so that every CTA gets the same bits. Every
// thread of every CTA of the cluster must call it.
__device__ double cluster_sum(double* part_slot, double* warp_slots, double v) {
  v = warp_sum(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (lane == 0) warp_slots[warp] = v;
  cta_sync();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kDrawThreads / 32; ++w) t += warp_slots[w];
    *part_slot = t;
  }
  cluster_sync();
  const uint32_t nrank = cluster_nctarank();
  const uint32_t addr = smem_u32(part_slot);
  double total = 0.0;
#pragma unroll
  for (int r = 0; r < 8; ++r)
    if (r < static_cast<int>(nrank)) total += ld_cluster_f64(map_shared_rank(addr, static_cast<uint32_t>(r)));
  cluster_sync();   // every CTA has read the slots before they are written again
  return total;
}

// Target of a test at one vocab entry after `n` rejections at the node:
// r_1 = p, r_{t+1} = max(r_t - q, 0) / Z_t (unchanged when Z_t = 0).
// Zinv[t] = 1 / Z[t] (0 when Z[t] = 0, which leaves r unchanged), taken once
// per rejection so the per-entry chain multiplies instead of dividing.
__device__ __forceinline__ double tree_target(float p, float q, const double* Zinv, int n) {
  double r = p;
  for (int t = 0; t < n; ++t)
    if (Zinv[t] > 0.0) r = fmax(r - static_cast<double>(q), 0.0) * Zinv[t];
  return r;
}

// One cluster per sequence; blockDim = kDrawThreads.
template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
    tree_finalize_kernel(const T* __restrict__ p_logits, const T* __restrict__ q_logits,
                         const TreeParams a) {
  extern __shared__ __align__(16) uint8_t dyn[];
  __shared__ DrawSmem sh;
  __shared__ int s_node[kTreeMaxN][kTreeMaxK + 1];   // trie node after j tokens of candidate i
  __shared__ int s_id[kTreeMaxN * kTreeMaxK];
  __shared__ int s_tok[kTreeMaxK];
  __shared__ double s_Z[kTreeMaxN];      // residual masses of the rejections at this node
  __shared__ double s_Zinv[kTreeMaxN];   // and their reciprocals (0 for a zero mass)
  __shared__ double s_part, s_warp[kDrawThreads / 32];
  __shared__ float s_stat[4];
  __shared__ int s_flag[4];   // [0] decision, [1] bad candidate, [2] trie nodes, [3] NaN
  __shared__ __align__(8) uint64_t s_bar;   // bulk copies of the staged rows
  uint32_t bar_phase = 0;

  if (threadIdx.x == 0) {
    pdl_trigger();
    mbar_init(smem_u32(&s_bar), 1);
    fence_mbar_init();
  }
  pdl_wait();
  const uint32_t nrank = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int b = blockIdx.x / nrank;
  const int N = a.N, k = a.k, V = a.V, R = a.R;
  const int nk = N * k;
  const uint64_t bg = a.seq_offset + static_cast<uint64_t>(b);
  const int32_t* cand = a.cands + static_cast<size_t>(b) * nk;
  int32_t* tok = a.out_tokens + static_cast<size_t>(b) * (k + 1);
  const float c = a.c;

  // 1. Trie numbering. rep(i, j) = the first candidate with the same j+1
  //    tokens; the first visits, in walk order (i, then j), get ids 1, 2, ...
  if (threadIdx.x == 0) {
    s_flag[1] = 0;
    s_flag[3] = 0;
  }
  cta_sync();
  for (int t = threadIdx.x; t < nk; t += blockDim.x) {
    const int i = t / k, j = t - i * k;
    const int x = cand[t];
    if (x < 0 || x >= V) atomicOr(&s_flag[1], 1);
    int rep = i;
    for (int i2 = 0; i2 < i && rep == i; ++i2) {
      bool same = true;
      for (int jj = 0; jj <= j && same; ++jj) same = cand[i2 * k + jj] == cand[i * k + jj];
      if (same) rep = i2;
    }
    s_node[i][j + 1] = rep;   // the representative for now
    s_id[t] = rep == i ? 1 : 0;
  }
  cta_sync();
  if (threadIdx.x == 0) {
    int run = 0;
    for (int t = 0; t < nk; ++t) s_id[t] = s_id[t] ? ++run : 0;
    s_flag[2] = run + 1;   // nodes, the root included
  }
  cta_sync();
  for (int t = threadIdx.x; t < nk; t += blockDim.x) {
    const int i = t / k, j = t - i * k;
    s_node[i][j + 1] = s_id[s_node[i][j + 1] * k + j];
  }
  for (int i = threadIdx.x; i < N; i += blockDim.x) s_node[i][0] = 0;
  cta_sync();

  // a candidate token outside [0, V), or more trie nodes than the R logit rows
  // given per sequence: flagged, outputs -1 (uniform over the cluster)
  auto give_up = [&](int32_t bits) {
    if (rank == 0) {
      if (threadIdx.x == 0) {
        a.accepted_len[b] = -1;
        a.out_count[b] = -1;
        raise_status(a.status, bits);
      }
      for (int i = threadIdx.x; i <= k; i += blockDim.x) tok[i] = -1;
    }
  };
  if (s_flag[1] || s_flag[2] > R) {
    give_up(kDevBadDraft);
    return;
  }

  int lo, len;
  chunk_range(V, static_cast<int>(nrank), static_cast<int>(rank), &lo, &len);
  T* zp = reinterpret_cast<T*>(dyn);
  T* zq = zp + a.chunk_elems;
  const size_t q_row0 = static_cast<size_t>(a.B) * R;
  int node = 0, n = 0;
  uint32_t live = N >= 32 ? 0xffffffffu : ((1u << N) - 1u);

  // 2. The walk, one depth at a time. Thread 0 of every CTA takes the same
  //    decisions from the same data; the residual masses are summed over the
  //    cluster in a fixed order, so every CTA follows the same path.
  for (int j = 0; j < k; ++j) {
    if (threadIdx.x == 0) {
      const float2 sp = row_stat(a.stats, b * R + node, a.chunks, c);
      const float2 sq = row_stat(a.stats, static_cast<int>(q_row0) + b * k + j, a.chunks, c);
      s_stat[0] = sp.x;
      s_stat[1] = sp.y;
      s_stat[2] = sq.x;
      s_stat[3] = sq.y;
      s_flag[3] = isnan(sp.y) || isnan(sq.y);
    }
    cta_sync();
    if (s_flag[3]) {
      give_up(kDevNaN);
      return;
    }
    const float Mp = s_stat[0], inv_sp = 1.f / s_stat[1];
    const float Mq = s_stat[2], inv_sq = 1.f / s_stat[3];
    const T* prow = p_logits + (static_cast<size_t>(b) * R + node) * V;
    const T* qrow = q_logits + (static_cast<size_t>(b) * k + j) * V;
    int nz = 0, accepted = -1;
    bool staged = false;
    for (int i = 0; i < N; ++i) {
      if (!((live >> i) & 1u)) continue;
      if (threadIdx.x == 0) {
        const int x = cand[i * k + j];
        const float px = fast_exp2((to_f32<T>(prow[x]) - Mp) * c) * inv_sp;
        const float qx = fast_exp2((to_f32<T>(qrow[x]) - Mq) * c) * inv_sq;
        const float r = static_cast<float>(tree_target(px, qx, s_Zinv, nz));
        const uint32_t idx = static_cast<uint32_t>(
            (bg * static_cast<uint64_t>(k) + static_cast<uint64_t>(j)) * static_cast<uint64_t>(N) +
            static_cast<uint64_t>(i));
        const float u1 = uniform24(philox_word0(a.seed, a.step, kStreamAccept, idx));
        s_flag[0] = (qx == 0.f) || (u1 * qx < r);
      }
      cta_sync();
      const bool acc = s_flag[0] != 0;
      cta_sync();   // read everywhere before thread 0 writes the next decision
      if (acc) {
        accepted = i;
        break;
      }
      // rejected: the residual mass Z of this test, over the whole vocabulary
      if (!staged) {
        bar_phase = stage_chunks(zp, prow + lo, zq, qrow + lo, len, &s_bar, bar_phase, a.status);
        staged = true;
      }
      double part = 0.0;
      for (int v = threadIdx.x; v < len; v += blockDim.x) {
        const float p = fast_exp2((to_f32<T>(zp[v]) - Mp) * c) * inv_sp;
        const float q = fast_exp2((to_f32<T>(zq[v]) - Mq) * c) * inv_sq;
        part += fmax(tree_target(p, q, s_Zinv, nz) - static_cast<double>(q), 0.0);
      }
      const double Z = cluster_sum(&s_part, s_warp, part);
      if (threadIdx.x == 0) {
        s_Z[nz] = Z;
        s_Zinv[nz] = Z > 0.0 ? 1.0 / Z : 0.0;
      }
      ++nz;
      cta_sync();
    }
    if (accepted >= 0) {
      const int x = cand[accepted * k + j];
      if (threadIdx.x == 0) s_tok[n] = x;
      ++n;
      node = s_node[accepted][j + 1];
      uint32_t next = 0;
      for (int i = 0; i < N; ++i)
        if (((live >> i) & 1u) && cand[i * k + j] == x) next |= 1u << i;
      live = next;
      cta_sync();
      continue;
    }
    // every live candidate rejected: draw from the last residual (stream 2)
    if (rank == 0) {
      if (threadIdx.x == 0) {
        a.accepted_len[b] = n;
        a.out_count[b] = n + 1;
      }
      for (int i = threadIdx.x; i <= k; i += blockDim.x)
        if (i != n) tok[i] = i < n ? s_tok[i] : -1;
    }
    const uint32_t idx2 = static_cast<uint32_t>(bg * static_cast<uint64_t>(k) + static_cast<uint64_t>(j));
    const double u = static_cast<double>(uniform24(philox_word0(a.seed, a.step, kStreamResidual, idx2)));
    const int last = nz - 1;
    auto w_res = [&](int v) {
      const float p = fast_exp2((to_f32<T>(zp[v]) - Mp) * c) * inv_sp;
      const float q = fast_exp2((to_f32<T>(zq[v]) - Mq) * c) * inv_sq;
      const double r = tree_target(p, q, s_Zinv, last);
      return static_cast<float>(s_Z[last] > 0.0 ? fmax(r - static_cast<double>(q), 0.0) : r);
    };
    bool zero = false;
    int token = cluster_draw(sh, w_res, lo, len, u, &zero);
    if (zero) {   // residual mass lost to rounding: draw from p of the node
      auto w_p = [&](int v) { return fast_exp2((to_f32<T>(zp[v]) - Mp) * c); };
      token = cluster_draw(sh, w_p, lo, len, u, &zero);
    }
    if (token >= 0 && threadIdx.x == 0) tok[n] = token;
    return;
  }

  // 3. All k positions accepted: the bonus token from p of the leaf (stream 3).
  if (rank == 0) {
    if (threadIdx.x == 0) {
      a.accepted_len[b] = k;
      a.out_count[b] = k + (a.bonus ? 1 : 0);
    }
    for (int i = threadIdx.x; i <= k; i += blockDim.x)
      if (i < k || !a.bonus) tok[i] = i < k ? s_tok[i] : -1;
  }
  if (!a.bonus) return;
  if (threadIdx.x == 0) {
    const float2 sp = row_stat(a.stats, b * R + node, a.chunks, c);
    s_stat[0] = sp.x;
    s_flag[3] = isnan(sp.y);
  }
  cta_sync();
  if (s_flag[3]) {
    give_up(kDevNaN);
    return;
  }
  const float Mp = s_stat[0];
  bar_phase = stage_chunks(zp, p_logits + (static_cast<size_t>(b) * R + node) * V + lo,
                           static_cast<T*>(nullptr), static_cast<const T*>(nullptr), len, &s_bar,
                           bar_phase, a.status);
  const uint32_t idx3 = static_cast<uint32_t>(bg * static_cast<uint64_t>(k) + static_cast<uint64_t>(k));
  const double u = static_cast<double>(uniform24(philox_word0(a.seed, a.step, kStreamBonus, idx3)));
  auto w_p = [&](int v) { return fast_exp2((to_f32<T>(zp[v]) - Mp) * c); };
  bool zero = false;
  const int token = cluster_draw(sh, w_p, lo, len, u, &zero);
  if (token >= 0 && threadIdx.x == 0) tok[k] = token;
}

// ------------------------------------------------------------------ distillation losses
//
// alpha * KL(p || q) + beta * TV(p, q) per row pair, p = softmax(z_teacher / T)
// (the clean, gate-0 rows), q = softmax(z_student / T) (the noisy, gate-1 rows)
// (hyper.ai page, section "方法": the distillation and total-variation
// losses), and the gradient w.r.t. the student logits:
//   (alpha (q - p) + beta q (s - sum_v s_v q_v) / 2) / (T rows),  s = sign(q - p).
// One cluster per row pair; each CTA stages its vocab chunk of both rows and
// makes three passes over it (partition sums, loss terms, gradient), the
// per-element arithmetic in float and every sum in double, with one exchange
// of CTA totals over the cluster after each of the first two (added in rank
// order, so every CTA holds the same bits).

struct DistillParams {
  int V, chunk_elems;
  float c;            // log2(e) / T
  float inv_t;        // 1 / T
  float alpha, beta;
  float grad_scale;   // 1 / (T rows)
  float* losses;      // [rows, 2]: KL, TV
  float* grad;        // [rows, V] or NULL
  int32_t* status;
};

template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
    distill_kernel(const T* __restrict__ z_teacher, const T* __restrict__ z_student,
                   const DistillParams a) {
  extern __shared__ __align__(16) uint8_t dyn[];
  constexpr int kWarps = kDrawThreads / 32;
  __shared__ float s_wm[kWarps][2];       // per warp: maxima (teacher, student)
  __shared__ double s_ws[kWarps][3];      // per warp: sums
  __shared__ float s_m[2];                // this CTA's maxima      } read by the
  __shared__ double s_s[2];               // and sums relative to them } whole cluster
  __shared__ double s_terms[3];           // this CTA's KL, sum |p - q|, sum s q
  __shared__ __align__(8) uint64_t s_bar;   // the chunks' bulk copies

  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const uint32_t nrank = cluster_nctarank();
  const uint32_t rank = cluster_ctarank();
  const int row = blockIdx.x / nrank;
  const int V = a.V;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int lo, len;
  chunk_range(V, static_cast<int>(nrank), static_cast<int>(rank), &lo, &len);
  T* zt = reinterpret_cast<T*>(dyn);
  T* zs = zt + a.chunk_elems;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&s_bar), 1);
    fence_mbar_init();
  }
  cta_sync();   // the barrier is initialised before anyone waits on it
  stage_chunks(zt, z_teacher + static_cast<size_t>(row) * V + lo, zs,
               z_student + static_cast<size_t>(row) * V + lo, len, &s_bar, 0u, a.status);
  const float c = a.c;

  // 1. both rows' maxima and partition sums: per warp the maxima, then each
  // thread's sums of 2^((z - m) c) relative to its warp's maxima (float), the
  // warps merged per CTA (double), the CTAs over the cluster in rank order
  // bf16 chunks are read as 16-byte vectors of 8 (the chunks start 16-byte
  // aligned in shared memory), two elements per instruction where the
  // arithmetic allows it; a ragged end of the chunk and f32 rows one by one
  constexpr bool kVec = std::is_same<T, __nv_bfloat16>::value;
  const int nvec = kVec ? len / 8 : 0;
  const int tail0 = nvec * 8;
  const uint4* vt = reinterpret_cast<const uint4*>(zt);
  const uint4* vs = reinterpret_cast<const uint4*>(zs);
  float mt = -INFINITY, ms = -INFINITY;
  bool nan = false;
  if (kVec) {   // maxima two at a time; a NaN makes the max NaN
    uint32_t mt2 = 0xFF80FF80u, ms2 = 0xFF80FF80u;
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
      const uint4 a = vt[i], b = vs[i];
      mt2 = bmax2_nan(mt2, bmax2_nan(bmax2_nan(a.x, a.y), bmax2_nan(a.z, a.w)));
      ms2 = bmax2_nan(ms2, bmax2_nan(bmax2_nan(b.x, b.y), bmax2_nan(b.z, b.w)));
    }
    const float t0 = bf16_lo(mt2), t1 = bf16_hi(mt2), s0 = bf16_lo(ms2), s1 = bf16_hi(ms2);
    nan = isnan(t0) || isnan(t1) || isnan(s0) || isnan(s1);
    mt = fmaxf(t0, t1);
    ms = fmaxf(s0, s1);
  }
  for (int i = tail0 + static_cast<int>(threadIdx.x); i < len; i += blockDim.x) {
    const float x = to_f32<T>(zt[i]), y = to_f32<T>(zs[i]);
    nan |= isnan(x) || isnan(y);
    mt = fmaxf(mt, x);
    ms = fmaxf(ms, y);
  }
  mt = warp_max(mt);
  ms = warp_max(ms);
  nan = __any_sync(0xffffffffu, nan);
  float st = 0.f, ss = 0.f;
  if (kVec) {
    const f32x2 c2 = f2_make(c, c), mt2 = f2_make(mt, mt), ms2 = f2_make(ms, ms);
    const bool dt = mt != -INFINITY, ds = ms != -INFINITY;
    f32x2 st2 = f2_make(0.f, 0.f), ss2 = f2_make(0.f, 0.f);
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
      const uint4 a = vt[i], b = vs[i];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float e0, e1;
        if (dt) {
          f2_split(f2_mul(f2_sub(f2_from_bf16x2(wa[q]), mt2), c2), e0, e1);
          st2 = f2_add(st2, f2_make(fast_exp2(e0), fast_exp2(e1)));
        }
        if (ds) {
          f2_split(f2_mul(f2_sub(f2_from_bf16x2(wb[q]), ms2), c2), e0, e1);
          ss2 = f2_add(ss2, f2_make(fast_exp2(e0), fast_exp2(e1)));
        }
      }
    }
    float a0, a1, b0, b1;
    f2_split(st2, a0, a1);
    f2_split(ss2, b0, b1);
    st = a0 + a1;
    ss = b0 + b1;
  }
  for (int i = tail0 + static_cast<int>(threadIdx.x); i < len; i += blockDim.x) {
    if (mt != -INFINITY) st += fast_exp2((to_f32<T>(zt[i]) - mt) * c);
    if (ms != -INFINITY) ss += fast_exp2((to_f32<T>(zs[i]) - ms) * c);
  }
  const double wst = warp_sum(static_cast<double>(st)), wss = warp_sum(static_cast<double>(ss));
  if (lane == 0) {
    s_wm[warp][0] = nan ? NAN : mt;
    s_wm[warp][1] = ms;
    s_ws[warp][0] = wst;
    s_ws[warp][1] = wss;
  }
  cta_sync();
  const double cd = static_cast<double>(c);
  if (threadIdx.x < 2) {   // thread 0: teacher, thread 1: student
    const int t = threadIdx.x;
    float m = -INFINITY;
    bool any = false;
    for (int w = 0; w < kWarps; ++w) {
      any |= isnan(s_wm[w][t]);
      m = fmaxf(m, s_wm[w][t]);
    }
    double sum = 0.0;
    for (int w = 0; w < kWarps; ++w)
      if (s_wm[w][t] != -INFINITY && !any)
        sum += s_ws[w][t] * exp2(static_cast<double>(s_wm[w][t] - m) * cd);
    s_m[t] = any ? NAN : m;
    s_s[t] = sum;
  }
  cluster_sync();   // exchange 1: every CTA's maxima and sums
  float Mt = -INFINITY, Ms = -INFINITY;
  bool any_nan = false;
  float cm[2][8];
  double csum[2][8];
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= static_cast<int>(nrank)) break;
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      cm[t][r] = ld_cluster_f32(map_shared_rank(smem_u32(&s_m[t]), static_cast<uint32_t>(r)));
      csum[t][r] = ld_cluster_f64(map_shared_rank(smem_u32(&s_s[t]), static_cast<uint32_t>(r)));
    }
    any_nan |= isnan(cm[0][r]);
    Mt = fmaxf(Mt, cm[0][r]);
    Ms = fmaxf(Ms, cm[1][r]);
  }
  if (any_nan) {   // uniform over the cluster
    cluster_sync();   // every CTA has read the others' slots before any leaves
    if (rank == 0 && threadIdx.x == 0) {
      a.losses[2 * row] = NAN;
      a.losses[2 * row + 1] = NAN;
      raise_status(a.status, kDevNaN);
    }
    if (a.grad)
      for (int i = threadIdx.x; i < len; i += blockDim.x)
        a.grad[static_cast<size_t>(row) * V + lo + i] = NAN;
    return;
  }
  double St = 0.0, Ss = 0.0;
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= static_cast<int>(nrank)) break;
    if (cm[0][r] != -INFINITY) St += csum[0][r] * exp2(static_cast<double>(cm[0][r] - Mt) * cd);
    if (cm[1][r] != -INFINITY) Ss += csum[1][r] * exp2(static_cast<double>(cm[1][r] - Ms) * cd);
  }

  // 2. KL, sum |p - q| and sum sign(q - p) q: per element in float (log p -
  // log q = (x - y) / T - dconst), per thread in float, then in double
  const float inv_st = static_cast<float>(1.0 / St), inv_ss = static_cast<float>(1.0 / Ss);
  const float inv_t = a.inv_t;
  const float dconst = static_cast<float>(static_cast<double>(Mt - Ms) * inv_t + (log(St) - log(Ss)));
  float k0 = 0.f, k1 = 0.f, k2 = 0.f;
  const f32x2 c2 = f2_make(c, c), Mt2 = f2_make(Mt, Mt), Ms2 = f2_make(Ms, Ms);
  const f32x2 ist2 = f2_make(inv_st, inv_st), iss2 = f2_make(inv_ss, inv_ss);
  // p and q of the two elements of bf16x2 words wx (teacher) and wy (student)
  auto pq2 = [&](uint32_t wx, uint32_t wy, f32x2* x, f32x2* y, f32x2* p, f32x2* q) {
    *x = f2_from_bf16x2(wx);
    *y = f2_from_bf16x2(wy);
    float ex0, ex1, ey0, ey1;
    f2_split(f2_mul(f2_sub(*x, Mt2), c2), ex0, ex1);
    f2_split(f2_mul(f2_sub(*y, Ms2), c2), ey0, ey1);
    *p = f2_mul(f2_make(fast_exp2(ex0), fast_exp2(ex1)), ist2);
    *q = f2_mul(f2_make(fast_exp2(ey0), fast_exp2(ey1)), iss2);
  };
  if (kVec) {
    const f32x2 it2 = f2_make(inv_t, inv_t), dc2 = f2_make(dconst, dconst);
    f32x2 K0 = f2_make(0.f, 0.f), K1 = K0, K2 = K0;
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
      const uint4 a = vt[i], b = vs[i];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f32x2 x, y, p, q;
        pq2(wa[j], wb[j], &x, &y, &p, &q);
        float p0, p1, q0, q1, t0, t1, d0, d1;
        f2_split(p, p0, p1);
        f2_split(q, q0, q1);
        f2_split(f2_sub(f2_mul(f2_sub(x, y), it2), dc2), t0, t1);
        K0 = f2_fma(p, f2_make(p0 > 0.f ? t0 : 0.f, p1 > 0.f ? t1 : 0.f), K0);   // 0 log 0 = 0
        f2_split(f2_sub(p, q), d0, d1);
        K1 = f2_add(K1, f2_make(fabsf(d0), fabsf(d1)));
        K2 = f2_add(K2, f2_make(q0 > p0 ? q0 : (q0 < p0 ? -q0 : 0.f), q1 > p1 ? q1 : (q1 < p1 ? -q1 : 0.f)));
      }
    }
    float u0, u1;
    f2_split(K0, u0, u1);
    k0 = u0 + u1;
    f2_split(K1, u0, u1);
    k1 = u0 + u1;
    f2_split(K2, u0, u1);
    k2 = u0 + u1;
  }
  for (int i = tail0 + static_cast<int>(threadIdx.x); i < len; i += blockDim.x) {
    const float x = to_f32<T>(zt[i]), y = to_f32<T>(zs[i]);
    const float p = fast_exp2((x - Mt) * c) * inv_st;
    const float q = fast_exp2((y - Ms) * c) * inv_ss;
    if (p > 0.f) k0 += p * ((x - y) * inv_t - dconst);
    k1 += fabsf(p - q);
    k2 += q > p ? q : (q < p ? -q : 0.f);
  }
  double v[3] = {warp_sum(static_cast<double>(k0)), warp_sum(static_cast<double>(k1)),
                 warp_sum(static_cast<double>(k2))};
  if (lane == 0)
#pragma unroll
    for (int i = 0; i < 3; ++i) s_ws[warp][i] = v[i];
  cta_sync();
  if (threadIdx.x < 3) {
    double t = 0.0;
    for (int w = 0; w < kWarps; ++w) t += s_ws[w][threadIdx.x];
    s_terms[threadIdx.x] = t;
  }
  cluster_sync();   // exchange 2: every CTA's terms
  double tot[3] = {0.0, 0.0, 0.0};
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    if (r >= static_cast<int>(nrank)) break;
#pragma unroll
    for (int i = 0; i < 3; ++i)
      tot[i] += ld_cluster_f64(map_shared_rank(smem_u32(&s_terms[i]), static_cast<uint32_t>(r)));
  }
  cluster_sync();   // every CTA has read the others' slots: nothing remote after this
  if (rank == 0 && threadIdx.x == 0) {
    a.losses[2 * row] = static_cast<float>(tot[0]);
    a.losses[2 * row + 1] = static_cast<float>(0.5 * tot[1]);
  }
  if (!a.grad) return;

  // 3. the gradient w.r.t. the student logits, this CTA's chunk (float)
  const float sq = static_cast<float>(tot[2]);
  const float ka = a.alpha * a.grad_scale;
  const float kb = 0.5f * a.beta * a.grad_scale;
  float* g = a.grad + static_cast<size_t>(row) * V + lo;
  if (kVec) {
    const f32x2 ka2 = f2_make(ka, ka), kb2 = f2_make(kb, kb), sq2 = f2_make(sq, sq);
    const bool g16 = (reinterpret_cast<uintptr_t>(g) & 15u) == 0;
    for (int i = threadIdx.x; i < nvec; i += blockDim.x) {
      const uint4 a = vt[i], b = vs[i];
      const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
      float out[8];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        f32x2 x, y, p, q;
        pq2(wa[j], wb[j], &x, &y, &p, &q);
        float p0, p1, q0, q1;
        f2_split(p, p0, p1);
        f2_split(q, q0, q1);
        const f32x2 sgn = f2_make(q0 > p0 ? 1.f : (q0 < p0 ? -1.f : 0.f),
                                  q1 > p1 ? 1.f : (q1 < p1 ? -1.f : 0.f));
        f2_split(f2_fma(f2_mul(kb2, q), f2_sub(sgn, sq2), f2_mul(ka2, f2_sub(q, p))), out[2 * j],
                 out[2 * j + 1]);
      }
      float* gi = g + 8 * i;
      if (g16) {
        reinterpret_cast<float4*>(gi)[0] = make_float4(out[0], out[1], out[2], out[3]);
        reinterpret_cast<float4*>(gi)[1] = make_float4(out[4], out[5], out[6], out[7]);
      } else {
#pragma unroll
        for (int j = 0; j < 8; ++j) gi[j] = out[j];
      }
    }
  }
  for (int i = tail0 + static_cast<int>(threadIdx.x); i < len; i += blockDim.x) {
    const float p = fast_exp2((to_f32<T>(zt[i]) - Mt) * c) * inv_st;
    const float q = fast_exp2((to_f32<T>(zs[i]) - Ms) * c) * inv_ss;
    const float sgn = q > p ? 1.f : (q < p ? -1.f : 0.f);
    g[i] = ka * (q - p) + kb * q * (sgn - sq);
  }
}

struct DraftParams {
  int k, V, chunks, chunk_len;
  TScale c;
  uint64_t seed, step, seq_offset;
  const DraftStat* stats;   // [rows, chunks] of the q rows
  int32_t* draft;
  int32_t* status;
};

constexpr int kDraftMaxChunks = 128;   // draft_chunks() never exceeds it

// Linear-sampler draw of one row, after row_stats_kernel has streamed the row
// once: the chunk totals w_c = s_c 2^((m_c - M) c) (M the row max) give the
// chunk that holds the threshold u0 * Z, Z = sum w_c (the last chunk with
// positive total whose exclusive prefix is <= u0 Z), and only that chunk is
// read again: per-thread contiguous segments of weights 2^((z - M) c), a block
// scan of the segment sums, then the owning thread walks its segment in
// ascending id. Every sum is taken in double from float weights. One CTA per
// row (B k rows); blockDim = kDrawThreads.
template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
    draft_draw_kernel(const T* __restrict__ q_logits, const DraftParams a) {
  __shared__ DrawSmem sh;
  __shared__ double s_tot[kDraftMaxChunks];
  __shared__ float s_M;
  __shared__ int s_bad, s_owner;
  __shared__ double s_tl;
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const int chunks = a.chunks;
  const TScale c = a.c;
  const DraftStat* st = a.stats + static_cast<size_t>(row) * chunks;
  if (threadIdx.x < 32) {
    float m = -INFINITY;
    bool nan = false;
    for (int i = threadIdx.x; i < chunks; i += 32) {
      const DraftStat v = st[i];
      nan |= isnan(v.m);
      m = fmaxf(m, v.m);
    }
    m = warp_max(m);
    nan = __any_sync(0xffffffffu, nan);
    if (threadIdx.x == 0) {
      s_M = m;
      s_bad = nan || m == -INFINITY;
    }
  }
  cta_sync();
  if (s_bad) {
    if (threadIdx.x == 0) {
      a.draft[row] = -1;
      raise_status(a.status, kDevNaN);
    }
    return;
  }
  const float M = s_M;
  // chunk totals relative to the row max: the rescale in double (exp2 of the
  // exact bf16 difference times c), so it adds no error of float size
  const double cd = static_cast<double>(c.hi) + static_cast<double>(c.lo);
  for (int i = threadIdx.x; i < chunks; i += blockDim.x) {
    const DraftStat v = st[i];
    s_tot[i] = v.m == -INFINITY ? 0.0 : v.s * exp2(static_cast<double>(v.m - M) * cd);
  }
  cta_sync();
  const int b = row / a.k, j = row - b * a.k;
  const uint64_t bg = a.seq_offset + static_cast<uint64_t>(b);
  const uint32_t idx = static_cast<uint32_t>(bg * static_cast<uint64_t>(a.k) + j);
  if (threadIdx.x == 0) {
    double Z = 0.0;
    for (int i = 0; i < chunks; ++i) Z += s_tot[i];
    const double thr = static_cast<double>(uniform24(philox_word0(a.seed, a.step, kStreamDraft, idx))) * Z;
    double pre = 0.0, own_pre = 0.0;
    int own = -1;
    for (int i = 0; i < chunks; ++i) {
      if (s_tot[i] > 0.0 && pre <= thr) {
        own = i;
        own_pre = pre;
      }
      pre += s_tot[i];
    }
    s_owner = own;
    s_tl = thr - own_pre;
  }
  cta_sync();
  const int own_chunk = s_owner;   // >= 0: the chunk holding the row max has total >= 1
  const int lo = own_chunk * a.chunk_len;
  const int len = min(a.V, lo + a.chunk_len) - lo;
  const T* z = q_logits + static_cast<size_t>(row) * a.V + lo;
  const int t = threadIdx.x;
  const int seg = (len + kDrawThreads - 1) / kDrawThreads;
  const int s0 = min(len, t * seg), s1 = min(len, s0 + seg);
  double my = 0.0;
  for (int i = s0; i < s1; ++i) my += static_cast<double>(fast_exp2((to_f32<T>(z[i]) - M) * c));
  block_scan(sh, my);
  const double tl = s_tl;
  const int own = block_max_index(sh, my > 0.0 && sh.prefix[t] <= tl);
  if (t == own) {
    const double tt = tl - sh.prefix[t];
    double run = 0.0;
    int pick = -1, last_nz = -1;
    for (int i = s0; i < s1; ++i) {
      const float w = fast_exp2((to_f32<T>(z[i]) - M) * c);
      if (w > 0.f) last_nz = i;
      run += static_cast<double>(w);
      if (run > tt) {
        pick = i;
        break;
      }
    }
    a.draft[row] = lo + (pick >= 0 ? pick : last_nz);
  } else if (own < 0 && t == 0) {
    // every recomputed weight of the chunk flushed to zero (its total is below
    // the float range): the chunk's first id with the row max
    int arg = 0;
    for (int i = 0; i < len; ++i)
      if (to_f32<T>(z[i]) == M) {
        arg = i;
        break;
      }
    a.draft[row] = lo + arg;
  }
}

// ------------------------------------------------------------------ vocabulary shards
//
// The vocabulary split over G devices, each holding the logits of its own
// contiguous shard [v0, v0 + Vs) (hyper.ai page, section "方法": the
// verification against the AR distribution needs the normaliser over the
// whole vocabulary and, for the residual and bonus draws, cumulative mass in
// vocabulary order). The kernels below compute each device's share; the
// exchanges between devices (all-gathers of a few floats per row, a max over
// the drawn token) are collectives issued by the caller:
//   vp_partials   per row of the shard: (m, s, z(d)) — max, sum of
//                 2^((z - m) c), and the drafted token's logit if held here;
//   vp_decide     from all shards' partials: acceptance and the first
//                 rejection n per sequence (the same on every device), the
//                 draw row and its merged statistics;
//   vp_masses     the draw row's residual mass and p mass over the shard;
//   vp_draw       from all shards' masses: the shard holding u Z in shard
//                 order draws inside its range (the others leave -1);
//   vp_draft_draw the next block's draft, the same owner rule on the draft
//                 rows' partials.

// Inverse-CDF draw inside one CTA over local ids [0, len): the smallest id
// whose inclusive cumulative weight (ascending id, summed in double) exceeds
// tl; the last id with positive weight when the total falls short of tl; -1
// when every weight is zero. Every thread calls it and gets the result.
template <typename WFn>
__device__ int block_draw(DrawSmem& sh, const WFn& wfn, int len, double tl) {
  const int t = threadIdx.x;
  const int seg = (len + kDrawThreads - 1) / kDrawThreads;
  const int s0 = min(len, t * seg), s1 = min(len, s0 + seg);
  double my = 0.0;
  for (int i = s0; i < s1; ++i) my += static_cast<double>(wfn(i));
  block_scan(sh, my);
  const int own = block_max_index(sh, my > 0.0 && sh.prefix[t] <= tl);
  if (t == 0) sh.token = -1;
  cta_sync();
  if (t == own) {
    const double tt = tl - sh.prefix[t];
    double run = 0.0;
    int pick = -1, last_nz = -1;
    for (int i = s0; i < s1; ++i) {
      const float w = wfn(i);
      if (w > 0.f) last_nz = i;
      run += static_cast<double>(w);
      if (run > tt) {
        pick = i;
        break;
      }
    }
    sh.token = pick >= 0 ? pick : last_nz;
  }
  cta_sync();
  return sh.token;
}

struct VpParams {
  int B, k, k_p, Vs, v0, V, G, rank;
  float c;      // log2(e) / T (verification)
  TScale cd;    // the same as a float pair (draft)
  uint64_t seed, step, seq_offset;
  const int32_t* draft;     // [B, k] global ids
  const float4* parts_p;    // [G, B k_p]: (m, s, z(d), 0) of the AR rows
  const float4* parts_q;    // [G, rows]: of the draft rows (verify: B k; next draft: B k)
  int32_t* accepted_len;
  int32_t* out_tokens;      // [B, k + 1]
  int32_t* out_count;
  int32_t* draw;            // [B]: draw position (n < k: residual, k: bonus) or -1
  float4* draw_stats;       // [B]: (Mp, Sp, Mq, Sq) of the draw row
  double2* masses;          // vp_masses: [B] of this shard; vp_draw: [G, B] of all shards
  int32_t* draft_out;       // vp_draft_draw: [rows]
  int32_t* status;
};

// Per row of the shard: (m, s, z(id), 0). id_kind 1: AR rows (row b k_p + j
// holds draft[b, j] for j < k, none for the bonus row); 2: draft rows (row i
// holds draft[i]); 0: none. One CTA per row.
template <typename T, typename C>
__global__ void __launch_bounds__(kStatThreads)
    vp_partials_kernel(const T* __restrict__ z, int Vs, int v0, const int32_t* __restrict__ draft,
                       int k, int k_p, int id_kind, C c, float4* __restrict__ out) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const T* zr = z + static_cast<size_t>(row) * Vs;
  const float2 st = block_row_stat<T>(zr, 0, Vs, c);
  if (threadIdx.x == 0) {
    int id = -1;
    if (id_kind == 1) {
      const int b = row / k_p, j = row - b * k_p;
      if (j < k) id = draft[b * k + j];
    } else if (id_kind == 2) {
      id = draft[row];
    }
    const float zid = (id >= v0 && id < v0 + Vs) ? to_f32<T>(zr[id - v0]) : -INFINITY;
    out[row] = make_float4(st.x, st.y, zid, 0.f);
  }
}

// Merged (M, S, z(id)) of one row over the G shards (shard order).
__device__ __forceinline__ float3 vp_merge(const float4* parts, int rows, int row, int G, float c) {
  float m = -INFINITY, s = 0.f, z = -INFINITY;
  bool nan = false;
  for (int g = 0; g < G; ++g) {
    const float4 v = parts[static_cast<size_t>(g) * rows + row];
    nan |= isnan(v.y);
    merge_stat(m, s, v.x, v.y, c);
    z = fmaxf(z, v.z);
  }
  return make_float3(m, nan ? NAN : s, z);
}

// One warp per sequence: lane j tests position j (as verify_finalize).
__global__ void __launch_bounds__(32) vp_decide_kernel(const VpParams a) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, j = threadIdx.x, k = a.k;
  const int rows_p = a.B * a.k_p, rows_q = a.B * k;
  const uint64_t bg = a.seq_offset + static_cast<uint64_t>(b);
  bool acc = true, bad = false, nan = false;
  if (j < k) {
    const int d = a.draft[b * k + j];
    bad = d < 0 || d >= a.V;
    const float3 sp = vp_merge(a.parts_p, rows_p, b * a.k_p + j, a.G, a.c);
    const float3 sq = vp_merge(a.parts_q, rows_q, b * k + j, a.G, a.c);
    nan = isnan(sp.y) || isnan(sq.y);
    if (!bad && !nan) {
      const float pd = sp.z > -INFINITY ? fast_exp2((sp.z - sp.x) * a.c) / sp.y : 0.f;
      const float qd = sq.z > -INFINITY ? fast_exp2((sq.z - sq.x) * a.c) / sq.y : 0.f;
      const uint32_t idx = static_cast<uint32_t>(bg * static_cast<uint64_t>(k) + j);
      const float u1 = uniform24(philox_word0(a.seed, a.step, kStreamAccept, idx));
      acc = (qd == 0.f) || (u1 * qd < pd);
    }
  }
  const uint32_t in_k = k >= 32 ? 0xffffffffu : ((1u << k) - 1u);
  const uint32_t rej = __ballot_sync(0xffffffffu, !acc) & in_k;
  const uint32_t badm = __ballot_sync(0xffffffffu, bad) & in_k;
  const uint32_t nanm = __ballot_sync(0xffffffffu, nan) & in_k;
  const int n = rej ? __ffs(rej) - 1 : k;
  int32_t* tok = a.out_tokens + static_cast<size_t>(b) * (k + 1);
  if (badm || nanm) {
    if (j == 0) {
      a.accepted_len[b] = -1;
      a.out_count[b] = -1;
      a.draw[b] = -1;
      raise_status(a.status, (badm ? kDevBadDraft : 0) | (nanm ? kDevNaN : 0));
    }
    for (int i = j; i <= k; i += 32) tok[i] = -1;
    return;
  }
  const int pos = n < k ? n : (a.k_p == k + 1 ? k : -1);
  for (int i = j; i <= k; i += 32) tok[i] = i < n ? a.draft[b * k + i] : -1;
  if (j == 0) {
    a.accepted_len[b] = n;
    a.out_count[b] = n + (pos >= 0 ? 1 : 0);
    a.draw[b] = pos;
    if (pos >= 0) {
      const float3 sp = vp_merge(a.parts_p, rows_p, b * a.k_p + pos, a.G, a.c);
      float3 sq = make_float3(0.f, 1.f, 0.f);
      if (pos < k) sq = vp_merge(a.parts_q, rows_q, b * k + pos, a.G, a.c);
      a.draw_stats[b] = make_float4(sp.x, sp.y, sq.x, sq.y);
    }
  }
}

// Sum of one double per thread over the CTA (valid in every thread).
__device__ __forceinline__ double block_sum(double v, double* slots) {
  v = warp_sum(v);
  if ((threadIdx.x & 31) == 0) slots[threadIdx.x >> 5] = v;
  cta_sync();
  double t = 0.0;
  for (int w = 0; w < kDrawThreads / 32; ++w) t += slots[w];
  cta_sync();
  return t;
}

// One CTA per sequence: (residual or bonus mass, p mass) of its draw row over the shard.
template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
    vp_masses_kernel(const T* __restrict__ p, const T* __restrict__ q, const VpParams a) {
  __shared__ double slots[kDrawThreads / 32];
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, pos = a.draw[b];
  if (pos < 0) {
    if (threadIdx.x == 0) a.masses[b] = make_double2(0.0, 0.0);
    return;
  }
  const bool residual = pos < a.k;
  const float4 st = a.draw_stats[b];
  const T* pr = p + (static_cast<size_t>(b) * a.k_p + pos) * a.Vs;
  const T* qr = q + (static_cast<size_t>(b) * a.k + (residual ? pos : 0)) * a.Vs;
  const float inv_sp = 1.f / st.y, inv_sq = residual ? 1.f / st.w : 0.f;
  double r = 0.0, pm = 0.0;
  for (int v = threadIdx.x; v < a.Vs; v += blockDim.x) {
    const float pv = fast_exp2((to_f32<T>(pr[v]) - st.x) * a.c) * inv_sp;
    const float qv = residual ? fast_exp2((to_f32<T>(qr[v]) - st.z) * a.c) * inv_sq : 0.f;
    r += static_cast<double>(fmaxf(pv - qv, 0.f));
    pm += static_cast<double>(pv);
  }
  r = block_sum(r, slots);
  pm = block_sum(pm, slots);
  if (threadIdx.x == 0) a.masses[b] = make_double2(residual ? r : pm, pm);
}

// Owner shard of a draw: the last shard with positive mass w(g) whose
// exclusive prefix (shard order) is <= u Z. Returns it; *tl = u Z - its prefix.
template <typename WFn>
__device__ __forceinline__ int vp_owner(const WFn& w, int G, double u, double* tl) {
  double Z = 0.0;
  for (int g = 0; g < G; ++g) Z += w(g);
  const double thr = u * Z;
  double pre = 0.0, own_pre = 0.0;
  int own = -1;
  for (int g = 0; g < G; ++g) {
    const double wg = w(g);
    if (wg > 0.0 && pre <= thr) {
      own = g;
      own_pre = pre;
    }
    pre += wg;
  }
  *tl = thr - own_pre;
  return own;
}

// One CTA per sequence with a draw: the owner shard writes the drawn token
// (global id) at out_tokens[b, pos]; the other shards leave it -1.
template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
    vp_draw_kernel(const T* __restrict__ p, const T* __restrict__ q, const VpParams a) {
  __shared__ DrawSmem sh;
  __shared__ int s_own;
  __shared__ double s_tl;
  __shared__ int s_res;
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, pos = a.draw[b], k = a.k;
  if (pos < 0) return;
  const bool residual = pos < k;
  if (threadIdx.x == 0) {
    double z0 = 0.0;
    for (int g = 0; g < a.G; ++g) z0 += a.masses[static_cast<size_t>(g) * a.B + b].x;
    const bool use_res = residual && z0 > 0.0;   // zero residual mass: draw from p
    auto w = [&](int g) {
      const double2 m = a.masses[static_cast<size_t>(g) * a.B + b];
      return use_res ? m.x : m.y;
    };
    const uint64_t bg = a.seq_offset + static_cast<uint64_t>(b);
    const uint32_t idx = static_cast<uint32_t>(bg * static_cast<uint64_t>(k) + pos);
    const double u = static_cast<double>(
        uniform24(philox_word0(a.seed, a.step, residual ? kStreamResidual : kStreamBonus, idx)));
    double tl = 0.0;
    s_own = vp_owner(w, a.G, u, &tl);
    s_tl = tl;
    s_res = use_res ? 1 : 0;
  }
  cta_sync();
  if (s_own != a.rank) return;   // uniform over the CTA
  const float4 st = a.draw_stats[b];
  const T* pr = p + (static_cast<size_t>(b) * a.k_p + pos) * a.Vs;
  const T* qr = q + (static_cast<size_t>(b) * k + (residual ? pos : 0)) * a.Vs;
  const float inv_sp = 1.f / st.y, inv_sq = residual ? 1.f / st.w : 0.f;
  const float c = a.c;
  int v;
  if (s_res) {
    auto w_res = [&](int i) {
      const float pv = fast_exp2((to_f32<T>(pr[i]) - st.x) * c) * inv_sp;
      const float qv = fast_exp2((to_f32<T>(qr[i]) - st.z) * c) * inv_sq;
      return fmaxf(pv - qv, 0.f);
    };
    v = block_draw(sh, w_res, a.Vs, s_tl);
  } else {
    auto w_p = [&](int i) { return fast_exp2((to_f32<T>(pr[i]) - st.x) * c) * inv_sp; };
    v = block_draw(sh, w_p, a.Vs, s_tl);
  }
  if (threadIdx.x == 0 && v >= 0) a.out_tokens[static_cast<size_t>(b) * (k + 1) + pos] = a.v0 + v;
}

// One CTA per draft row: from all shards' partials of the row (taken with the
// float-pair scale), the owner shard draws d ~ softmax(z / T) inside its range
// (stream 0, index (seq_offset + b) k + j); the others write -1.
template <typename T>
__global__ void __launch_bounds__(kDrawThreads)
    vp_draft_draw_kernel(const T* __restrict__ q, const VpParams a) {
  __shared__ DrawSmem sh;
  __shared__ int s_own;
  __shared__ double s_tl;
  __shared__ float s_M;
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  const int row = blockIdx.x;
  const int rows = a.B * a.k;
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    bool nan = false;
    for (int g = 0; g < a.G; ++g) {
      const float4 v = a.parts_q[static_cast<size_t>(g) * rows + row];
      nan |= isnan(v.y);
      M = fmaxf(M, v.x);
    }
    s_own = -2;
    if (nan || M == -INFINITY) {
      a.draft_out[row] = -1;
      raise_status(a.status, kDevNaN);
    } else {
      const double cdd = static_cast<double>(a.cd.hi) + static_cast<double>(a.cd.lo);
      auto w = [&](int g) {
        const float4 v = a.parts_q[static_cast<size_t>(g) * rows + row];
        return v.x == -INFINITY ? 0.0
                                : static_cast<double>(v.y) * exp2(static_cast<double>(v.x - M) * cdd);
      };
      const int b = row / a.k, j = row - b * a.k;
      const uint64_t bg = a.seq_offset + static_cast<uint64_t>(b);
      const uint32_t idx = static_cast<uint32_t>(bg * static_cast<uint64_t>(a.k) + j);
      const double u = static_cast<double>(uniform24(philox_word0(a.seed, a.step, kStreamDraft, idx)));
      double tl = 0.0;
      s_own = vp_owner(w, a.G, u, &tl);
      s_tl = tl;
      s_M = M;
      if (s_own != a.rank) a.draft_out[row] = -1;
    }
  }
  cta_sync();
  if (s_own != a.rank) return;   // uniform over the CTA
  const T* zr = q + static_cast<size_t>(row) * a.Vs;
  const float M = s_M;
  const TScale c = a.cd;
  auto w = [&](int i) { return fast_exp2((to_f32<T>(zr[i]) - M) * c); };
  const int v = block_draw(sh, w, a.Vs, s_tl);
  if (threadIdx.x == 0) a.draft_out[row] = v >= 0 ? a.v0 + v : -1;
}

__global__ void philox_kernel(uint64_t seed, uint64_t step, uint32_t stream, uint32_t index0,
                              int64_t n, uint32_t* words, float* u) {
  if (threadIdx.x == 0) pdl_trigger();
  pdl_wait();
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint32_t w = philox_word0(seed, step, stream, index0 + static_cast<uint32_t>(i));
    if (words) words[i] = w;
    if (u) u[i] = uniform24(w);
  }
}

// Cluster width for a vocabulary: enough CTAs that one chunk (two rows of
// logits) fits comfortably in shared memory, at most 8 (portable).
int draw_cluster(int V, int esz, int* chunk_elems) {
  int n = 1;
  while (n < 8 && (static_cast<int64_t>((V + n - 1) / n) * esz * 2 > 48 * 1024)) n <<= 1;
  int per = (V + n - 1) / n;
  per = (per + 7) & ~7;
  *chunk_elems = per;
  return n;
}

template <typename Kern, typename... Args>
uno_status launch_cluster(Kern kern, int grid, int cluster, size_t smem, cudaStream_t s,
                          Args... args) {
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(draw smem)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(kDrawThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, static_cast<unsigned>(cluster), 1, 1);
  cfg.attrs = attr;
  e = cudaLaunchKernelEx(&cfg, kern, args...);
  if (e != cudaSuccess) return cuda_error(e, "sampler launch");
  return UNO_OK;
}

int stat_chunks(int rows, int V) {
  const int target = 4 * device_sm_count();
  int c = (target + rows - 1) / rows;
  c = std::min(c, std::max(1, V / 2048));
  return std::max(1, c);
}

}  // namespace

size_t verify_workspace(int32_t B, int32_t k, int32_t k_p, int32_t V) {
  const int rows = B * k_p + B * k;
  const int chunks = stat_chunks(rows, V);
  return static_cast<size_t>(rows) * chunks * sizeof(float2);
}

uno_status verify_launch(const VerifyArgs& a, void* ws, cudaStream_t s) {
  const int rows = a.B * a.k_p + a.B * a.k;
  const int chunks = stat_chunks(rows, a.V);
  const int chunk_len = ((a.V + chunks - 1) / chunks + 7) & ~7;
  const float c = make_scale(a.temperature);
  float2* stats = static_cast<float2*>(ws);
  const int esz = a.dt == UNO_F32 ? 4 : 2;
  int chunk_elems = 0;
  const int cl = draw_cluster(a.V, esz, &chunk_elems);
  FinalizeParams fp{};
  fp.B = a.B;
  fp.k = a.k;
  fp.k_p = a.k_p;
  fp.V = a.V;
  fp.chunks = chunks;
  fp.c = c;
  fp.seed = a.seed;
  fp.step = a.step;
  fp.seq_offset = a.seq_offset;
  fp.draft = a.draft;
  fp.stats = stats;
  fp.accepted_len = a.accepted_len;
  fp.out_tokens = a.out_tokens;
  fp.out_count = a.out_count;
  fp.status = a.dev_status;
  fp.chunk_elems = chunk_elems;
  // bf16 rows whose every 8-id vector is 16-byte aligned are read in place by
  // the draw: no staging, so many more clusters fit on the GPU at once
  fp.direct = a.dt == UNO_BF16 && a.V % 8 == 0 &&
              ((reinterpret_cast<uintptr_t>(a.p_logits) | reinterpret_cast<uintptr_t>(a.q_logits)) & 15u) == 0;
  const size_t smem = fp.direct ? 0 : static_cast<size_t>(chunk_elems) * esz * 2;
  const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(rows) * chunks));
  cudaError_t e;
  if (a.dt == UNO_F32) {
    e = launch_kernel(row_stats_kernel<float>, grid, dim3(kStatThreads), 0, s, 1,
                      static_cast<const float*>(a.p_logits), static_cast<const float*>(a.q_logits),
                      a.B * a.k_p, a.V, chunks, chunk_len, c, stats);
  } else {
    e = launch_kernel(row_stats_kernel<__nv_bfloat16>, grid, dim3(kStatThreads), 0, s, 1,
                      static_cast<const __nv_bfloat16*>(a.p_logits),
                      static_cast<const __nv_bfloat16*>(a.q_logits), a.B * a.k_p, a.V, chunks,
                      chunk_len, c, stats);
  }
  if (e != cudaSuccess) return cuda_error(e, "row_stats launch");
  if (a.dt == UNO_F32)
    return launch_cluster(verify_finalize_kernel<float>, a.B * cl, cl, smem, s,
                          static_cast<const float*>(a.p_logits),
                          static_cast<const float*>(a.q_logits), fp);
  return launch_cluster(verify_finalize_kernel<__nv_bfloat16>, a.B * cl, cl, smem, s,
                        static_cast<const __nv_bfloat16*>(a.p_logits),
                        static_cast<const __nv_bfloat16*>(a.q_logits), fp);
}

size_t tree_verify_workspace(int32_t B, int32_t k, int32_t R, int32_t V) {
  const int rows = B * R + B * k;
  const int chunks = stat_chunks(rows, V);
  return static_cast<size_t>(rows) * chunks * sizeof(float2);
}

uno_status tree_verify_launch(const TreeVerifyArgs& a, void* ws, cudaStream_t s) {
  const int rows = a.B * a.R + a.B * a.k;
  const int chunks = stat_chunks(rows, a.V);
  const int chunk_len = ((a.V + chunks - 1) / chunks + 7) & ~7;
  const float c = make_scale(a.temperature);
  float2* stats = static_cast<float2*>(ws);
  const int esz = a.dt == UNO_F32 ? 4 : 2;
  int chunk_elems = 0;
  const int cl = draw_cluster(a.V, esz, &chunk_elems);
  TreeParams tp{};
  tp.B = a.B;
  tp.N = a.N;
  tp.k = a.k;
  tp.R = a.R;
  tp.V = a.V;
  tp.chunks = chunks;
  tp.bonus = a.bonus ? 1 : 0;
  tp.c = c;
  tp.seed = a.seed;
  tp.step = a.step;
  tp.seq_offset = a.seq_offset;
  tp.cands = a.cands;
  tp.stats = stats;
  tp.accepted_len = a.accepted_len;
  tp.out_tokens = a.out_tokens;
  tp.out_count = a.out_count;
  tp.status = a.dev_status;
  tp.chunk_elems = chunk_elems;
  const size_t smem = static_cast<size_t>(chunk_elems) * esz * 2;
  const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(rows) * chunks));
  cudaError_t e;
  if (a.dt == UNO_F32) {
    e = launch_kernel(row_stats_kernel<float>, grid, dim3(kStatThreads), 0, s, 1,
                      static_cast<const float*>(a.p_logits), static_cast<const float*>(a.q_logits),
                      a.B * a.R, a.V, chunks, chunk_len, c, stats);
  } else {
    e = launch_kernel(row_stats_kernel<__nv_bfloat16>, grid, dim3(kStatThreads), 0, s, 1,
                      static_cast<const __nv_bfloat16*>(a.p_logits),
                      static_cast<const __nv_bfloat16*>(a.q_logits), a.B * a.R, a.V, chunks,
                      chunk_len, c, stats);
  }
  if (e != cudaSuccess) return cuda_error(e, "row_stats launch");
  if (a.dt == UNO_F32)
    return launch_cluster(tree_finalize_kernel<float>, a.B * cl, cl, smem, s,
                          static_cast<const float*>(a.p_logits),
                          static_cast<const float*>(a.q_logits), tp);
  return launch_cluster(tree_finalize_kernel<__nv_bfloat16>, a.B * cl, cl, smem, s,
                        static_cast<const __nv_bfloat16*>(a.p_logits),
                        static_cast<const __nv_bfloat16*>(a.q_logits), tp);
}

uno_status distill_launch(const DistillArgs& a, cudaStream_t s) {
  const int esz = a.dt == UNO_F32 ? 4 : 2;
  int chunk_elems = 0;
  const int cl = draw_cluster(a.V, esz, &chunk_elems);
  DistillParams dp{};
  dp.V = a.V;
  dp.chunk_elems = chunk_elems;
  dp.c = make_scale(a.temperature);
  dp.inv_t = 1.f / a.temperature;
  dp.alpha = a.alpha;
  dp.beta = a.beta;
  dp.grad_scale = 1.f / (a.temperature * static_cast<float>(a.rows));
  dp.losses = a.losses;
  dp.grad = a.grad;
  dp.status = a.dev_status;
  const size_t smem = static_cast<size_t>(chunk_elems) * esz * 2;
  if (a.dt == UNO_F32)
    return launch_cluster(distill_kernel<float>, a.rows * cl, cl, smem, s,
                          static_cast<const float*>(a.z_teacher),
                          static_cast<const float*>(a.z_student), dp);
  return launch_cluster(distill_kernel<__nv_bfloat16>, a.rows * cl, cl, smem, s,
                        static_cast<const __nv_bfloat16*>(a.z_teacher),
                        static_cast<const __nv_bfloat16*>(a.z_student), dp);
}

// Vocabulary chunks of the draft's stats pass: kSubLen ids each, one warp
// per chunk, so the draw re-reads 1 / chunks of each row.
int draft_chunks(int rows, int V) {
  (void)rows;
  return (V + kSubLen - 1) / kSubLen;
}

size_t draft_workspace(int32_t B, int32_t k, int32_t V) {
  const int rows = B * k;
  return static_cast<size_t>(rows) * draft_chunks(rows, V) * sizeof(DraftStat);
}

uno_status draft_launch(const DraftArgs& a, void* ws, cudaStream_t s) {
  const int rows = a.B * a.k;
  const int chunks = draft_chunks(rows, a.V);
  if (chunks > kDraftMaxChunks) return set_error(UNO_ERR_UNSUPPORTED, "vocabulary too large for the draft");
  const int chunk_len = kSubLen;
  const TScale c = make_tscale(a.temperature);
  DraftStat* stats = static_cast<DraftStat*>(ws);
  DraftParams dp{};
  dp.k = a.k;
  dp.V = a.V;
  dp.chunks = chunks;
  dp.chunk_len = chunk_len;
  dp.c = c;
  dp.seed = a.seed;
  dp.step = a.step;
  dp.seq_offset = a.seq_offset;
  dp.stats = stats;
  dp.draft = a.draft;
  dp.status = a.dev_status;
  const int64_t warps = static_cast<int64_t>(rows) * chunks;
  const dim3 grid(static_cast<unsigned>((warps + kStatThreads / 32 - 1) / (kStatThreads / 32)));
  cudaError_t e;
  if (a.dt == UNO_F32) {
    const float* q = static_cast<const float*>(a.q_logits);
    e = launch_kernel(draft_stats_kernel<float>, grid, dim3(kStatThreads), 0, s, 1, q, rows, a.V,
                      chunks, c, stats);
    if (e == cudaSuccess)
      e = launch_kernel(draft_draw_kernel<float>, dim3(rows), dim3(kDrawThreads), 0, s, 1, q, dp);
  } else {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q_logits);
    const bool staged = (reinterpret_cast<uintptr_t>(q) & 15u) == 0 && a.V % 8 == 0;
    if (staged) {
      const uint32_t smem = kStagedWarps * kDraftSlots * kDraftSlotBytes;
      const int64_t per_cta = kStagedWarps;
      const int ctas = static_cast<int>(std::max<int64_t>(
          1, std::min<int64_t>(device_sm_count(), (warps + per_cta - 1) / per_cta)));
      e = cudaFuncSetAttribute(draft_stats_staged_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               static_cast<int>(smem));
      if (e == cudaSuccess)
        e = launch_kernel(draft_stats_staged_kernel, dim3(ctas), dim3(kStagedThreads), smem, s, 1, q,
                          rows, a.V, chunks, c, stats, a.dev_status);
    } else {
      e = launch_kernel(draft_stats_kernel<__nv_bfloat16>, grid, dim3(kStatThreads), 0, s, 1, q,
                        rows, a.V, chunks, c, stats);
    }
    if (e == cudaSuccess)
      e = launch_kernel(draft_draw_kernel<__nv_bfloat16>, dim3(rows), dim3(kDrawThreads), 0, s, 1,
                        q, dp);
  }
  if (e != cudaSuccess) return cuda_error(e, "draft launch");
  return UNO_OK;
}

namespace {
VpParams vp_params(const VpArgs& a) {
  VpParams p{};
  p.B = a.B;
  p.k = a.k;
  p.k_p = a.k_p;
  p.Vs = a.Vs;
  p.v0 = a.v0;
  p.V = a.V;
  p.G = a.G;
  p.rank = a.rank;
  p.c = make_scale(a.temperature);
  p.cd = make_tscale(a.temperature);
  p.seed = a.seed;
  p.step = a.step;
  p.seq_offset = a.seq_offset;
  p.draft = a.draft;
  p.parts_p = reinterpret_cast<const float4*>(a.parts_p);
  p.parts_q = reinterpret_cast<const float4*>(a.parts_q);
  p.accepted_len = a.accepted_len;
  p.out_tokens = a.out_tokens;
  p.out_count = a.out_count;
  p.draw = a.draw;
  p.draw_stats = reinterpret_cast<float4*>(a.draw_stats);
  p.masses = reinterpret_cast<double2*>(a.masses);
  p.draft_out = a.draft_out;
  p.status = a.dev_status;
  return p;
}
}  // namespace

uno_status vp_partials_launch(uno_dtype dt, int rows, int Vs, int v0, const void* z,
                              const int32_t* draft, int k, int k_p, int id_kind, bool precise,
                              float temperature, float* out, cudaStream_t s) {
  if (rows == 0) return UNO_OK;
  float4* o = reinterpret_cast<float4*>(out);
  cudaError_t e;
  const float c = make_scale(temperature);
  const TScale cd = make_tscale(temperature);
  if (dt == UNO_F32) {
    const float* zz = static_cast<const float*>(z);
    e = precise ? launch_kernel(vp_partials_kernel<float, TScale>, dim3(rows), dim3(kStatThreads), 0, s,
                                1, zz, Vs, v0, draft, k, k_p, id_kind, cd, o)
                : launch_kernel(vp_partials_kernel<float, float>, dim3(rows), dim3(kStatThreads), 0, s,
                                1, zz, Vs, v0, draft, k, k_p, id_kind, c, o);
  } else {
    const __nv_bfloat16* zz = static_cast<const __nv_bfloat16*>(z);
    e = precise ? launch_kernel(vp_partials_kernel<__nv_bfloat16, TScale>, dim3(rows),
                                dim3(kStatThreads), 0, s, 1, zz, Vs, v0, draft, k, k_p, id_kind, cd, o)
                : launch_kernel(vp_partials_kernel<__nv_bfloat16, float>, dim3(rows),
                                dim3(kStatThreads), 0, s, 1, zz, Vs, v0, draft, k, k_p, id_kind, c, o);
  }
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "vocab-shard partials launch");
}

uno_status vp_decide_launch(const VpArgs& a, cudaStream_t s) {
  if (a.B == 0) return UNO_OK;
  const cudaError_t e = launch_kernel(vp_decide_kernel, dim3(a.B), dim3(32), 0, s, 1, vp_params(a));
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "vocab-shard decide launch");
}

uno_status vp_masses_launch(const VpArgs& a, cudaStream_t s) {
  if (a.B == 0) return UNO_OK;
  cudaError_t e;
  if (a.dt == UNO_F32)
    e = launch_kernel(vp_masses_kernel<float>, dim3(a.B), dim3(kDrawThreads), 0, s, 1,
                      static_cast<const float*>(a.p), static_cast<const float*>(a.q), vp_params(a));
  else
    e = launch_kernel(vp_masses_kernel<__nv_bfloat16>, dim3(a.B), dim3(kDrawThreads), 0, s, 1,
                      static_cast<const __nv_bfloat16*>(a.p), static_cast<const __nv_bfloat16*>(a.q),
                      vp_params(a));
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "vocab-shard masses launch");
}

uno_status vp_draw_launch(const VpArgs& a, cudaStream_t s) {
  if (a.B == 0) return UNO_OK;
  cudaError_t e;
  if (a.dt == UNO_F32)
    e = launch_kernel(vp_draw_kernel<float>, dim3(a.B), dim3(kDrawThreads), 0, s, 1,
                      static_cast<const float*>(a.p), static_cast<const float*>(a.q), vp_params(a));
  else
    e = launch_kernel(vp_draw_kernel<__nv_bfloat16>, dim3(a.B), dim3(kDrawThreads), 0, s, 1,
                      static_cast<const __nv_bfloat16*>(a.p), static_cast<const __nv_bfloat16*>(a.q),
                      vp_params(a));
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "vocab-shard draw launch");
}

uno_status vp_draft_draw_launch(const VpArgs& a, cudaStream_t s) {
  const int rows = a.B * a.k;
  if (rows == 0) return UNO_OK;
  cudaError_t e;
  if (a.dt == UNO_F32)
    e = launch_kernel(vp_draft_draw_kernel<float>, dim3(rows), dim3(kDrawThreads), 0, s, 1,
                      static_cast<const float*>(a.q), vp_params(a));
  else
    e = launch_kernel(vp_draft_draw_kernel<__nv_bfloat16>, dim3(rows), dim3(kDrawThreads), 0, s, 1,
                      static_cast<const __nv_bfloat16*>(a.q), vp_params(a));
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "vocab-shard draft launch");
}

uno_status philox_launch(uint64_t seed, uint64_t step, uint32_t stream_id, uint32_t index0,
                         int64_t n, uint32_t* words, float* u, cudaStream_t s) {
  if (n == 0) return UNO_OK;
  const int threads = 256;
  const int64_t blocks = std::min<int64_t>((n + threads - 1) / threads, 8 * device_sm_count());
  const cudaError_t e = launch_kernel(philox_kernel, dim3(static_cast<unsigned>(blocks)),
                                      dim3(threads), 0, s, 1, seed, step, stream_id, index0, n,
                                      words, u);
  if (e != cudaSuccess) return cuda_error(e, "philox launch");
  return UNO_OK;
}

}  // namespace uno

// ---------------------------------------------------------------- verify without allocation
//
// uno_psi_verify_noalloc keeps the per-(logit row, vocab chunk) stats in a
// static device array of this file instead of a caller workspace. It serves
// callers that cannot allocate device memory where they verify: a decode loop
// that must not stall on the device-wide synchronisation cudaMalloc/cudaFree
// may cause, or a host runtime that owns the logits and output buffers but no
// device allocator. The pages describe no such variant.
namespace uno {
namespace {

constexpr size_t kNoAllocStatsBytes = size_t{2} << 20;   // 2 MiB: 262,144 (m, s) pairs
constexpr int kNoAllocMaxDevices = 64;

// Every entry a call reads is written earlier in the same call (row stats
// kernel before the finalize kernel, ordered on one stream), so the array
// needs no starting value and is never cleared.
static __device__ __align__(256) float2 g_noalloc_stats[kNoAllocStatsBytes / sizeof(float2)];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_stats on the current device; looked up once per
// device (the lookup may load this library's module onto the device).
uno_status noalloc_scratch(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_error(e, "cudaGetDevice");
  if (dev < 0 || dev >= kNoAllocMaxDevices)
    return set_error(UNO_ERR_UNSUPPORTED, "device %d: the static verify scratch serves devices 0..%d",
                     dev, kNoAllocMaxDevices - 1);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_stats);
    if (e != cudaSuccess) return cuda_error(e, "cudaGetSymbolAddress of the static verify scratch");
    if (!p) return set_error(UNO_ERR_CUDA, "static verify scratch has a NULL device address");
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return UNO_OK;
}

}  // namespace
}  // namespace uno

extern "C" uno_status uno_psi_verify_noalloc(uno_dtype dt, int32_t B, int32_t k, int32_t k_p,
                                             int32_t V, const void* p_logits,
                                             const void* q_logits, const int32_t* draft,
                                             float temperature, uint64_t seed, uint64_t step,
                                             uint64_t seq_offset, int32_t* accepted_len,
                                             int32_t* out_tokens, int32_t* out_count,
                                             int32_t* dev_status, void* stream) {
  using namespace uno;
  const size_t need = uno_psi_verify_workspace(B, k, k_p, V);
  if (need > kNoAllocStatsBytes)
    return set_error(UNO_ERR_UNSUPPORTED,
                     "uno_psi_verify_noalloc: B=%d k=%d k_p=%d V=%d needs %zu bytes of stats "
                     "scratch, the static scratch holds %zu; call uno_psi_verify with a workspace",
                     B, k, k_p, V, need, kNoAllocStatsBytes);
  void* ws = nullptr;
  const uno_status s = noalloc_scratch(&ws);
  if (s != UNO_OK) return s;
  // Argument checks, kernels and results are those of uno_psi_verify.
  return uno_psi_verify(dt, B, k, k_p, V, p_logits, q_logits, draft, temperature, seed, step,
                        seq_offset, accepted_len, out_tokens, out_count, dev_status, ws,
                        kNoAllocStatsBytes, stream);
}
