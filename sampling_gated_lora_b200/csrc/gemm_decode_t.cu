// Gated-LoRA linear for decode-size batches with the rank-r activations
// computed once per linear (bf16, M <= 32 rows, r <= 128):
//
//   t = scale * gate (.) (x A^T)          lora_down_dec_kernel
//   y = x W^T + t Bl^T                    gemm_dect_kernel
//
// (the gated LoRA of hyper.ai page, section "方法": the adapter is off on the
// verify rows and on for the draft rows of one forward pass).
//
// Why two launches. A kernel that computes the adapter term inside every
// weight tile re-reads A (r x K) in each of the N/128 feature tiles, as many
// bytes as W for a 4096 x 4096 linear, and the A tiles take half of each
// pipeline stage; timestamps inside such a kernel showed its main loop held
// to ~68 GB/s per SM by the bytes it could keep in flight. Here t is
// computed once, spread over the SMs, and the weight kernel's stages carry W
// and x only.
//
// lora_down_dec_kernel: CTA (j-block of 8 adapter rows, K-slice s); a
// cluster of S CTAs covers K. Each CTA copies its rows of A (constant) into
// shared memory before it waits for the writer of x, then stages its x
// slice; warp w takes adapter row 8 jb + w, lane l the token rows
// l, l + 32, ...; the cluster adds the S partial sums through distributed
// shared memory in rank order (no atomics: the result does not depend on
// timing) and writes t rounded to bf16.
//
// gemm_dect_kernel: the weight rows fill the 128-row MMA side, the tokens the
// N side (16 or 32); K is split over a cluster of CTAs. The CTA of K-slice 0
// first adds Bl t^T (its Bl rows and the t tile, r/64 K-blocks), then every
// CTA streams its W slice through a ring of W + x stages, and the cluster sums
// the CTAs' accumulators through distributed shared memory. Shared memory is
// held to about half an SM, so the next launch's CTAs can start on an SM
// while this launch's CTA drains; the CTAs of other K-slices use the Bl / t
// space as extra stages.
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace uno {

namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;                          // MMA M
constexpr int kHalf = 64;
constexpr int kRowBytes = 128;                      // 64 bf16 of K per row
constexpr uint32_t kTileBytes = kRows * kRowBytes;  // 16 KB
constexpr int kPartPad = 4;
constexpr uint32_t kSmemHalfSm = 110u * 1024u;      // shared memory of one CTA

// ------------------------------------------------------------------ t = s g (x A^T)

constexpr int kDownThreads = 256;
constexpr int kDownRows = 8;        // adapter rows per CTA (one per warp)
constexpr int kDownMaxM = 32;       // token rows (one per lane)
constexpr int kDownPad = 8;         // bf16 of padding per staged x row

struct DownDecParams {
  const __nv_bfloat16* x;
  const __nv_bfloat16* A[kMaxGroups];
  __nv_bfloat16* t;
  const uint8_t* gate;
  int M, K, r, G, ldt, kslice, gate_row0;
  float scale;
};

__global__ void __launch_bounds__(kDownThreads)
    lora_down_dec_kernel(const DownDecParams p) {
  extern __shared__ __align__(16) uint8_t dsm[];
  __shared__ __align__(8) uint64_t abar;
  const int jb = blockIdx.x;
  const int S = static_cast<int>(gridDim.y);
  const int s = blockIdx.y;
  const int k0 = s * p.kslice;
  const int kl = max(0, min(p.K, k0 + p.kslice) - k0);
  const int J = p.G * p.r;
  const int stride = p.kslice + kDownPad;   // staged x row, in bf16
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(dsm);
  __nv_bfloat16* as = xs + static_cast<size_t>(p.M) * stride;
  float* part = reinterpret_cast<float*>(as + static_cast<size_t>(kDownRows) * p.kslice);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // rows of A (constant): bulk copies into shared memory before the wait
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&abar), 1);
    fence_mbar_init();
  }
  cta_sync();
  if (threadIdx.x == 0) {
    pdl_trigger();
    int n = 0;
    for (int w = 0; w < kDownRows; ++w) n += (jb * kDownRows + w < J && kl > 0) ? 1 : 0;
    mbar_arrive_expect_tx(smem_u32(&abar), static_cast<uint32_t>(n * kl * 2));
    for (int w = 0; w < kDownRows; ++w) {
      const int j = jb * kDownRows + w;
      if (j >= J || kl == 0) continue;
      const int gi = j / p.r;   // constant indices: the parameter array stays out of local memory
      const __nv_bfloat16* Ag = gi == 0 ? p.A[0] : (gi == 1 ? p.A[1] : p.A[2]);
      const __nv_bfloat16* src = Ag + static_cast<size_t>(j % p.r) * p.K + k0;
      bulk_load(smem_u32(as + static_cast<size_t>(w) * p.kslice), src, static_cast<uint32_t>(kl * 2),
                smem_u32(&abar));
    }
  }
  pdl_wait();
  // the x slice: 16-byte vectors (K and kslice are multiples of 8)
  const int nv = kl / 8;
  for (int i = threadIdx.x; i < p.M * nv; i += kDownThreads) {
    const int m = i / nv, c = i - m * nv;
    *reinterpret_cast<uint4*>(xs + static_cast<size_t>(m) * stride + 8 * c) =
        *reinterpret_cast<const uint4*>(p.x + static_cast<size_t>(m) * p.K + k0 + 8 * c);
  }
  const bool got = mbar_wait(smem_u32(&abar), 0);
  cta_sync();
  float acc = 0.f;
  const int j = jb * kDownRows + warp;
  if (got && j < J && lane < p.M) {
    const __nv_bfloat16* ar = as + static_cast<size_t>(warp) * p.kslice;
    const __nv_bfloat16* xr = xs + static_cast<size_t>(lane) * stride;
    for (int c = 0; c < kl; c += 8) {
      const uint4 av = *reinterpret_cast<const uint4*>(ar + c);
      const uint4 xv = *reinterpret_cast<const uint4*>(xr + c);
      acc += bf16_lo(av.x) * bf16_lo(xv.x) + bf16_hi(av.x) * bf16_hi(xv.x) +
             bf16_lo(av.y) * bf16_lo(xv.y) + bf16_hi(av.y) * bf16_hi(xv.y) +
             bf16_lo(av.z) * bf16_lo(xv.z) + bf16_hi(av.z) * bf16_hi(xv.z) +
             bf16_lo(av.w) * bf16_lo(xv.w) + bf16_hi(av.w) * bf16_hi(xv.w);
    }
  }
  if (!got && threadIdx.x == 0) raise_status(nullptr, kDevTimeout);
  part[lane * kDownRows + warp] = acc;   // [token][adapter row] of this K-slice
  cluster_sync();
  // the cluster's S partials, in rank order; CTA rank q writes its share of the outputs
  const uint32_t q = cluster_ctarank();
  const int outs = kDownMaxM * kDownRows;
  const int per = (outs + S - 1) / S;
  for (int e = static_cast<int>(q) * per + threadIdx.x; e < min(outs, (static_cast<int>(q) + 1) * per);
       e += kDownThreads) {
    const int m = e / kDownRows, w = e - m * kDownRows;
    const int jj = jb * kDownRows + w;
    if (m >= p.M || jj >= J) continue;
    float sum = 0.f;
    for (int rk = 0; rk < S; ++rk)
      sum += ld_cluster_f32(map_shared_rank(smem_u32(part + e), static_cast<uint32_t>(rk)));
    const float g = p.gate ? static_cast<float>(p.gate[m]) : (m >= p.gate_row0 ? 1.f : 0.f);
    p.t[static_cast<size_t>(m) * p.ldt + jj] = __float2bfloat16_rn(p.scale * g * sum);
  }
  cluster_sync();   // every CTA has read the others' partials before any exits
}

// ------------------------------------------------------------------ y = x W^T + t Bl^T

struct DectParams {
  GemmArgs a;
  int bn, tmem_cols, kb_per_split, splits, nkr;
  int stages0, stages;          // ring stages of K-slice 0 and of the others
  uint32_t stage_bytes, bl_off, tq_off, bar_off;
};
static_assert(sizeof(DectParams) <= kLaunchParamBytes, "DectParams must fit GemmLaunch::params");

__device__ __forceinline__ void epi_bar() { named_sync(1, 128); }

template <bool kSilu>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_dect_kernel(const __grid_constant__ TensorMaps tm, const DectParams p) {
  constexpr int kT = kSilu ? 2 : 1;   // adapters per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
  const GemmArgs& a = p.a;
  const int bn = p.bn;
  const int ft = blockIdx.y, split = blockIdx.z;
  const bool adapter = split == 0 && p.nkr > 0;
  const int S = adapter ? p.stages0 : p.stages;   // K-slices without the adapter use its space
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* empty = full + p.stages;
  uint64_t* accum = empty + p.stages;
  uint64_t* adfull = accum + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  constexpr uint32_t x_off = kTileBytes;   // within a stage: W | x

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = group_of(a, ft);
  const int feat0 = (ft - a.g[g].tile0) * (kSilu ? kHalf : kRows);
  const int tok0 = blockIdx.x * bn;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accum), 1);
    mbar_init(smem_u32(adfull), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  cta_sync();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();

  const int nkb = a.nkb_main;
  const int kb0 = split * p.kb_per_split;
  const int kb1 = min(nkb, kb0 + p.kb_per_split);
  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(a.status, kDevTimeout);
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    const uint32_t bl = smem_u32(smem + p.bl_off), tq = smem_u32(smem + p.tq_off);
    if (adapter) {   // Bl rows of this tile (constant) now, t after the wait
      const uint32_t fb = smem_u32(adfull);
      mbar_arrive_expect_tx(fb, static_cast<uint32_t>(kT * p.nkr) *
                                    (kTileBytes + static_cast<uint32_t>(bn) * kRowBytes));
      for (int h = 0; h < kT; ++h)
        for (int kb = 0; kb < p.nkr; ++kb) {
          const uint32_t dst = bl + static_cast<uint32_t>(h * p.nkr + kb) * kTileBytes;
          if (kSilu) {   // gate rows then up rows; the other adapter's half reads zeros
            tma_load_2d(dst, &tm.b[0], kb * 64, h == 0 ? feat0 : a.g[0].b_rows, fb);
            tma_load_2d(dst + kTileBytes / 2, &tm.b[1], kb * 64, h == 1 ? feat0 : a.g[1].b_rows, fb);
          } else {
            tma_load_2d(dst, &tm.b[g], kb * 64, feat0, fb);
          }
        }
    }
    auto load_w = [&](int kb, uint32_t st, uint32_t fb) {
      const int kc = kb * 64;
      if (kSilu) {
        tma_load_2d(st, &tm.w[0], kc, feat0, fb);
        tma_load_2d(st + kTileBytes / 2, &tm.w[1], kc, feat0, fb);
      } else {
        tma_load_2d(st, &tm.w[g], kc, feat0, fb);
      }
    };
    const uint32_t tx = kTileBytes + static_cast<uint32_t>(bn) * kRowBytes;
    const int pre = min(S, kb1 - kb0);
    for (int q = 0; q < pre; ++q) {
      const uint32_t st = smem_u32(smem + q * p.stage_bytes);
      mbar_arrive_expect_tx(smem_u32(&full[q]), tx);
      load_w(kb0 + q, st, smem_u32(&full[q]));
    }
    pdl_wait();
    if (adapter)
      for (int h = 0; h < kT; ++h)
        for (int kb = 0; kb < p.nkr; ++kb)
          tma_load_2d(tq + static_cast<uint32_t>((h * p.nkr + kb) * bn * kRowBytes), &tm.t,
                      a.g[kSilu ? h : g].t_col + kb * 64, tok0, smem_u32(adfull));
    for (int q = 0; q < pre; ++q)
      tma_load_2d(smem_u32(smem + q * p.stage_bytes) + x_off, &tm.x, (kb0 + q) * 64, tok0,
                  smem_u32(&full[q]));
    int it = pre;
    for (int kb = kb0 + pre; kb < kb1; ++kb, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1u;
      if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u) || *abort_flag) {
        fail();
        break;
      }
      const uint32_t st = smem_u32(smem + s * p.stage_bytes);
      const uint32_t fb = smem_u32(&full[s]);
      mbar_arrive_expect_tx(fb, tx);
      load_w(kb, st, fb);
      tma_load_2d(st + x_off, &tm.x, kb * 64, tok0, fb);
    }
    prefetch_next(a.pf, static_cast<long long>(blockIdx.y) * gridDim.z + blockIdx.z,
                  static_cast<long long>(gridDim.y) * gridDim.z);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_f32acc(kRows, bn, false);
    uint32_t acc_flag = 0;
    bool ok = true;
    if (adapter) {   // D = Bl t^T first: t is ready as soon as x is
      if (mbar_wait(smem_u32(adfull), 0)) {
        tc_fence_after();
        const uint32_t bl = smem_u32(smem + p.bl_off), tq = smem_u32(smem + p.tq_off);
        for (int h = 0; h < kT; ++h)
          for (int kb = 0; kb < p.nkr; ++kb) {
            const uint64_t bd = sdesc_k_sw128(bl + static_cast<uint32_t>(h * p.nkr + kb) * kTileBytes);
            const uint64_t td = sdesc_k_sw128(tq + static_cast<uint32_t>((h * p.nkr + kb) * bn * kRowBytes));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              mma_ss<false>(tmem, bd + 2 * kk, td + 2 * kk, idesc, acc_flag);
              acc_flag = 1;
            }
          }
      } else {
        fail();
        ok = false;
      }
    }
    int it = 0;
    for (int kb = kb0; ok && kb < kb1; ++kb, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1u;
      if (!mbar_wait(smem_u32(&full[s]), ph)) {
        fail();
        break;
      }
      tc_fence_after();
      const uint32_t st = smem_u32(smem + s * p.stage_bytes);
      const uint64_t xd = sdesc_k_sw128(st + x_off);
      const uint64_t wd = sdesc_k_sw128(st);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        mma_ss<false>(tmem, wd + 2 * kk, xd + 2 * kk, idesc, acc_flag);
        acc_flag = 1;
      }
      mma_commit(smem_u32(&empty[s]));
    }
    mma_commit(smem_u32(accum));
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int i = quarter * 32 + lane;   // TMEM lane: feature row of D
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    pdl_wait();
    bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(accum), 0));
    if (!ok && lane == 0) fail();
    tc_fence_after();
    // an empty K-slice (no K-blocks and no adapter) accumulated nothing: zeros
    const bool empty_slice = kb1 <= kb0 && !adapter;
    float* stage = reinterpret_cast<float*>(smem);   // the stage ring is free now
    const uint32_t trow = tmem + lane_base;
    auto ld16 = [&](int c, float (&v)[16]) {
      if (empty_slice) {
#pragma unroll
        for (int j = 0; j < 16; ++j) v[j] = 0.f;
      } else {
        tmem_ld16(trow + c, v);
      }
    };
    if (p.splits == 1) {
      if (!kSilu) {
        if (ok) {
          for (int c = 0; c < bn; c += 16) {
            float v[16];
            ld16(c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) epi_store1<__nv_bfloat16>(a, g, tok0 + c + j, feat0 + i, v[j]);
          }
        }
      } else {
        const int R = bn * (kHalf + 1);
        const int f = i & (kHalf - 1);
        float* dst = stage + (i < kHalf ? 0 : R);
        if (ok) {
          for (int c = 0; c < bn; c += 16) {
            float v[16];
            ld16(c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[(c + j) * (kHalf + 1) + f] = v[j];
          }
        }
        epi_bar();
        if (ok) {
          for (int j = i >> 6; j < bn; j += 2)
            epi_store1<__nv_bfloat16>(a, 0, tok0 + j, feat0 + f,
                                      silu_f(stage[j * (kHalf + 1) + f]) * stage[R + j * (kHalf + 1) + f]);
        }
      }
    } else {
      for (int c = 0; c < bn; c += 16) {
        float v[16];
        ld16(c, v);
        if (!ok) {
#pragma unroll
          for (int j = 0; j < 16; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) stage[(c + j) * (kRows + kPartPad) + i] = v[j];
      }
    }
  }

  if (p.splits > 1) {
    cluster_sync();
    const uint32_t rank = cluster_ctarank();
    const int Sp = p.splits;
    const int groups = kSilu ? bn * (kRows / 8) : bn * (kRows / 4);
    const int chunk = (groups + Sp - 1) / Sp;
    const int e0 = static_cast<int>(rank) * chunk;
    const int e1 = min(groups, e0 + chunk);
    const uint32_t part0 = smem_u32(smem);
    // unrolled to the largest cluster (8) with constant indices: registers, not stack
    uint32_t peer[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) peer[r] = map_shared_rank(part0, r < Sp ? r : 0);
    auto sum4 = [&](uint32_t off) {
      float4 v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < Sp) v[r] = ld_cluster_f32x4(peer[r] + off);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < Sp) {
          acc.x += v[r].x; acc.y += v[r].y; acc.z += v[r].z; acc.w += v[r].w;
        }
      return acc;
    };
    for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += kThreads) {
      if (!kSilu) {
        const int j = e / (kRows / 4), i4 = e % (kRows / 4);
        const float4 acc = sum4(static_cast<uint32_t>((j * (kRows + kPartPad) + 4 * i4) * 4));
        epi_store4<__nv_bfloat16>(a, g, tok0 + j, feat0 + 4 * i4, acc);
      } else {
        const int j = e / (kRows / 8), f4 = e % (kRows / 8);
        const uint32_t row = static_cast<uint32_t>(j * (kRows + kPartPad));
        const float4 gv = sum4((row + 4 * f4) * 4);
        const float4 uv = sum4((row + kHalf + 4 * f4) * 4);
        epi_store4<__nv_bfloat16>(a, 0, tok0 + j, feat0 + 4 * f4,
                                  make_float4(silu_f(gv.x) * uv.x, silu_f(gv.y) * uv.y,
                                              silu_f(gv.z) * uv.z, silu_f(gv.w) * uv.w));
      }
    }
    cluster_sync();
  }

  tc_fence_before();
  cta_sync();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

// Shared-memory plan: Bl and t tiles, the ring, the barriers. Returns the
// ring stages of K-slice 0 (0 when even two do not fit).
int dect_plan(bool silu, int bn, int nkr, uint32_t* stage_bytes, uint32_t* ad_bytes) {
  const int kT = silu ? 2 : 1;
  *stage_bytes = (kTileBytes + static_cast<uint32_t>(bn) * kRowBytes + 1023u) & ~1023u;
  *ad_bytes = static_cast<uint32_t>(kT * nkr) * (kTileBytes + static_cast<uint32_t>(bn) * kRowBytes);
  const uint32_t budget = kSmemHalfSm - 2048u;   // barriers and alignment slack
  if (*ad_bytes + 2 * *stage_bytes > budget) return 0;
  return std::min(8, static_cast<int>((budget - *ad_bytes) / *stage_bytes));
}

}  // namespace

bool gemm_dect_suits(const GemmProblem& pb) {
  if (pb.dt != UNO_BF16 || pb.M < 1 || pb.M > kDownMaxM || pb.r > 128 || !pb.t) return false;
  if (pb.mode != kEpiStore && pb.mode != kEpiAdd && pb.mode != kEpiSiluPair) return false;
  const bool silu = pb.mode == kEpiSiluPair;
  const int bn = round_up(static_cast<int>(pb.M), 16);
  uint32_t sb, ab;
  if (dect_plan(silu, bn, (pb.r + 63) / 64, &sb, &ab) < 2) return false;
  // one wave: at most two CTAs per SM over all feature tiles and K-slices
  int64_t tiles = 0;
  const int ftile = silu ? kHalf : kRows;
  if (silu) tiles = (pb.g[0].N + ftile - 1) / ftile;
  else
    for (int i = 0; i < pb.ngroups; ++i) tiles += (pb.g[i].N + ftile - 1) / ftile;
  return tiles <= 2 * device_sm_count();
}

uno_status gemm_dect_prepare(const GemmProblem& pb, GemmLaunch* out) {
  const bool silu = pb.mode == kEpiSiluPair;
  const int bn = round_up(static_cast<int>(pb.M), 16);
  const int feat_tile = silu ? kHalf : kRows;
  DectParams dp{};
  dp.a = make_gemm_args(pb, feat_tile, kRowBytes);
  const int feat_tiles = feature_tiles(dp.a, feat_tile);
  if (feat_tiles > 65535) return set_error(UNO_ERR_UNSUPPORTED, "N too large for the tile grid");
  dp.bn = bn;
  dp.nkr = pb.r > 0 ? (pb.r + 63) / 64 : 0;
  uint32_t ad_bytes = 0;
  const int s0 = dect_plan(silu, bn, dp.nkr, &dp.stage_bytes, &ad_bytes);
  if (s0 < 2) return set_error(UNO_ERR_UNSUPPORTED, "decode tile does not fit");
  const uint32_t budget = kSmemHalfSm - 2048u;
  dp.stages0 = s0;
  dp.stages = std::min(8, static_cast<int>(budget / dp.stage_bytes));
  const uint32_t ring = static_cast<uint32_t>(dp.stages) * dp.stage_bytes;
  const uint32_t need_part = static_cast<uint32_t>(bn * (kRows + kPartPad) * 4);
  const uint32_t need_silu = static_cast<uint32_t>(2 * bn * (kHalf + 1) * 4);
  if (need_part > static_cast<uint32_t>(s0) * dp.stage_bytes ||
      need_silu > static_cast<uint32_t>(s0) * dp.stage_bytes)
    return set_error(UNO_ERR_UNSUPPORTED, "decode epilogue does not fit");
  // K-slice 0 keeps Bl and t past its s0 stages; the others use that space as stages
  dp.bl_off = static_cast<uint32_t>(s0) * dp.stage_bytes;
  dp.tq_off = dp.bl_off + static_cast<uint32_t>((silu ? 2 : 1) * dp.nkr) * kTileBytes;
  dp.bar_off = (std::max(ring, dp.bl_off + ad_bytes) + 15u) & ~15u;
  dp.tmem_cols = 32;
  while (dp.tmem_cols < bn) dp.tmem_cols <<= 1;
  const int smem = static_cast<int>(dp.bar_off + 8 * (2 * dp.stages + 2) + 16 + 1024);

  // split K so that the feature tiles times the K-slices cover the SMs (a
  // cluster per feature tile, at most 8 CTAs)
  const int sms = device_sm_count();
  const int nkb = dp.a.nkb_main;
  int splits = std::max(1, std::min({8, sms / std::max(1, feat_tiles), nkb}));
  int kb_per = (nkb + splits - 1) / splits;
  splits = (nkb + kb_per - 1) / kb_per;
  dp.kb_per_split = kb_per;
  dp.splits = splits;

  uno_status s;
  TensorMaps& tm = out->tm;
  if ((s = make_map(&tm.x, pb.dt, pb.x, pb.K, pb.M, pb.K, static_cast<uint32_t>(bn))) != UNO_OK) return s;
  if (pb.r > 0) {
    if ((s = make_map(&tm.t, pb.dt, pb.t, pb.ldt, pb.M, pb.ldt, static_cast<uint32_t>(bn))) != UNO_OK)
      return s;
  } else {
    tm.t = tm.x;
  }
  const uint32_t wbox = silu ? kHalf : kRows;
  for (int i = 0; i < kMaxGroups; ++i) {
    const int gi = i < pb.ngroups ? i : 0;
    const GemmGroup& G = pb.g[gi];
    if ((s = make_map(&tm.w[i], pb.dt, G.W, pb.K, G.N, pb.K, wbox)) != UNO_OK) return s;
    if (pb.r > 0) {
      if ((s = make_map(&tm.b[i], pb.dt, G.Bl, pb.r, G.N, pb.r, wbox)) != UNO_OK) return s;
    } else {
      tm.b[i] = tm.w[i];
    }
    tm.a[i] = tm.w[i];
  }
  std::memcpy(out->params, &dp, sizeof(dp));
  out->kind = 3;
  out->kb_per_split = dp.kb_per_split;
  out->swap = silu ? 1 : 0;   // kernel variant
  out->grid_x = 1;
  out->grid_y = feat_tiles;
  out->splits = splits;
  out->smem_bytes = smem;
  out->dtype = pb.dt;
  return UNO_OK;
}

uno_status gemm_dect_run(const GemmLaunch& l, cudaStream_t stream) {
  void* fn = l.swap ? reinterpret_cast<void*>(&gemm_dect_kernel<true>)
                    : reinterpret_cast<void*>(&gemm_dect_kernel<false>);
  cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, l.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(decode gemm smem)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid_x, l.grid_y, l.splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = l.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, 1, 1, static_cast<unsigned>(l.splits));
  cfg.attrs = attr;
  DectParams dp;
  std::memcpy(&dp, l.params, sizeof(dp));
  void* args[2] = {const_cast<TensorMaps*>(&l.tm), &dp};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_error(e, "decode GEMM launch");
  return UNO_OK;
}

// ---------------------------------------------------------------- the down-projection launch

bool lora_down_dec_suits(int64_t M, int64_t K, int32_t r, int G) {
  if (M < 1 || M > kDownMaxM || r < 1 || r > 128 || G < 1 || G > kMaxGroups || K % 8) return false;
  return true;
}

uno_status lora_down_dec_launch(const DownDecArgs& d, cudaStream_t s) {
  DownDecParams p{};
  p.x = static_cast<const __nv_bfloat16*>(d.x);
  for (int i = 0; i < kMaxGroups; ++i)
    p.A[i] = static_cast<const __nv_bfloat16*>(d.A[i < d.G ? i : 0]);
  p.t = static_cast<__nv_bfloat16*>(d.t);
  p.gate = d.gate;
  p.M = static_cast<int>(d.M);
  p.K = static_cast<int>(d.K);
  p.r = d.r;
  p.G = d.G;
  p.ldt = static_cast<int>(d.ldt);
  p.gate_row0 = static_cast<int>(d.gate_row0 < d.M ? d.gate_row0 : d.M);
  p.scale = d.scale;
  const int J = d.G * d.r;
  const int nj = (J + kDownRows - 1) / kDownRows;
  // K-slices: a cluster of up to 8, enough CTAs for two per SM in all
  int S = std::max(1, std::min(8, (2 * device_sm_count() + nj - 1) / nj));
  S = std::min(S, static_cast<int>((d.K + 63) / 64));
  p.kslice = round_up(static_cast<int>((d.K + S - 1) / S), 64);
  S = static_cast<int>((d.K + p.kslice - 1) / p.kslice);
  const size_t smem = static_cast<size_t>(p.M) * (p.kslice + kDownPad) * 2 +
                      static_cast<size_t>(kDownRows) * p.kslice * 2 + kDownMaxM * kDownRows * 4;
  if (smem > 200 * 1024) return set_error(UNO_ERR_UNSUPPORTED, "decode down-projection does not fit");
  cudaError_t e = cudaFuncSetAttribute(lora_down_dec_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(down smem)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(static_cast<unsigned>(nj), static_cast<unsigned>(S), 1);
  cfg.blockDim = dim3(kDownThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, 1, static_cast<unsigned>(S), 1);
  cfg.attrs = attr;
  e = cudaLaunchKernelEx(&cfg, lora_down_dec_kernel, p);
  if (e != cudaSuccess) return cuda_error(e, "decode down-projection launch");
  return UNO_OK;
}

}  // namespace uno
