// Fused gated-LoRA linear for decode-size batches (bf16, M <= 256, r <= 128).
//
//   y_g = x W_g^T + (scale * gate (.) (x A_g^T)) Bl_g^T
//   (the gated LoRA adapter of hyper.ai, section "方法": the adapter is off
//   on the verify rows and on for the draft rows of the same forward pass)
//
// One launch does both projections of the adapter. The weight rows fill the
// 128-row MMA side and the tokens the N side (16..128); K is split across a
// thread-block cluster so that every SM streams a slice of W. Each CTA
//   1. accumulates D = W_s x_s^T and T = A_s x_s^T over its K-slice s
//      (two TMEM accumulators; A and Bl are constant and are fetched before
//      the kernel waits for the writer of x);
//   2. turns T into the bf16 operand t_s = scale * gate * T_s, written by the
//      epilogue warps straight into shared memory in the 128-byte-swizzled
//      K-major layout the tensor core reads;
//   3. adds Bl t_s^T into D with one more MMA pass (r/64 K-blocks);
// and the cluster then sums the CTAs' D through distributed shared memory.
// Because the adapter term is linear in x, the sum of the per-slice terms is
// the full adapter term; t_s is rounded to bf16 per slice.
// silu-pair tiles hold 64 gate rows then the same 64 up rows; they keep a T
// accumulator per adapter and use zero-padded Bl tiles so each half only
// receives its own adapter.
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace uno {

namespace {

constexpr int kThreads = 192;
constexpr int kRows = 128;                      // MMA M
constexpr int kHalf = 64;
constexpr int kRowBytes = 128;                  // 64 bf16 of K per row
constexpr uint32_t kTileBytes = kRows * kRowBytes;   // 16 KB: one 128-row K-block tile
constexpr int kPartPad = 4;

struct DecParams {
  GemmArgs a;
  int bn, stages, tmem_cols, kb_per_split, splits, nkr;
  uint32_t stage_bytes, bl_off, tq_off, bar_off;
};
static_assert(sizeof(DecParams) <= 256, "DecParams must fit GemmLaunch::params");

__device__ __forceinline__ void epi_bar() { named_sync(1, 128); }

template <bool kSilu>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_dec_kernel(const __grid_constant__ TensorMaps tm, const DecParams p) {
  constexpr int kT = kSilu ? 2 : 1;   // T accumulators (adapters) per tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
  const GemmArgs& a = p.a;
  const int bn = p.bn;
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + p.bar_off);
  uint64_t* empty = full + S;
  uint64_t* accum = empty + S;
  uint64_t* blfull = accum + 1;
  uint64_t* tqready = accum + 2;
  uint64_t* accum2 = accum + 3;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const uint32_t x_off = kTileBytes * (1 + kT);   // within a stage: W | A_0 [| A_1] | x

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ft = blockIdx.y, split = blockIdx.z;
  const int g = group_of(a, ft);
  const int feat0 = (ft - a.g[g].tile0) * (kSilu ? kHalf : kRows);
  const int tok0 = blockIdx.x * bn;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accum), 1);
    mbar_init(smem_u32(blfull), 1);
    mbar_init(smem_u32(tqready), 4);
    mbar_init(smem_u32(accum2), 1);
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
    // adapter up-projection tiles Bl (constant): rows of this tile's features
    {
      const uint32_t bl = smem_u32(smem + p.bl_off);
      const uint32_t fb = smem_u32(blfull);
      mbar_arrive_expect_tx(fb, static_cast<uint32_t>(kT * p.nkr) * kTileBytes);
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
    auto load_const = [&](int kb, uint32_t st, uint32_t fb) {   // W and A of K-block kb
      const int kc = kb * 64;
      if (kSilu) {
        tma_load_2d(st, &tm.w[0], kc, feat0, fb);
        tma_load_2d(st + kTileBytes / 2, &tm.w[1], kc, feat0, fb);
        tma_load_2d(st + kTileBytes, &tm.a[0], kc, 0, fb);
        tma_load_2d(st + 2 * kTileBytes, &tm.a[1], kc, 0, fb);
      } else {
        tma_load_2d(st, &tm.w[g], kc, feat0, fb);
        tma_load_2d(st + kTileBytes, &tm.a[g], kc, 0, fb);
      }
    };
    const uint32_t tx = kTileBytes * (1 + kT) + static_cast<uint32_t>(bn) * kRowBytes;
    const int pre = min(S, kb1 - kb0);
    for (int q = 0; q < pre; ++q) {
      const uint32_t st = smem_u32(smem + q * p.stage_bytes);
      mbar_arrive_expect_tx(smem_u32(&full[q]), tx);
      load_const(kb0 + q, st, smem_u32(&full[q]));
    }
    pdl_wait();
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
      load_const(kb, st, fb);
      tma_load_2d(st + x_off, &tm.x, kb * 64, tok0, fb);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_f32acc(kRows, bn, false);
    int it = 0;
    bool ok = true;
    for (int kb = kb0; kb < kb1; ++kb, ++it) {
      const int s = it % S;
      const uint32_t ph = (it / S) & 1u;
      if (!mbar_wait(smem_u32(&full[s]), ph)) {
        fail();
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t st = smem_u32(smem + s * p.stage_bytes);
      const uint64_t xd = sdesc_k_sw128(st + x_off);
      const uint64_t wd = sdesc_k_sw128(st);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_ss<false>(tmem, wd + 2 * kk, xd + 2 * kk, idesc, (it > 0 || kk > 0) ? 1u : 0u);
#pragma unroll
      for (int h = 0; h < kT; ++h) {
        const uint64_t ad = sdesc_k_sw128(st + kTileBytes * (1 + h));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_ss<false>(tmem + static_cast<uint32_t>(bn * (1 + h)), ad + 2 * kk, xd + 2 * kk, idesc,
                        (it > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(smem_u32(&empty[s]));
    }
    mma_commit(smem_u32(accum));
    // adapter up-projection: D += Bl t^T once the epilogue has staged t
    if (ok && mbar_wait(smem_u32(blfull), 0) && mbar_wait(smem_u32(tqready), 0)) {
      tc_fence_after();
      const uint32_t bl = smem_u32(smem + p.bl_off), tq = smem_u32(smem + p.tq_off);
      for (int h = 0; h < kT; ++h)
        for (int kb = 0; kb < p.nkr; ++kb) {
          const uint64_t bd = sdesc_k_sw128(bl + static_cast<uint32_t>(h * p.nkr + kb) * kTileBytes);
          const uint64_t td =
              sdesc_k_sw128(tq + static_cast<uint32_t>((h * p.nkr + kb) * bn * kRowBytes));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) mma_ss<false>(tmem, bd + 2 * kk, td + 2 * kk, idesc, 1u);
        }
    } else if (ok) {
      fail();
    }
    mma_commit(smem_u32(accum2));
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;
    const int i = quarter * 32 + lane;   // TMEM lane: feature row of D, adapter row j of T
    const uint32_t lane_base = static_cast<uint32_t>(quarter * 32) << 16;
    pdl_wait();
    bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(accum), 0));
    tc_fence_after();
    // T -> t = scale * gate * T as bf16, K-major, 128-byte swizzled: row = token m,
    // K index = adapter row j (K-block j / 64, 16-byte chunk (j % 64) / 8).
    const uint32_t tq = smem_u32(smem + p.tq_off);
    for (int h = 0; h < kT; ++h) {
      for (int c = 0; c < bn; c += 16) {
        float v[16];
        tmem_ld16(tmem + lane_base + static_cast<uint32_t>(bn * (1 + h) + c), v);
        if (ok && i < p.nkr * 64) {
          const int kbq = i >> 6, jj = i & 63;
          const uint32_t tile = tq + static_cast<uint32_t>((h * p.nkr + kbq) * bn * kRowBytes);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int m = c + e;
            const float val = v[e] * a.scale * row_gate(a, tok0 + m);
            const uint32_t addr = tile + static_cast<uint32_t>(m * kRowBytes) +
                                  static_cast<uint32_t>((((jj >> 3) ^ (m & 7)) << 4) + ((jj & 7) << 1));
            const __nv_bfloat16 bv = __float2bfloat16_rn(val);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(addr),
                         "h"(*reinterpret_cast<const unsigned short*>(&bv))
                         : "memory");
          }
        }
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(tqready));
    ok = __all_sync(0xffffffffu, ok && mbar_wait(smem_u32(accum2), 0));
    if (!ok && lane == 0) fail();
    tc_fence_after();
    float* stage = reinterpret_cast<float*>(smem);   // the stage ring is free now
    const uint32_t trow = tmem + lane_base;
    if (p.splits == 1) {
      if (!kSilu) {
        if (ok) {
          for (int c = 0; c < bn; c += 16) {
            float v[16];
            tmem_ld16(trow + c, v);
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
            tmem_ld16(trow + c, v);
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
    } else if (ok) {
      for (int c = 0; c < bn; c += 16) {
        float v[16];
        tmem_ld16(trow + c, v);
#pragma unroll
        for (int j = 0; j < 16; ++j) stage[(c + j) * (kRows + kPartPad) + i] = v[j];
      }
    }
  }

  if (p.splits > 1) {
    cluster_sync_converged();
    const uint32_t rank = cluster_ctarank();
    const int Sp = p.splits;
    const int groups = kSilu ? bn * (kRows / 8) : bn * (kRows / 4);
    const int chunk = (groups + Sp - 1) / Sp;
    const int e0 = static_cast<int>(rank) * chunk;
    const int e1 = min(groups, e0 + chunk);
    const uint32_t part0 = smem_u32(smem);
    // unrolled to the largest cluster (8) with constant indices, so the peer
    // addresses and partials stay in registers and all loads go out at once
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
    cluster_sync_converged();
  }

  tc_fence_before();
  cta_sync_converged();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

int pow2_at_least(int v) {
  int c = 32;
  while (c < v) c <<= 1;
  return c;
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

void* dec_kernel(bool silu) {
  return silu ? reinterpret_cast<void*>(&gemm_dec_kernel<true>)
              : reinterpret_cast<void*>(&gemm_dec_kernel<false>);
}

int64_t dec_max_clusters(bool silu, int cluster, int smem) {
  static std::mutex mu;
  static std::map<std::tuple<bool, int, int>, int64_t> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(silu, cluster, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  void* fn = dec_kernel(silu);
  int n = 0;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(1, 1, cluster);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = cluster;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, fn, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 1 << 20;
    }
  }
  cache[key] = n;
  return n;
}

}  // namespace

namespace {

// Shared-memory plan of a fused decode launch: stages, or 0 when it does not fit.
int dec_stages(const GemmProblem& pb, int bn, uint32_t* stage_bytes, uint32_t* bl_bytes,
               uint32_t* tq_bytes) {
  const int kT = pb.mode == kEpiSiluPair ? 2 : 1;
  const int nkr = (pb.r + 63) / 64;
  *stage_bytes = (static_cast<uint32_t>(kTileBytes * (1 + kT) + bn * kRowBytes) + 1023u) & ~1023u;
  *bl_bytes = static_cast<uint32_t>(kT * nkr) * kTileBytes;
  *tq_bytes = static_cast<uint32_t>(kT * nkr * bn * kRowBytes);
  const uint32_t budget = 218u * 1024u;
  if (*bl_bytes + *tq_bytes >= budget) return 0;
  return std::min(8, static_cast<int>((budget - *bl_bytes - *tq_bytes) / *stage_bytes));
}

}  // namespace

bool gemm_dec_suits(const GemmProblem& pb) {
  if (pb.dt != UNO_BF16 || pb.M < 1 || pb.M > 256 || pb.r < 1 || pb.r > 128) return false;
  if (pb.mode != kEpiStore && pb.mode != kEpiAdd && pb.mode != kEpiSiluPair) return false;
  for (int i = 0; i < pb.ngroups; ++i)
    if (!pb.A[i]) return false;
  const bool silu = pb.mode == kEpiSiluPair;
  const int bn = round_up(static_cast<int>(pb.M), 16);
  if (bn > (silu ? 32 : 128)) return false;
  // one CTA per SM: the tiles must fit in one wave, with a pipeline of >= 3 stages
  int64_t tiles = 0;
  const int ft = silu ? kHalf : kRows;
  if (silu) tiles = (pb.g[0].N + ft - 1) / ft;
  else
    for (int i = 0; i < pb.ngroups; ++i) tiles += (pb.g[i].N + ft - 1) / ft;
  uint32_t sb, blb, tqb;
  return tiles <= device_sm_count() && dec_stages(pb, bn, &sb, &blb, &tqb) >= 3;
}

uno_status gemm_dec_prepare(const GemmProblem& pb, GemmLaunch* out) {
  const bool silu = pb.mode == kEpiSiluPair;
  const int kT = silu ? 2 : 1;
  const int bn = round_up(static_cast<int>(pb.M), 16);
  const int feat_tile = silu ? kHalf : kRows;
  DecParams dp{};
  dp.a = make_gemm_args(pb, feat_tile, kRowBytes);
  const int feat_tiles = feature_tiles(dp.a, feat_tile);
  if (feat_tiles > 65535) return set_error(UNO_ERR_UNSUPPORTED, "N too large for the tile grid");
  dp.bn = bn;
  dp.nkr = (pb.r + 63) / 64;
  uint32_t bl_bytes, tq_bytes;
  const int stages = dec_stages(pb, bn, &dp.stage_bytes, &bl_bytes, &tq_bytes);
  if (stages < 2) return set_error(UNO_ERR_UNSUPPORTED, "fused decode tile does not fit");
  dp.stages = stages;
  const uint32_t ring = stages * dp.stage_bytes;
  const uint32_t need_part = static_cast<uint32_t>(bn * (kRows + kPartPad) * 4);
  const uint32_t need_silu = static_cast<uint32_t>(2 * bn * (kHalf + 1) * 4);
  if (need_part > ring || need_silu > ring)
    return set_error(UNO_ERR_UNSUPPORTED, "fused decode epilogue does not fit");
  dp.bl_off = ring;
  dp.tq_off = ring + bl_bytes;
  dp.bar_off = (dp.tq_off + tq_bytes + 15u) & ~15u;
  dp.tmem_cols = pow2_at_least((1 + kT) * bn);
  const int smem = static_cast<int>(dp.bar_off + 8 * (2 * stages + 4) + 16 + 1024);

  // one CTA per SM; split K so the grid covers the SMs, with every cluster resident
  const int sms = device_sm_count();
  const int nkb = dp.a.nkb_main;
  int splits = std::max(1, std::min({8, sms / std::max(1, feat_tiles), nkb}));
  while (splits > 1 && dec_max_clusters(silu, splits, smem) < feat_tiles) --splits;
  int kb_per = (nkb + splits - 1) / splits;
  splits = (nkb + kb_per - 1) / kb_per;
  dp.kb_per_split = kb_per;
  dp.splits = splits;

  uno_status s;
  TensorMaps& tm = out->tm;
  if ((s = make_map(&tm.x, pb.dt, pb.x, pb.K, pb.M, pb.K, static_cast<uint32_t>(bn))) != UNO_OK)
    return s;
  tm.t = tm.x;
  const uint32_t wbox = silu ? kHalf : kRows;
  for (int i = 0; i < kMaxGroups; ++i) {
    const int gi = i < pb.ngroups ? i : 0;
    const GemmGroup& G = pb.g[gi];
    if ((s = make_map(&tm.w[i], pb.dt, G.W, pb.K, G.N, pb.K, wbox)) != UNO_OK) return s;
    if ((s = make_map(&tm.b[i], pb.dt, G.Bl, pb.r, G.N, pb.r, wbox)) != UNO_OK) return s;
    if ((s = make_map(&tm.a[i], pb.dt, pb.A[gi], pb.K, pb.r, pb.K, kRows)) != UNO_OK) return s;
  }
  std::memcpy(out->params, &dp, sizeof(dp));
  out->kind = 2;
  out->swap = silu ? 1 : 0;   // kernel variant
  out->grid_x = 1;
  out->grid_y = feat_tiles;
  out->splits = splits;
  out->smem_bytes = smem;
  out->dtype = pb.dt;
  return UNO_OK;
}

uno_status gemm_dec_run(const GemmLaunch& l, cudaStream_t stream) {
  void* fn = dec_kernel(l.swap != 0);
  cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, l.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(decode gemm smem)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid_x, l.grid_y, l.splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = l.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, 1, 1, static_cast<unsigned>(l.splits));
  cfg.attrs = attr;
  DecParams dp;
  std::memcpy(&dp, l.params, sizeof(dp));
  void* args[2] = {const_cast<TensorMaps*>(&l.tm), &dp};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_error(e, "decode GEMM launch");
  return UNO_OK;
}

}  // namespace uno
