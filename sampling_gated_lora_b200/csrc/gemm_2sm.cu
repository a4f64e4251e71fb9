// Persistent CTA-pair gated GEMM for large M (bf16, sm_100a).
//
//   y_g = x W_g^T + t_g Bl_g^T   (t_g = the gated LoRA down-projection, folded
//   in as extra K-blocks, so W streams once — the gated adapter of hyper.ai,
//   section "方法"); up to three groups share x. In silu-pair tiles the 256
//   B rows are 128 gate rows (CTA 0's half) and the same 128 up rows (CTA 1's
//   half), so every CTA's accumulator holds gate and up side by side and the
//   epilogue writes silu(gate) * up.
//
// One cluster of two CTAs on one TPC computes 256 x 256 output tiles with
// tcgen05.mma.cta_group::2 (M = 256, N = 256, K = 16): CTA r of the pair
// holds tokens [128 r, 128 r + 128) of the tile's A side and features
// [128 r, 128 r + 128) of its B side, and its TMEM receives its 128 token rows
// across all 256 features. Per K-block each CTA loads 32 KB (vs 48 KB for a
// 128 x 256 single-CTA tile of the same output per CTA), which is what keeps
// the shared-memory fill rate within L2 bandwidth at full tensor rate.
//
// Roles (192 threads per CTA):
//   warp 0 lane 0 (both CTAs): TMA producer of this CTA's operand halves; the
//     loads signal the leader CTA's full barrier, which the leader's producer
//     arms with the bytes of both halves;
//   warp 1 lane 0 (leader only): MMA issuer; each stage is released to both
//     producers by a commit to each CTA's empty barrier;
//   warps 2..5 (both CTAs): epilogue from TMEM, then a release of the TMEM
//     buffer to the leader's accumulator-empty barrier.
// Two 256-column TMEM accumulators let the epilogue of tile i overlap the
// mainloop of tile i+1. Tiles are visited token-block fastest so concurrent
// pairs share W tiles (and x stays resident in L2).
#include <algorithm>
#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace uno {

namespace {

constexpr int kThreads = 192;
constexpr int kHalf = 128;                  // rows per CTA per operand
constexpr int kTile = 256;                  // tile edge (M and N) per pair
constexpr uint32_t kHalfBytes = kHalf * 128;   // one 128-row, 128-byte K-block half
constexpr uint32_t kStageBytes = 2 * kHalfBytes;
constexpr int kAccCols = 256;

struct PairParams {
  GemmArgs a;
  int tiles_m, num_tiles;
  int stages;
};
static_assert(sizeof(PairParams) <= kLaunchParamBytes, "PairParams must fit GemmLaunch::params");

__global__ void __launch_bounds__(kThreads, 1)
    gemm_pair_kernel(const __grid_constant__ TensorMaps tm, const PairParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
  const int S = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * kStageBytes);
  uint64_t* empty = full + S;
  uint64_t* accf = empty + S;     // [2]
  uint64_t* acce = accf + 2;      // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acce + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0 = leader, 1 = peer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1;
  const int num_pairs = gridDim.x >> 1;
  const GemmArgs& a = p.a;
  const bool silu = a.mode == kEpiSiluPair;
  const int nkb = a.nkb_main + (silu ? 2 : 1) * a.nkb_r;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&accf[b]), 1);
      mbar_init(smem_u32(&acce[b]), 8);   // 4 epilogue warps x 2 CTAs
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(smem_u32(tmem_slot), 2 * kAccCols);
    tmem_relinquish_pair();
  }
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tm.x);
    tma_prefetch_desc(&tm.w[0]);
  }
  tc_fence_before();
  cluster_sync();   // barriers of both CTAs initialised, TMEM allocated in both
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) pdl_trigger();

  auto fail = [&]() {
    *abort_flag = 1;
    raise_status(a.status, kDevTimeout);
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    // The first stages' weight halves are constant: they are issued before
    // waiting for the kernel that writes the activations.
    int it = 0;
    bool ok = true;
    int pre = 0;   // k-blocks of the first tile whose W half went out early
    bool waited = false;
    for (int tile = pair; ok && tile < p.num_tiles; tile += num_pairs) {
      const int mb = tile % p.tiles_m, ft = tile / p.tiles_m;
      const int g = group_of(a, ft);
      const int m0 = mb * kTile + static_cast<int>(rank) * kHalf;
      // B rows of this CTA's half: its 128 features of group g, or (silu) the
      // tile's 128 features of group `rank` (gate for CTA 0, up for CTA 1)
      const int gb = silu ? static_cast<int>(rank) : g;
      const int n0 = silu ? ft * kHalf : (ft - a.g[g].tile0) * kTile + static_cast<int>(rank) * kHalf;
      auto load_b = [&](int kb, uint32_t sb, uint32_t fb) {
        if (kb < a.nkb_main) {
          tma_load_2d_pair(sb, &tm.w[gb], kb * 64, n0, fb);
        } else {
          const int l = kb - a.nkb_main;
          const int h = silu ? l / a.nkb_r : 0;
          const int j = silu ? l % a.nkb_r : l;
          // silu: the other group's adapter rows are read past the end (zeros)
          const int row = (silu && h != static_cast<int>(rank)) ? a.g[gb].b_rows : n0;
          tma_load_2d_pair(sb, &tm.b[gb], j * 64, row, fb);
        }
      };
      auto load_a = [&](int kb, uint32_t sa, uint32_t fb) {
        if (kb < a.nkb_main) {
          tma_load_2d_pair(sa, &tm.x, kb * 64, m0, fb);
        } else {
          const int l = kb - a.nkb_main;
          const int h = silu ? l / a.nkb_r : 0;
          const int j = silu ? l % a.nkb_r : l;
          tma_load_2d_pair(sa, &tm.t, a.g[silu ? h : g].t_col + j * 64, m0, fb);
        }
      };
      if (tile == pair) {
        pre = min(S, nkb);
        for (int q = 0; q < pre; ++q) {
          const uint32_t sa = smem_u32(smem + q * kStageBytes);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[q]), 2 * kStageBytes);
          load_b(q, sa + kHalfBytes, map_shared_rank(smem_u32(&full[q]), 0));
        }
        if (!a.x_ready) {
          pdl_wait();
          waited = true;
        }
        for (int q = 0; q < pre; ++q) {
          if (!waited && q >= a.nkb_main) {
            pdl_wait();
            waited = true;
          }
          load_a(q, smem_u32(smem + q * kStageBytes), map_shared_rank(smem_u32(&full[q]), 0));
        }
        it = pre;
      }
      for (int kb = (tile == pair) ? pre : 0; kb < nkb; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u) || *abort_flag) {
          fail();
          ok = false;
          break;
        }
        const uint32_t fb = map_shared_rank(smem_u32(&full[s]), 0);
        if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), 2 * kStageBytes);
        const uint32_t sa = smem_u32(smem + s * kStageBytes);
        if (!waited && kb >= a.nkb_main) {
          pdl_wait();
          waited = true;
        }
        load_a(kb, sa, fb);
        load_b(kb, sa + kHalfBytes, fb);
      }
    }
    if (!waited) pdl_wait();
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    const uint32_t idesc = idesc_f32acc(kTile, kTile, false);
    int it = 0, lt = 0;
    bool ok = true;
    for (int tile = pair; ok && tile < p.num_tiles; tile += num_pairs, ++lt) {
      const int b = lt & 1;
      const uint32_t aph = (lt >> 1) & 1u;
      if (!mbar_wait_cluster(smem_u32(&acce[b]), aph ^ 1u)) {
        fail();
        break;
      }
      tc_fence_after();
      const uint32_t dacc = tmem + static_cast<uint32_t>(b * kAccCols);
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(smem_u32(&full[s]), ph)) {
          fail();
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t sa = smem_u32(smem + s * kStageBytes);
        const uint64_t ad = sdesc_k_sw128(sa);
        const uint64_t bd = sdesc_k_sw128(sa + kHalfBytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_pair_bf16(dacc, ad + static_cast<uint64_t>(2 * kk), bd + static_cast<uint64_t>(2 * kk),
                        idesc, (kb > 0 || kk > 0) ? 1u : 0u);
        const uint32_t eb = smem_u32(&empty[s]);
        mma_commit_pair(map_shared_rank(eb, 0));
        mma_commit_pair(map_shared_rank(eb, 1));
      }
      const uint32_t fb = smem_u32(&accf[b]);
      mma_commit_pair(map_shared_rank(fb, 0));
      mma_commit_pair(map_shared_rank(fb, 1));
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue (both CTAs)
    if (!a.x_ready) pdl_wait();
    const int quarter = warp & 3;
    const int i = quarter * 32 + lane;
    int lt = 0;
    for (int tile = pair; tile < p.num_tiles; tile += num_pairs, ++lt) {
      const int b = lt & 1;
      const uint32_t aph = (lt >> 1) & 1u;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&accf[b]), aph));
      if (!ok) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after();
      const int mb = tile % p.tiles_m, ft = tile / p.tiles_m;
      const int g = group_of(a, ft);
      const int m = mb * kTile + static_cast<int>(rank) * kHalf + i;
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(b * kAccCols);
      if (!silu) {
        const int nb0 = (ft - a.g[g].tile0) * kTile;
        for (int c = 0; c < kTile; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          if (nb0 + c < a.g[g].N) epi_store16<__nv_bfloat16>(a, g, m, nb0 + c, v);
        }
      } else {
        const int f0 = ft * kHalf;
        for (int c = 0; c < kHalf; c += 16) {
          float gv[16], uv[16];
          tmem_ld16(trow + c, gv);
          tmem_ld16(trow + kHalf + c, uv);
#pragma unroll
          for (int j = 0; j < 16; ++j) gv[j] = silu_f(gv[j]) * uv[j];
          if (f0 + c < a.g[0].N) epi_store16<__nv_bfloat16>(a, 0, m, f0 + c, gv);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(map_shared_rank(smem_u32(&acce[b]), 0));
    }
  }

  // Everything issued has been waited for by the epilogues (or given up on);
  // meet the peer before freeing the pair's TMEM.
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 2 * kAccCols);
  }
}

}  // namespace

bool gemm_pair_suits(const GemmProblem& pb) {
  if (pb.dt != UNO_BF16 || pb.M <= 256 || pb.mode == kEpiRowScale) return false;
  if (pb.mode == kEpiSiluPair) return true;
  int64_t ntiles = 0;
  for (int i = 0; i < pb.ngroups; ++i) ntiles += (pb.g[i].N + kTile - 1) / kTile;
  const int64_t tiles = ((pb.M + kTile - 1) / kTile) * ntiles;
  // two or more full token tiles already beat the one-CTA kernel (measured
  // at M = 544..800); just above 256 rows the one-CTA kernel's split-K wins
  return tiles >= device_sm_count() / 2 || pb.M >= 512;
}

uno_status gemm_pair_prepare(const GemmProblem& pb, GemmLaunch* out) {
  const bool silu = pb.mode == kEpiSiluPair;
  const int tile_n = silu ? kHalf : kTile;
  PairParams pp{};
  pp.a = make_gemm_args(pb, tile_n, 128);
  pp.tiles_m = static_cast<int>((pb.M + kTile - 1) / kTile);
  const int64_t tiles = static_cast<int64_t>(pp.tiles_m) * feature_tiles(pp.a, tile_n);
  if (tiles > (1ll << 30)) return set_error(UNO_ERR_UNSUPPORTED, "too many tiles");
  pp.num_tiles = static_cast<int>(tiles);
  pp.stages = 6;
  uno_status s;
  TensorMaps& tm = out->tm;
  if ((s = make_map(&tm.x, pb.dt, pb.x, pb.K, pb.M, pb.K, kHalf)) != UNO_OK) return s;
  if (pb.r > 0) {
    if ((s = make_map(&tm.t, pb.dt, pb.t, pb.ldt, pb.M, pb.ldt, kHalf)) != UNO_OK) return s;
  } else {
    tm.t = tm.x;
  }
  for (int i = 0; i < kMaxGroups; ++i) {
    const GemmGroup& G = pb.g[i < pb.ngroups ? i : 0];
    if ((s = make_map(&tm.w[i], pb.dt, G.W, pb.K, G.N, pb.K, kHalf)) != UNO_OK) return s;
    if (pb.r > 0) {
      if ((s = make_map(&tm.b[i], pb.dt, G.Bl, pb.r, G.N, pb.r, kHalf)) != UNO_OK) return s;
    } else {
      tm.b[i] = tm.w[i];
    }
  }
  std::memcpy(out->params, &pp, sizeof(pp));
  const int pairs = std::max(1, std::min<int>(device_sm_count() / 2, pp.num_tiles));
  out->kind = 1;
  out->swap = 0;
  out->grid_x = 2 * pairs;
  out->grid_y = 1;
  out->splits = 1;
  out->smem_bytes = static_cast<int>(pp.stages * kStageBytes + 1024 + 256);
  out->dtype = pb.dt;
  return UNO_OK;
}

uno_status gemm_pair_run(const GemmLaunch& l, cudaStream_t stream) {
  void* fn = reinterpret_cast<void*>(&gemm_pair_kernel);
  cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, l.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(pair smem)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid_x, 1, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = l.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, 2, 1, 1);
  cfg.attrs = attr;
  PairParams pp;
  std::memcpy(&pp, l.params, sizeof(pp));
  void* args[2] = {const_cast<TensorMaps*>(&l.tm), &pp};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_error(e, "pair GEMM launch");
  return UNO_OK;
}

}  // namespace uno
