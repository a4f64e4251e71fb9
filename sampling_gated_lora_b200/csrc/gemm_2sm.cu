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
// pairs share W tiles (and x stays resident in L2). For deep tiles whose count
// would leave the last round part-empty, the K-blocks of the last tiles are
// shared out evenly (stream-K); the two pairs that cut a tile meet through
// fp32 partial sums and flags in the caller's workspace.
//
// Down tiles. When the kernel also computes t (r <= 128), the work list opens
// with the down tiles of every 256-row token block:
// t[:, g r + j] = scale * gate(m) * (x A_g^T)[m, j], the same K-loop over x
// with adapter rows on the B side. Groups go two to a tile (A_2j in CTA 0's
// half, A_2j+1 in CTA 1's, an N = 256 MMA); an odd last group takes a
// 256 x 128 tile (64 of its rows per CTA, an N = 128 MMA). The epilogue
// stores t in bf16 and adds one per epilogue warp to the token block's
// counter; a main tile's producer waits for that count (bounded)
// before its first adapter K-block only. Every pair takes its down tiles
// before its main tiles and down tiles wait for nothing, so the waits end.
// One launch replaces the separate down-projection launch, whose CTAs held
// SMs that the pairs could not use while it ran.
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
// Stream-K partial sum of one epilogue warp: 32 accumulator rows x 256 columns,
// column-major so that a warp's 32 lanes touch 128 contiguous bytes.
constexpr uint32_t kSkWarpFloats = 32 * kAccCols;
constexpr uint32_t kSkWarpBytes = kSkWarpFloats * 4;

struct PairParams {
  GemmArgs a;
  int tiles_m, num_tiles;
  int stages;
  // Tiles [0, dp_tiles) are visited whole, round-robin over the pairs. The
  // K-block iterations of the remaining tiles (sk_iters in all, the tiles
  // taken in order) are shared out evenly, stream-K style: pair p takes
  // iterations [p I / P, (p + 1) I / P).
  int dp_tiles;
  long long sk_iters;
  float* sk_part;       // [pairs][2 CTAs][4 epilogue warps][256 columns][32 rows] fp32
  int32_t* sk_flag;     // [pairs][2 CTAs][4 epilogue warps], zero once the predecessor is done
  // Down tiles [0, down_tiles): groups 2j and 2j + 1 (j = tile / tiles_m),
  // token block tile % tiles_m (0 when t comes from an earlier launch); main
  // tile i is tile down_tiles + i.
  int down_tiles, down_expect, r, ldt;
  __nv_bfloat16* t;
  int32_t* t_ready;     // [tiles_m] finished down-tile epilogue warps per token block
};
static_assert(sizeof(PairParams) <= kLaunchParamBytes, "PairParams must fit GemmLaunch::params");

// The work of one pair: its whole tiles, then its stream-K share cut at tile
// boundaries. Each share spans at least one tile's worth of K-blocks (the
// stream-K tiles number at least as many as the pairs), so a tile that two
// shares cut has exactly two parts: the first (kb0 = 0, kb1 < nkb) ends pair
// p's share, the second (kb0 > 0, kb1 = nkb) begins pair p + 1's. A share is
// walked as: the tiles wholly inside it, then its first part (the head, which
// starts at K-block 0), then its second part (the tail) last. Every pair
// enters its share at the same time, so at any moment the pairs stand at one
// of a few common K offsets (the heads and whole tiles at the offset of the
// clock, the tails at the clock minus a constant), and the tiles they run at
// once share their x and W K-slices in L2; walked in index order instead, the
// parts start at scattered K offsets and the same slices stream from HBM once
// per pair. The head's pair hands its partial sum to pair p + 1, which adds it
// when it finishes the tile with the tail, its last item (its stage ring is
// idle then).
struct WorkCursor {
  int tile;
  int phase;              // stream-K share: 0 whole tiles, 1 head, 2 tail, 3 done
  long long it, it_end;   // the share [it, it_end) in K-block iterations
  long long w, w_end;     // its whole tiles [w, w_end) (tile aligned)
};

__device__ __forceinline__ WorkCursor work_begin(const PairParams& p, int pair, int pairs, int nkb) {
  WorkCursor c;
  c.tile = pair;
  c.phase = 0;
  c.it = p.sk_iters * pair / pairs;
  c.it_end = p.sk_iters * (pair + 1) / pairs;
  c.w = (c.it + nkb - 1) / nkb * nkb;
  c.w_end = max(c.w, c.it_end / nkb * nkb);
  return c;
}

template <bool kDown>
__device__ __forceinline__ bool work_next(const PairParams& p, int pairs, int nkb, WorkCursor& c,
                                          int& tile, int& kb0, int& kb1) {
  if (c.tile < p.dp_tiles) {
    tile = c.tile;
    kb0 = 0;
    kb1 = kDown && tile < p.down_tiles ? p.a.nkb_main : nkb;
    c.tile += pairs;
    return true;
  }
  if (c.it >= c.it_end) return false;
  if (c.phase == 0) {   // the tiles wholly inside the share
    if (c.w < c.w_end) {
      tile = p.dp_tiles + static_cast<int>(c.w / nkb);
      kb0 = 0;
      kb1 = nkb;
      c.w += nkb;
      return true;
    }
    c.phase = 1;
  }
  if (c.phase == 1) {   // the head: the first part of the tile the share ends in
    c.phase = 2;
    if (c.it_end % nkb != 0) {
      const long long rel = c.it_end / nkb;
      tile = p.dp_tiles + static_cast<int>(rel);
      kb0 = 0;
      kb1 = static_cast<int>(c.it_end - rel * nkb);
      return true;
    }
  }
  if (c.phase == 2) {   // the tail: the second part of the tile the share starts in
    c.phase = 3;
    if (c.it % nkb != 0) {
      const long long rel = c.it / nkb;
      tile = p.dp_tiles + static_cast<int>(rel);
      kb0 = static_cast<int>(c.it - rel * nkb);
      kb1 = nkb;
      return true;
    }
  }
  return false;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Token block, feature tile (main) or first group (down) of a work item;
// `wide`: a down tile with two groups.
struct TileId {
  bool down, wide;
  int mb, ft, g;
};

template <bool kDown>
__device__ __forceinline__ TileId tile_id(const PairParams& p, int tile) {
  TileId t;
  t.down = kDown && tile < p.down_tiles;
  t.wide = false;
  if (t.down) {
    t.mb = tile % p.tiles_m;
    t.g = 2 * (tile / p.tiles_m);
    t.wide = t.g + 1 < p.a.ngroups;
    t.ft = 0;
  } else {
    const int mt = kDown ? tile - p.down_tiles : tile;
    t.mb = mt % p.tiles_m;
    t.ft = mt / p.tiles_m;
    t.g = group_of(p.a, t.ft);
  }
  return t;
}

// kDown: the launch has down tiles (a separate instance, so that launches
// without them run none of their code).
template <bool kDown>
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
  uint64_t* skbar = acce + 2;     // [4] stream-K partial sums copied in, one per epilogue warp
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(skbar + 4);
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
    for (int q = 0; q < 4; ++q) mbar_init(smem_u32(&skbar[q]), 1);
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
    bool first = true;
    bool waited = false;
    WorkCursor wc = work_begin(p, pair, num_pairs, nkb);
    int tile, kb0, kb1;
    while (ok && work_next<kDown>(p, num_pairs, nkb, wc, tile, kb0, kb1)) {
      const TileId id = tile_id<kDown>(p, tile);
      const int mb = id.mb, ft = id.ft, g = id.g;
      const int m0 = mb * kTile + static_cast<int>(rank) * kHalf;
      // a down tile's B side: 64 rows of A_g per CTA
      const uint32_t tx = id.down && !id.wide ? 3 * kHalfBytes : 2 * kStageBytes;
      bool t_seen = !kDown;   // t of this token block is complete
      // B rows of this CTA's half: its 128 features of group g, or (silu) the
      // tile's 128 features of group `rank` (gate for CTA 0, up for CTA 1)
      const int gb = silu ? static_cast<int>(rank) : g;
      const int n0 = silu ? ft * kHalf : (ft - a.g[g].tile0) * kTile + static_cast<int>(rank) * kHalf;
      auto load_b = [&](int kb, uint32_t sb, uint32_t fb) {
        if (id.down) {   // wide: A_{g + rank}, all rows; else rows [64 rank, 64 rank + 64) of A_g
          if (id.wide)
            tma_load_2d_pair(sb, &tm.a[g + static_cast<int>(rank)], kb * 64, 0, fb);
          else
            tma_load_2d_pair(sb, &tm.a[g], kb * 64, static_cast<int>(rank) * (kHalf / 2), fb);
        } else if (kb < a.nkb_main) {
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
      auto load_a = [&](int kb, uint32_t sa, uint32_t fb) -> bool {
        if (kb < a.nkb_main) {
          tma_load_2d_pair(sa, &tm.x, kb * 64, m0, fb);
        } else {
          if (!t_seen) {   // the down tiles of this token block wrote t with generic stores
            if (!counter_wait(p.t_ready + mb, p.down_expect)) return false;
            fence_proxy_async_global();
            t_seen = true;
          }
          const int l = kb - a.nkb_main;
          const int h = silu ? l / a.nkb_r : 0;
          const int j = silu ? l % a.nkb_r : l;
          tma_load_2d_pair(sa, &tm.t, a.g[silu ? h : g].t_col + j * 64, m0, fb);
        }
        return true;
      };
      int kb_next = kb0;
      if (first) {
        // k-blocks of the first work item whose W half goes out early
        first = false;
        const int pre = min(S, kb1 - kb0);
        for (int q = 0; q < pre; ++q) {
          const uint32_t sa = smem_u32(smem + q * kStageBytes);
          if (leader) mbar_arrive_expect_tx(smem_u32(&full[q]), tx);
          load_b(kb0 + q, sa + kHalfBytes, map_shared_rank(smem_u32(&full[q]), 0));
        }
        if (!a.x_ready) {
          pdl_wait();
          waited = true;
        }
        for (int q = 0; q < pre; ++q) {
          if (!waited && kb0 + q >= a.nkb_main) {
            pdl_wait();
            waited = true;
          }
          if (!load_a(kb0 + q, smem_u32(smem + q * kStageBytes), map_shared_rank(smem_u32(&full[q]), 0))) {
            fail();
            ok = false;
            break;
          }
        }
        if (!ok) break;
        it = pre;
        kb_next = kb0 + pre;
      }
      for (int kb = kb_next; kb < kb1; ++kb, ++it) {
        const int s = it % S;
        const uint32_t ph = (it / S) & 1u;
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u) || *abort_flag) {
          fail();
          ok = false;
          break;
        }
        const uint32_t fb = map_shared_rank(smem_u32(&full[s]), 0);
        if (leader) mbar_arrive_expect_tx(smem_u32(&full[s]), tx);
        const uint32_t sa = smem_u32(smem + s * kStageBytes);
        if (!waited && kb >= a.nkb_main) {
          pdl_wait();
          waited = true;
        }
        if (!load_a(kb, sa, fb)) {
          fail();
          ok = false;
          break;
        }
        load_b(kb, sa + kHalfBytes, fb);
      }
    }
    if (!waited) pdl_wait();
  } else if (warp == 1 && lane == 0 && leader) {
    // ------------------------------------------------------------ MMA issuer (leader)
    const uint32_t idesc = idesc_f32acc(kTile, kTile, false);
    const uint32_t idesc_down = idesc_f32acc(kTile, kHalf, false);
    int it = 0, lt = 0;
    bool ok = true;
    WorkCursor wc = work_begin(p, pair, num_pairs, nkb);
    int tile, kb0, kb1;
    for (; ok && work_next<kDown>(p, num_pairs, nkb, wc, tile, kb0, kb1); ++lt) {
      const int b = lt & 1;
      const uint32_t aph = (lt >> 1) & 1u;
      if (!mbar_wait_cluster(smem_u32(&acce[b]), aph ^ 1u)) {
        fail();
        break;
      }
      tc_fence_after();
      const uint32_t dacc = tmem + static_cast<uint32_t>(b * kAccCols);
      const TileId id = tile_id<kDown>(p, tile);
      const uint32_t id_k = id.down && !id.wide ? idesc_down : idesc;
      for (int kb = kb0; kb < kb1; ++kb, ++it) {
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
                        id_k, (kb > kb0 || kk > 0) ? 1u : 0u);
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
    WorkCursor wc = work_begin(p, pair, num_pairs, nkb);
    int tile, kb0, kb1;
    for (; work_next<kDown>(p, num_pairs, nkb, wc, tile, kb0, kb1); ++lt) {
      const int b = lt & 1;
      const uint32_t aph = (lt >> 1) & 1u;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(&accf[b]), aph));
      if (!ok) {
        if (lane == 0) fail();
        break;
      }
      tc_fence_after();
      const TileId id = tile_id<kDown>(p, tile);
      const int mb = id.mb, ft = id.ft, g = id.g;
      const int m = mb * kTile + static_cast<int>(rank) * kHalf + i;
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16) +
                            static_cast<uint32_t>(b * kAccCols);
      if (id.down) {
        // t[m, g r + j] = scale * gate(m) * acc[128 (g - id.g) + j], j < r, in bf16
        const float f = m < a.M ? a.scale * row_gate(a, m) : 0.f;
        for (int gg = 0; gg < (id.wide ? 2 : 1); ++gg) {
          __nv_bfloat16* dst = p.t + static_cast<size_t>(m) * p.ldt + a.g[g + gg].t_col;
          for (int c = 0; c < p.r; c += 16) {
            float v[16];
            tmem_ld16(trow + static_cast<uint32_t>(gg * kHalf + c), v);
            if (m < a.M) {
#pragma unroll
              for (int h = 0; h < 2; ++h) {
                if (c + 8 * h >= p.r) break;
                uint4 w;
                w.x = pack_bf16x2(f * v[8 * h + 0], f * v[8 * h + 1]);
                w.y = pack_bf16x2(f * v[8 * h + 2], f * v[8 * h + 3]);
                w.z = pack_bf16x2(f * v[8 * h + 4], f * v[8 * h + 5]);
                w.w = pack_bf16x2(f * v[8 * h + 6], f * v[8 * h + 7]);
                *reinterpret_cast<uint4*>(dst + c + 8 * h) = w;
              }
            }
          }
        }
        // t is read by the main tiles' bulk tensor copies (the async proxy)
        fence_proxy_async_global();
        __threadfence();
        __syncwarp();
        if (lane == 0) counter_add_release(p.t_ready + mb, 1);
      } else if (kb1 < nkb) {
        // first part of a stream-K tile (this pair's head): hand this warp's
        // partial sum (its 32 rows, all 256 columns) to the next pair, which
        // finishes the tile. The partial sums are shared by the launches of a
        // stream and the flags cleared by the preceding launch: both wait
        // until that launch has finished.
        const int fi = (pair * 2 + static_cast<int>(rank)) * 4 + quarter;
        float* part = p.sk_part + static_cast<size_t>(fi) * kSkWarpFloats;
        pdl_wait();
        for (int c = 0; c < kTile; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) part[(c + j) * 32 + lane] = v[j];
        }
        fence_proxy_async_global();   // the reader copies them with the async proxy
        __threadfence();
        __syncwarp();
        if (lane == 0) flag_release(p.sk_flag + fi, 1);
      } else {
        // a whole tile, or the second part of a stream-K tile (the pair's last
        // work item, so the stage ring is idle): copy the previous pair's
        // partial sum for this warp's rows into shared memory, then add it
        const float* part = nullptr;
        if (kb0 > 0) {
          const int fi = ((pair - 1) * 2 + static_cast<int>(rank)) * 4 + quarter;
          pdl_wait();   // the flags were cleared by the preceding launch
          bool got = __all_sync(0xffffffffu, flag_wait(p.sk_flag + fi, 1));
          const uint32_t dst = smem_u32(smem + static_cast<uint32_t>(quarter) * kSkWarpBytes);
          if (got) {
            if (lane == 0) {
              // the partial sums were stored through the generic proxy; the
              // bulk copy reads through the async proxy
              fence_proxy_async_global();
              mbar_arrive_expect_tx(smem_u32(&skbar[quarter]), kSkWarpBytes);
              bulk_load(dst, p.sk_part + static_cast<size_t>(fi) * kSkWarpFloats, kSkWarpBytes,
                        smem_u32(&skbar[quarter]));
            }
            got = __all_sync(0xffffffffu, mbar_wait(smem_u32(&skbar[quarter]), 0));
          }
          if (got)
            part = reinterpret_cast<const float*>(smem + static_cast<uint32_t>(quarter) * kSkWarpBytes);
          else if (lane == 0)
            fail();
        }
        // the folded RMSNorm of the input rows (1 without one)
        const float rs = in_row_scale(a, m);
        if (!silu) {
          const int nb0 = (ft - a.g[g].tile0) * kTile;
          float sq = 0.f;
          float* sqp = a.out_ss ? &sq : nullptr;
          for (int c = 0; c < kTile; c += 16) {
            float v[16];
            tmem_ld16(trow + c, v);
            if (part) {
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] += part[(c + j) * 32 + lane];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) v[j] *= rs;
            if (nb0 + c < a.g[g].N) epi_store16<__nv_bfloat16>(a, g, m, nb0 + c, v, sqp);
          }
          // this tile's share of the stored rows' sums of squares (group 0 only)
          if (a.out_ss && m < a.M)
            a.out_ss[static_cast<size_t>(m) * a.out_ss_cols + (ft - a.g[g].tile0)] = sq;
        } else {
          const int f0 = ft * kHalf;
          for (int c = 0; c < kHalf; c += 16) {
            float gv[16], uv[16];
            tmem_ld16(trow + c, gv);
            tmem_ld16(trow + kHalf + c, uv);
            if (part) {
#pragma unroll
              for (int j = 0; j < 16; ++j) {
                gv[j] += part[(c + j) * 32 + lane];
                uv[j] += part[(kHalf + c + j) * 32 + lane];
              }
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) gv[j] = silu_f(gv[j] * rs) * (uv[j] * rs);
            if (f0 + c < a.g[0].N) epi_store16<__nv_bfloat16>(a, 0, m, f0 + c, gv);
          }
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
  cluster_sync_converged();
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

int pair_sk_slots() { return std::max(1, device_sm_count() / 2); }

size_t pair_sk_part_bytes() {
  return static_cast<size_t>(pair_sk_slots()) * 2 * kTile * kHalf * sizeof(float);
}

size_t pair_sk_flag_bytes() { return static_cast<size_t>(pair_sk_slots()) * 2 * 4 * sizeof(int32_t); }

size_t pair_t_ready_bytes(int64_t M) {
  return static_cast<size_t>((M + kTile - 1) / kTile) * sizeof(int32_t);
}

uno_status gemm_pair_prepare(const GemmProblem& pb, GemmLaunch* out) {
  const bool silu = pb.mode == kEpiSiluPair;
  const int tile_n = silu ? kHalf : kTile;
  PairParams pp{};
  pp.a = make_gemm_args(pb, tile_n, 128);
  pp.tiles_m = static_cast<int>((pb.M + kTile - 1) / kTile);
  // t computed here: down tiles ahead of the main tiles, for 16 or more token
  // blocks (M > 3840) when the down tiles fit in the pairs that the last round
  // of main tiles leaves idle (same number of rounds). Same-box A/B on the
  // Qwen3-8B-shaped step: 3 % faster at M = 4352 (B = 256), where every linear
  // passes; taken at every M it was 3-4 % slower at M = 1088 and 2176. There
  // the separate down-projection is short and hides under the previous
  // launch's tail, while the main tiles of the first round wait for t here
  // (~7 us: a down tile streams as long a K-loop as a main tile).
  const int main_tiles = static_cast<int>(std::min<int64_t>(
      static_cast<int64_t>(pp.tiles_m) * feature_tiles(pp.a, tile_n), 1ll << 30));
  const int all_pairs = std::max(1, device_sm_count() / 2);
  const int down_per_block = (pb.ngroups + 1) / 2;   // two groups per down tile
  const int n_down = pp.tiles_m * down_per_block;
  bool down = pb.t_ready && pb.t && pb.r > 0 && pb.r <= kHalf && pp.tiles_m >= 16 &&
              (main_tiles + all_pairs - 1) / all_pairs ==
                  (main_tiles + n_down + all_pairs - 1) / all_pairs;
  for (int i = 0; i < pb.ngroups; ++i) down = down && pb.A[i];
  if (down && reinterpret_cast<uintptr_t>(pb.t_ready) % 4)
    return set_error(UNO_ERR_INVALID_ARG, "t counters must be 4-byte aligned");
  pp.down_tiles = down ? n_down : 0;
  pp.down_expect = 8 * down_per_block;               // 8 epilogue warps per down tile
  pp.r = pb.r;
  pp.ldt = static_cast<int>(pb.ldt);
  pp.t = down ? static_cast<__nv_bfloat16*>(const_cast<void*>(pb.t)) : nullptr;
  pp.t_ready = down ? pb.t_ready : nullptr;
  if (down) pp.a.x_ready = 0;   // x comes from the launch right before
  const int64_t tiles = static_cast<int64_t>(pp.tiles_m) * feature_tiles(pp.a, tile_n) + pp.down_tiles;
  if (tiles > (1ll << 30)) return set_error(UNO_ERR_UNSUPPORTED, "too many tiles");
  pp.num_tiles = static_cast<int>(tiles);
  pp.stages = 6;
  uno_status s;
  TensorMaps& tm = out->tm;
  for (int i = 0; i < kMaxGroups; ++i) {
    if (down) {   // A_g, rows >= r read zeros: 128 rows in one CTA (paired groups) or 64 in each
      const bool single = i == pb.ngroups - 1 && pb.ngroups % 2 == 1;
      if ((s = make_map(&tm.a[i], pb.dt, pb.A[i < pb.ngroups ? i : 0], pb.K, pb.r, pb.K,
                        single ? kHalf / 2 : kHalf)) != UNO_OK)
        return s;
    } else {
      std::memset(&tm.a[i], 0, sizeof(tm.a[i]));
    }
  }
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
  const int pairs = std::max(1, std::min<int>(device_sm_count() / 2, pp.num_tiles));
  // Stream-K: when the whole tiles would leave the last round part-empty
  // (rem of the pairs busy), the last `pairs + rem` tiles are shared out by
  // K-blocks instead, so every pair ends at the same time. Taken for deep
  // tiles only (>= 128 K-blocks, e.g. 12288 -> 4096 at M = 4352: 419 -> 396 us
  // on one B200): with 64-block tiles a part-empty last round runs its tiles
  // faster (fewer pairs share the L2), and splitting them measured no gain.
  // Not worth the hand-over of partial sums when the last round is nearly full.
  const int nkb = pp.a.nkb_main + (silu ? 2 : 1) * pp.a.nkb_r;
  const int rem = pp.num_tiles % pairs;
  // the finishing pair stages the partial sums in its idle stage ring
  static_assert(4 * kSkWarpBytes <= 6 * kStageBytes, "partial sums must fit the stage ring");
  pp.dp_tiles = pp.num_tiles;
  pp.sk_iters = 0;
  out->sk_flag = nullptr;
  out->sk_flag_bytes = 0;
  if (pb.sk_part && pb.sk_flag && pairs <= pb.sk_slots && rem > 0 && 5 * rem <= 4 * pairs &&
      nkb >= 128 && pp.num_tiles - (pairs + rem) >= pp.down_tiles) {
    const int sk_tiles = pairs + rem;
    pp.dp_tiles = pp.num_tiles - sk_tiles;
    pp.sk_iters = static_cast<long long>(sk_tiles) * nkb;
    pp.sk_part = pb.sk_part;
    pp.sk_flag = pb.sk_flag;
    out->sk_flag = pb.sk_flag;
    out->sk_flag_bytes = pair_sk_flag_bytes();
  }
  out->computes_t = down;
  out->t_ready = pp.t_ready;
  out->t_ready_bytes = down ? pair_t_ready_bytes(pb.M) : 0;
  std::memcpy(out->params, &pp, sizeof(pp));
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
  PairParams pp;
  std::memcpy(&pp, l.params, sizeof(pp));
  void* fn = pp.down_tiles > 0 ? reinterpret_cast<void*>(&gemm_pair_kernel<true>)
                               : reinterpret_cast<void*>(&gemm_pair_kernel<false>);
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
  void* args[2] = {const_cast<TensorMaps*>(&l.tm), &pp};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_error(e, "pair GEMM launch");
  return UNO_OK;
}

}  // namespace uno
