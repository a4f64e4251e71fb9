// Gated-LoRA GEMM on the 5th-generation tensor cores (sm_100a), one CTA per tile.
//
//   y_g = x W_g^T + t_g Bl_g^T,   t_g = scale * gate (.) (x A_g^T)
//   (the gated LoRA adapter: hyper.ai page, section "方法" — an adapter on
//   every AR matrix, switched per row)
//
// The adapter's up-projection is folded into the same accumulator as extra
// K-steps: the K loop runs over [x | t] against [W | Bl], so W streams from
// HBM exactly once and the LoRA term costs r/64 extra K-blocks. The gated
// down-projection t is the same kernel with epilogue kEpiRowScale. One launch
// covers up to three output groups that share x (q|k|v, or their
// down-projections); kEpiSiluPair fuses silu(gate) * up.
//
// Structure of one CTA (192 threads):
//   warp 0, one lane : TMA producer — 128-byte-swizzled K-major tiles of both
//                      operands into a ring of shared-memory stages;
//   warp 1, one lane : MMA issuer — tcgen05.mma (kind::f16 for bf16,
//                      kind::tf32 for f32), M = 128, N = bn, fp32 accumulator
//                      in TMEM; tcgen05.commit frees each stage;
//   warps 2..5       : epilogue — tcgen05.ld of the accumulator (each warp
//                      reads its 32-lane quarter), convert, store.
// Operand roles: the "P" operand fills the 128 MMA rows, the "Q" operand the
// bn MMA columns. Normal: P = tokens (x), Q = features (W). "Swap" (decode
// batches and the down-projections): P = features, Q = tokens (16..256 per
// tile). In swap silu-pair tiles the 128 feature rows are 64 gate rows then
// the same 64 up rows. Small problems split K across a thread-block cluster;
// the partial tiles are summed through distributed shared memory (no global
// scratch, no atomics, no spin waits).
#include <algorithm>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>
#include <type_traits>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace uno {

namespace {

constexpr int kGemmThreads = 192;
constexpr int kTileP = 128;         // MMA M
constexpr int kRowBytes = 128;      // one K-block row of either operand (64 bf16 / 32 f32)
constexpr int kMaxStages = 12;
// Split-K partial tiles in shared memory (fp32, padded rows):
//   non-swapped: part[i][bn + 4]   (one row per accumulator lane = token)
//   swapped:     part[j][128 + 4]  (one row per token column; lanes = features)
// so the reduction reads 16-byte groups of 4 consecutive lanes or columns.
constexpr int kPartPad = 4;
constexpr int kHalfP = kTileP / 2;

struct Gemm1Params {
  GemmArgs a;
  int bn;                 // Q rows per tile (multiple of 16, <= 256)
  int stages;
  int tmem_cols;
  int kb_per_split, splits;
  int32_t* zero_flags;    // cleared by CTA (0,0,0) after its wait (or NULL); 16-byte aligned
  int zero_words;         // a multiple of 4
};
static_assert(sizeof(Gemm1Params) <= 256, "Gemm1Params must fit GemmLaunch::params");

__host__ __device__ constexpr uint32_t stage_bytes_for(int bn) {
  return ((kTileP + bn) * kRowBytes + 1023u) & ~1023u;
}

__device__ __forceinline__ void epi_bar() { named_sync(1, 128); }

template <typename T, bool kSwap>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm1_kernel(const __grid_constant__ TensorMaps tm, const Gemm1Params p) {
  constexpr bool kTf32 = std::is_same<T, float>::value;
  constexpr int kBKe = kRowBytes / static_cast<int>(sizeof(T));  // elements per K-block
  constexpr int kKSteps = kRowBytes / 32;                          // MMAs per K-block (32 B of K each)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
  const GemmArgs& a = p.a;
  const int bn = p.bn;
  const uint32_t p_bytes = kTileP * kRowBytes;
  const uint32_t q_bytes = static_cast<uint32_t>(bn) * kRowBytes;
  const uint32_t st_bytes = stage_bytes_for(bn);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + p.stages * st_bytes);
  uint64_t* full = bars;
  uint64_t* empty = bars + p.stages;
  uint64_t* accum = bars + 2 * p.stages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* consumed = abort_flag + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const bool silu = a.mode == kEpiSiluPair;   // swap tiles only
  const int ft = blockIdx.y, split = blockIdx.z;
  const int g = group_of(a, ft);
  const int feat_rows = kSwap ? (silu ? kHalfP : kTileP) : bn;
  const int feat0 = (ft - a.g[g].tile0) * feat_rows;        // first feature of the tile in group g
  const int tok0 = blockIdx.x * (kSwap ? bn : kTileP);      // first token of the tile

  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(accum), 1);
    *abort_flag = 0;
    *consumed = 0;
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
  if (threadIdx.x == 0 && a.mode != kEpiRowScale) pdl_trigger();

  const int nkb_lora = silu ? 2 * a.nkb_r : a.nkb_r;
  const int nkb = a.nkb_main + nkb_lora;
  const int kb0 = split * p.kb_per_split;
  const int kb1 = min(nkb, kb0 + p.kb_per_split);
  int issued = 0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    // The weight (feature) operand of the first stages is constant: issue it
    // before waiting for the kernel that writes the activations.
    auto load_feat = [&](int kb, uint32_t s_feat, uint32_t fb) {
      if (kb < a.nkb_main) {
        const int kc = kb * kBKe;
        if (silu) {
          tma_load_2d(s_feat, &tm.w[0], kc, feat0, fb);
          tma_load_2d(s_feat + kHalfP * kRowBytes, &tm.w[1], kc, feat0, fb);
        } else {
          tma_load_2d(s_feat, &tm.w[g], kc, feat0, fb);
        }
      } else {
        const int l = kb - a.nkb_main;
        const int h = silu ? l / a.nkb_r : 0;           // silu: 0 = gate block, 1 = up block
        const int j = silu ? l % a.nkb_r : l;
        if (silu) {
          // the other half's adapter rows are read past the end: zeros
          tma_load_2d(s_feat, &tm.b[0], j * kBKe, h == 0 ? feat0 : a.g[0].b_rows, fb);
          tma_load_2d(s_feat + kHalfP * kRowBytes, &tm.b[1], j * kBKe,
                      h == 1 ? feat0 : a.g[1].b_rows, fb);
        } else {
          tma_load_2d(s_feat, &tm.b[g], j * kBKe, feat0, fb);
        }
      }
    };
    auto load_tok = [&](int kb, uint32_t s_tok, uint32_t fb) {
      if (kb < a.nkb_main) {
        tma_load_2d(s_tok, &tm.x, kb * kBKe, tok0, fb);
      } else {
        const int l = kb - a.nkb_main;
        const int h = silu ? l / a.nkb_r : 0;
        const int j = silu ? l % a.nkb_r : l;
        tma_load_2d(s_tok, &tm.t, a.g[silu ? h : g].t_col + j * kBKe, tok0, fb);
      }
    };
    // Down-projections (kEpiRowScale) let their dependent start only once
    // they have waited for the writer of their own input; a main GEMM so
    // launched (x_ready) reads x at once and waits only before reading t.
    const bool down = a.mode == kEpiRowScale;
    bool waited = false;
    auto wait_pred = [&]() {
      if (!waited) {
        pdl_wait();
        waited = true;
        if (p.zero_flags && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0)
          for (int w = 0; w < p.zero_words; w += 4)
            *reinterpret_cast<int4*>(p.zero_flags + w) = make_int4(0, 0, 0, 0);
        if (down) pdl_trigger();
      }
    };
    const int pre = min(p.stages, kb1 - kb0);
    for (int q = 0; q < pre; ++q) {
      const uint32_t sp = smem_u32(smem + q * st_bytes);
      const uint32_t fb = smem_u32(&full[q]);
      mbar_arrive_expect_tx(fb, p_bytes + q_bytes);
      load_feat(kb0 + q, kSwap ? sp : sp + p_bytes, fb);
    }
    for (int q = 0; q < pre; ++q) {
      const int kb = kb0 + q;
      if (!a.x_ready || kb >= a.nkb_main) wait_pred();
      const uint32_t sp = smem_u32(smem + q * st_bytes);
      load_tok(kb, kSwap ? sp + p_bytes : sp, smem_u32(&full[q]));
    }
    issued = pre;
    for (int kb = kb0 + pre; kb < kb1; ++kb, ++issued) {
      const int s = issued % p.stages;
      const uint32_t ph = (issued / p.stages) & 1u;
      if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u)) {
        *abort_flag = 1;
        raise_status(a.status, kDevTimeout);
        break;
      }
      if (*abort_flag) break;
      const uint32_t sp = smem_u32(smem + s * st_bytes);
      const uint32_t fb = smem_u32(&full[s]);
      mbar_arrive_expect_tx(fb, p_bytes + q_bytes);
      load_feat(kb, kSwap ? sp : sp + p_bytes, fb);
      if (kb >= a.nkb_main) wait_pred();
      load_tok(kb, kSwap ? sp + p_bytes : sp, fb);
    }
    if (down) wait_pred();   // a CTA with no K-blocks still triggers
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_f32acc(kTileP, bn, kTf32);
    int it = 0;
    for (int kb = kb0; kb < kb1; ++kb, ++it) {
      const int s = it % p.stages;
      const uint32_t ph = (it / p.stages) & 1u;
      if (!mbar_wait(smem_u32(&full[s]), ph)) {
        *abort_flag = 1;
        raise_status(a.status, kDevTimeout);
        break;
      }
      tc_fence_after();
      const uint32_t sp = smem_u32(smem + s * st_bytes);
      const uint64_t ad = sdesc_k_sw128(sp);
      const uint64_t bd = sdesc_k_sw128(sp + p_bytes);
#pragma unroll
      for (int kk = 0; kk < kKSteps; ++kk) {
        // +32 bytes of K inside the swizzled 128-byte rows = +2 in the encoded address
        mma_ss<kTf32>(tmem, ad + static_cast<uint64_t>(2 * kk), bd + static_cast<uint64_t>(2 * kk),
                      idesc, (it > 0 || kk > 0) ? 1u : 0u);
      }
      mma_commit(smem_u32(&empty[s]));
      *consumed = it + 1;
    }
    mma_commit(smem_u32(accum));
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3;            // TMEM lanes this warp may read
    const int i = quarter * 32 + lane;       // accumulator row
    if (!a.x_ready) pdl_wait();
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(accum), 0));
    if (!ok && lane == 0) {
      *abort_flag = 1;
      raise_status(a.status, kDevTimeout);
    }
    tc_fence_after();
    const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
    float* stage = reinterpret_cast<float*>(smem);   // the stage ring is free now
    if (p.splits == 1) {
      if (!kSwap) {
        if (ok) {
          for (int c = 0; c < bn; c += 16) {
            float v[16];
            tmem_ld16(trow + c, v);
            epi_store16<T>(a, g, tok0 + i, feat0 + c, v);
          }
        }
      } else if (!silu) {
        if (ok) {
          for (int c = 0; c < bn; c += 16) {
            float v[16];
            tmem_ld16(trow + c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) epi_store1<T>(a, g, tok0 + c + j, feat0 + i, v[j]);
          }
        }
      } else {
        // lanes 0..63 hold gate, 64..127 the matching up features: stage both
        // through shared memory, then every thread forms silu(gate) * up
        const int R = bn * (kHalfP + 1);
        const int f = i & (kHalfP - 1);
        float* dst = stage + (i < kHalfP ? 0 : R);
        if (ok) {
          for (int c = 0; c < bn; c += 16) {
            float v[16];
            tmem_ld16(trow + c, v);
#pragma unroll
            for (int j = 0; j < 16; ++j) dst[(c + j) * (kHalfP + 1) + f] = v[j];
          }
        }
        epi_bar();
        if (ok) {
          for (int j = i >> 6; j < bn; j += 2) {
            const float gv = stage[j * (kHalfP + 1) + f];
            const float uv = stage[R + j * (kHalfP + 1) + f];
            epi_store1<T>(a, 0, tok0 + j, feat0 + f, silu_f(gv) * uv);
          }
        }
      }
    } else if (ok) {
      for (int c = 0; c < bn; c += 16) {
        float v[16];
        tmem_ld16(trow + c, v);
        if (kSwap) {
#pragma unroll
          for (int j = 0; j < 16; ++j) stage[(c + j) * (kTileP + kPartPad) + i] = v[j];
        } else {
          float4* row = reinterpret_cast<float4*>(stage + i * (bn + kPartPad) + c);
#pragma unroll
          for (int q = 0; q < 4; ++q)
            row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
  }

  if (p.splits > 1) {
    // Sum the cluster's partial tiles. CTA `rank` reduces a contiguous range
    // of 4-element groups, reading the same group from every CTA.
    cluster_sync_converged();
    const uint32_t rank = cluster_ctarank();
    const int S = p.splits;
    const int groups = kSwap ? (silu ? bn * (kTileP / 8) : bn * (kTileP / 4)) : kTileP * bn / 4;
    const int chunk = (groups + S - 1) / S;
    const int e0 = static_cast<int>(rank) * chunk;
    const int e1 = min(groups, e0 + chunk);
    const uint32_t part0 = smem_u32(smem);
    // unrolled to the largest cluster (8) with constant indices, so the peer
    // addresses and partials stay in registers and all loads go out at once
    uint32_t peer[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) peer[r] = map_shared_rank(part0, r < S ? r : 0);
    auto sum4 = [&](uint32_t off) {
      float4 v[8];
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < S) v[r] = ld_cluster_f32x4(peer[r] + off);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int r = 0; r < 8; ++r)
        if (r < S) {
          acc.x += v[r].x; acc.y += v[r].y; acc.z += v[r].z; acc.w += v[r].w;
        }
      return acc;
    };
    for (int e = e0 + static_cast<int>(threadIdx.x); e < e1; e += kGemmThreads) {
      if (!kSwap) {
        const int i = e / (bn / 4), j4 = e % (bn / 4);
        const float4 acc = sum4(static_cast<uint32_t>((i * (bn + kPartPad) + 4 * j4) * 4));
        epi_store4<T>(a, g, tok0 + i, feat0 + 4 * j4, acc);
      } else if (!silu) {
        const int j = e / (kTileP / 4), i4 = e % (kTileP / 4);
        const float4 acc = sum4(static_cast<uint32_t>((j * (kTileP + kPartPad) + 4 * i4) * 4));
        epi_store4<T>(a, g, tok0 + j, feat0 + 4 * i4, acc);
      } else {
        const int j = e / (kTileP / 8), f4 = e % (kTileP / 8);
        const uint32_t row = static_cast<uint32_t>(j * (kTileP + kPartPad));
        const float4 gv = sum4((row + 4 * f4) * 4);
        const float4 uv = sum4((row + kHalfP + 4 * f4) * 4);
        epi_store4<T>(a, 0, tok0 + j, feat0 + 4 * f4,
                      make_float4(silu_f(gv.x) * uv.x, silu_f(gv.y) * uv.y, silu_f(gv.z) * uv.z,
                                  silu_f(gv.w) * uv.w));
      }
    }
    cluster_sync_converged();
  }

  // Drain: if the MMA side gave up, wait (bounded) for TMA copies still in flight.
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int it = *consumed; it < issued; ++it)
      mbar_wait(smem_u32(&full[it % p.stages]), (it / p.stages) & 1u, kWaitLimitNs / 4);
  }
  tc_fence_before();
  cta_sync_converged();   // every warp is done with TMEM before it is freed
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

template <typename T, bool kSwap>
void* kernel_ptr() {
  return reinterpret_cast<void*>(&gemm1_kernel<T, kSwap>);
}

void* pick_kernel(uno_dtype dt, bool swap) {
  if (dt == UNO_F32) return swap ? kernel_ptr<float, true>() : kernel_ptr<float, false>();
  return swap ? kernel_ptr<__nv_bfloat16, true>() : kernel_ptr<__nv_bfloat16, false>();
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

// How many clusters of `cluster` CTAs (cluster along z) of kernel `fn` with
// `smem` bytes of dynamic shared memory the GPU can hold at once (cached).
int64_t max_active_clusters(void* fn, int cluster, int smem) {
  static std::mutex mu;
  static std::map<std::tuple<void*, int, int>, int> cache;
  std::lock_guard<std::mutex> lock(mu);
  const auto key = std::make_tuple(fn, cluster, smem);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  int n = 0;
  if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(1, 1, cluster);
    cfg.blockDim = dim3(kGemmThreads, 1, 1);
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
      n = 1 << 20;   // unknown: do not restrict
    }
  }
  cache[key] = n;
  return n;
}

int pow2_at_least(int v) {
  int c = 32;
  while (c < v) c <<= 1;
  return c;
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

}  // namespace

uno_status make_map(CUtensorMap* tm, uno_dtype dt, const void* base, uint64_t inner, uint64_t rows,
                    uint64_t row_stride_elems, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const uint32_t esz = dt == UNO_F32 ? 4u : 2u;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {row_stride_elems * esz};
  const cuuint32_t box[2] = {kRowBytes / esz, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r =
      fn(tm, dt == UNO_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
         const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS)
    return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d): inner=%llu rows=%llu",
                     static_cast<int>(r), static_cast<unsigned long long>(inner),
                     static_cast<unsigned long long>(rows));
  return UNO_OK;
}

int device_sm_count() {
  static int n = [] {
    int dev = 0, v = 148;
    if (cudaGetDevice(&dev) == cudaSuccess)
      cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v;
  }();
  return n;
}

uno_status gemm_prepare(const GemmProblem& pb, GemmLaunch* out) {
  out->sk_flag = nullptr;
  out->sk_flag_bytes = 0;
  out->t_ready = nullptr;
  out->t_ready_bytes = 0;
  out->computes_t = false;
  if (pb.ngroups < 1 || pb.ngroups > kMaxGroups)
    return set_error(UNO_ERR_INVALID_ARG, "1..3 output groups per GEMM launch");
  if (pb.mode == kEpiSiluPair && (pb.ngroups != 2 || pb.g[0].N != pb.g[1].N))
    return set_error(UNO_ERR_INVALID_ARG, "silu-pair needs two groups of equal width");
  if (pb.zero_flags && (pb.mode != kEpiRowScale || pb.M <= 256 || pb.zero_words % 4 ||
                        reinterpret_cast<uintptr_t>(pb.zero_flags) % 16))
    return set_error(UNO_ERR_INVALID_ARG, "only a large-batch down-projection clears flags");
  if (gemm_pair_suits(pb)) return gemm_pair_prepare(pb, out);
  if (gemm_dec_suits(pb)) return gemm_dec_prepare(pb, out);
  if (pb.mode == kEpiSiluPair && pb.M > 256)
    return set_error(UNO_ERR_UNSUPPORTED, "silu-pair with M > 256 needs the bf16 pair kernel");
  const int esz = pb.dt == UNO_F32 ? 4 : 2;
  (void)esz;
  const int sms = device_sm_count();
  const int64_t M = pb.M;
  if (M > (1ll << 30)) return set_error(UNO_ERR_UNSUPPORTED, "M too large");
  const bool silu = pb.mode == kEpiSiluPair;

  // Tile shape: decode batches and the rank-r down-projections put the
  // weight rows on the 128-row MMA side ("swap").
  const bool swap = M <= 256 || pb.mode == kEpiRowScale;
  int bn, tok_tiles;
  if (swap) {
    // decode batches: one token tile of up to 256; down-projections of large
    // batches: 128-token tiles (more tiles to spread over the SMs)
    const int tile = M <= 256 ? 256 : 128;
    tok_tiles = static_cast<int>((M + tile - 1) / tile);
    bn = round_up(static_cast<int>((M + tok_tiles - 1) / tok_tiles), 16);
  } else {
    tok_tiles = static_cast<int>((M + kTileP - 1) / kTileP);
    int64_t ntiles256 = 0;
    for (int i = 0; i < pb.ngroups; ++i) ntiles256 += (pb.g[i].N + 255) / 256;
    bn = (tok_tiles * ntiles256 >= sms) ? 256 : 128;
  }
  const int feat_tile = swap ? (silu ? kHalfP : kTileP) : bn;
  GemmArgs ga = make_gemm_args(pb, feat_tile, kRowBytes);
  const int feat_tiles = feature_tiles(ga, feat_tile);
  if (feat_tiles > 65535) return set_error(UNO_ERR_UNSUPPORTED, "N too large for the tile grid");

  const int nkb = ga.nkb_main + (silu ? 2 : 1) * ga.nkb_r;

  // Shared memory: ~96 KB for narrow decode tiles, ~200 KB otherwise. (Shared
  // memory would fit two or three narrow CTAs per SM; the swap variant's 142
  // registers a thread allow two.)
  // Down-projections of large batches take the full ring: their cluster grid
  // is sized to one CTA per SM, and each CTA streams a long K-slice whose
  // rate is set by the bytes it keeps in flight.
  const uint32_t st = stage_bytes_for(bn);
  const bool narrow = bn <= 64;
  const uint32_t budget = narrow ? 96u * 1024u : 200u * 1024u;
  int stages = std::min<int>(kMaxStages, static_cast<int>(budget / st));
  stages = std::max(stages, 2);
  const int per_sm = narrow ? std::max(1, static_cast<int>((228u * 1024u) / (stages * st + 2048u)))
                            : 1;

  // Split K across a cluster when the tile grid cannot fill the GPU.
  const int64_t tiles = static_cast<int64_t>(tok_tiles) * feat_tiles;
  int splits = 1;
  const int64_t capacity = static_cast<int64_t>(sms) * per_sm;
  if (tiles < capacity) {
    splits = static_cast<int>(std::min<int64_t>(8, capacity / tiles));
    splits = std::max(1, std::min(splits, nkb / 2));
  }
  // every cluster of the launch must be resident at once: cap the split by
  // the number of clusters of that size the GPU can hold
  while (splits > 1 &&
         max_active_clusters(pick_kernel(pb.dt, swap), splits,
                             static_cast<int>(stages * st + 1024 + 64 + 16 * (2 * stages + 1))) <
             tiles)
    --splits;
  int kb_per = (nkb + splits - 1) / splits;
  splits = (nkb + kb_per - 1) / kb_per;   // every split gets >= 1 K-block
  // the split-K partial tile (and the silu hand-over) must fit in the stage ring
  const uint32_t part_bytes = static_cast<uint32_t>(
      (swap ? bn * (kTileP + kPartPad) : kTileP * (bn + kPartPad)) * 4);
  const uint32_t silu_bytes = static_cast<uint32_t>(2 * bn * (kHalfP + 1) * 4);
  if (splits > 1 && part_bytes > stages * st) {
    splits = 1;
    kb_per = nkb;
  }
  if (silu && splits == 1 && silu_bytes > stages * st)
    return set_error(UNO_ERR_UNSUPPORTED, "silu-pair tile does not fit shared memory");

  Gemm1Params gp{};
  gp.a = ga;
  gp.bn = bn;
  gp.stages = stages;
  gp.tmem_cols = pow2_at_least(bn);
  gp.kb_per_split = kb_per;
  gp.splits = splits;
  gp.zero_flags = pb.zero_flags;
  gp.zero_words = pb.zero_words;

  const uint32_t tok_box = swap ? static_cast<uint32_t>(bn) : kTileP;
  const uint32_t feat_box = swap ? static_cast<uint32_t>(feat_tile) : static_cast<uint32_t>(bn);
  uno_status s;
  TensorMaps& tm = out->tm;
  if ((s = make_map(&tm.x, pb.dt, pb.x, pb.K, M, pb.K, tok_box)) != UNO_OK) return s;
  if (pb.r > 0) {
    if ((s = make_map(&tm.t, pb.dt, pb.t, pb.ldt, M, pb.ldt, tok_box)) != UNO_OK) return s;
  } else {
    tm.t = tm.x;
  }
  for (int i = 0; i < kMaxGroups; ++i) {
    const GemmGroup& G = pb.g[i < pb.ngroups ? i : 0];
    if ((s = make_map(&tm.w[i], pb.dt, G.W, pb.K, G.N, pb.K, feat_box)) != UNO_OK) return s;
    if (pb.r > 0) {
      if ((s = make_map(&tm.b[i], pb.dt, G.Bl, pb.r, G.N, pb.r, feat_box)) != UNO_OK) return s;
    } else {
      tm.b[i] = tm.w[i];
    }
  }
  std::memcpy(out->params, &gp, sizeof(gp));
  out->kind = 0;
  out->swap = swap;
  out->grid_x = tok_tiles;
  out->grid_y = feat_tiles;
  out->splits = splits;
  out->smem_bytes = static_cast<int>(stages * st + 1024 + 64 + 16 * (2 * stages + 1));
  out->dtype = pb.dt;
  return UNO_OK;
}

uno_status gemm_run(const GemmLaunch& l, cudaStream_t stream) {
  if (l.kind == 1) return gemm_pair_run(l, stream);
  if (l.kind == 2) return gemm_dec_run(l, stream);
  void* fn = pick_kernel(static_cast<uno_dtype>(l.dtype), l.swap != 0);
  cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, l.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(gemm smem)");
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid_x, l.grid_y, l.splits);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = l.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  cfg.numAttrs = launch_attrs(attr, 1, 1, static_cast<unsigned>(l.splits));
  cfg.attrs = attr;
  Gemm1Params gp;
  std::memcpy(&gp, l.params, sizeof(gp));
  void* args[2] = {const_cast<TensorMaps*>(&l.tm), &gp};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_error(e, "gated GEMM launch");
  return UNO_OK;
}

}  // namespace uno
