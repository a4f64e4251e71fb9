// Gated-LoRA GEMM on the 5th-generation tensor cores (sm_100a).
//
//   y = x W^T + t Bl^T,   t = scale * g (.) (x A^T)   (the gated LoRA adapter:
//   hyper.ai page, section "方法" — adapter on every AR matrix, gated per row)
//
// The adapter's up-projection is folded into the same accumulator as extra
// K-steps: the K loop runs over [x | t] against [W | Bl], so W streams from
// HBM exactly once and the LoRA term costs r/64 extra K-blocks. The gated
// down-projection t is the same kernel with epilogue kEpiRowScale.
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
// bn MMA columns. Large M: P = tokens (x), Q = features (W). Small M
// ("swap"): P = features (W), Q = tokens (x), so a decode batch of 9..256
// rows still fills the 128-row MMA. Small problems split K across a thread
// block cluster; the partial tiles are summed through distributed shared
// memory (no global scratch, no atomics, no spin waits).
#include <algorithm>
#include <cstring>
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
// so the reduction reads 16-byte groups of 4 consecutive output features.
constexpr int kPartPad = 4;

struct GemmParams {
  EpiArgs e;
  int bn;                 // Q rows per tile (multiple of 16, <= 256)
  int stages;
  int tmem_cols;
  int nkb_main, nkb_lora, kb_per_split, splits;
  int32_t* status;
};
static_assert(sizeof(GemmParams) <= 128, "GemmParams must fit GemmLaunch::params");

__host__ __device__ constexpr uint32_t stage_bytes_for(int bn) {
  return ((kTileP + bn) * kRowBytes + 1023u) & ~1023u;
}

template <typename T, bool kSwap>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gated_gemm_kernel(const __grid_constant__ CUtensorMap tm_x,
                      const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_t,
                      const __grid_constant__ CUtensorMap tm_b, const GemmParams p) {
  constexpr bool kTf32 = std::is_same<T, float>::value;
  constexpr int kBKe = kRowBytes / static_cast<int>(sizeof(T));  // elements per K-block
  constexpr int kKSteps = kRowBytes / 32;                          // MMAs per K-block (32 B of K each)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023u) & ~static_cast<uintptr_t>(1023u));
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
  const int tok_tile = blockIdx.x, feat_tile = blockIdx.y, split = blockIdx.z;
  const int p_row0 = kSwap ? feat_tile * kTileP : tok_tile * kTileP;
  const int q_row0 = kSwap ? tok_tile * bn : feat_tile * bn;

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
  if (warp == 1 && lane == 0) {
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_w);
    if (p.nkb_lora) {
      tma_prefetch_desc(&tm_t);
      tma_prefetch_desc(&tm_b);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int nkb = p.nkb_main + p.nkb_lora;
  const int kb0 = split * p.kb_per_split;
  const int kb1 = min(nkb, kb0 + p.kb_per_split);
  int issued = 0;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    for (int kb = kb0; kb < kb1; ++kb, ++issued) {
      const int s = issued % p.stages;
      const uint32_t ph = (issued / p.stages) & 1u;
      if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u)) {
        *abort_flag = 1;
        raise_status(p.status, kDevTimeout);
        break;
      }
      if (*abort_flag) break;
      const uint32_t sp = smem_u32(smem + s * st_bytes);
      const uint32_t sq = sp + p_bytes;
      const uint32_t fb = smem_u32(&full[s]);
      mbar_arrive_expect_tx(fb, p_bytes + q_bytes);
      const bool lora = kb >= p.nkb_main;
      const int kc = (lora ? kb - p.nkb_main : kb) * kBKe;
      const CUtensorMap* tok_map = lora ? &tm_t : &tm_x;
      const CUtensorMap* feat_map = lora ? &tm_b : &tm_w;
      if (kSwap) {
        tma_load_2d(sp, feat_map, kc, p_row0, fb);
        tma_load_2d(sq, tok_map, kc, q_row0, fb);
      } else {
        tma_load_2d(sp, tok_map, kc, p_row0, fb);
        tma_load_2d(sq, feat_map, kc, q_row0, fb);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_f32acc(kTileP, bn, kTf32);
    int it = 0;
    for (int kb = kb0; kb < kb1; ++kb, ++it) {
      const int s = it % p.stages;
      const uint32_t ph = (it / p.stages) & 1u;
      if (!mbar_wait(smem_u32(&full[s]), ph)) {
        *abort_flag = 1;
        raise_status(p.status, kDevTimeout);
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
    const bool ok = __all_sync(0xffffffffu, mbar_wait(smem_u32(accum), 0));
    if (!ok && lane == 0) {
      *abort_flag = 1;
      raise_status(p.status, kDevTimeout);
    }
    tc_fence_after();
    if (ok) {
      const uint32_t trow = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
      if (p.splits == 1) {
        for (int c = 0; c < bn; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          if (!kSwap) {
            const int m = p_row0 + i, n0 = q_row0 + c;
            if (m < p.e.M) {
              if (n0 + 16 <= p.e.N) {
                epi_store16_row<T>(p.e, m, n0, v);
              } else {
#pragma unroll
                for (int j = 0; j < 16; ++j) epi_store1<T, kSwap>(p.e, p_row0, q_row0, i, c + j, v[j]);
              }
            }
          } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) epi_store1<T, kSwap>(p.e, p_row0, q_row0, i, c + j, v[j]);
          }
        }
      } else {
        float* part = reinterpret_cast<float*>(smem);   // the stage ring is free now
        for (int c = 0; c < bn; c += 16) {
          float v[16];
          tmem_ld16(trow + c, v);
          if (kSwap) {
#pragma unroll
            for (int j = 0; j < 16; ++j) part[(c + j) * (kTileP + kPartPad) + i] = v[j];
          } else {
            float4* row = reinterpret_cast<float4*>(part + i * (bn + kPartPad) + c);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              row[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
          }
        }
      }
    }
  }

  if (p.splits > 1) {
    // Sum the cluster's partial tiles. The tile is cut into groups of 4
    // consecutive output features; CTA `rank` reduces a contiguous range of
    // groups, reading the same group from every CTA of the cluster.
    cluster_sync();
    const uint32_t rank = cluster_ctarank();
    const int S = p.splits;
    const int groups = kTileP * bn / 4;
    const int chunk = (groups + S - 1) / S;
    const int g0 = static_cast<int>(rank) * chunk;
    const int g1 = min(groups, g0 + chunk);
    const uint32_t part0 = smem_u32(smem);
    uint32_t peer[8];
    for (int r = 0; r < S; ++r) peer[r] = map_shared_rank(part0, r);
    for (int g = g0 + static_cast<int>(threadIdx.x); g < g1; g += kGemmThreads) {
      int m, n;
      uint32_t off;
      if (kSwap) {
        const int j = g / (kTileP / 4), i4 = g % (kTileP / 4);
        off = static_cast<uint32_t>((j * (kTileP + kPartPad) + 4 * i4) * 4);
        m = q_row0 + j;
        n = p_row0 + 4 * i4;
      } else {
        const int i = g / (bn / 4), j4 = g % (bn / 4);
        off = static_cast<uint32_t>((i * (bn + kPartPad) + 4 * j4) * 4);
        m = p_row0 + i;
        n = q_row0 + 4 * j4;
      }
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int r = 0; r < S; ++r) {
        const float4 v = ld_cluster_f32x4(peer[r] + off);
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      if (m < p.e.M && n < p.e.N) epi_store4<T>(p.e, m, n, acc);
    }
    cluster_sync();
  }

  // Drain: if the MMA side gave up, wait (bounded) for TMA copies still in flight.
  if (warp == 0 && lane == 0 && *abort_flag) {
    for (int it = *consumed; it < issued; ++it)
      mbar_wait(smem_u32(&full[it % p.stages]), (it / p.stages) & 1u, kWaitLimitNs / 4);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
  }
}

// ---------------------------------------------------------------- host side

template <typename T, bool kSwap>
void* kernel_ptr() {
  return reinterpret_cast<void*>(&gated_gemm_kernel<T, kSwap>);
}

void* pick_kernel(uno_dtype dt, bool swap) {
  if (dt == UNO_F32) return swap ? kernel_ptr<float, true>() : kernel_ptr<float, false>();
  return swap ? kernel_ptr<__nv_bfloat16, true>() : kernel_ptr<__nv_bfloat16, false>();
}

int round_up(int v, int m) { return (v + m - 1) / m * m; }

int pow2_at_least(int v) {
  int c = 32;
  while (c < v) c <<= 1;
  return c;
}

}  // namespace

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

// Row-major [rows, inner] tensor, box = 128 bytes of K x box_rows rows, 128-byte swizzle.
uno_status make_map(CUtensorMap* tm, uno_dtype dt, const void* base, uint64_t inner, uint64_t rows,
                    uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return set_error(UNO_ERR_CUDA, "cuTensorMapEncodeTiled is not available");
  const uint32_t esz = dt == UNO_F32 ? 4u : 2u;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {inner * esz};
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
  if (gemm_pair_suits(pb)) return gemm_pair_prepare(pb, out);
  const int esz = pb.dt == UNO_F32 ? 4 : 2;
  const int bke = kRowBytes / esz;
  const int sms = device_sm_count();
  const int64_t M = pb.M, N = pb.N;
  if (M > (1ll << 30) || N > (1ll << 30)) return set_error(UNO_ERR_UNSUPPORTED, "M or N too large");

  // Tile shape: small M puts the weight rows on the 128-row MMA side.
  const bool swap = M <= 256;
  int bn, grid_x, grid_y;
  if (swap) {
    bn = round_up(static_cast<int>(M), 16);
    grid_x = 1;
    grid_y = static_cast<int>((N + kTileP - 1) / kTileP);
  } else {
    const int64_t tiles_tok = (M + kTileP - 1) / kTileP;
    bn = (tiles_tok * ((N + 255) / 256) >= sms) ? 256 : 128;
    grid_x = static_cast<int>(tiles_tok);
    grid_y = static_cast<int>((N + bn - 1) / bn);
  }
  if (grid_y > 65535) return set_error(UNO_ERR_UNSUPPORTED, "N too large for the tile grid");

  const int nkb_main = static_cast<int>((pb.K + bke - 1) / bke);
  const int nkb_lora = pb.r > 0 ? (pb.r + bke - 1) / bke : 0;
  const int nkb = nkb_main + nkb_lora;

  // Shared memory: ~96 KB (two or three CTAs per SM) for narrow decode tiles,
  // ~200 KB otherwise.
  const uint32_t st = stage_bytes_for(bn);
  const bool narrow = bn <= 64;
  const uint32_t budget = narrow ? 96u * 1024u : 200u * 1024u;
  int stages = std::min<int>(kMaxStages, static_cast<int>(budget / st));
  stages = std::max(stages, 2);
  const int per_sm = narrow ? std::max(1, static_cast<int>((228u * 1024u) / (stages * st + 2048u)))
                            : 1;

  // Split K across a cluster when the tile grid cannot fill the GPU.
  const int64_t tiles = static_cast<int64_t>(grid_x) * grid_y;
  int splits = 1;
  const int64_t capacity = static_cast<int64_t>(sms) * per_sm;
  if (tiles < capacity) {
    splits = static_cast<int>(std::min<int64_t>(8, capacity / tiles));
    splits = std::max(1, std::min(splits, nkb / 2));
  }
  int kb_per = (nkb + splits - 1) / splits;
  splits = (nkb + kb_per - 1) / kb_per;   // every split gets >= 1 K-block
  // the split-K partial tile must fit in the stage ring
  const uint32_t part_bytes = static_cast<uint32_t>(
      (swap ? bn * (kTileP + kPartPad) : kTileP * (bn + kPartPad)) * 4);
  if (splits > 1 && part_bytes > stages * st) {
    splits = 1;
    kb_per = nkb;
  }

  GemmParams gp{};
  gp.e = epi_args(pb);
  gp.bn = bn;
  gp.stages = stages;
  gp.tmem_cols = pow2_at_least(bn);
  gp.nkb_main = nkb_main;
  gp.nkb_lora = nkb_lora;
  gp.kb_per_split = kb_per;
  gp.splits = splits;
  gp.status = nullptr;

  const uint32_t tok_box = swap ? static_cast<uint32_t>(bn) : kTileP;
  const uint32_t feat_box = swap ? kTileP : static_cast<uint32_t>(bn);
  uno_status s;
  if ((s = make_map(&out->tm[0], pb.dt, pb.x, pb.K, M, tok_box)) != UNO_OK) return s;
  if ((s = make_map(&out->tm[1], pb.dt, pb.W, pb.K, N, feat_box)) != UNO_OK) return s;
  if (pb.r > 0) {
    if ((s = make_map(&out->tm[2], pb.dt, pb.t, pb.r, M, tok_box)) != UNO_OK) return s;
    if ((s = make_map(&out->tm[3], pb.dt, pb.Bl, pb.r, N, feat_box)) != UNO_OK) return s;
  } else {
    out->tm[2] = out->tm[0];
    out->tm[3] = out->tm[1];
  }
  std::memcpy(out->params, &gp, sizeof(gp));
  out->kind = 0;
  out->swap = swap;
  out->grid_x = grid_x;
  out->grid_y = grid_y;
  out->splits = splits;
  out->smem_bytes = static_cast<int>(stages * st + 1024 + 64 + 16 * (2 * stages + 1));
  out->dtype = pb.dt;
  return UNO_OK;
}

uno_status gemm_run(const GemmLaunch& l, cudaStream_t stream) {
  if (l.kind == 1) return gemm_pair_run(l, stream);
  void* fn = pick_kernel(static_cast<uno_dtype>(l.dtype), l.swap != 0);
  cudaError_t e =
      cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, l.smem_bytes);
  if (e != cudaSuccess) return cuda_error(e, "cudaFuncSetAttribute(gemm smem)");
  if (l.splits > 1) {
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    (void)e;
  }
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid_x, l.grid_y, l.splits);
  cfg.blockDim = dim3(kGemmThreads, 1, 1);
  cfg.dynamicSmemBytes = l.smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  if (l.splits > 1) {
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = l.splits;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
  GemmParams gp;
  std::memcpy(&gp, l.params, sizeof(gp));
  void* args[5] = {const_cast<CUtensorMap*>(&l.tm[0]), const_cast<CUtensorMap*>(&l.tm[1]),
                   const_cast<CUtensorMap*>(&l.tm[2]), const_cast<CUtensorMap*>(&l.tm[3]), &gp};
  e = cudaLaunchKernelExC(&cfg, fn, args);
  if (e != cudaSuccess) return cuda_error(e, "gated GEMM launch");
  return UNO_OK;
}

}  // namespace uno
