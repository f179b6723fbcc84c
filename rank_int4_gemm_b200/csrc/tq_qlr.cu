// tq_qlr.cu -- the down projection of the INT4 low-rank branch on
// 5th-generation tensor cores, straight from the activation codes.
//
// TwinQuant (Figure 4, both low-rank components quantized): X L1 is taken
// from the rotated per-token INT4 activation codes and the INT4 codes of
// H^T L1 (per column), accumulated in INT32, dequantized with s_x s_L1 and
// requantized per token to INT4 for the up projection.  For a tile of 128
// tokens
//
//   acc[t][j] = sum_k qx[t][k] qL1[j][k]      (tcgen05.mma kind::i8, exact)
//
// with both operands staged by TMA one code per byte.  A cluster of C CTAs
// splits K; each CTA sends the partial row of every token to the CTA that
// owns the token (distributed shared memory, rows split evenly), and the
// owner sums the C partials (integers: exact in any order), dequantizes
// v = s_x[t] s_L1[j] acc and requantizes the row: scale max|v| / 7 and
// RoundClip(v 7 / max|v|) with ties to even, in the same fp32 operations as
// the stand-alone requantization kernel.  Ranks above 256 (the widest MMA)
// run in column chunks that store the INT32 sums instead.
//
// Warp 0: TMA producer.  Warp 1: TMEM allocation and MMA issue.  Warps 2-5:
// TMEM readers (warp w reads lanes 32*(w%4)..), then the owners' rows.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "tq_act_common.cuh"
#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

namespace {

constexpr int kTok = 128;                        // tokens per tile (MMA M)
constexpr int kKb = 128;                         // codes per k-block (one 128-byte row)
constexpr uint32_t kTileX = kTok * kKb;          // bytes of one staged code tile
// Stages: at most kMaxNS within kStageBudget.  Small on purpose: with about
// 96 KB a CTA can become resident beside the activation kernel's CTAs while
// they finish (programmatic dependent launch); eight 24 KB stages measured
// slower at every shape, four as fast as any.
constexpr int kMaxNS = 4;
constexpr uint32_t kStageBudget = 192 * 1024;
constexpr int kMaxRn = 256;                      // columns of one launch (MMA N)
constexpr int kMaxC = 8;                         // CTAs per cluster along K
constexpr int kEpiFirstWarp = 2;
constexpr int kThreads = 32 * (kEpiFirstWarp + 4);

struct QlrParams {
  const float* s_x;        // [M] activation scales
  const float* s_L1;       // [r] scales of the L1 codes (whole rank)
  __nv_bfloat16* XL1q;     // [M][rn] requantized codes as bf16 integers, or null
  float* s_xl1;            // [M] their scales
  int32_t* acc_out;        // [M][r_ld] INT32 sums at column r_off (chunked ranks), or null
  uint32_t* status;        // timeout report
  int M, kb_total, nb;     // k-blocks in total and per CTA
  int rn, r_ld, r_off;     // columns of this launch, row stride of acc_out, first column
  int ns;                  // stages
  uint32_t tmem_cols;      // power of two >= max(32, rn)
};

__host__ __device__ constexpr uint32_t stage_bytes(int rn) {
  return kTileX + (uint32_t)rn * kKb;
}
__host__ __device__ constexpr int num_stages(int rn) {
  return (int)(kStageBudget / stage_bytes(rn)) < kMaxNS ? (int)(kStageBudget / stage_bytes(rn))
                                                        : kMaxNS;
}
// [stages][barriers: full, empty, acc_full][tmem slot, abort flag]
__host__ __device__ constexpr uint32_t smem_bytes(int rn) {
  return (uint32_t)num_stages(rn) * stage_bytes(rn) + (2 * kMaxNS + 1) * 8 + 8;
}
// receive area of the cluster reduction, [C][rows per owner][rn + 4] int32
// (padded rows: the 16-byte stores of 32 consecutive rows spread over the
// banks); it reuses the stages once every CTA's MMAs are done
__host__ __device__ constexpr uint32_t recv_bytes(int rn, int C) {
  return (uint32_t)C * (uint32_t)((kTok + C - 1) / C) * (uint32_t)(rn + 4) * 4u;
}
static_assert(num_stages(kMaxRn) >= 2, "stages");
static_assert(recv_bytes(kMaxRn, kMaxC) <= num_stages(kMaxRn) * stage_bytes(kMaxRn), "receive area");
static_assert(recv_bytes(16, kMaxC) <= num_stages(16) * stage_bytes(16), "receive area");

__device__ __forceinline__ void cluster_arrive_rel() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
    xl1_codes_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_l1, const QlrParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  const uint32_t stage = stage_bytes(p.rn);
  const int ns = p.ns;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + (uint32_t)ns * stage);
  uint64_t* empty = full + kMaxNS;
  uint64_t* acc_full = empty + kMaxNS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int tile = blockIdx.y;
  const int kb0 = (int)crank * p.nb;
  const int nb = max(0, min(p.nb, p.kb_total - kb0));  // k-blocks of this CTA

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < ns; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_x);
    tma_prefetch_desc(&map_l1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, p.tmem_cols);
    tmem_relinquish();
  }
  pdl_wait();                // the codes and s_x come from the preceding kernel
  cluster_arrive_relaxed();  // B0: this CTA is running
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();

  if (warp == 0) {
    // ======================================================== TMA producer
    cluster_wait_acquire();  // B0
    if (lane == 0) {
      const uint64_t pol = policy_evict_last();  // the codes are read again by the GEMM
      for (int i = 0; i < nb; ++i) {
        const int s = i % ns;
        if (!mbar_wait(&empty[s], ((uint32_t)(i / ns) & 1u) ^ 1u, p.status, abort_flag)) break;
        mbar_arrive_expect_tx(&full[s], stage);
        uint8_t* st = smem + (uint32_t)s * stage;
        const int x = (kb0 + i) * kKb;
        tma_load_2d(st, &map_x, &full[s], x, tile * kTok, pol);
        tma_load_2d(st + kTileX, &map_l1, &full[s], x, p.r_off, pol);
      }
    }
    __syncwarp();
    cluster_arrive_rel();  // B2
    cluster_wait_acquire();
    cluster_arrive_rel();  // B3
    cluster_wait_acquire();
  } else if (warp == 1) {
    // ========================================================== MMA issuer
    cluster_wait_acquire();  // B0
    const uint32_t idesc = idesc_i8_s32(p.rn);
    for (int i = 0; i < nb; ++i) {
      const int s = i % ns;
      if (!mbar_wait(&full[s], (uint32_t)(i / ns) & 1u, p.status, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = base + (uint32_t)s * stage;
        const uint64_t da = sdesc_sw128(st);
        const uint64_t db = sdesc_sw128(st + kTileX);
#pragma unroll
        for (int kk = 0; kk < kKb / 32; ++kk)  // K = 32 codes (32 bytes) per MMA
          mma_i8(tmem, da + 2 * kk, db + 2 * kk, idesc, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(acc_full);
    __syncwarp();
    cluster_arrive_rel();  // B2
    cluster_wait_acquire();
    cluster_arrive_rel();  // B3
    cluster_wait_acquire();
  } else {
    // ===================================================== TMEM readers
    const int q = warp & 3;         // TMEM lane quarter
    const int row = q * 32 + lane;  // token row of the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const int rpo = (kTok + (int)csize - 1) / (int)csize;  // rows per owner
    const uint32_t rs = (uint32_t)p.rn + 4u;                // receive row stride (words)
    cluster_wait_acquire();  // B0
    const bool ok = __all_sync(kFull, mbar_wait(acc_full, 0u, p.status, abort_flag));
    cluster_arrive_rel();    // B2: this CTA's MMAs are done, its stages may be written
    cluster_wait_acquire();
    if (ok) {
      tc_fence_after();
      const int owner = row / rpo;
      const uint32_t dst =
          dsmem_map(base + ((uint32_t)((int)crank * rpo + row - owner * rpo) * rs) * 4u,
                    (uint32_t)owner);
      for (int c0 = 0; c0 < p.rn; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + (uint32_t)c0 + lane_off, v);
        tmem_ld_wait();
        if (nb == 0) {  // no k-block here: the accumulator was never written
#pragma unroll
          for (int e = 0; e < 16; ++e) v[e] = 0u;
        }
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          asm volatile("st.shared::cluster.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst + (uint32_t)(c0 + e) * 4u),
                       "r"(v[e]), "r"(v[e + 1]), "r"(v[e + 2]), "r"(v[e + 3])
                       : "memory");
      }
    }
    cluster_arrive_rel();  // B3: partials delivered
    cluster_wait_acquire();
    if (!*abort_flag) {
      // this CTA's rows, one warp per row, lane + 32 i the columns
      const int row0 = (int)crank * rpo;
      const int nrow = min(rpo, kTok - row0);
      const int32_t* recv = reinterpret_cast<const int32_t*>(smem);
      for (int rr = warp - kEpiFirstWarp; rr < nrow; rr += 4) {
        const int gr = tile * kTok + row0 + rr;
        if (gr >= p.M) break;
        constexpr int kPer = kMaxRn / 32;
        int acc[kPer];
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int j = lane + 32 * i;
          acc[i] = 0;
          if (j < p.rn)
            for (int z = 0; z < (int)csize; ++z) acc[i] += recv[(size_t)(z * rpo + rr) * rs + j];
        }
        if (p.acc_out) {
#pragma unroll
          for (int i = 0; i < kPer; ++i) {
            const int j = lane + 32 * i;
            if (j < p.rn) p.acc_out[(size_t)gr * p.r_ld + p.r_off + j] = acc[i];
          }
          continue;
        }
        const float sx = __ldg(p.s_x + gr);
        float v[kPer];
        float amax = 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int j = lane + 32 * i;
          v[i] = 0.f;
          if (j < p.rn) {
            v[i] = sx * __ldg(p.s_L1 + p.r_off + j) * (float)acc[i];
            amax = fmaxf(amax, fabsf(v[i]));
          }
        }
        amax = warp_max(amax);
        const float inv = amax > 0.f ? 7.f / amax : 0.f;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
          const int j = lane + 32 * i;
          if (j < p.rn)
            p.XL1q[(size_t)gr * p.rn + j] = __float2bfloat16_rn((float)quant_code(v[i], inv));
        }
        if (lane == 0) p.s_xl1[gr] = amax / 7.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, p.tmem_cols);
  }
}

// One launch: columns [r_off, r_off + rn) of X L1 (rn <= kMaxRn, a multiple
// of 16), requantized when acc_out is null (then rn is the whole rank).
cudaError_t launch_xl1_one(const int8_t* Xq8, const int8_t* qL1, int M, int K, int r, int r_off,
                           int rn, const float* s_x, const float* s_L1, uint16_t* XL1q,
                           float* s_xl1, int32_t* acc_out, uint32_t* status,
                           cudaStream_t stream) {
  QlrParams p{};
  p.s_x = s_x;
  p.s_L1 = s_L1;
  p.XL1q = reinterpret_cast<__nv_bfloat16*>(XL1q);
  p.s_xl1 = s_xl1;
  p.acc_out = acc_out;
  p.status = status;
  p.M = M;
  p.kb_total = K / kKb;
  p.rn = rn;
  p.r_ld = r;
  p.r_off = r_off;
  p.ns = num_stages(rn);
  p.tmem_cols = 32;
  while (p.tmem_cols < (uint32_t)rn) p.tmem_cols <<= 1;
  const int tiles = (M + kTok - 1) / kTok;
  // a cluster of C CTAs along K per 128-token tile: about one CTA per SM;
  // every CTA of the cluster gets at least one k-block
  int C = std::max(1, std::min(std::min(kMaxC, p.kb_total), num_sms() / tiles));
  p.nb = (p.kb_total + C - 1) / C;
  C = (p.kb_total + p.nb - 1) / p.nb;
  const uint32_t smem = smem_bytes(rn) + 1024u;
  if (recv_bytes(rn, C) > (uint32_t)p.ns * stage_bytes(rn)) return cudaErrorInvalidValue;
  static uint64_t attr_set = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set >> dev & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(xl1_codes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)(smem_bytes(kMaxRn) + 1024u));
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  CUtensorMap map_x, map_l1;
  if (!encode_tiled_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_UINT8, Xq8, (uint64_t)K, (uint64_t)M,
                       (uint64_t)K, kKb, kTok, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tiled_2d(&map_l1, CU_TENSOR_MAP_DATA_TYPE_UINT8, qL1, (uint64_t)K, (uint64_t)r,
                       (uint64_t)K, kKb, (uint32_t)rn, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, tiles, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = tuning().pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, xl1_codes_kernel, map_x, map_l1, p);
}

}  // namespace

cudaError_t launch_xl1_codes(const int8_t* Xq8, const int8_t* qL1, const float* s_x,
                             const float* s_L1, int M, int K, int r, uint16_t* XL1q, float* s_xl1,
                             int32_t* acc, uint32_t* status, cudaStream_t stream) {
  if (M <= 0 || K <= 0 || K % kKb != 0 || r <= 0 || r % 16 != 0) return cudaErrorInvalidValue;
  if (r <= kMaxRn)
    return launch_xl1_one(Xq8, qL1, M, K, r, 0, r, s_x, s_L1, XL1q, s_xl1, nullptr, status,
                          stream);
  for (int off = 0; off < r; off += kMaxRn)
    if (cudaError_t e = launch_xl1_one(Xq8, qL1, M, K, r, off, std::min(kMaxRn, r - off), s_x,
                                       s_L1, nullptr, nullptr, acc, status, stream))
      return e;
  return launch_requant_xl1(acc, s_x, s_L1, M, r, XL1q, s_xl1, stream);
}

}  // namespace tq
