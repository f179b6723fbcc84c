// tq_gemm.cu -- the W4A4 + low-rank GEMM on 5th-generation tensor cores.
//
// One CTA computes a 128 x BN output tile (128 = MMA M, the "P" operand;
// BN = MMA N, the "Q" operand), optionally over a slice of K (split-K):
//
//   warp 4  TMA producer: streams packed int4 tiles of P and Q (64 bytes =
//           128 codes per row per k-block) into a staging ring.
//   warps 0-3 converters: expand int4 -> int8 in shared memory, written
//           straight into the 128-byte-swizzled K-major layout tcgen05 reads
//           (tcgen05 has no dense int4 kind).  A nibble n becomes the byte
//           16*n, so both operands are scaled by 16 and the INT32 accumulator
//           holds 256 * sum(qx qw) exactly (|acc| <= 256*49*K < 2^31 for
//           K <= 32768); the epilogue shifts it back.  For the low-rank
//           branch they also stage bf16(XL1) and L2^T chunks (64 wide).
//   warp 5  MMA issuer: tcgen05.mma kind::i8 into an INT32 TMEM accumulator
//           and, for the low-rank chunks, kind::f16 (bf16 in, fp32
//           accumulate) into a second TMEM accumulator.
//   warps 0-3 epilogue: tcgen05.ld both accumulators and compute
//           Y = s_p s_q acc + lr in fp32, store bf16 (TwinQuant's single
//           shared epilogue).  With split-K each CTA publishes its INT32
//           partial; the last CTA of a tile sums them in split order (exact,
//           deterministic) and finishes the tile.
//
// Prefill (M > 128): P = activations (tokens), Q = weights.  Decode
// (M <= 128): operands swapped, P = weights (channels fill the 128 TMEM
// lanes), Q = tokens (BN = 16..128), so the weight stream uses the whole MMA.
//
// No TMA multicast is used anywhere.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdio>

#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

Tuning& tuning() {
  static Tuning t;
  return t;
}

namespace {

constexpr int kBM = 128;         // MMA M
constexpr int kKB = 128;         // codes per k-block (one 128-byte int8 row)
constexpr int kPackedRow = 64;   // packed bytes per row per k-block
constexpr int kLrChunk = 64;     // bf16 columns per low-rank chunk (128 bytes)
constexpr int kEpiThreads = 128;  // warps 0-3: TMEM lanes 0-127, the epilogue

struct GemmParams {
  const float* s_p;
  const float* s_q;
  const float* xl1;               // [M][r] fp32
  const __nv_bfloat16* l2t;       // [N][r] bf16
  int rows_p, rows_q, K, r;
  int kb_total, kb_per_split, splits;
  __nv_bfloat16* Y;
  int ldy;                        // = N
  int32_t* acc_out;               // debug accumulators [M][N] or null
  uint32_t* status;               // device status word
  int use_lr;                     // r > 0 and Y requested
};

constexpr int kKBS = 2;          // k-blocks per TMA stage: 128-byte rows, 128B swizzle
constexpr int kMaxSplits = 8;    // split-K cluster size limit (portable clusters)

template <int BN, int NSTG, int NOPS, bool RECV>
struct SmemLayout {
  static constexpr uint32_t kRowsPQ = kBM + BN;
  static constexpr uint32_t kOpP = kBM * 128;        // int8 / bf16 operand P
  static constexpr uint32_t kOpStage = kRowsPQ * 128;  // P then Q, multiple of 1024
  static constexpr uint32_t kStgP = kBM * 128;       // packed P rows (2 k-blocks each)
  static constexpr uint32_t kStgStage = kRowsPQ * 128;
  static constexpr uint32_t kOpBase = 0;
  static constexpr uint32_t kStgBase = kOpBase + NOPS * kOpStage;
  static constexpr uint32_t kRingEnd = kStgBase + NSTG * kStgStage;
  // split-K receive area: INT32 partials [S][BN][ceil(128/S)] and the
  // low-rank tile [BN][ceil(128/S)] -- (S+1) * BN * ceil(128/S) * 4 bytes,
  // at most 2 * BN * 128 * 4 (S = 1).  Dedicated (RECV) or the freed rings.
  static constexpr uint32_t kRecvBytes = 2u * BN * kBM * 4u;
  static constexpr uint32_t kRecvBase = RECV ? kRingEnd : 0u;
  static constexpr uint32_t kScaleBase = kRingEnd + (RECV ? kRecvBytes : 0u);  // fp32 [128 + BN]
  static constexpr uint32_t kBarBase = kScaleBase + kRowsPQ * 4u;
  // barriers: stg_full, stg_empty, op_full, op_empty, acc_full
  static constexpr uint32_t kNumBars = 2 * NSTG + 2 * NOPS + 1;
  static constexpr uint32_t kMiscBase = kBarBase + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscBase + 32;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-B alignment
  static_assert(kOpStage % 1024 == 0 && kStgStage % 1024 == 0, "1024-B aligned stages");
  static_assert(NOPS >= kKBS, "a staged stage feeds kKBS operand slots");
  // single split (prefill): bf16 tile [128][BN + 8] in the freed rings
  static constexpr uint32_t kYRow = BN * 2 + 16;
  static constexpr uint32_t kYBytes = kBM * kYRow;
};

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ int ld_shared_s32(uint32_t addr) {
  int v;
  asm volatile("ld.shared.s32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ float ld_shared_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void dsmem_st_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void cluster_arrive() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Rows of a 128-row tile owned by split `o` of `S` in the split-K reduction:
// row r belongs to split floor(r * S / 128).
__device__ __forceinline__ int owned_lo(int o, int S) { return (o * kBM + S - 1) / S; }

// Sum of the NACC rotating INT32 accumulators for 16 columns, unscaled
// (each MMA operand carries a factor 16, so the sum is 256 x the codes' dot).
template <int NACC, int BN>
__device__ __forceinline__ void tmem_acc16(uint32_t taddr, int (&out)[16]) {
  uint32_t a[16];
  tmem_ld16(taddr, a);
  if constexpr (NACC == 1) {
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) out[j] = ((int)a[j]) >> 8;
  } else {
    uint32_t b[16];
    tmem_ld16(taddr + BN, b);
    if constexpr (NACC == 4) {
      uint32_t c[16], d[16];
      tmem_ld16(taddr + 2 * BN, c);
      tmem_ld16(taddr + 3 * BN, d);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j)
        out[j] = ((int)a[j] + (int)b[j] + (int)c[j] + (int)d[j]) >> 8;
    } else {
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) out[j] = ((int)a[j] + (int)b[j]) >> 8;
    }
  }
}

// One 128 x BN output tile over k-blocks [split*kb_per_split, ...).  SWAP
// kernels are launched as clusters of `splits` CTAs along z; the CTAs of a
// cluster combine their INT32 partials through distributed shared memory.
// Warps 0..CW-1 convert (warps 0-3 also run the epilogue), warp CW is the TMA
// producer, warp CW+1 allocates TMEM and issues the MMAs.
template <int BN, bool SWAP, int NSTG, int NOPS, int NACC, bool RECV, int CW>
__global__ void __launch_bounds__(32 * (CW + 2), 1)
    w4a4_lr_gemm_kernel(const __grid_constant__ CUtensorMap map_p,
                        const __grid_constant__ CUtensorMap map_q, const GemmParams prm) {
  using L = SmemLayout<BN, NSTG, NOPS, RECV>;
  constexpr int kRows = kBM + BN;
  constexpr int kConvThreads = 32 * CW;
  constexpr int kProducerWarp = CW, kMmaWarp = CW + 1;
  static_assert(CW >= 4, "warps 0-3 own the TMEM lanes of the epilogue");
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarBase);
  uint64_t* stg_full = bars;
  uint64_t* stg_empty = bars + NSTG;
  uint64_t* op_full = bars + 2 * NSTG;
  uint64_t* op_empty = bars + 2 * NSTG + NOPS;
  uint64_t* acc_full = bars + 2 * NSTG + 2 * NOPS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMiscBase);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMiscBase + 4);
  float* sc = reinterpret_cast<float*>(smem + L::kScaleBase);  // s_p [128], s_q [BN]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile_p = blockIdx.x, tile_q = blockIdx.y, split = blockIdx.z;
  const int kb0 = split * prm.kb_per_split;
  const int n_kb = min(prm.kb_total - kb0, prm.kb_per_split);
  const int n_st = (n_kb + kKBS - 1) / kKBS;       // staged (TMA) stages
  const bool do_lr = prm.use_lr && split == 0;
  const int n_lr = do_lr ? (prm.r + kLrChunk - 1) / kLrChunk : 0;
  const int n_ops = n_lr + n_kb;                   // operand stages: low-rank first
  constexpr uint32_t kCols = NACC * BN + BN;
  constexpr uint32_t kTmemCols = kCols <= 32 ? 32 : kCols <= 64 ? 64 : kCols <= 128 ? 128
                                 : kCols <= 256 ? 256 : 512;
  const int pre = min(n_st, NSTG);

  // Warp 4, lane 0 initialises the barriers and immediately starts streaming
  // the first NSTG stages of weights, which do not depend on the preceding
  // kernel (programmatic dependent launch), while warp 5 allocates TMEM.
  if (warp == kProducerWarp && lane == 0) {
    for (int i = 0; i < NSTG; ++i) {
      mbar_init(&stg_full[i], 1);
      mbar_init(&stg_empty[i], kConvThreads);
    }
    for (int i = 0; i < NOPS; ++i) {
      mbar_init(&op_full[i], kConvThreads);
      mbar_init(&op_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(SWAP ? &map_p : &map_q);
    const uint64_t pol_w = policy_evict_first();
    for (int i = 0; i < pre; ++i) {
      uint8_t* sp = smem + L::kStgBase + i * L::kStgStage;
      mbar_arrive_expect_tx(&stg_full[i], L::kStgStage);
      const int x = (kb0 + i * kKBS) * kPackedRow;
      if (SWAP)
        tma_load_2d(sp, &map_p, &stg_full[i], x, tile_p * kBM, pol_w);
      else
        tma_load_2d(sp + L::kStgP, &map_q, &stg_full[i], x, tile_q * BN, pol_w);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  // split-K clusters with a dedicated receive area: announce this CTA now;
  // the epilogue waits for every peer before its first remote store
  if constexpr (SWAP && RECV) cluster_arrive_relaxed();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_lr = tmem_base + NACC * BN;  // fp32, BN columns
  constexpr int kScPer = (kRows + kEpiThreads - 1) / kEpiThreads;
  float sc_reg[kScPer];
#pragma unroll
  for (int u = 0; u < kScPer; ++u) sc_reg[u] = 0.f;

  if (warp == kProducerWarp) {
    // ------------------------------------------------------ TMA producer
    const uint64_t pol_w = policy_evict_first();
    const uint64_t pol_a = policy_evict_last();
    if (lane == 0) {
      pdl_wait();  // activations come from the preceding kernel
      for (int i = 0; i < pre; ++i) {
        uint8_t* sp = smem + L::kStgBase + i * L::kStgStage;
        const int x = (kb0 + i * kKBS) * kPackedRow;
        if (SWAP)
          tma_load_2d(sp + L::kStgP, &map_q, &stg_full[i], x, tile_q * BN, pol_a);
        else
          tma_load_2d(sp, &map_p, &stg_full[i], x, tile_p * kBM, pol_a);
      }
    }
    __syncwarp();
    for (int i = pre; i < n_st; ++i) {
      const int s = i % NSTG;
      const uint32_t ph = (uint32_t)(i / NSTG) & 1u;
      if (!mbar_wait(&stg_empty[s], ph ^ 1u, prm.status, abort_flag)) break;
      if (lane == 0) {
        uint8_t* sp = smem + L::kStgBase + s * L::kStgStage;
        mbar_arrive_expect_tx(&stg_full[s], L::kStgStage);
        const int x = (kb0 + i * kKBS) * kPackedRow;
        tma_load_2d(sp, &map_p, &stg_full[s], x, tile_p * kBM, SWAP ? pol_w : pol_a);
        tma_load_2d(sp + L::kStgP, &map_q, &stg_full[s], x, tile_q * BN, SWAP ? pol_a : pol_w);
      }
      __syncwarp();
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------- MMA issuer
    const uint32_t id_i8 = idesc_i8_s32(BN);
    const uint32_t id_bf = idesc_bf16_f32(BN);
    for (int i = 0; i < n_ops; ++i) {
      const int s = i % NOPS;
      const uint32_t ph = (uint32_t)(i / NOPS) & 1u;
      if (!mbar_wait(&op_full[s], ph, prm.status, abort_flag)) break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t a_addr = base + L::kOpBase + s * L::kOpStage;
        const uint64_t da = sdesc_sw128(a_addr);
        const uint64_t db = sdesc_sw128(a_addr + L::kOpP);
        if (i >= n_lr) {
          const int kbi = i - n_lr;
          // 4 x K=32 int8 per 128-byte row, rotating over NACC accumulators
          // so that consecutive small-N MMAs do not wait on each other
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(tmem_base + (kk % NACC) * BN, da + 2 * kk, db + 2 * kk, id_i8,
                   (kbi > 0 || kk >= NACC) ? 1u : 0u);
        } else {
          const int nk = min(kLrChunk, prm.r - i * kLrChunk) / 16;
          for (int kk = 0; kk < nk; ++kk)  // K=16 bf16 = 32 bytes per step
            mma_bf16(tmem_lr, da + 2 * kk, db + 2 * kk, id_bf, (i > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&op_empty[s]);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(acc_full);
    __syncwarp();
  } else {
    // ---------------------------------------------------------- converters
    const int tid = threadIdx.x;  // 0..kConvThreads-1
    pdl_wait();
    // scales of this tile's rows and columns, for the epilogue: loaded now,
    // stored to shared memory after the main loop (the load latency hides
    // under the weight stream)
#pragma unroll
    for (int u = 0; u < kScPer; ++u) {
      const int i = tid + u * kEpiThreads;
      float v = 0.f;
      if (!prm.acc_out && i < kRows && tid < kEpiThreads) {
        if (i < kBM) {
          const int g = tile_p * kBM + i;
          if (g < prm.rows_p) v = __ldg(prm.s_p + g);
        } else {
          const int g = tile_q * BN + (i - kBM);
          if (g < prm.rows_q) v = __ldg(prm.s_q + g);
        }
      }
      sc_reg[u] = v;
    }
    bool alive = true;
    // low-rank chunks first; each thread issues all its global loads before
    // any of its shared-memory stores
    for (int i = 0; i < n_lr && alive; ++i) {
      const int s = i % NOPS;
      if (!mbar_wait(&op_empty[s], ((uint32_t)(i / NOPS) & 1u) ^ 1u, prm.status, abort_flag)) {
        alive = false;
        break;
      }
      const uint32_t op_p = base + L::kOpBase + s * L::kOpStage;
      constexpr int kPer = (kRows * 8 + kConvThreads - 1) / kConvThreads;
      constexpr int kBatch = 8;
      for (int b0 = 0; b0 < kPer; b0 += kBatch) {
        uint4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int c = tid + (b0 + u) * kConvThreads;
          v[u] = make_uint4(0u, 0u, 0u, 0u);
          if (b0 + u < kPer && c < kRows * 8) {
            const int row = c >> 3, jj = c & 7;
            const bool on_p = row < kBM;
            const int rr = on_p ? row : row - kBM;
            const int g_row = on_p ? tile_p * kBM + rr : tile_q * BN + rr;
            const int g_lim = on_p ? prm.rows_p : prm.rows_q;
            const int col0 = i * kLrChunk + jj * 8;
            if (g_row < g_lim && col0 < prm.r) {
              if (on_p != SWAP) {  // XL1 (fp32) sits on the token side
                const float4* src =
                    reinterpret_cast<const float4*>(prm.xl1 + (size_t)g_row * prm.r + col0);
                const float4 a = __ldg(src), b = __ldg(src + 1);
                v[u] = make_uint4(pack_bf16x2(a.x, a.y), pack_bf16x2(a.z, a.w),
                                  pack_bf16x2(b.x, b.y), pack_bf16x2(b.z, b.w));
              } else {
                v[u] = __ldg(reinterpret_cast<const uint4*>(prm.l2t + (size_t)g_row * prm.r + col0));
              }
            }
          }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int c = tid + (b0 + u) * kConvThreads;
          if (b0 + u < kPer && c < kRows * 8) {
            const int row = c >> 3, jj = c & 7;
            // P rows then Q rows: one operand stage is laid out as rows 0..127
            // of P followed by the BN rows of Q, each 128-byte swizzled
            st_shared_v4(op_p + sw128_offset((uint32_t)row, (uint32_t)jj), v[u]);
          }
        }
      }
      fence_proxy_async_smem();
      mbar_arrive(&op_full[s]);
    }
    // int4 -> int8: a thread expands one 128-code row segment (64 packed
    // bytes, 4 swizzled chunks of the staged row) into the 8 chunks of the
    // operand row, 16 * code per byte.  One k-block (one operand slot) at a
    // time, so the expansion of k-block i+1 overlaps the MMAs of k-block i.
    for (int st = 0; st < n_st && alive; ++st) {
      const int sg_slot = st % NSTG;
      if (!mbar_wait(&stg_full[sg_slot], (uint32_t)(st / NSTG) & 1u, prm.status, abort_flag)) break;
      const int nsub = min(kKBS, n_kb - st * kKBS);
      const uint32_t sg = base + L::kStgBase + sg_slot * L::kStgStage;
      for (int sub = 0; sub < nsub; ++sub) {
        const int i = n_lr + st * kKBS + sub;
        if (!mbar_wait(&op_empty[i % NOPS], ((uint32_t)(i / NOPS) & 1u) ^ 1u, prm.status,
                       abort_flag)) {
          alive = false;
          break;
        }
        const uint32_t dst0 = base + L::kOpBase + (uint32_t)(i % NOPS) * L::kOpStage;
        for (int row = tid; row < kRows; row += kConvThreads) {
          const uint32_t x7 = (uint32_t)row & 7u;
          const uint32_t src = sg + (uint32_t)row * 128u;
          uint4 w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w[q] = ld_shared_v4(src + (((uint32_t)(sub * 4 + q) ^ x7) << 4));
          const uint32_t dst = dst0 + (uint32_t)row * 128u;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 lo, hi;
            lo.x = (w[q].x << 4) & 0xF0F0F0F0u;
            lo.y = (w[q].y << 4) & 0xF0F0F0F0u;
            lo.z = (w[q].z << 4) & 0xF0F0F0F0u;
            lo.w = (w[q].w << 4) & 0xF0F0F0F0u;
            hi.x = w[q].x & 0xF0F0F0F0u;
            hi.y = w[q].y & 0xF0F0F0F0u;
            hi.z = w[q].z & 0xF0F0F0F0u;
            hi.w = w[q].w & 0xF0F0F0F0u;
            st_shared_v4(dst + (((uint32_t)(2 * q) ^ x7) << 4), lo);
            st_shared_v4(dst + (((uint32_t)(2 * q + 1) ^ x7) << 4), hi);
          }
        }
        fence_proxy_async_smem();
        mbar_arrive(&op_full[i % NOPS]);
      }
      if (!alive) break;
      mbar_arrive(&stg_empty[sg_slot]);
    }
  }

  // -------------------------------------------------------------- epilogue
  // Warps 0-3 read TMEM (warp w owns lanes 32w..32w+31 = tile rows).
  const bool is_epi = warp < 4;
  const int row = warp * 32 + lane;
  const int gp = tile_p * kBM + row;
  const uint32_t t_row = (uint32_t)(warp * 32) << 16;
  bool ok = true;
  if (is_epi) {
#pragma unroll
    for (int u = 0; u < kScPer; ++u)
      if (threadIdx.x + u * kEpiThreads < kRows) sc[threadIdx.x + u * kEpiThreads] = sc_reg[u];
    named_bar_sync(2, kEpiThreads);  // scales visible to every epilogue thread
    ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0u, prm.status, abort_flag));
    tc_fence_after();
  }

  if constexpr (SWAP) {
    // Split-K over the cluster: row r of the tile belongs to split
    // r * S / 128; every split pushes its INT32 partial rows (and split 0 its
    // low-rank rows) into the owner's shared memory with remote stores, then
    // each owner reduces its rows in split order (exact, deterministic).
    static_assert(RECV || L::kRecvBytes <= L::kRingEnd, "split-K partials must fit in the rings");
    const int S = prm.splits;
    const int owner = (row * S) >> 7;
    const int lo_o = owned_lo(owner, S);
    const int rows_max = (kBM + S - 1) / S;
    const uint32_t owner_base = dsmem_map(base + L::kRecvBase, (uint32_t)owner);
    const uint32_t dst_i = owner_base + (uint32_t)((split * BN * rows_max + (row - lo_o)) * 4);
    const uint32_t dst_f = owner_base + (uint32_t)((S * BN * rows_max + (row - lo_o)) * 4);
    if constexpr (!RECV) cluster_arrive();  // this CTA's rings are free now
    auto push16 = [&](int cb) {
      int acc[16];
      tmem_acc16<NACC, BN>(tmem_base + t_row + cb, acc);
      uint32_t af[16];
      if (do_lr) {
        tmem_ld16(tmem_lr + t_row + cb, af);
        tmem_ld_wait();
      }
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        dsmem_st_u32(dst_i + (uint32_t)((cb + j) * rows_max * 4), (uint32_t)acc[j]);
        if (do_lr) dsmem_st_u32(dst_f + (uint32_t)((cb + j) * rows_max * 4), af[j]);
      }
    };
    cluster_wait();  // every peer is running (RECV) / has freed its rings (!RECV)
    if (is_epi && ok) {
      for (int cb = 0; cb < BN; cb += 16) push16(cb);
    }
    cluster_sync();    // all partials delivered
    if (is_epi && !*abort_flag) {
      const int me = split;
      const int lo_m = owned_lo(me, S);
      const int rows_m = owned_lo(me + 1, S) - lo_m;
      const uint32_t red_i = base + L::kRecvBase;                       // int [S][BN][rows_max]
      const uint32_t red_f = red_i + (uint32_t)(S * BN * rows_max) * 4u;  // fp32 [BN][rows_max]
      const uint32_t scs = smem_u32(sc);
      for (int idx = threadIdx.x; idx < BN * rows_m; idx += kEpiThreads) {
        const int col = idx / rows_m, rr = idx - col * rows_m;
        const int g_p = tile_p * kBM + lo_m + rr, g_q = tile_q * BN + col;
        // all shared-memory loads of this element first, then the sums
        int part[kMaxSplits];
#pragma unroll
        for (int z = 0; z < kMaxSplits; ++z)
          part[z] = z < S ? ld_shared_s32(red_i + (uint32_t)(((z * BN + col) * rows_max + rr) * 4))
                          : 0;
        const float s_p = ld_shared_f32(scs + (uint32_t)(lo_m + rr) * 4u);
        const float s_q = ld_shared_f32(scs + (uint32_t)(kBM + col) * 4u);
        const float lr = prm.use_lr ? ld_shared_f32(red_f + (uint32_t)((col * rows_max + rr) * 4)) : 0.f;
        if (g_p >= prm.rows_p || g_q >= prm.rows_q) continue;
        int acc = 0;
#pragma unroll
        for (int z = 0; z < kMaxSplits; ++z) acc += part[z];  // split order
        // out[m][n] with m = token (Q side), n = channel (P side)
        if (prm.acc_out) {
          prm.acc_out[(size_t)g_q * prm.ldy + g_p] = acc;
        } else {
          prm.Y[(size_t)g_q * prm.ldy + g_p] = __float2bfloat16_rn(s_p * s_q * (float)acc + lr);
        }
      }
    }
  } else {
    static_assert(L::kYBytes <= L::kRingEnd, "the bf16 output tile must fit in the rings");
    if (is_epi && ok) {
      if (prm.acc_out) {
        for (int cb = 0; cb < BN; cb += 16) {
          int acc[16];
          tmem_acc16<NACC, BN>(tmem_base + t_row + cb, acc);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int gq = tile_q * BN + cb + j;
            if (gp < prm.rows_p && gq < prm.rows_q) prm.acc_out[(size_t)gp * prm.ldy + gq] = acc[j];
          }
        }
      } else {
        // y = s_x s_w acc + lr in fp32 -> bf16 tile in shared memory, then
        // coalesced 16-byte stores of whole rows.
        const float sp = sc[row];
        const uint32_t ys = base + (uint32_t)row * L::kYRow;
        for (int cb = 0; cb < BN; cb += 16) {
          int acc[16];
          tmem_acc16<NACC, BN>(tmem_base + t_row + cb, acc);
          uint32_t af[16];
          if (do_lr) {
            tmem_ld16(tmem_lr + t_row + cb, af);
            tmem_ld_wait();
          }
          uint32_t pk[8];
#pragma unroll
          for (int j = 0; j < 16; j += 2) {
            float y0 = sp * sc[kBM + cb + j] * (float)acc[j];
            float y1 = sp * sc[kBM + cb + j + 1] * (float)acc[j + 1];
            if (do_lr) {
              y0 += __uint_as_float(af[j]);
              y1 += __uint_as_float(af[j + 1]);
            }
            pk[j / 2] = pack_bf16x2(y0, y1);
          }
          st_shared_v4(ys + cb * 2, make_uint4(pk[0], pk[1], pk[2], pk[3]));
          st_shared_v4(ys + cb * 2 + 16, make_uint4(pk[4], pk[5], pk[6], pk[7]));
        }
        named_bar_sync(1, kEpiThreads);
        constexpr int kChunksPerRow = BN / 8;
        for (int c = threadIdx.x; c < kBM * kChunksPerRow; c += kEpiThreads) {
          const int rr = c / kChunksPerRow, cc = c % kChunksPerRow;
          const int g_p = tile_p * kBM + rr, g_q = tile_q * BN + cc * 8;
          if (g_p >= prm.rows_p || g_q >= prm.rows_q) continue;  // N % 8 == 0
          const uint4 v = ld_shared_v4(base + (uint32_t)rr * L::kYRow + cc * 16);
          *reinterpret_cast<uint4*>(prm.Y + (size_t)g_p * prm.ldy + g_q) = v;
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// ------------------------------------------------------------------ host

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Packed int4 matrix [rows][K/2] bytes, box = 128 bytes (two k-blocks) x box_rows,
// landing 128-byte swizzled in shared memory.
bool make_packed_map(CUtensorMap* m, const uint8_t* ptr, int rows, int K, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {(cuuint32_t)(kPackedRow * kKBS), (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct Plan {
  bool swap;
  int bn;
  int splits;
  int kb_per_split;
  int tiles_p, tiles_q;
};

int num_sms_cached() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}


Plan make_plan(int M, int N, int K) {
  Plan p{};
  const int kb = K / kKB;
  if (M <= 128) {
    // Decode: weights on the MMA M side, split K over a cluster so that about
    // one CTA per SM streams weights.
    p.swap = true;
    p.bn = M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
    p.tiles_p = (N + kBM - 1) / kBM;
    p.tiles_q = (M + p.bn - 1) / p.bn;
    int s = tuning().split_k;
    if (s <= 0) s = std::max(1, num_sms_cached() / (p.tiles_p * p.tiles_q));
    s = std::max(1, std::min(std::min(s, kb), kMaxSplits));
    p.kb_per_split = (kb + s - 1) / s;
    // whole staged stages per split when that keeps the split count
    const int kbs = kKBS;
    const int rounded = (p.kb_per_split + kbs - 1) / kbs * kbs;
    if ((kb + rounded - 1) / rounded == (kb + p.kb_per_split - 1) / p.kb_per_split)
      p.kb_per_split = rounded;
    p.splits = (kb + p.kb_per_split - 1) / p.kb_per_split;
  } else {
    p.swap = false;
    p.bn = 256;
    p.tiles_p = (M + kBM - 1) / kBM;
    p.tiles_q = (N + p.bn - 1) / p.bn;
    p.splits = 1;
    p.kb_per_split = kb;
  }
  return p;
}

template <int BN, bool SWAP, int NSTG, int NOPS, int NACC, bool RECV, int CW>
cudaError_t launch_variant(const GemmArgs& a, const Plan& pl, const GemmParams& prm,
                           cudaStream_t stream) {
  using L = SmemLayout<BN, NSTG, NOPS, RECV>;
  CUtensorMap map_p, map_q;
  const uint8_t* P = SWAP ? a.Wq : a.Xq;
  const uint8_t* Q = SWAP ? a.Xq : a.Wq;
  if (!make_packed_map(&map_p, P, prm.rows_p, a.K, kBM)) return cudaErrorInvalidValue;
  if (!make_packed_map(&map_q, Q, prm.rows_q, a.K, BN)) return cudaErrorInvalidValue;
  auto kern = w4a4_lr_gemm_kernel<BN, SWAP, NSTG, NOPS, NACC, RECV, CW>;
  static uint64_t attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set >> dev & 1u)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.tiles_p, pl.tiles_q, pl.splits);
  cfg.blockDim = dim3(32 * (CW + 2), 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = tuning().pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = SWAP ? pl.splits : 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, map_p, map_q, prm);
}

}  // namespace

int num_sms() { return num_sms_cached(); }

bool encode_tiled_2d(CUtensorMap* m, CUtensorMapDataType dtype, const void* ptr, uint64_t inner,
                     uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                     CUtensorMapSwizzle swizzle) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dtype, 2, const_cast<void*>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

size_t gemm_workspace_bytes(int M, int N, int K, int r) {
  (void)M; (void)N; (void)K; (void)r;
  return 256;  // the device status word (split-K partials live in shared memory)
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t stream) {
  const bool debug = a.acc_out != nullptr;
  const Plan pl = make_plan(a.M, a.N, a.K);
  if (a.ws_bytes < gemm_workspace_bytes(a.M, a.N, a.K, a.r)) return cudaErrorInvalidValue;
  GemmParams prm{};
  prm.s_p = pl.swap ? a.s_w : a.s_x;
  prm.s_q = pl.swap ? a.s_x : a.s_w;
  prm.xl1 = a.XL1;
  prm.l2t = reinterpret_cast<const __nv_bfloat16*>(a.L2t);
  prm.rows_p = pl.swap ? a.N : a.M;
  prm.rows_q = pl.swap ? a.M : a.N;
  prm.K = a.K;
  prm.r = a.r;
  prm.kb_total = a.K / kKB;
  prm.kb_per_split = pl.kb_per_split;
  prm.splits = pl.splits;
  prm.Y = reinterpret_cast<__nv_bfloat16*>(a.Y);
  prm.ldy = a.N;
  prm.acc_out = a.acc_out;
  prm.status = reinterpret_cast<uint32_t*>(a.ws);
  prm.use_lr = (a.r > 0 && !debug) ? 1 : 0;
  //                                BN  SWAP  NSTG NOPS NACC RECV  CW
  if (!pl.swap) return launch_variant<256, false, 2, 2, 1, false, 8>(a, pl, prm, stream);
  switch (pl.bn) {
    case 16: return launch_variant<16, true, 4, 4, 1, true, 8>(a, pl, prm, stream);
    case 32: return launch_variant<32, true, 4, 4, 1, true, 8>(a, pl, prm, stream);
    case 64: return launch_variant<64, true, 4, 4, 1, false, 8>(a, pl, prm, stream);
    default: return launch_variant<128, true, 2, 4, 1, false, 8>(a, pl, prm, stream);
  }
}

}  // namespace tq
