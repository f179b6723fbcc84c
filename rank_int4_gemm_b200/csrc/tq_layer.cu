// tq_layer.cu -- the whole decode layer (M <= 16 tokens) in one kernel.
//
//   Y = dequant( Q4(X H) . Q4(H^T R) ) + bf16(X L1) L2
//
// Per output tile of 128 channels, a cluster of S CTAs splits K (split-K).
// CTA z owns k-blocks [z*kbps, ...) of K.  Its warps:
//
//   warps 0-7   activation: read the tokens' slice of X straight from L2,
//               Sylvester transform (the same warp butterflies as
//               tq_quantize_act, so the codes are the same bits), partial
//               absmax, X.L1 partial on mma.sync; the cluster exchanges
//               absmax and X.L1 partials through distributed shared memory;
//               then the token codes are written as int8 (16 * code) straight
//               into the MMA's B operand.  Warps 0-3 run the epilogue.
//   warps 8-11  expand the streamed int4 weights to int8 operand tiles and,
//               in split 0, stage the L2^T rows of the tile.
//   warp 12     TMA producer of the packed weights (started before the
//               kernel waits on its predecessor: weights never depend on it).
//   warp 13     TMEM allocation and MMA issue: kind::i8 for the codes,
//               kind::f16 for the low-rank branch (split 0).
//
// The epilogue is the split-K reduction of the GEMM kernel: each split pushes
// its INT32 partial rows to the row's owner CTA, owners reduce in split order
// and store Y.  Nothing goes through global memory except X, the weights and
// Y.  No TMA multicast.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "tq_act_common.cuh"
#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

namespace {

constexpr int kBM = 128;           // channels per tile (MMA M)
constexpr int kBN = 16;            // tokens (MMA N)
constexpr int kKB = 128;           // codes per k-block
constexpr int kPackedRow = 64;     // packed bytes per row per k-block
constexpr int kKBS = 2;            // k-blocks per TMA stage (128-byte swizzled rows)
constexpr int kNSTG = 2;           // TMA stages
constexpr int kNOPS = 2;           // int8 operand slots
constexpr int kMaxKb = 8;          // k-blocks per CTA (slice <= 1024 columns)
constexpr int kMaxSplits = 4;     // split-K cluster size limit of this kernel
constexpr int kMaxR = 64;          // low-rank width handled here
constexpr int kE = 16;             // values per lane per warp pass
constexpr int kW = 32 * kE;        // 512 columns per warp pass
constexpr int kL1Chunk = 256;      // L1^T columns per staged chunk
constexpr int kActWarps = 8, kConvWarps = 4;
constexpr int kProducerWarp = 12, kMmaWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr int kActThreads = kActWarps * 32;
constexpr int kConvThreads = kConvWarps * 32;
constexpr int kEpiThreads = 128;

struct LayerParams {
  const __nv_bfloat16* X;    // [M][K]
  const __nv_bfloat16* L1t;  // [r][K]
  const float* s_w;          // [N]
  const __nv_bfloat16* L2t;  // [N][r]
  __nv_bfloat16* Y;          // [M][N]
  uint32_t* status;
  int M, N, K, r, b;
  int kb_total, kb_per_split, splits;
  float scale_mul;           // 1 / (7 sqrt(b))
};

// Shared-memory map (offsets from the 1024-aligned base).
struct Smem {
  static constexpr uint32_t kStg = kBM * 128;                 // one TMA stage
  static constexpr uint32_t kOp = kBM * 128;                  // one int8 weight k-block
  static constexpr uint32_t kStgBase = 0;
  static constexpr uint32_t kOpBase = kStgBase + kNSTG * kStg;  // also the L2^T tile (split 0)
  static constexpr uint32_t kBBase = kOpBase + kNOPS * kOp;   // token codes [kb][16][128]
  static constexpr uint32_t kBBytes = kMaxKb * kBN * 128;
  static constexpr uint32_t kLrBBase = kBBase + kBBytes;      // bf16(XL1) [16][64], SW128
  static constexpr uint32_t kXBase = kLrBBase + kBN * 128;    // X slice [16][1024 + 8] bf16
  static constexpr uint32_t kXStride = kMaxKb * kKB + 8;      // bf16 elements per row
  static constexpr uint32_t kXBytes = kBN * kXStride * 2;
  static constexpr uint32_t kL1Base = kXBase + kXBytes;       // L1^T chunks [4|2][r][256 + 8]
  static constexpr uint32_t kL1Stride = kL1Chunk + 8;         // bf16 elements per row
  static constexpr uint32_t kL1Bytes = 2 * kMaxR * kL1Stride * 2;
  static constexpr uint32_t kXRecv = kL1Base + kL1Bytes;      // XL1 partials [S][16][r] fp32
  static constexpr uint32_t kXRecvBytes = kMaxSplits * kBN * kMaxR * 4;
  static constexpr uint32_t kKRecv = kXRecv + kXRecvBytes;    // split-K [S][16][rows], lr [16][rows]
  static constexpr uint32_t kKRecvBytes = 2 * kBN * kBM * 4;  // largest at S = 1
  static constexpr uint32_t kAmax = kKRecv + kKRecvBytes;     // [S][16] + [16]
  static constexpr uint32_t kScale = kAmax + (kMaxSplits + 1) * kBN * 4;  // s_w [128]
  static constexpr uint32_t kBar = kScale + kBM * 4;
  // barriers: stg_full, stg_empty, op_full, op_empty, b_ready, lr_ready, acc_full
  static constexpr uint32_t kNumBars = 2 * kNSTG + 2 * kNOPS + 3;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kMisc + 32;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};
static_assert(Smem::kAlloc <= 227 * 1024, "fused layer shared memory");

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
__device__ __forceinline__ void dsmem_st_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
__device__ __forceinline__ int owned_lo(int o, int S) { return (o * kBM + S - 1) / S; }

// 16-byte chunk j (0..7) of row `row` of a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw_off(uint32_t row, uint32_t j) {
  return row * 128u + ((j ^ (row & 7u)) << 4);
}

__global__ void __launch_bounds__(kThreads, 1)
    w4a4_lr_layer_decode_kernel(const __grid_constant__ CUtensorMap map_w, const LayerParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  using S_ = Smem;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S_::kBar);
  uint64_t* stg_full = bars;
  uint64_t* stg_empty = bars + kNSTG;
  uint64_t* op_full = bars + 2 * kNSTG;
  uint64_t* op_empty = bars + 2 * kNSTG + kNOPS;
  uint64_t* b_ready = bars + 2 * kNSTG + 2 * kNOPS;
  uint64_t* lr_ready = b_ready + 1;
  uint64_t* acc_full = b_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S_::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S_::kMisc + 4);
  float* amax_all = reinterpret_cast<float*>(smem + S_::kAmax);  // [S][16]
  float* amax_row = amax_all + kMaxSplits * kBN;                  // [16]
  float* sw_tile = reinterpret_cast<float*>(smem + S_::kScale);   // s_w of the tile

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.z;
  const int S = p.splits;
  const int kb0 = split * p.kb_per_split;
  const int n_kb = min(p.kb_total - kb0, p.kb_per_split);
  const int n_st = (n_kb + kKBS - 1) / kKBS;
  const int kbase = kb0 * kKB;           // first column of this CTA's slice
  const int slice = n_kb * kKB;
  const bool do_lr = p.r > 0 && split == 0;
  constexpr uint32_t kTmemCols = 32;     // INT32 [16] + fp32 low-rank [16]

  // ---------------------------------------------------------------- prologue
  if (warp == kProducerWarp && lane == 0) {
    for (int i = 0; i < kNSTG; ++i) {
      mbar_init(&stg_full[i], 1);
      mbar_init(&stg_empty[i], kConvThreads);
    }
    for (int i = 0; i < kNOPS; ++i) {
      mbar_init(&op_full[i], kConvThreads);
      mbar_init(&op_empty[i], 1);
    }
    mbar_init(b_ready, kActThreads);
    mbar_init(lr_ready, kActThreads + kConvThreads);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&map_w);
    const uint64_t pol = policy_evict_first();
    for (int i = 0; i < min(n_st, kNSTG); ++i) {
      mbar_arrive_expect_tx(&stg_full[i], S_::kStg);
      tma_load_2d(smem + S_::kStgBase + i * S_::kStg, &map_w, &stg_full[i],
                  (kb0 + i * kKBS) * kPackedRow, tile * kBM, pol);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  cluster_arrive_relaxed();  // B0: this CTA is running
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_acc = *tmem_slot;
  const uint32_t tmem_lr = tmem_acc + kBN;

  if (warp < kActWarps) {
    // =================================================== activation warps
    const int tid = threadIdx.x;  // 0..255
    // L1^T chunks 0 and 1 of this slice (a weight: needs no predecessor)
    const int n_l1 = (p.r > 0) ? slice / kL1Chunk : 0;
    // chunk buffers of r rows: all chunks of the slice fit when r <= 32
    const int l1_bufs = (p.r <= kMaxR / 2) ? 4 : 2;
    const uint32_t l1_buf_bytes = (uint32_t)p.r * S_::kL1Stride * 2u;
    auto stage_l1 = [&](int ci) {
      const uint32_t dst = base + S_::kL1Base + (uint32_t)(ci % l1_bufs) * l1_buf_bytes;
      const int cpr = kL1Chunk / 8;
      for (int c = tid; c < p.r * cpr; c += kActThreads) {
        const int j = c / cpr, cc = c - j * cpr;
        const __nv_bfloat16* src = p.L1t + (size_t)j * p.K + kbase + ci * kL1Chunk + cc * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                         dst + (uint32_t)(j * S_::kL1Stride + cc * 8) * 2u),
                     "l"(src)
                     : "memory");
      }
      cp_async_commit();
    };
    for (int ci = 0; ci < min(n_l1, l1_bufs); ++ci) stage_l1(ci);
    // scales of the tile's channels (weights: no predecessor)
    for (int i = tid; i < kBM; i += kActThreads) {
      const int g = tile * kBM + i;
      sw_tile[i] = g < p.N ? __ldg(p.s_w + g) : 0.f;
    }

    pdl_wait();  // X comes from the preceding kernel

    // ---- X slice [16][slice] -> shared memory (rows past M are zero)
    __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem + S_::kXBase);
    {
      const int cpr = slice / 8;  // 16-byte chunks per row
      for (int c = tid; c < kBN * cpr; c += kActThreads) {
        const int row = c / cpr, cc = c - row * cpr;
        const bool ok = row < p.M;
        const __nv_bfloat16* src = p.X + (size_t)(ok ? row : 0) * p.K + kbase + cc * 8;
        cp_async16(xs + (size_t)row * S_::kXStride + cc * 8, src, ok);
      }
      cp_async_commit();
      cp_async_wait<0>();  // also completes the L1^T chunks staged above
      named_bar_sync(3, kActThreads);
    }

    // ---- transform of tokens warp and warp + 8 over this slice; values kept
    const int np = slice / kW;  // 1 or 2 passes of 512 columns
    float v[2][2][kE];
    float amax[2] = {0.f, 0.f};
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int row = warp + 8 * t;
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        if (ps < np) {
          load_row_values<kE>(xs + (size_t)row * S_::kXStride + ps * kW + lane * kE, v[t][ps]);
          fwht_warp<kE>(v[t][ps], p.b);
#pragma unroll
          for (int i = 0; i < kE; ++i) amax[t] = fmaxf(amax[t], fabsf(v[t][ps][i]));
        }
      }
      amax[t] = warp_max(amax[t]);
    }
    cluster_wait_acquire();  // B0 complete: every peer is running
    if (lane < S) {
      dsmem_st_f32(dsmem_map(smem_u32(&amax_all[split * kBN + warp]), (uint32_t)lane), amax[0]);
      dsmem_st_f32(dsmem_map(smem_u32(&amax_all[split * kBN + warp + 8]), (uint32_t)lane),
                   amax[1]);
    }

    // ---- X L1 partial over the slice: warp w takes k16-steps w, w+8, ...;
    //      A fragments (tokens x k) straight from global, B from L1^T chunks
    if (n_l1 > 0) {
      const int ntiles = p.r / 8;
      float acc[kMaxR / 8][4];
#pragma unroll
      for (int t = 0; t < kMaxR / 8; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
      const int r0 = lane >> 2, c0 = 2 * (lane & 3);
      // warp w owns k16-steps w and w + 8 of every 256-column chunk
      const uint32_t xs_base = smem_u32(xs);
      for (int ci = 0; ci < n_l1; ci += 2) {
        if (l1_bufs == 2) {
          cp_async_wait<0>();
          named_bar_sync(3, kActThreads);
        }
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          if (ci + cc < n_l1) {
            const uint32_t l1b = base + S_::kL1Base + (uint32_t)((ci + cc) % l1_bufs) * l1_buf_bytes;
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
              const int ks = warp + 8 * k2;
              uint32_t a[4];
              {
                const int mat = lane >> 3, rin = lane & 7;
                const int rr = rin + (mat & 1) * 8;
                const int col = (ci + cc) * kL1Chunk + ks * 16 + (mat >> 1) * 8;
                ldmatrix_x4(a, xs_base + (uint32_t)((rr * S_::kXStride + col) * 2));
              }
#pragma unroll
              for (int t = 0; t < kMaxR / 8; ++t) {
                if (t < ntiles) {
                  uint32_t bb[2];
                  const int l = lane & 15;
                  const int jr = t * 8 + (l & 7);
                  const int c2 = ks * 16 + (l >> 3) * 8;
                  ldmatrix_x2(bb, l1b + (uint32_t)((jr * S_::kL1Stride + c2) * 2));
                  mma_16816(acc[t], a, bb);
                }
              }
            }
          }
        }
        if (l1_bufs == 2 && ci + 2 < n_l1) {
          named_bar_sync(3, kActThreads);  // both buffers consumed
          stage_l1(ci + 2);
          if (ci + 3 < n_l1) stage_l1(ci + 3);
        }
      }
      // cross-warp sum in a fixed order through the (still unused) token-code
      // area: warps 0-3 write, warps 4-7 add, then warp pairs are summed
      float* red = reinterpret_cast<float*>(smem + S_::kBBase);  // [4][16][r]
      if (warp < 4) {
#pragma unroll
        for (int t = 0; t < kMaxR / 8; ++t)
          if (t < ntiles) {
            float* d = red + (warp * kBN) * p.r;
            d[r0 * p.r + t * 8 + c0] = acc[t][0];
            d[r0 * p.r + t * 8 + c0 + 1] = acc[t][1];
            d[(r0 + 8) * p.r + t * 8 + c0] = acc[t][2];
            d[(r0 + 8) * p.r + t * 8 + c0 + 1] = acc[t][3];
          }
      }
      named_bar_sync(3, kActThreads);
      if (warp >= 4) {
#pragma unroll
        for (int t = 0; t < kMaxR / 8; ++t)
          if (t < ntiles) {
            float* d = red + ((warp - 4) * kBN) * p.r;
            d[r0 * p.r + t * 8 + c0] += acc[t][0];
            d[r0 * p.r + t * 8 + c0 + 1] += acc[t][1];
            d[(r0 + 8) * p.r + t * 8 + c0] += acc[t][2];
            d[(r0 + 8) * p.r + t * 8 + c0 + 1] += acc[t][3];
          }
      }
      named_bar_sync(3, kActThreads);
      // this CTA's partial [16][r] -> split 0's receive area, slot `split`
      const uint32_t dst0 = dsmem_map(base + S_::kXRecv, 0u);
      for (int idx = tid; idx < kBN * p.r; idx += kActThreads) {
        const float s4 = (red[idx] + red[kBN * p.r + idx]) + (red[2 * kBN * p.r + idx] + red[3 * kBN * p.r + idx]);
        dsmem_st_f32(dst0 + (uint32_t)((split * kBN * p.r + idx) * 4), s4);
      }
    }

    cluster_arrive_release();  // B1: absmax and X L1 partials delivered
    cluster_wait_acquire();

    // ---- token absmax, then the codes of this slice as int8 B operand
    if (tid < kBN) {
      float m = 0.f;
      for (int c = 0; c < S; ++c) m = fmaxf(m, amax_all[c * kBN + tid]);
      amax_row[tid] = m;
    }
    named_bar_sync(3, kActThreads);
#pragma unroll
    for (int t = 0; t < 2; ++t) {
      const int row = warp + 8 * t;
      const float am = amax_row[row];
      const float inv = am > 0.f ? 7.f / am : 0.f;
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        if (ps < np) {
          // this lane's 16 codes = one 16-byte chunk of the operand row
          uint32_t w4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint32_t wv = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
              wv |= ((uint32_t)(quant_code(v[t][ps][4 * q + j], inv) << 4) & 0xFFu) << (8 * j);
            w4[q] = wv;
          }
          const int col = ps * kW + lane * kE;  // within the slice
          const int kb = col / kKB, j = (col % kKB) / 16;
          st_shared_v4(base + S_::kBBase + (uint32_t)(kb * kBN * 128) + sw_off((uint32_t)row, (uint32_t)j),
                       make_uint4(w4[0], w4[1], w4[2], w4[3]));
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(b_ready);

    // ---- split 0: X L1 = sum of the splits' partials (split order), bf16
    //      into the low-rank B operand
    if (do_lr) {
      const uint32_t xr = base + S_::kXRecv;
      for (int c = tid; c < kBN * 8; c += kActThreads) {  // 16 rows x 8 chunks
        const int row = c >> 3, j = c & 7;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
        if (j * 8 < p.r) {
          for (int z = 0; z < S; ++z)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] += ld_shared_f32(xr + (uint32_t)(((z * kBN + row) * p.r + j * 8 + e) * 4));
        }
        st_shared_v4(base + S_::kLrBBase + sw_off((uint32_t)row, (uint32_t)j),
                     make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
      }
      fence_proxy_async_smem();
    }
    if (p.r > 0) mbar_arrive(lr_ready);
  } else if (warp < kActWarps + kConvWarps) {
    // ==================================================== weight converters
    const int tid = threadIdx.x - kActThreads;  // 0..127
    cluster_wait_acquire();    // B0
    cluster_arrive_release();  // B1 (nothing to publish from these warps)
    bool alive = true;
    for (int st = 0; st < n_st && alive; ++st) {
      const int sg_slot = st % kNSTG;
      if (!mbar_wait(&stg_full[sg_slot], (uint32_t)(st / kNSTG) & 1u, p.status, abort_flag)) break;
      const int nsub = min(kKBS, n_kb - st * kKBS);
      const uint32_t sg = base + S_::kStgBase + sg_slot * S_::kStg;
      for (int sub = 0; sub < nsub; ++sub) {
        const int i = st * kKBS + sub;
        if (!mbar_wait(&op_empty[i % kNOPS], ((uint32_t)(i / kNOPS) & 1u) ^ 1u, p.status,
                       abort_flag)) {
          alive = false;
          break;
        }
        const uint32_t dst0 = base + S_::kOpBase + (uint32_t)(i % kNOPS) * S_::kOp;
        for (int row = tid; row < kBM; row += kConvThreads) {
          const uint32_t x7 = (uint32_t)row & 7u;
          const uint32_t src = sg + (uint32_t)row * 128u;
          uint4 w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) w[q] = ld_shared_v4(src + (((uint32_t)(sub * 4 + q) ^ x7) << 4));
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
        mbar_arrive(&op_full[i % kNOPS]);
      }
      if (!alive) break;
      mbar_arrive(&stg_empty[sg_slot]);
    }
    // split 0: the tile's L2^T rows [128][r] bf16 -> the next operand slot,
    // the A operand of the low-rank MMA
    if (alive && do_lr) {
      const int i = n_kb;
      if (mbar_wait(&op_empty[i % kNOPS], ((uint32_t)(i / kNOPS) & 1u) ^ 1u, p.status, abort_flag)) {
        const uint32_t dst0 = base + S_::kOpBase + (uint32_t)(i % kNOPS) * S_::kOp;
        for (int c = tid; c < kBM * 8; c += kConvThreads) {
          const int row = c >> 3, j = c & 7;
          const int g = tile * kBM + row;
          uint4 val = make_uint4(0u, 0u, 0u, 0u);
          if (g < p.N && j * 8 < p.r)
            val = __ldg(reinterpret_cast<const uint4*>(p.L2t + (size_t)g * p.r + j * 8));
          st_shared_v4(dst0 + sw_off((uint32_t)row, (uint32_t)j), val);
        }
        fence_proxy_async_smem();
      }
    }
    if (p.r > 0) mbar_arrive(lr_ready);
    cluster_wait_acquire();
  } else if (warp == kProducerWarp) {
    // =========================================================== producer
    cluster_wait_acquire();    // B0
    cluster_arrive_release();  // B1
    const uint64_t pol = policy_evict_first();
    for (int i = kNSTG; i < n_st; ++i) {
      const int s = i % kNSTG;
      if (!mbar_wait(&stg_empty[s], ((uint32_t)(i / kNSTG) & 1u) ^ 1u, p.status, abort_flag)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&stg_full[s], S_::kStg);
        tma_load_2d(smem + S_::kStgBase + s * S_::kStg, &map_w, &stg_full[s],
                    (kb0 + i * kKBS) * kPackedRow, tile * kBM, pol);
      }
      __syncwarp();
    }
    cluster_wait_acquire();
  } else {
    // ========================================================== MMA issuer
    cluster_wait_acquire();    // B0
    cluster_arrive_release();  // B1
    const uint32_t id_i8 = idesc_i8_s32(kBN);
    const uint32_t id_bf = idesc_bf16_f32(kBN);
    bool alive = mbar_wait(b_ready, 0u, p.status, abort_flag);
    for (int i = 0; i < n_kb && alive; ++i) {
      const int s = i % kNOPS;
      if (!mbar_wait(&op_full[s], (uint32_t)(i / kNOPS) & 1u, p.status, abort_flag)) {
        alive = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        const uint64_t da = sdesc_sw128(base + S_::kOpBase + s * S_::kOp);
        const uint64_t db = sdesc_sw128(base + S_::kBBase + (uint32_t)(i * kBN * 128));
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          mma_i8(tmem_acc, da + 2 * kk, db + 2 * kk, id_i8, (i > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&op_empty[s]);
      }
      __syncwarp();
    }
    if (alive && do_lr && mbar_wait(lr_ready, 0u, p.status, abort_flag)) {
      tc_fence_after();
      if (lane == 0) {
        const uint64_t da = sdesc_sw128(base + S_::kOpBase + (uint32_t)(n_kb % kNOPS) * S_::kOp);
        const uint64_t db = sdesc_sw128(base + S_::kLrBBase);
        for (int kk = 0; kk < p.r / 16; ++kk)
          mma_bf16(tmem_lr, da + 2 * kk, db + 2 * kk, id_bf, kk > 0 ? 1u : 0u);
      }
      __syncwarp();
    }
    if (lane == 0) mma_commit(acc_full);
    __syncwarp();
    cluster_wait_acquire();
  }

  // ------------------------------------------------------------- epilogue
  // Warps 0-3 read TMEM (warp w owns lanes 32w.. = channel rows of the tile).
  const bool is_epi = warp < 4;
  const int row = warp * 32 + lane;
  const uint32_t t_row = (uint32_t)(warp * 32) << 16;
  const int owner = (row * S) >> 7;
  const int lo_o = owned_lo(owner, S);
  const int rows_max = (kBM + S - 1) / S;
  if (is_epi) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0u, p.status, abort_flag));
    tc_fence_after();
    if (ok) {
      uint32_t ai[16], af[16];
      tmem_ld16(tmem_acc + t_row, ai);
      if (do_lr) tmem_ld16(tmem_lr + t_row, af);
      tmem_ld_wait();
      const uint32_t ob = dsmem_map(base + S_::kKRecv, (uint32_t)owner);
      const uint32_t dst_i = ob + (uint32_t)((split * kBN * rows_max + (row - lo_o)) * 4);
      const uint32_t dst_f = ob + (uint32_t)((S * kBN * rows_max + (row - lo_o)) * 4);
#pragma unroll
      for (int j = 0; j < kBN; ++j) {
        dsmem_st_u32(dst_i + (uint32_t)(j * rows_max * 4), (uint32_t)(((int)ai[j]) >> 8));
        if (do_lr) dsmem_st_u32(dst_f + (uint32_t)(j * rows_max * 4), af[j]);
      }
    }
  }
  cluster_sync();  // B2: every split's partial rows delivered
  if (is_epi && !*abort_flag) {
    const int lo_m = owned_lo(split, S);
    const int rows_m = owned_lo(split + 1, S) - lo_m;
    const uint32_t red_i = base + S_::kKRecv;
    const uint32_t red_f = red_i + (uint32_t)(S * kBN * rows_max) * 4u;
    for (int idx = threadIdx.x; idx < kBN * rows_m; idx += kEpiThreads) {
      const int col = idx / rows_m, rr = idx - col * rows_m;  // col = token
      const int g_n = tile * kBM + lo_m + rr;
      int part[kMaxSplits];
#pragma unroll
      for (int z = 0; z < kMaxSplits; ++z)
        part[z] = z < S ? ld_shared_s32(red_i + (uint32_t)(((z * kBN + col) * rows_max + rr) * 4)) : 0;
      const float lr = p.r > 0 ? ld_shared_f32(red_f + (uint32_t)((col * rows_max + rr) * 4)) : 0.f;
      if (col >= p.M || g_n >= p.N) continue;
      int acc = 0;
#pragma unroll
      for (int z = 0; z < kMaxSplits; ++z) acc += part[z];  // split order
      const float s_x = amax_row[col] * p.scale_mul;
      p.Y[(size_t)col * p.N + g_n] = __float2bfloat16_rn(s_x * sw_tile[lo_m + rr] * (float)acc + lr);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem_acc, kTmemCols);
  }
}

}  // namespace

bool layer_decode_supported(int M, int N, int K, int r, int had_block) {
  (void)N;
  return M >= 1 && M <= kBN && r <= kMaxR && K % kW == 0 && had_block <= kW &&
         K / kKB <= kMaxKb * kMaxSplits;
}

cudaError_t launch_layer_decode(const LayerArgs& a, cudaStream_t stream) {
  LayerParams p{};
  p.X = reinterpret_cast<const __nv_bfloat16*>(a.X);
  p.L1t = reinterpret_cast<const __nv_bfloat16*>(a.L1t);
  p.s_w = a.s_w;
  p.L2t = reinterpret_cast<const __nv_bfloat16*>(a.L2t);
  p.Y = reinterpret_cast<__nv_bfloat16*>(a.Y);
  p.status = reinterpret_cast<uint32_t*>(a.ws);
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.r = a.r;
  p.b = a.had_block;
  p.scale_mul = (float)(1.0 / (7.0 * sqrt((double)a.had_block)));
  p.kb_total = a.K / kKB;
  const int tiles = (a.N + kBM - 1) / kBM;
  // splits: about one CTA per SM, each split a whole number of 512-column
  // warp passes (4 k-blocks) and at most kMaxKb k-blocks
  int s = tuning().split_k;
  if (s <= 0) s = std::max(1, num_sms() / tiles);
  s = std::max(1, std::min(s, kMaxSplits));
  int kbps = (p.kb_total + s - 1) / s;
  kbps = (kbps + 3) / 4 * 4;
  if (kbps > kMaxKb) return cudaErrorInvalidValue;
  p.kb_per_split = kbps;
  p.splits = (p.kb_total + kbps - 1) / kbps;
  CUtensorMap map_w;
  if (!encode_tiled_2d(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, (uint64_t)(a.K / 2),
                       (uint64_t)a.N, (uint64_t)(a.K / 2), (uint32_t)(kPackedRow * kKBS),
                       (uint32_t)kBM, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  static uint64_t attr_set = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set >> dev & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(w4a4_lr_layer_decode_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)Smem::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(tiles, 1, p.splits);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = Smem::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = tuning().pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = p.splits;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, w4a4_lr_layer_decode_kernel, map_w, p);
}

}  // namespace tq
