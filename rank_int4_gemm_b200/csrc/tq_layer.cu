// tq_layer.cu -- the whole decode layer (M <= 16 tokens) in one kernel.
//
//   Y = dequant( Q4(X H) . Q4(H^T R) ) + bf16(X L1) L2
//
// Per output tile of 128 channels, a cluster of S CTAs splits K (split-K);
// CTA z owns k-blocks [z*kbps, ...) of K, at most 1024 columns.  Its warps:
//
//   warps 0-15  activation, warp t = token t: the token's slice of X is
//               staged once in shared memory; Sylvester transform (the warp
//               butterflies of tq_quantize_act, so the codes are the same
//               bits) and partial absmax, exchanged across the cluster through
//               distributed shared memory.  While that exchange completes
//               the same warps compute the slice's X.L1 partial on mma.sync
//               (L1^T fragments are fetched into registers while X lands)
//               and push it to split 0; then the rotated values, kept in
//               registers, become the codes, written as int8 (16 * code)
//               straight into the MMA's B operand.  Warps 0-3 run the
//               epilogue.
//   warps 16-19 expand the int4 weights into one int8 operand slot per
//               k-block (the whole slice is requested at CTA start and lands
//               packed in the odd slots), all before the token codes exist,
//               so the MMAs run back to back.  In split 0 they also place the
//               tile's L2^T rows (the low-rank A operand).
//   warp 16     also issues the weight TMAs in the prologue (before the
//               kernel waits on its predecessor: weights never depend on it),
//               allocates TMEM and issues the MMAs: kind::i8 for the codes,
//               kind::f16 for the low-rank branch (split 0).
//
// Cluster barriers, all threads of all CTAs in order: B0 (every CTA is
// running), B1 (absmax partials delivered), B2 (X.L1 partials delivered),
// B3 (split-K partial rows delivered).  The epilogue is the GEMM kernel's
// split-K reduction: each split pushes its INT32 partial rows to the row's
// owner CTA, owners reduce in split order and store Y.  Nothing goes through
// global memory except X, the weights, L1^T, L2^T, s_w and Y.  No TMA
// multicast.
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
constexpr int kNSTG = 4;           // TMA stages (2 k-blocks each): the whole slice at CTA start
constexpr int kMaxKb = 8;          // k-blocks per CTA (slice <= 1024 columns)
constexpr int kMaxSplits = 4;      // split-K cluster size limit of this kernel
constexpr int kMaxR = 32;          // low-rank width handled here
constexpr int kE = 16;             // values per lane per warp pass
constexpr int kW = 32 * kE;        // 512 columns per warp pass
constexpr int kActWarps = 16, kConvWarps = 4;
// the first converter warp also issues the prologue TMAs, owns the TMEM
// allocation and issues the MMAs (20 warps: five per SM sub-partition, so each
// thread may hold up to 96 registers)
constexpr int kIssueWarp = kActWarps;
constexpr int kThreads = (kActWarps + kConvWarps) * 32;
constexpr int kActThreads = kActWarps * 32;
constexpr int kConvThreads = kConvWarps * 32;
constexpr int kEpiThreads = 128;
constexpr int kMaxBPair = 8;       // X L1 k-step pairs per warp (B fragments held in registers)

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
  // kMaxKb int8 weight k-blocks, one slot each; stage s (2 packed k-blocks,
  // 128-byte swizzled rows) lands in slot 2s+1 and is expanded in place
  static constexpr uint32_t kOp = kBM * 128;
  static constexpr uint32_t kStg = kBM * 128;
  static constexpr uint32_t kOpBase = 0;
  static constexpr uint32_t kBBase = kOpBase + kMaxKb * kOp;  // token codes [kb][16][128]
  static constexpr uint32_t kBBytes = kMaxKb * kBN * 128;
  static constexpr uint32_t kLrBBase = kBBase + kBBytes;      // bf16(XL1) [16][64], SW128
  static constexpr uint32_t kLrABase = (kLrBBase + kBN * 128 + 1023u) & ~1023u;  // L2^T [128][64]
  static constexpr uint32_t kXBase = kLrABase + kBM * 128;    // X slice [16][1024] bf16, swizzled
  static constexpr uint32_t kXRow = kMaxKb * kKB * 2;         // bytes per X row
  static constexpr uint32_t kXBytes = kBN * kXRow;
  // split-K partials [S][16][rows] + low-rank [16][rows]; before the epilogue
  // the X L1 k-part partials [KP][16][r]
  static constexpr uint32_t kKRecv = kXBase + kXBytes;
  static constexpr uint32_t kKRecvBytes = 2 * kBN * kBM * 4;  // largest at S = 1
  static constexpr uint32_t kXRecv = kKRecv + kKRecvBytes;    // XL1 partials [S][16][r] fp32
  static constexpr uint32_t kXRecvBytes = kMaxSplits * kBN * kMaxR * 4;
  static constexpr uint32_t kAmax = kXRecv + kXRecvBytes;     // [S][16] + [16]
  static constexpr uint32_t kScale = kAmax + (kMaxSplits + 1) * kBN * 4;  // s_w [128]
  static constexpr uint32_t kBar = kScale + kBM * 4;
  // barriers: stg_full[kNSTG], op_full[kMaxKb], b_ready, lr_ready, acc_full
  static constexpr uint32_t kNumBars = kNSTG + kMaxKb + 3;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kMisc + 32;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};
static_assert(Smem::kAlloc <= 227 * 1024, "fused layer shared memory");
static_assert(kActWarps * kBN * 8 * 4 <= Smem::kKRecvBytes, "X L1 k-part partials");

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
__device__ __forceinline__ void st_shared_f32(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
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
__device__ __forceinline__ uint32_t ldg_u32(const __nv_bfloat16* p) {
  return __ldg(reinterpret_cast<const unsigned int*>(p));
}
__device__ __forceinline__ int owned_lo(int o, int S) { return (o * kBM + S - 1) / S; }

// 16-byte chunk j (0..7) of row `row` of a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw_off(uint32_t row, uint32_t j) {
  return row * 128u + ((j ^ (row & 7u)) << 4);
}
// 16-byte chunk c (0..127) of row `row` (0..15) of the staged X slice; the
// chunk index is XORed with the row so that the 8 rows of an ldmatrix land
// in different banks.
__device__ __forceinline__ uint32_t x_off(uint32_t row, uint32_t c) {
  return row * Smem::kXRow + ((c ^ (row & 7u)) << 4);
}

// This lane's kE = 16 consecutive values of token `row`, columns
// col0 .. col0 + 15 of the staged slice, as fp32.
__device__ __forceinline__ void load_x16(uint32_t xbase, int row, int col0, float (&v)[kE]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const uint4 u = ld_shared_v4(xbase + x_off((uint32_t)row, (uint32_t)(col0 / 8 + h)));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      v[8 * h + 2 * j] = __uint_as_float(w[j] << 16);
      v[8 * h + 2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
    }
  }
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
  uint64_t* op_full = bars + kNSTG;
  uint64_t* b_ready = op_full + kMaxKb;
  uint64_t* lr_ready = b_ready + 1;
  uint64_t* acc_full = b_ready + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S_::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S_::kMisc + 4);
  const uint32_t amax_all = base + S_::kAmax;                 // [S][16] fp32
  const uint32_t amax_row = amax_all + kMaxSplits * kBN * 4;  // [16] fp32
  float* sw_tile = reinterpret_cast<float*>(smem + S_::kScale);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x, split = blockIdx.z;
  const int S = p.splits;
  const int kb0 = split * p.kb_per_split;
  const int n_kb = min(p.kb_total - kb0, p.kb_per_split);
  const int n_st = (n_kb + kKBS - 1) / kKBS;
  const int kbase = kb0 * kKB;           // first column of this CTA's slice
  const int slice = n_kb * kKB;          // 512 or 1024 columns
  const bool do_lr = p.r > 0 && split == 0;
  constexpr uint32_t kTmemCols = 32;     // INT32 [16] + fp32 low-rank [16]

  pdl_launch_dependents();  // the next layer may start staging its weights
  // ---------------------------------------------------------------- prologue
  if (warp == kIssueWarp && lane == 0) {
    for (int i = 0; i < kNSTG; ++i) mbar_init(&stg_full[i], 1);
    for (int i = 0; i < kMaxKb; ++i) mbar_init(&op_full[i], kConvThreads);
    mbar_init(b_ready, kActThreads);
    mbar_init(lr_ready, kActThreads + kConvThreads);
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&map_w);
    const uint64_t pol = policy_evict_first();
    for (int i = 0; i < n_st; ++i) {  // the whole slice, into the odd slots
      mbar_arrive_expect_tx(&stg_full[i], S_::kStg);
      tma_load_2d(smem + S_::kOpBase + (2 * i + 1) * S_::kOp, &map_w, &stg_full[i],
                  (kb0 + i * kKBS) * kPackedRow, tile * kBM, pol);
    }
  }
  if (warp == kIssueWarp) {
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
    const int tid = threadIdx.x;  // 0..511
    const int g = lane >> 2, c = lane & 3;
    // X L1 work split: warp = (n-tile nt, k-part kp); KP k-parts of kspp
    // k-steps (16 columns) each
    const int ntiles = p.r / 8;
    const int KP = ntiles > 0 ? kActWarps / ntiles : 1;
    const bool xl1_warp = ntiles > 0 && warp < ntiles * KP;
    const int nt = ntiles > 0 ? warp % ntiles : 0, kp = ntiles > 0 ? warp / ntiles : 0;
    const int kspp = (slice / 16) / KP;
    pdl_wait();  // X comes from the preceding kernel

    // ---- X slice [16][slice] -> shared memory (rows past M are zero)
    const uint32_t xbase = base + S_::kXBase;
    {
      const int cpr = slice / 8;  // 16-byte chunks per row
      for (int ch = tid; ch < kBN * cpr; ch += kActThreads) {
        const int row = ch / cpr, cc = ch - row * cpr;
        const bool ok = row < p.M;
        const __nv_bfloat16* src = p.X + (size_t)(ok ? row : 0) * p.K + kbase + cc * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         xbase + x_off((uint32_t)row, (uint32_t)cc)),
                     "l"(src), "r"(ok ? 16u : 0u)
                     : "memory");
      }
      cp_async_commit();
    }
    // L1^T fragments of this warp's k-steps, fetched while X lands.  Inside
    // each pair of k-steps (32 columns) lane (g, c) takes columns 8c .. 8c+7
    // of both operands, so one 16-byte load gives its B fragments for the
    // pair: mma k-step 0 uses columns 8c + {0,1 | 2,3}, k-step 1 uses
    // 8c + {4,5 | 6,7} (the same bijection on A and B, so every product
    // X[t][k] L1[k][j] is summed exactly once).
    uint4 bq[kMaxBPair];
#pragma unroll
    for (int i = 0; i < kMaxBPair; ++i) {
      bq[i] = make_uint4(0u, 0u, 0u, 0u);
      if (xl1_warp && 2 * i < kspp)
        bq[i] = __ldg(reinterpret_cast<const uint4*>(
            p.L1t + (size_t)(nt * 8 + g) * p.K + kbase + 32 * (kp * kspp / 2 + i) + 8 * c));
    }
    cp_async_wait<0>();
    named_bar_sync(1, kActThreads);

    // ---- transform of token `warp` over the slice (kept in registers),
    //      partial absmax
    const int np = slice / kW;  // 1 or 2 warp passes
    float v[2][kE];
    float amax = 0.f;
#pragma unroll
    for (int ps = 0; ps < 2; ++ps) {
      if (ps < np) {
        load_x16(xbase, warp, ps * kW + lane * kE, v[ps]);
        fwht_warp<kE>(v[ps], p.b);
#pragma unroll
        for (int i = 0; i < kE; ++i) amax = fmaxf(amax, fabsf(v[ps][i]));
      }
    }
    amax = warp_max(amax);
    cluster_wait_acquire();  // B0 complete: every peer is running
    if (lane < S)
      dsmem_st_f32(dsmem_map(amax_all + (uint32_t)((split * kBN + warp) * 4), (uint32_t)lane), amax);
    cluster_arrive_release();  // B1: this CTA's absmax partials delivered
    cluster_wait_acquire();  // B1 complete

    // ---- codes of token `warp` as the int8 B operand (16 * code: the code's
    //      low nibble in the high nibble)
    {
      float am = 0.f;
#pragma unroll
      for (int z = 0; z < kMaxSplits; ++z)
        if (z < S) am = fmaxf(am, ld_shared_f32(amax_all + (uint32_t)((z * kBN + warp) * 4)));
      if (lane == 0) st_shared_f32(amax_row + (uint32_t)(warp * 4), am);
      const CodeScale cs = code_scale(am);
#pragma unroll
      for (int ps = 0; ps < 2; ++ps) {
        if (ps < np) {
          if (cs.pre != 1.f) {
#pragma unroll
            for (int i = 0; i < kE; ++i) v[ps][i] *= cs.pre;
          }
          uint32_t w4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            w4[q] = (low_bytes4(code_bits(v[ps][4 * q], cs.inv), code_bits(v[ps][4 * q + 1], cs.inv),
                                code_bits(v[ps][4 * q + 2], cs.inv), code_bits(v[ps][4 * q + 3], cs.inv))
                     << 4) &
                    0xF0F0F0F0u;
          const int col = ps * kW + lane * kE;  // within the slice
          const int kb = col / kKB, j = (col % kKB) / 16;
          st_shared_v4(base + S_::kBBase + (uint32_t)(kb * kBN * 128) + sw_off((uint32_t)warp, (uint32_t)j),
                       make_uint4(w4[0], w4[1], w4[2], w4[3]));
        }
      }
    }
    fence_proxy_async_smem();
    mbar_arrive(b_ready);

    // ---- X L1 partial over the slice (mma.sync, overlapping the integer
    //      MMAs): A fragments from the staged X, B from the registers
    const uint32_t part = base + S_::kKRecv;  // [KP][16][r] fp32
    if (xl1_warp) {
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int i = 0; i < kMaxBPair; ++i) {
        if (2 * i < kspp) {
          const uint32_t q = (uint32_t)(4 * (kp * kspp / 2 + i) + c);  // 16-byte chunk of the slice
          const uint4 x0 = ld_shared_v4(xbase + x_off((uint32_t)g, q));
          const uint4 x8 = ld_shared_v4(xbase + x_off((uint32_t)(g + 8), q));
          const uint32_t a0[4] = {x0.x, x8.x, x0.y, x8.y}, b0[2] = {bq[i].x, bq[i].y};
          const uint32_t a1[4] = {x0.z, x8.z, x0.w, x8.w}, b1[2] = {bq[i].z, bq[i].w};
          mma_16816(acc[0], a0, b0);
          mma_16816(acc[1], a1, b1);
        }
      }
      // C fragment: tokens g and g + 8, columns nt*8 + 2c, +1
      const uint32_t d0 = part + (uint32_t)(((kp * kBN + g) * p.r + nt * 8 + 2 * c) * 4);
      const uint32_t d1 = d0 + (uint32_t)(8 * p.r * 4);
      st_shared_f32(d0, acc[0][0] + acc[1][0]);
      st_shared_f32(d0 + 4, acc[0][1] + acc[1][1]);
      st_shared_f32(d1, acc[0][2] + acc[1][2]);
      st_shared_f32(d1 + 4, acc[0][3] + acc[1][3]);
    }
    named_bar_sync(1, kActThreads);
    // k-parts summed in order; this CTA's partial [16][r] -> split 0's
    // receive area, slot `split`
    if (ntiles > 0 && tid < kBN * p.r) {
      float s = 0.f;
      for (int k = 0; k < KP; ++k) s += ld_shared_f32(part + (uint32_t)((k * kBN * p.r + tid) * 4));
      dsmem_st_f32(dsmem_map(base + S_::kXRecv + (uint32_t)((split * kBN * p.r + tid) * 4), 0u), s);
    }
    cluster_arrive_release();  // B2: this CTA's X L1 partial delivered
    cluster_wait_acquire();

    // ---- split 0: X L1 = sum of the splits' partials (split order), bf16
    //      into the low-rank B operand [16][64] (columns past r are zero)
    if (do_lr) {
      if (tid < kBN * 8) {
        const int row = tid >> 3, j = tid & 7;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
        if (j * 8 < p.r) {
          const uint32_t xr = base + S_::kXRecv + (uint32_t)((row * p.r + j * 8) * 4);
          for (int z = 0; z < S; ++z)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] += ld_shared_f32(xr + (uint32_t)((z * kBN * p.r + e) * 4));
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
    // split 0: the tile's L2^T row `tid` ([r] bf16, r <= 32: 4 chunks),
    // fetched now and placed once its operand slot is free
    uint4 l2row[kMaxR / 8];
    // the scale of channel `tid`, for the epilogue (stored after the loop, so
    // that no thread waits on this load early)
    const float sw = (tile * kBM + tid < p.N) ? __ldg(p.s_w + tile * kBM + tid) : 0.f;
#pragma unroll
    for (int j = 0; j < kMaxR / 8; ++j) {
      l2row[j] = make_uint4(0u, 0u, 0u, 0u);
      const int gn = tile * kBM + tid;
      if (do_lr && gn < p.N && j * 8 < p.r)
        l2row[j] = __ldg(reinterpret_cast<const uint4*>(p.L2t + (size_t)gn * p.r + j * 8));
    }
    cluster_wait_acquire();    // B0
    cluster_arrive_release();  // B1 (nothing to publish from these warps)
    // split 0: the tile's L2^T rows -> the low-rank A operand
    if (do_lr) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(base + S_::kLrABase + sw_off((uint32_t)tid, (uint32_t)j),
                     j < kMaxR / 8 ? l2row[j] : make_uint4(0u, 0u, 0u, 0u));
      fence_proxy_async_smem();
    }
    // int4 -> int8, in place: each thread expands its row of the stage's
    // first k-block into slot 2s, reads the second, and once all four warps
    // have read the packed rows, writes the second into slot 2s+1
    for (int st = 0; st < n_st; ++st) {
      if (!mbar_wait(&stg_full[st], 0u, p.status, abort_flag)) break;
      const uint32_t x7 = (uint32_t)tid & 7u;
      const uint32_t src = base + S_::kOpBase + (uint32_t)(2 * st + 1) * S_::kOp + (uint32_t)tid * 128u;
      auto expand = [&](const uint4 (&w)[4], int slot) {
        const uint32_t dst = base + S_::kOpBase + (uint32_t)slot * S_::kOp + (uint32_t)tid * 128u;
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
      };
      uint4 w[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = ld_shared_v4(src + (((uint32_t)q ^ x7) << 4));
      expand(w, 2 * st);  // slot 2s holds nothing yet
#pragma unroll
      for (int q = 0; q < 4; ++q) w[q] = ld_shared_v4(src + (((uint32_t)(4 + q) ^ x7) << 4));
      named_bar_sync(2, kConvThreads);  // every row of the packed stage is read
      expand(w, 2 * st + 1);
      fence_proxy_async_smem();
      mbar_arrive(&op_full[2 * st]);
      mbar_arrive(&op_full[2 * st + 1]);
    }
    cluster_wait_acquire();    // B1
    cluster_arrive_release();  // B2
    if (p.r > 0) mbar_arrive(lr_ready);
    sw_tile[tid] = sw;         // read by the epilogue after B3
    if (warp == kIssueWarp) {
      // ======================================================== MMA issue
      const uint32_t id_i8 = idesc_i8_s32(kBN);
      const uint32_t id_bf = idesc_bf16_f32(kBN);
      bool alive = mbar_wait(b_ready, 0u, p.status, abort_flag);
      for (int i = 0; i < n_kb && alive; ++i) {
        if (!mbar_wait(&op_full[i], 0u, p.status, abort_flag)) {
          alive = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = sdesc_sw128(base + S_::kOpBase + (uint32_t)i * S_::kOp);
          const uint64_t db = sdesc_sw128(base + S_::kBBase + (uint32_t)(i * kBN * 128));
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_i8(tmem_acc, da + 2 * kk, db + 2 * kk, id_i8, (i > 0 || kk > 0) ? 1u : 0u);
        }
        __syncwarp();
      }
      if (alive && do_lr && mbar_wait(lr_ready, 0u, p.status, abort_flag)) {
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = sdesc_sw128(base + S_::kLrABase);
          const uint64_t db = sdesc_sw128(base + S_::kLrBBase);
          for (int kk = 0; kk < p.r / 16; ++kk)
            mma_bf16(tmem_lr, da + 2 * kk, db + 2 * kk, id_bf, kk > 0 ? 1u : 0u);
        }
        __syncwarp();
      }
      if (lane == 0) mma_commit(acc_full);
      __syncwarp();
    }
    cluster_wait_acquire();  // B2
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
  cluster_sync();  // B3: every split's partial rows delivered
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
      const float s_x = ld_shared_f32(amax_row + (uint32_t)(col * 4)) * p.scale_mul;
      p.Y[(size_t)col * p.N + g_n] = __float2bfloat16_rn(s_x * sw_tile[lo_m + rr] * (float)acc + lr);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kIssueWarp) {
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
