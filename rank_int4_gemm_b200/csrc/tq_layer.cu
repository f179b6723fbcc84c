// tq_layer.cu -- the whole decode layer (M <= 16 tokens) in one kernel.
//
//   Y = dequant( Q4(X H) . Q4(H^T R) ) + bf16(X L1) L2
//
// Per output tile of 128 channels, a cluster of S CTAs splits K (split-K);
// CTA z owns k-blocks [z*kbps, ...) of K, at most 8 blocks of 128 columns.
//
// The rotation runs on the tensor cores.  The slice of X is staged as a
// 128-row bf16 operand whose row (t, j) = 8 t + j is token t's k-block j
// (128 columns), so one kind::f16 MMA chain of M = N = K = 128 against the
// block-diagonal Sylvester matrix (+-1 entries, Hadamard blocks of b <= 128
// columns, generated in shared memory) gives every rotated value of the
// slice, exact products accumulated in fp32, in TMEM.  The int4 weights are
// expanded into TMEM as the integer MMA's A operand, so the expanded weights
// never pass through shared memory.
//
//   warps 0-15  activation: stage X (cp.async), one thread issues the
//               rotation MMAs; warp w reads TMEM lanes 32 (w % 4) .. (the
//               rows of tokens 4 (w % 4) .. +3) and columns 32 (w / 4) ..;
//               partial absmax per token, exchanged across the cluster
//               through distributed shared memory; the rotated values, kept
//               in registers, become the codes, written as int8 (16 * code)
//               into the integer MMA's B operand.  Then the slice's X.L1
//               partial on mma.sync (L1^T fragments fetched into registers
//               while X lands), pushed to split 0.  Warps 0-3 run the
//               epilogue.
//   warps 16-19 expand the streamed int4 weights (the whole slice is
//               requested at CTA start) into TMEM; in split 0 they also place
//               the tile's L2^T rows (the low-rank A operand).
//   warp 16     also issues the weight TMAs in the prologue (before the
//               kernel waits on its predecessor: weights never depend on it),
//               allocates TMEM and issues the integer MMAs (kind::i8, A from
//               TMEM, tokens as N = 16) and the low-rank MMAs (kind::f16,
//               split 0).
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
constexpr int kMaxB = 128;         // Hadamard block limit (one MMA row = one block)
constexpr int kSplitCols = 512;    // a split covers a multiple of 4 k-blocks
constexpr int kActWarps = 16, kConvWarps = 4;
// the first converter warp also issues the prologue TMAs, owns the TMEM
// allocation and issues the integer MMAs (20 warps: five per SM
// sub-partition, so each thread may hold up to 96 registers)
constexpr int kIssueWarp = kActWarps;
constexpr int kThreads = (kActWarps + kConvWarps) * 32;
constexpr int kActThreads = kActWarps * 32;
constexpr int kConvThreads = kConvWarps * 32;
constexpr int kEpiThreads = 128;
constexpr int kMaxBPair = 8;       // X L1 k-step pairs per warp (B fragments held in registers)

// TMEM columns (512 allocated; one CTA per SM)
constexpr uint32_t kColRot = 0;    // fp32 rotated slice, [128 rows (t, j)][128]
constexpr uint32_t kColW = 128;    // int8 weights, 32 columns per k-block
constexpr uint32_t kColAcc = 384;  // INT32 accumulator [16 tokens]
constexpr uint32_t kColLr = 400;   // fp32 low-rank accumulator [16 tokens]
constexpr uint32_t kTmemCols = 512;

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

// Shared-memory map (offsets from the 1024-aligned base).  The two K halves
// (64 columns each) of the 128-column operands are separate 128-byte
// swizzled tiles.
struct Smem {
  static constexpr uint32_t kHalf = 128 * 128;               // [128 rows][128 B]
  static constexpr uint32_t kXBase = 0;                      // X rows (t, j) [2][128][128 B]
  // Hadamard tiles P, Q [64 rows][128 B] (Q = -P, used when b = 128)
  static constexpr uint32_t kHTile = 64 * 128;
  static constexpr uint32_t kHBase = kXBase + 2 * kHalf;
  static constexpr uint32_t kStg = kBM * 128;                // one TMA stage (2 packed k-blocks)
  static constexpr uint32_t kWBase = kHBase + 4 * kHTile;    // packed weights [kNSTG]
  static constexpr uint32_t kBBase = kWBase + kNSTG * kStg;  // token codes [kb][16][128]
  static constexpr uint32_t kBBytes = kMaxKb * kBN * 128;
  static constexpr uint32_t kLrABase = kBBase + kBBytes;     // L2^T [128][128 B], SW128
  static constexpr uint32_t kLrBBase = kLrABase + kBM * 128; // bf16(XL1) [16][128 B], SW128
  // split-K partials [S][16][rows] + low-rank [16][rows]; before the epilogue
  // the X L1 k-part partials [KP][16][r]
  static constexpr uint32_t kKRecv = kLrBBase + kBN * 128;
  static constexpr uint32_t kKRecvBytes = 2 * kBN * kBM * 4;  // largest at S = 1
  static constexpr uint32_t kXRecv = kKRecv + kKRecvBytes;    // XL1 partials [S][16][r] fp32
  static constexpr uint32_t kXRecvBytes = kMaxSplits * kBN * kMaxR * 4;
  static constexpr uint32_t kAmax = kXRecv + kXRecvBytes;     // [S][4][16] + [16]
  static constexpr uint32_t kScale = kAmax + (kMaxSplits * 4 + 1) * kBN * 4;  // s_w [128]
  static constexpr uint32_t kBar = kScale + kBM * 4;
  // barriers: stg_full[kNSTG], rot_full, w_full, b_ready, lr_ready, acc_full, h_ready
  static constexpr uint32_t kNumBars = kNSTG + 6;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kMisc + 32;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};
static_assert(Smem::kAlloc <= 227 * 1024, "fused layer shared memory");
static_assert(kActWarps * kBN * 8 * 4 <= Smem::kKRecvBytes, "X L1 k-part partials");
static_assert(Smem::kWBase % 1024 == 0 && Smem::kBBase % 1024 == 0 &&
                  Smem::kLrABase % 1024 == 0 && Smem::kLrBBase % 1024 == 0,
              "1024-byte aligned operand tiles");

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
__device__ __forceinline__ int owned_lo(int o, int S) { return (o * kBM + S - 1) / S; }

// 16-byte chunk j (0..7) of row `row` of a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw_off(uint32_t row, uint32_t j) {
  return row * 128u + ((j ^ (row & 7u)) << 4);
}
// 16-byte chunk q (0..127: columns 8q .. 8q+7 of the slice) of token t in
// the staged X operand: row 8t + q/16 (k-block), K half (q/8) & 1.
__device__ __forceinline__ uint32_t xa_off(uint32_t t, uint32_t q) {
  return ((q >> 3) & 1u) * Smem::kHalf + sw_off(t * 8u + (q >> 4), q & 7u);
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
  uint64_t* rot_full = bars + kNSTG;
  uint64_t* w_full = rot_full + 1;
  uint64_t* b_ready = rot_full + 2;
  uint64_t* lr_ready = rot_full + 3;
  uint64_t* acc_full = rot_full + 4;
  uint64_t* h_ready = rot_full + 5;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S_::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S_::kMisc + 4);
  const uint32_t amax_all = base + S_::kAmax;                     // [S][4][16] fp32
  const uint32_t amax_row = amax_all + kMaxSplits * 4 * kBN * 4;  // [16] fp32
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

  pdl_launch_dependents();  // the next layer may start staging its weights
  // ---------------------------------------------------------------- prologue
  if (warp == kIssueWarp && lane == 0) {
    for (int i = 0; i < kNSTG; ++i) mbar_init(&stg_full[i], 1);
    mbar_init(rot_full, 1);
    mbar_init(w_full, kConvThreads);
    mbar_init(b_ready, kActThreads);
    mbar_init(lr_ready, kActThreads + kConvThreads);
    mbar_init(acc_full, 1);
    mbar_init(h_ready, kConvThreads);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&map_w);
    const uint64_t pol = policy_evict_first();
    for (int i = 0; i < n_st; ++i) {  // the whole slice
      mbar_arrive_expect_tx(&stg_full[i], S_::kStg);
      tma_load_2d(smem + S_::kWBase + i * S_::kStg, &map_w, &stg_full[i],
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
  const uint32_t tmem = *tmem_slot;

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

    // ---- X slice -> the rotation's A operand (rows of tokens past M are zero)
    const uint32_t xbase = base + S_::kXBase;
    {
      const int cpr = slice / 8;  // 16-byte chunks per token
      for (int ch = tid; ch < kBN * cpr; ch += kActThreads) {
        const int row = ch / cpr, q = ch - row * cpr;
        const bool ok = row < p.M;
        const __nv_bfloat16* src = p.X + (size_t)(ok ? row : 0) * p.K + kbase + q * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(
                         xbase + xa_off((uint32_t)row, (uint32_t)q)),
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
    // ---- X rows of k-blocks past a short slice: zero (while X lands)
    {
      const int nz = kMaxKb - n_kb;  // k-blocks past the slice, per token
      for (int ch = tid; ch < kBN * nz * 16; ch += kActThreads) {
        const int t = ch / (nz * 16), rem = ch - t * nz * 16;
        const int j = n_kb + (rem >> 4), cc = rem & 15;
        st_shared_v4(base + S_::kXBase + (uint32_t)(cc >> 3) * S_::kHalf +
                         sw_off((uint32_t)(t * 8 + j), (uint32_t)(cc & 7)),
                     make_uint4(0u, 0u, 0u, 0u));
      }
    }
    cp_async_wait<0>();
    fence_proxy_async_smem();  // X and zero rows -> tensor core reads
    named_bar_sync(1, kActThreads);

    // ---- rotation: D[(t, j)][n] = sum_k X[t][128 j + k] H[k][n], in two
    //      halves of 64 output columns.  For b = 128, H = [[P, P], [P, -P]]
    //      with P the Sylvester matrix of order 64 (k or n >= 64 sets bit 6,
    //      which adds 1 to popcount(n & k) only when both do); for b <= 64,
    //      H = diag(P, P) with P block-diagonal, and the off-diagonal
    //      quadrants are skipped.
    if (tid == 0) {
      mbar_wait(h_ready, 0u, p.status, abort_flag);
      tc_fence_after();
      const uint32_t id = idesc_bf16_f32(64);
      const uint64_t dp = sdesc_sw128(base + S_::kHBase);
      const uint64_t dq = sdesc_sw128(base + S_::kHBase + S_::kHTile);
      const bool full = p.b == kMaxB;
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        uint32_t acc = 0u;
#pragma unroll
        for (int kh = 0; kh < 2; ++kh) {
          if (!full && kh != nh) continue;
          const uint64_t da = sdesc_sw128(xbase + (uint32_t)kh * S_::kHalf);
          const uint64_t db = (full && nh == 1 && kh == 1) ? dq : dp;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            mma_bf16(tmem + kColRot + 64u * (uint32_t)nh, da + 2 * kk, db + 2 * kk, id, acc);
            acc = 1u;
          }
        }
      }
      mma_commit(rot_full);
    }
    // this thread's row of D: token t, k-block j, columns 32 cq .. 32 cq + 31
    const int q4 = warp & 3, cq = warp >> 2;
    const int t = 4 * q4 + (lane >> 3), j = lane & 7;
    float v[32];
    {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(rot_full, 0u, p.status, abort_flag));
      tc_fence_after();
      uint32_t u[32];
      if (ok) {
        tmem_ld32(tmem + kColRot + 32u * (uint32_t)cq + ((uint32_t)(32 * q4) << 16), u);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) u[i] = 0u;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(u[i]);
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    // over the token's 8 rows (lanes 8 (t % 4) ..)
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    cluster_wait_acquire();  // B0 complete: every peer is running
    if (j < S)
      dsmem_st_f32(dsmem_map(amax_all + (uint32_t)(((split * 4 + cq) * kBN + t) * 4), (uint32_t)j),
                   amax);
    cluster_arrive_release();  // B1: this CTA's absmax partials delivered
    cluster_wait_acquire();    // B1 complete

    // ---- codes of (t, j, columns 32 cq ..) as the int8 B operand (16 * code:
    //      the code's low nibble in the high nibble)
    {
      float am = 0.f;
#pragma unroll
      for (int z = 0; z < kMaxSplits; ++z)
        if (z < S)
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4)
            am = fmaxf(am, ld_shared_f32(amax_all + (uint32_t)(((z * 4 + c4) * kBN + t) * 4)));
      if (cq == 0 && j == 0) st_shared_f32(amax_row + (uint32_t)(t * 4), am);
      const CodeScale cs = code_scale(am);
      if (cs.pre != 1.f) {
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] *= cs.pre;
      }
      if (j < n_kb) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w4[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float* x = v + 16 * h + 4 * q;
            w4[q] = (low_bytes4(code_bits(x[0], cs.inv), code_bits(x[1], cs.inv),
                                code_bits(x[2], cs.inv), code_bits(x[3], cs.inv))
                     << 4) &
                    0xF0F0F0F0u;
          }
          st_shared_v4(base + S_::kBBase + (uint32_t)(j * kBN * 128) +
                           sw_off((uint32_t)t, (uint32_t)(2 * cq + h)),
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
          const uint4 x0 = ld_shared_v4(xbase + xa_off((uint32_t)g, q));
          const uint4 x8 = ld_shared_v4(xbase + xa_off((uint32_t)(g + 8), q));
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
        const int row = tid >> 3, jj = tid & 7;
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = 0.f;
        if (jj * 8 < p.r) {
          const uint32_t xr = base + S_::kXRecv + (uint32_t)((row * p.r + jj * 8) * 4);
          for (int z = 0; z < S; ++z)
#pragma unroll
            for (int e = 0; e < 8; ++e)
              f[e] += ld_shared_f32(xr + (uint32_t)((z * kBN * p.r + e) * 4));
        }
        st_shared_v4(base + S_::kLrBBase + sw_off((uint32_t)row, (uint32_t)jj),
                     make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]),
                                pack_bf16x2(f[4], f[5]), pack_bf16x2(f[6], f[7])));
      }
      fence_proxy_async_smem();
    }
    if (p.r > 0) mbar_arrive(lr_ready);
  } else {
    // ==================================================== weight converters
    const int tid = threadIdx.x - kActThreads;  // 0..127: channel row = TMEM lane
    // split 0: the tile's L2^T row `tid` ([r] bf16, r <= 32: 4 chunks)
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
    // the Hadamard tiles of the rotation (idle time: the weights are still
    // in flight).  P[n][k] (n, k < 64) = (-1)^popcount(n & k & m) inside the
    // diagonal blocks of min(b, 64) columns, m = min(b, 64) - 1; Q = -P.
    // One 16-byte chunk (k = k0 .. k0+7, k0 % 8 == 0) at a time: for blocks
    // of 8 or more columns the chunk lies in one block or none, and the
    // parity of n & k splits into that of n & k0 and that of n & e
    // (e = k - k0), read from an 8-entry pattern table indexed by n & 7.
    {
      const int bm = min(p.b, 64) - 1;
      const int n_chunks = (p.b == kMaxB ? 2 : 1) * 64 * 8;
      constexpr unsigned long long kParity8 = 0x963C5AF066CCAA00ull;  // byte m: bit e = parity(m & e)
      for (int ch = tid; ch < n_chunks; ch += kConvThreads) {
        const int q = ch >> 9, n = (ch >> 3) & 63, c8 = ch & 7;
        const int k0 = c8 * 8;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if (bm >= 7) {
          if (((n ^ k0) & ~bm) == 0) {
            const uint32_t flip = ((__popc((unsigned)(n & k0 & bm)) & 1) ^ q) ? 0xFFu : 0u;
            const uint32_t bits = ((uint32_t)(kParity8 >> (8 * (n & 7))) & 0xFFu) ^ flip;
#pragma unroll
            for (int e = 0; e < 4; ++e)
              w[e] = 0x3F803F80u | (((bits >> (2 * e)) & 1u) << 15) |
                     (((bits >> (2 * e + 1)) & 1u) << 31);
          }
        } else {  // blocks of 1, 2 or 4 columns: element by element
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int k = k0 + e;
            if (((n ^ k) & ~bm) == 0)
              w[e >> 1] |= ((__popc((unsigned)(n & k & bm)) & 1) ? 0xBF80u : 0x3F80u) << (16 * (e & 1));
          }
        }
        st_shared_v4(base + S_::kHBase + (uint32_t)q * S_::kHTile + sw_off((uint32_t)n, (uint32_t)c8),
                     make_uint4(w[0], w[1], w[2], w[3]));
      }
      fence_proxy_async_smem();
      mbar_arrive(h_ready);
    }
    cluster_wait_acquire();    // B0
    cluster_arrive_release();  // B1 (nothing to publish from these warps)
    if (do_lr) {
#pragma unroll
      for (int j = 0; j < 8; ++j)
        st_shared_v4(base + S_::kLrABase + sw_off((uint32_t)tid, (uint32_t)j),
                     j < kMaxR / 8 ? l2row[j] : make_uint4(0u, 0u, 0u, 0u));
      fence_proxy_async_smem();
    }
    // int4 -> int8 into TMEM: row `tid` of each k-block becomes 32 columns of
    // lane `tid` (column c holds codes 4c .. 4c+3 as 16 * code; within a
    // 16-byte packed group, byte i holds code i in its low nibble and code
    // i + 16 in its high nibble)
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const uint32_t x7 = (uint32_t)tid & 7u;
    for (int st = 0; st < n_st; ++st) {
      if (!__all_sync(0xffffffffu, mbar_wait(&stg_full[st], 0u, p.status, abort_flag))) break;
      const uint32_t src = base + S_::kWBase + (uint32_t)st * S_::kStg + (uint32_t)tid * 128u;
      uint4 w[8];
#pragma unroll
      for (int q = 0; q < 8; ++q) w[q] = ld_shared_v4(src + (((uint32_t)q ^ x7) << 4));
#pragma unroll
      for (int sub = 0; sub < kKBS; ++sub) {
        if (st * kKBS + sub < n_kb) {
          uint32_t e32[32];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint4 ww = w[4 * sub + c4];
            const uint32_t wv[4] = {ww.x, ww.y, ww.z, ww.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              e32[8 * c4 + e] = (wv[e] << 4) & 0xF0F0F0F0u;
              e32[8 * c4 + 4 + e] = wv[e] & 0xF0F0F0F0u;
            }
          }
          tmem_st32(tmem + kColW + 32u * (uint32_t)(st * kKBS + sub) + lane_off, e32);
        }
      }
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(w_full);
    cluster_wait_acquire();    // B1
    cluster_arrive_release();  // B2
    if (p.r > 0) mbar_arrive(lr_ready);
    sw_tile[tid] = sw;         // read by the epilogue after B3
    if (warp == kIssueWarp) {
      // ======================================================== MMA issue
      const uint32_t id_i8 = idesc_i8_s32(kBN);
      const uint32_t id_bf = idesc_bf16_f32(kBN);
      bool alive = mbar_wait(b_ready, 0u, p.status, abort_flag) &&
                   mbar_wait(w_full, 0u, p.status, abort_flag) && !*abort_flag;
      if (alive) {
        tc_fence_after();
        if (lane == 0) {
          for (int i = 0; i < n_kb; ++i) {
            const uint64_t db = sdesc_sw128(base + S_::kBBase + (uint32_t)(i * kBN * 128));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_i8_tmem_a(tmem + kColAcc, tmem + kColW + 32u * (uint32_t)i + 8u * (uint32_t)kk,
                            db + 2 * kk, id_i8, (i > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (alive && do_lr && mbar_wait(lr_ready, 0u, p.status, abort_flag)) {
        tc_fence_after();
        if (lane == 0) {
          const uint64_t da = sdesc_sw128(base + S_::kLrABase);
          const uint64_t db = sdesc_sw128(base + S_::kLrBBase);
          for (int kk = 0; kk < p.r / 16; ++kk)
            mma_bf16(tmem + kColLr, da + 2 * kk, db + 2 * kk, id_bf, kk > 0 ? 1u : 0u);
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
      tmem_ld16(tmem + kColAcc + t_row, ai);
      if (do_lr) tmem_ld16(tmem + kColLr + t_row, af);
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
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool layer_decode_supported(int M, int N, int K, int r, int had_block) {
  (void)N;
  return M >= 1 && M <= kBN && r <= kMaxR && K % kSplitCols == 0 && had_block >= 1 &&
         had_block <= kMaxB && K / kKB <= kMaxKb * kMaxSplits;
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
  // groups (4 k-blocks) and at most kMaxKb k-blocks
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
