// tq_decode.cu -- the whole decode layer (M <= 16 tokens) in one kernel,
// sized so that the CTAs of two consecutive layers share every SM.
//
//   Y = dequant( Q4(X H) . Q4(H^T R) ) + bf16(X L1) L2
//
// Why this shape.  A decode layer reads ~9 MB (the int4 weights) and does
// little arithmetic, so its time is the latency of its dependency chain
// (X -> rotation -> per-token absmax across all of K -> codes -> integer
// MMAs -> split-K reduction -> Y) plus the time to bring the weights on
// chip.  The weights do not depend on the preceding kernel, so each CTA
// requests and expands them before its programmatic-dependent-launch wait.
// A CTA uses ~103 KB of shared memory, 256 TMEM columns and <= 112
// registers per thread, so a second CTA (the next layer's) fits on the same
// SM: while one layer runs its chain, the next one's weights stream in.
//
// Grid: one cluster of C = K / 256 CTAs per group of G = 128 T output
// channels.  CTA z of a cluster owns columns [256 z, 256 z + 256) of K for
// all G channels (T tiles of 128), and after the split-K exchange it owns
// channels [ceil(z G / C), ceil((z + 1) G / C)) of the output.
//
//   warps 0-7  (workers)
//     1. expand the group's int4 weights of this K slice (16 * code, int8):
//        tiles 0-2 into TMEM (the integer MMA's A operand), tile 3 into
//        shared memory (128-byte swizzled K-major);
//     2. rotate X: warp w holds tokens w and w + 8, each lane 8 consecutive
//        values, the same in-register and shuffle butterflies as the
//        activation kernel (so codes and scales equal tq_quantize_act's);
//        partial absmax per token to every CTA of the cluster;
//     3. X L1 partial over the slice on mma.sync, to the owner of each
//        token (token t belongs to CTA t % C), who sums the C partials in
//        cluster order, rounds to bf16 and sends the row to every CTA;
//     4. codes with the cluster-wide absmax (RoundClip, ties to even) into
//        the MMA's B operand;
//     5. read the INT32 accumulators and send each channel's 16 sums (as
//        int16: they are 16 x sum q q with |sum| <= 49 * 256) to the
//        channel's owner;
//     6. owners: split-K sum in cluster order, s_w s_x acc + bf16(X L1) L2,
//        store bf16 Y.
//   warp 8  (control)
//     barriers, weight and L1^T TMA (before the PDL wait), TMEM, the PDL
//     wait and the X TMA, then the integer MMAs (kind::i8, M = 128 channels,
//     N = 16 tokens, K = 32).
//
// All exchanges between CTAs are st.async stores completing as transaction
// bytes on the receiver's mbarrier (no cluster-wide barrier on the chain).
// Every wait is bounded; a CTA whose wait gives up records the timeout and
// still executes every barrier, so no peer is left waiting.  No TMA
// multicast.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "tq_act_common.cuh"
#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

namespace {

constexpr int kMT = 16;          // tokens (MMA N)
constexpr int kSlice = 256;      // columns of K per CTA (two 128-column k-blocks)
constexpr int kMaxC = 16;        // cluster size limit: K <= 4096
constexpr int kMaxT = 4;         // 128-channel tiles per CTA
constexpr int kTmemTiles = 3;    // tiles whose expanded weights live in TMEM
constexpr int kMaxR = 64;        // low-rank width handled here (0, 16, 32 or 64)
constexpr int kWorkers = 256;    // warps 0-7
constexpr int kCtrlWarp = 8;
constexpr int kThreads = kWorkers + 32;
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kColAcc = 192;  // INT32 accumulators: tile j at 192 + 16 j

struct DecodeParams {
  const float* s_w;          // [N]
  const __nv_bfloat16* L2t;  // [N][r]
  __nv_bfloat16* Y;          // [M][N]
  uint32_t* status;
  int8_t* dbg_codes;         // [M][K] activation codes, or null
  float* dbg_sx;             // [M] scales, or null
  int32_t* dbg_acc;          // [M][N] integer sums, or null
  const uint32_t* signs;     // randomized Hadamard sign masks [n_rht][K / 32], or null
  int M, N, K, r, b;
  int C;                     // CTAs per cluster (K / 256)
  int T;                     // 128-channel tiles per CTA
  float scale_mul;           // 1 / (7 sqrt(b))
  int n_rht;                 // composed randomized Hadamards (masks)
};

// Shared-memory map (offsets from the 1024-aligned base), for rank R.
template <int R>
struct Sm {
  static constexpr int kRr = R > 16 ? R : 16;                 // L1^T rows staged
  static constexpr uint32_t kWTile = 128 * 128;               // packed tile [128][128 B], SW128
  static constexpr uint32_t kW = 0;                           // [T] packed tiles
  static constexpr uint32_t kA3 = 0;                          // tile 3 int8 [2 k-blocks][128][128 B]
  static constexpr uint32_t kA3Block = 128 * 128;
  static constexpr uint32_t kKRecv = 32 * 1024;               // split-K sums [C][per_max][16] int16
  static constexpr uint32_t kKRecvMax = 17 * 1024;
  static constexpr uint32_t kX = 64 * 1024;                   // X [4 chunks of 64 cols][16][128 B]
  static constexpr uint32_t kXChunk = kMT * 128;
  static constexpr uint32_t kL1 = kX + 4 * kXChunk;           // L1^T [4 chunks][R][128 B]
  static constexpr uint32_t kL1Chunk = kRr * 128;
  // rank 64: chunk 3 of L1^T goes to the weight staging's tail, free once
  // the weights are expanded (above the split-K area), so that two CTAs
  // still share an SM
  static constexpr int kL1Here = R == 64 ? 3 : 4;
  static constexpr uint32_t kL1Hi = 50 * 1024;
  static constexpr uint32_t kB = kL1 + kL1Here * kL1Chunk;    // codes [2 k-blocks][16][128 B]
  static constexpr uint32_t kBBlock = kMT * 128;
  static constexpr uint32_t kAmax = kB + 2 * kBBlock;         // [C][16] fp32
  // [C][tpo][r] fp32: C ceil(16 / C) <= 30 token slots (C = 15); rank 64
  // takes only clusters that divide 16 (16 slots)
  static constexpr uint32_t kXl1Recv = kAmax + kMaxC * kMT * 4;
  static constexpr uint32_t kXl1RecvBytes = 4096;
  static constexpr uint32_t kXl1Part = kXl1Recv + kXl1RecvBytes;  // [KP][16][r] fp32
  static constexpr uint32_t kXl1B = kXl1Part + 4096;          // bf16 X L1 [16][r]
  static constexpr uint32_t kSx = kXl1B + kMT * kRr * 2;      // s_x [16], partial absmax [16]
  static constexpr uint32_t kBar = kSx + 2 * kMT * 4;
  static constexpr uint32_t kNumBars = 12;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
  static_assert((R == 64 ? 16 : 30) * kRr * 4 <= kXl1RecvBytes &&
                    (8 / (kRr / 8 > 8 ? 8 : kRr / 8)) * kMT * kRr * 4 <= 4096,
                "X L1 exchange buffers");
  static_assert(R != 64 || (kL1Hi >= kKRecv + kKRecvMax && kL1Hi + kL1Chunk <= kX &&
                            kL1Hi % 1024 == 0),
                "L1^T chunk 3 between the split-K area and X");
  static_assert(kKRecv + kKRecvMax <= kX, "split-K area inside the weight staging");
  static_assert(kA3 + 2 * kA3Block <= kKRecv, "tile 3 below the split-K area");
  static_assert(kX % 1024 == 0 && kL1 % 1024 == 0 && kB % 1024 == 0 && kXChunk % 1024 == 0 &&
                    kL1Chunk % 1024 == 0 && kBBlock % 1024 == 0,
                "1024-byte aligned swizzled tiles");
};
// two CTAs per SM (228 KB of shared memory per SM, 1 KB reserved per CTA):
// the second slot of an SM takes the next layer's CTA (one CTA per SM
// measured 17.5 against 10.6 us per layer at rank 32)
static_assert(2 * (Sm<32>::kAlloc + 1024) <= 228 * 1024, "two CTAs per SM");
static_assert(2 * (Sm<64>::kAlloc + 1024) <= 228 * 1024, "two CTAs per SM at rank 64");
template <int R>
constexpr int kCtasPerSm = 2;

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void sts64(uint32_t addr, uint32_t a, uint32_t b) {
  asm volatile("st.shared.v2.u32 [%0], {%1,%2};" ::"r"(addr), "r"(a), "r"(b) : "memory");
}
__device__ __forceinline__ float ldsf(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void stsf(uint32_t addr, float v) {
  asm volatile("st.shared.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}
__device__ __forceinline__ void bar_sync_workers() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWorkers) : "memory");
}
// A wait of all worker warps: one lane polls the mbarrier (sleeping between
// polls), the others block on a hardware barrier, so that waiting warps
// (also those of the next layer's CTA on this SM) take no issue slots.
// Returns the same verdict to every worker.
template <bool kCluster>
__device__ __forceinline__ bool workers_wait(uint64_t* bar, uint32_t* status,
                                             volatile int* abort_flag, int* verdict) {
  if (threadIdx.x == 0) {
    const bool ok = kCluster ? mbar_wait_cluster(bar, 0u, status, abort_flag)
                             : mbar_wait(bar, 0u, status, abort_flag);
    *verdict = ok ? 1 : 0;
  }
  bar_sync_workers();
  const bool ok = *reinterpret_cast<volatile int*>(verdict) != 0;
  bar_sync_workers();  // the verdict slot may be reused by the next wait
  return ok;
}
__device__ __forceinline__ uint4 ldg_nc_v4(const void* ptr) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(ptr));
  return v;
}
__device__ __forceinline__ float ldg_nc_f32(const float* ptr) {
  float v;
  asm volatile("ld.global.nc.f32 %0, [%1];" : "=f"(v) : "l"(ptr));
  return v;
}
__device__ __forceinline__ void cluster_arrive_rel() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ uint32_t bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}
// int4 -> int8 (16 * code) of one 16-byte packed chunk (codes 32c .. 32c+31:
// byte i holds code i in its low nibble and code i + 16 in its high nibble):
// lo = codes 0..15, hi = codes 16..31, four per 32-bit word.
__device__ __forceinline__ void expand16(uint4 w, uint4& lo, uint4& hi) {
  lo = make_uint4((w.x << 4) & 0xF0F0F0F0u, (w.y << 4) & 0xF0F0F0F0u, (w.z << 4) & 0xF0F0F0F0u,
                  (w.w << 4) & 0xF0F0F0F0u);
  hi = make_uint4(w.x & 0xF0F0F0F0u, w.y & 0xF0F0F0F0u, w.z & 0xF0F0F0F0u, w.w & 0xF0F0F0F0u);
}

// kRhtN: composed randomized Hadamards (n_rht > 1 masks); a separate
// instantiation, so that the single-transform kernels carry none of it.
template <int R, bool kRhtN>
__global__ void __launch_bounds__(kThreads, kCtasPerSm<R>)
    w4a4_lr_decode_kernel(const __grid_constant__ CUtensorMap map_w,
                          const __grid_constant__ CUtensorMap map_x,
                          const __grid_constant__ CUtensorMap map_l1, const DecodeParams p) {
  using S = Sm<R>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* w_full = bars + 0;       // weight tiles (TMA)
  uint64_t* x_full = bars + 1;       // X slice (TMA)
  uint64_t* l1_full = bars + 2;      // L1^T slice (TMA)
  uint64_t* amax_bar = bars + 3;     // partial absmax from every CTA (st.async)
  uint64_t* xl1p_bar = bars + 4;     // X L1 partials of owned tokens (st.async)
  uint64_t* xl1b_bar = bars + 5;     // bf16 X L1 rows from their owners (st.async)
  uint64_t* codes_ready = bars + 6;  // workers: weights in TMEM / smem, codes in smem
  uint64_t* part_bar = bars + 7;     // split-K sums of owned channels (st.async)
  uint64_t* acc_full = bars + 8;     // [kMaxT]: tile j's MMAs done (commit)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + S::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + S::kMisc + 4);
  int* verdict = reinterpret_cast<int*>(smem + S::kMisc + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int C = p.C;
  const uint32_t crank = cluster_ctarank();
  const int G = p.T * 128;
  const int n0 = blockIdx.y * G;                 // first channel of this group
  const int kbase = (int)crank * kSlice;         // first column of this CTA's slice
  const int t_valid = min(p.T, (p.N - n0 + 127) / 128);
  const int per_max = (G + C - 1) / C;
  const int own_lo = ((int)crank * G + C - 1) / C;
  const int per = (((int)crank + 1) * G + C - 1) / C - own_lo;
  const int tpo = (kMT + C - 1) / C;             // tokens per owner, at most
  const int own_tok = p.M > (int)crank ? (p.M - (int)crank + C - 1) / C : 0;
  const int r = R;

  pdl_launch_dependents();  // the next layer may start staging its weights
  if (threadIdx.x == kCtrlWarp * 32) {
    mbar_init(w_full, 1);
    mbar_init(x_full, 1);
    mbar_init(l1_full, 1);
    mbar_init(amax_bar, 1);
    mbar_init(xl1p_bar, 1);
    mbar_init(xl1b_bar, 1);
    mbar_init(codes_ready, kWorkers);
    for (int j = 0; j < kMaxT; ++j) mbar_init(&acc_full[j], 1);
    mbar_init(part_bar, 1);
    *abort_flag = 0;
    // the bytes the other CTAs of the cluster will store here
    mbar_arrive_expect_tx(amax_bar, (uint32_t)(C * kMT * 4));
    mbar_arrive_expect_tx(xl1p_bar, (uint32_t)(r > 0 ? C * own_tok * r * 4 : 0));
    mbar_arrive_expect_tx(xl1b_bar, (uint32_t)(r > 0 ? p.M * r * 2 : 0));
    mbar_arrive_expect_tx(part_bar, (uint32_t)(C * per * kMT * 2));
    fence_barrier_init();
    fence_proxy_async_smem();
    tma_prefetch_desc(&map_w);
    tma_prefetch_desc(&map_x);
    const uint64_t pol_w = policy_evict_first();
    // weights and L1^T never depend on the preceding kernel: requested now
    mbar_arrive_expect_tx(w_full, (uint32_t)(t_valid * S::kWTile));
    for (int j = 0; j < t_valid; ++j)
      tma_load_2d(smem + S::kW + j * S::kWTile, &map_w, w_full, kbase / 2, n0 + 128 * j, pol_w);
    if (r > 0) {
      tma_prefetch_desc(&map_l1);
      const uint64_t pol_l = policy_evict_last();  // every group reads the same L1^T
      mbar_arrive_expect_tx(l1_full, (uint32_t)(4 * r * 128));
      for (int cc = 0; cc < S::kL1Here; ++cc)
        tma_load_2d(smem + S::kL1 + cc * S::kL1Chunk, &map_l1, l1_full, kbase + 64 * cc, 0,
                    pol_l);
    }
  }
  if (warp == kCtrlWarp) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  cluster_arrive_relaxed();  // B0: this CTA is running, its barriers initialised
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t idesc = idesc_i8_s32(kMT);

  if (warp == kCtrlWarp) {
    // ============================================================ control
    if (lane == 0) {
      pdl_wait();  // X comes from the preceding kernel
      mbar_arrive_expect_tx(x_full, 4 * S::kXChunk);
      const uint64_t pol_x = policy_evict_first();
      for (int cc = 0; cc < 4; ++cc)
        tma_load_2d(smem + S::kX + cc * S::kXChunk, &map_x, x_full, kbase + 64 * cc, 0, pol_x);
      const bool ok = mbar_wait(codes_ready, 0u, p.status, abort_flag) && !*abort_flag;
      tc_fence_after();
      // tile by tile (measured faster than interleaving the tiles'
      // accumulators), each tile committed on its own, so that its sums
      // leave for their owners while the next tiles compute
      for (int j = 0; j < kMaxT; ++j) {
        if (ok && j < t_valid) {
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const uint64_t db = sdesc_sw128(base + S::kB + (uint32_t)kb * S::kBBlock);
            const uint64_t da = sdesc_sw128(base + S::kA3 + (uint32_t)kb * S::kA3Block);
            const uint32_t d = tmem + kColAcc + 16u * (uint32_t)j;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t accum = (kb > 0 || kk > 0) ? 1u : 0u;
              if (j < kTmemTiles)
                mma_i8_tmem_a(d, tmem + 64u * (uint32_t)j + 32u * (uint32_t)kb + 8u * (uint32_t)kk,
                              db + 2 * kk, idesc, accum);
              else
                mma_i8(d, da + 2 * kk, db + 2 * kk, idesc, accum);
            }
          }
        }
        mma_commit(&acc_full[j]);  // also on the abort path: the waiters are released
      }
    }
    __syncwarp();
    cluster_wait_acquire();  // B0 (nothing remote from this warp)
    cluster_arrive_rel();    // teardown barrier: nothing to send
  } else {
    // ============================================================ workers
    const int tid = threadIdx.x;  // 0..255
    const int q = warp & 3, h = warp >> 2;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const int row = 32 * q + lane;  // channel within a tile = TMEM lane

    // ---- 1. weights int4 -> int8 (16 * code): tiles h and h + 2
    bool ok = workers_wait<false>(w_full, p.status, abort_flag, verdict);
    uint4 t3[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) t3[c] = make_uint4(0u, 0u, 0u, 0u);
    if (ok) {
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int j = h + 2 * jj;
        if (j >= t_valid) continue;
        const uint32_t src = base + S::kW + (uint32_t)j * S::kWTile;
        if (j < kTmemTiles) {
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t e[32];
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
              const int c = 4 * half + c4;
              uint4 lo, hi;
              expand16(lds128(src + sw128_offset((uint32_t)row, (uint32_t)c)), lo, hi);
              e[8 * c4 + 0] = lo.x; e[8 * c4 + 1] = lo.y; e[8 * c4 + 2] = lo.z; e[8 * c4 + 3] = lo.w;
              e[8 * c4 + 4] = hi.x; e[8 * c4 + 5] = hi.y; e[8 * c4 + 6] = hi.z; e[8 * c4 + 7] = hi.w;
            }
            tmem_st32(tmem + 64u * (uint32_t)j + 32u * (uint32_t)half + lane_off, e);
          }
        } else {
#pragma unroll
          for (int c = 0; c < 8; ++c) t3[c] = lds128(src + sw128_offset((uint32_t)row, (uint32_t)c));
        }
      }
    }
    bar_sync_workers();  // tiles 0 and 1 are read: their staging may be overwritten
    if constexpr (S::kL1Here < 4) {
      // the packed tiles 2 and 3 are read too: L1^T chunk 3 into their tail
      // (its bytes were counted on l1_full with the others)
      if (tid == 0) {
        fence_proxy_async_smem();
        tma_load_2d(smem + S::kL1Hi, &map_l1, l1_full, kbase + 192, 0, policy_evict_last());
      }
    }
    if (ok && h == 1 && t_valid > kTmemTiles) {
      // tile 3: packed chunk c -> int8 chunks 2 (c % 4), +1 of k-block c / 4
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        uint4 lo, hi;
        expand16(t3[c], lo, hi);
        const uint32_t dst = base + S::kA3 + (uint32_t)(c >> 2) * S::kA3Block;
        sts128(dst + sw128_offset((uint32_t)row, (uint32_t)(2 * (c & 3))), lo);
        sts128(dst + sw128_offset((uint32_t)row, (uint32_t)(2 * (c & 3) + 1)), hi);
      }
    }
    tmem_st_wait();

    // ---- 2. rotation of tokens warp and warp + 8, partial absmax
    ok = workers_wait<false>(x_full, p.status, abort_flag, verdict) && ok;
    float v[2][8];
    float am_part[2] = {0.f, 0.f};
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t = warp + 8 * tt;
      const uint4 u = lds128(base + S::kX + (uint32_t)(lane >> 3) * S::kXChunk +
                             sw128_offset((uint32_t)t, (uint32_t)(lane & 7)));
      const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[tt][2 * e] = __uint_as_float(w4[e] << 16);
        v[tt][2 * e + 1] = __uint_as_float(w4[e] & 0xFFFF0000u);
      }
    }
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      apply_signs<8>(v[tt], p.signs, kbase + 8 * lane);  // x D (randomized Hadamard)
      fwht_warp<8>(v[tt], p.b);
    }
    if constexpr (kRhtN) {  // composed randomized Hadamards: D_2 H, D_3 H
      for (int i = 1; i < p.n_rht; ++i) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt) {
          apply_signs<8>(v[tt], p.signs + (size_t)i * (p.K / 32), kbase + 8 * lane);
          fwht_warp<8>(v[tt], p.b);
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      float a = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[tt][i]));
      am_part[tt] = a;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
      am_part[0] = fmaxf(am_part[0], __shfl_xor_sync(0xffffffffu, am_part[0], o));
      am_part[1] = fmaxf(am_part[1], __shfl_xor_sync(0xffffffffu, am_part[1], o));
    }
    const uint32_t amax_stage = base + S::kSx + kMT * 4;  // this CTA's partials [16]
    if (lane == 0) {
      stsf(amax_stage + (uint32_t)(warp * 4), am_part[0]);
      stsf(amax_stage + (uint32_t)((warp + 8) * 4), am_part[1]);
    }
    cluster_wait_acquire();  // B0 complete: every peer is running
    bar_sync_workers();
    if (ok && tid < C * 4) {  // peer tid / 4 gets floats 4 (tid % 4) .. +3
      const uint32_t z = (uint32_t)(tid >> 2), qq = (uint32_t)(tid & 3);
      st_async_v4(dsmem_map(base + S::kAmax + (crank * kMT + 4u * qq) * 4u, z),
                  lds128(amax_stage + 16u * qq), dsmem_map(smem_u32(amax_bar), z));
    }

    // ---- 3. codes with the cluster-wide absmax -> the MMAs may start
    ok = workers_wait<true>(amax_bar, p.status, abort_flag, verdict) && ok;
#pragma unroll
    for (int tt = 0; tt < 2; ++tt) {
      const int t = warp + 8 * tt;
      float am = 0.f;
#pragma unroll
      for (int z = 0; z < kMaxC; ++z)
        if (z < C) am = fmaxf(am, ldsf(base + S::kAmax + (uint32_t)((z * kMT + t) * 4)));
      const CodeScale cs = code_scale(am);
      if (cs.pre != 1.f) {
#pragma unroll
        for (int i = 0; i < 8; ++i) v[tt][i] *= cs.pre;
      }
      uint32_t cb[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) cb[i] = code_bits(v[tt][i], cs.inv);
      const uint32_t lo = low_bytes4(cb[0], cb[1], cb[2], cb[3]);
      const uint32_t hi = low_bytes4(cb[4], cb[5], cb[6], cb[7]);
      // columns 8 lane .. +7: k-block lane / 16, byte (lane % 16) * 8 of the row
      sts64(base + S::kB + (uint32_t)(lane >> 4) * S::kBBlock +
                sw128_offset((uint32_t)t, (uint32_t)((lane & 15) >> 1)) + 8u * (uint32_t)(lane & 1),
            lo, hi);
      if (p.dbg_codes && t < p.M)
        *reinterpret_cast<uint2*>(p.dbg_codes + (size_t)t * p.K + kbase + 8 * lane) = make_uint2(lo, hi);
      if (lane == 0) {
        stsf(base + S::kSx + (uint32_t)(t * 4), am * p.scale_mul);
        if (p.dbg_sx && crank == 0 && t < p.M) p.dbg_sx[t] = am * p.scale_mul;
      }
    }
    fence_proxy_async_smem();  // codes and tile 3 -> tensor core reads
    tc_fence_before();         // TMEM weight stores -> the MMA issuer
    mbar_arrive(codes_ready);

    // ---- 4. X L1 partial over the slice (while the integer MMAs run) ->
    //         the owner of each token
    if constexpr (R > 0) {
      constexpr int kNt = R / 8;             // 8-column tiles of the rank: 2, 4 or 8
      constexpr int kKP = 8 / kNt;           // k-parts: 4, 2 or 1
      constexpr int kSteps = (kSlice / 16) / kKP;
      constexpr int kGrp = kSteps < 8 ? kSteps : 8;  // operands held at once
      const bool l1_ok = workers_wait<false>(l1_full, p.status, abort_flag, verdict);
      ok = ok && l1_ok;
      const int nt = warp % kNt, kp = warp / kNt;
      float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
#pragma unroll
      for (int g0 = 0; g0 < kSteps; g0 += kGrp) {
        uint32_t a[kGrp][4], bb[kGrp][2];
#pragma unroll
        for (int s3 = 0; s3 < kGrp; ++s3) {
          const int kk = (kp * kSteps + g0 + s3) * 16;
          const int mat = lane >> 3, trow = (lane & 7) + (mat & 1) * 8;
          const int ka = kk + (mat >> 1) * 8;
          ldmatrix_x4(a[s3], base + S::kX + (uint32_t)(ka >> 6) * S::kXChunk +
                                 sw128_offset((uint32_t)trow, (uint32_t)((ka & 63) >> 3)));
          const int l = lane & 15;
          const int jr = nt * 8 + (l & 7), kb2 = kk + (l >> 3) * 8;
          const int l1c = kb2 >> 6;  // 64-column chunk of the slice
          ldmatrix_x2(bb[s3], base + ((l1c < S::kL1Here) ? S::kL1 + (uint32_t)l1c * S::kL1Chunk : S::kL1Hi) +
                                  sw128_offset((uint32_t)jr, (uint32_t)((kb2 & 63) >> 3)));
        }
#pragma unroll
        for (int s3 = 0; s3 < kGrp; ++s3) mma_16816(acc[(g0 + s3) & 1], a[s3], bb[s3]);
      }
      // C fragment: tokens lane / 4 and lane / 4 + 8, columns nt 8 + 2 (lane % 4), +1
      const uint32_t part = base + S::kXl1Part;
      const int trw = lane >> 2, cc = nt * 8 + 2 * (lane & 3);
      stsf(part + (uint32_t)(((kp * kMT + trw) * R + cc) * 4), acc[0][0] + acc[1][0]);
      stsf(part + (uint32_t)(((kp * kMT + trw) * R + cc + 1) * 4), acc[0][1] + acc[1][1]);
      stsf(part + (uint32_t)(((kp * kMT + trw + 8) * R + cc) * 4), acc[0][2] + acc[1][2]);
      stsf(part + (uint32_t)(((kp * kMT + trw + 8) * R + cc + 1) * 4), acc[0][3] + acc[1][3]);
      bar_sync_workers();
      // k-parts summed in order; token t's row -> CTA t % C, slot (crank, t / C)
      constexpr int kR4 = R / 4;
      if (tid < kMT * kR4) {
        const int t = tid / kR4, c4 = tid - t * kR4;
        if (t < p.M) {
          uint4 u[kKP];
#pragma unroll
          for (int k = 0; k < kKP; ++k) u[k] = lds128(part + (uint32_t)(((k * kMT + t) * R + 4 * c4) * 4));
          float f[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int k = 0; k < kKP; ++k) {
            f[0] += __uint_as_float(u[k].x);
            f[1] += __uint_as_float(u[k].y);
            f[2] += __uint_as_float(u[k].z);
            f[3] += __uint_as_float(u[k].w);
          }
          const uint32_t owner = (uint32_t)(t % C);
          const uint32_t slot = (crank * (uint32_t)tpo + (uint32_t)(t / C)) * (uint32_t)R + 4u * c4;
          if (ok)
            st_async_v4(dsmem_map(base + S::kXl1Recv + slot * 4u, owner),
                        make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]),
                                   __float_as_uint(f[2]), __float_as_uint(f[3])),
                        dsmem_map(smem_u32(xl1p_bar), owner));
        }
      }

      // ---- 4b. owned tokens: X L1 = sum of the C partials (cluster order),
      //          bf16, to every CTA
      if (own_tok > 0) {
        const bool got = workers_wait<true>(xl1p_bar, p.status, abort_flag, verdict);
        constexpr int kR8 = R / 8;
        if (tid < own_tok * kR8) {
          const int li = tid / kR8, c8 = tid - li * kR8;
          const int t = (int)crank + C * li;
          float f[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) f[e] = 0.f;
#pragma unroll
          for (int z = 0; z < kMaxC; ++z) {
            if (z < C) {
              const uint32_t src = base + S::kXl1Recv + (uint32_t)(((z * tpo + li) * R + 8 * c8) * 4);
              const uint4 a0 = lds128(src), b0 = lds128(src + 16);
              f[0] += __uint_as_float(a0.x); f[1] += __uint_as_float(a0.y);
              f[2] += __uint_as_float(a0.z); f[3] += __uint_as_float(a0.w);
              f[4] += __uint_as_float(b0.x); f[5] += __uint_as_float(b0.y);
              f[6] += __uint_as_float(b0.z); f[7] += __uint_as_float(b0.w);
            }
          }
          const uint4 val = make_uint4(bf16x2(f[0], f[1]), bf16x2(f[2], f[3]), bf16x2(f[4], f[5]),
                                       bf16x2(f[6], f[7]));
          if (ok && got)
            for (int z = 0; z < C; ++z)
              st_async_v4(dsmem_map(base + S::kXl1B + (uint32_t)((t * R + 8 * c8) * 2), (uint32_t)z),
                          val, dsmem_map(smem_u32(xl1b_bar), (uint32_t)z));
        }
      }
    }

    // owner-side operands of the epilogue, loaded while the MMAs run: item
    // `tid` is channel tid % per, tokens 4 (tid / per) .. +3
    const bool fast_epi = per <= 64 && (kWorkers % per) == 0;
    const int c_own = fast_epi ? tid % per : 0;
    const int n_own = n0 + own_lo + c_own;
    // (rank 64 loads its L2^T row in the epilogue: held through the MMAs
    // its 32 registers would spill)
    constexpr int kPre = (R > 0 && R <= 32) ? R / 8 : 1;
    float sw_own = 0.f;
    uint4 l2_own[kPre];
#pragma unroll
    for (int i = 0; i < kPre; ++i) l2_own[i] = make_uint4(0u, 0u, 0u, 0u);
    if (fast_epi && tid < 4 * per && n_own < p.N) {
      sw_own = ldg_nc_f32(p.s_w + n_own);
      if constexpr (R > 0 && R <= 32) {
#pragma unroll
        for (int i = 0; i < R / 8; ++i) l2_own[i] = ldg_nc_v4(p.L2t + (size_t)n_own * R + 8 * i);
      }
    }

    // ---- 5. accumulators -> the channel's owner (int16 sums of this slice),
    //         each tile as soon as its MMAs are done
#pragma unroll
    for (int jj = 0; jj < 2; ++jj) {
      const int j = h + 2 * jj;
      if (j >= p.T) continue;  // warp-uniform
      // one lane of each warp polls; its warp-mates take its verdict
      bool got = true;
      if (lane == 0) got = mbar_wait(&acc_full[j], 0u, p.status, abort_flag);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      ok = ok && got;
      tc_fence_after();
      uint32_t a[16];
      if (j < t_valid && ok) {
        tmem_ld16(tmem + kColAcc + 16u * (uint32_t)j + lane_off, a);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) a[i] = 0u;
      }
      uint32_t pk[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        pk[i] = ((uint32_t)(((int)a[2 * i]) >> 4) & 0xFFFFu) | ((uint32_t)(((int)a[2 * i + 1]) >> 4) << 16);
      const int rg = 128 * j + row;             // channel within the group
      const int o = (rg * C) / G;               // its owner
      const int lo_o = (o * G + C - 1) / C;
      const uint32_t dst = dsmem_map(base + S::kKRecv +
                                         (uint32_t)(((int)crank * per_max + (rg - lo_o)) * kMT * 2),
                                     (uint32_t)o);
      const uint32_t rb = dsmem_map(smem_u32(part_bar), (uint32_t)o);
      if (ok) {
        st_async_v4(dst, make_uint4(pk[0], pk[1], pk[2], pk[3]), rb);
        st_async_v4(dst + 16u, make_uint4(pk[4], pk[5], pk[6], pk[7]), rb);
      }
    }

    // ---- 6. owner epilogue: Y[t][n] for the owned channels, four tokens
    //         per item (the waits' named barriers also make s_x of every
    //         token, written in step 3 by other threads, visible here)
    ok = workers_wait<true>(part_bar, p.status, abort_flag, verdict) && ok;
    if (R > 0) ok = workers_wait<true>(xl1b_bar, p.status, abort_flag, verdict) && ok;
    if (ok) {
      const int items = per * 4;
      for (int it = tid; it < items; it += kWorkers) {
        const int c = it % per, tq4 = it / per;
        const int n = n0 + own_lo + c;
        if (n >= p.N || 4 * tq4 >= p.M) continue;
        // split-K sums of tokens 4 tq4 .. +3: one 8-byte load per split
        int acc4[4] = {0, 0, 0, 0};
        uint2 u[kMaxC];
#pragma unroll
        for (int z = 0; z < kMaxC; ++z) {
          u[z] = make_uint2(0u, 0u);
          if (z < C) {
            const uint32_t ad = base + S::kKRecv + (uint32_t)(((z * per_max + c) * kMT + 4 * tq4) * 2);
            asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(u[z].x), "=r"(u[z].y) : "r"(ad));
          }
        }
#pragma unroll
        for (int z = 0; z < kMaxC; ++z) {  // split order
          acc4[0] += (int)(short)(u[z].x & 0xFFFFu);
          acc4[1] += ((int)u[z].x) >> 16;
          acc4[2] += (int)(short)(u[z].y & 0xFFFFu);
          acc4[3] += ((int)u[z].y) >> 16;
        }
        float sw = sw_own;
        uint4 l2[R > 0 ? R / 8 : 1];
        if constexpr (R > 0 && R <= 32) {
#pragma unroll
          for (int i = 0; i < R / 8; ++i) l2[i] = l2_own[i];
        }
        if (!fast_epi) sw = ldg_nc_f32(p.s_w + n);
        if (!fast_epi || R > 32) {
#pragma unroll
          for (int i = 0; i < R / 8; ++i) l2[i] = ldg_nc_v4(p.L2t + (size_t)n * R + 8 * i);
        }
#pragma unroll
        for (int e4 = 0; e4 < 4; ++e4) {
          const int t = 4 * tq4 + e4;
          if (t >= p.M) break;
          float lr = 0.f;
          if constexpr (R > 0) {
            const uint32_t xr = base + S::kXl1B + (uint32_t)(t * R * 2);
#pragma unroll
            for (int i = 0; i < R / 8; ++i) {
              const uint4 xa = lds128(xr + 16u * (uint32_t)i);
              const uint32_t xw[4] = {xa.x, xa.y, xa.z, xa.w};
              const uint32_t lw[4] = {l2[i].x, l2[i].y, l2[i].z, l2[i].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                lr = fmaf(__uint_as_float(xw[e] << 16), __uint_as_float(lw[e] << 16), lr);
                lr = fmaf(__uint_as_float(xw[e] & 0xFFFF0000u), __uint_as_float(lw[e] & 0xFFFF0000u), lr);
              }
            }
          }
          const float s_x = ldsf(base + S::kSx + (uint32_t)(t * 4));
          p.Y[(size_t)t * p.N + n] = __float2bfloat16_rn(sw * s_x * (float)acc4[e4] + lr);
          if (p.dbg_acc) p.dbg_acc[(size_t)t * p.N + n] = acc4[e4];
        }
      }
    }
    // every store this thread makes into other CTAs has been issued: the
    // teardown's cluster barrier only waits for the peers to get here
    cluster_arrive_rel();
  }

  // ---- teardown: no peer writes here any more (every incoming byte was
  // waited for), and every peer has issued its last store
  tc_fence_before();
  __syncthreads();
  cluster_wait_acquire();
  if (warp == kCtrlWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool layer_decode2_supported(int M, int N, int K, int r, int had_block) {
  (void)N;
  // rank 64: clusters that divide 16 (its X L1 exchange holds 16 token slots)
  return M >= 1 && M <= kMT && (r == 0 || r == 16 || r == 32 || (r == 64 && K > 0 && K % kSlice == 0 && 16 % (K / kSlice) == 0)) &&
         K % kSlice == 0 && K / kSlice <= kMaxC && had_block >= 1 && had_block <= kSlice;
}

cudaError_t launch_layer_decode2(const LayerArgs& a, cudaStream_t stream, int8_t* dbg_codes,
                                 float* dbg_sx, int32_t* dbg_acc) {
  if (!layer_decode2_supported(a.M, a.N, a.K, a.r, a.had_block)) return cudaErrorInvalidValue;
  DecodeParams p{};
  p.s_w = a.s_w;
  p.L2t = reinterpret_cast<const __nv_bfloat16*>(a.L2t);
  p.Y = reinterpret_cast<__nv_bfloat16*>(a.Y);
  p.status = reinterpret_cast<uint32_t*>(a.ws);
  p.dbg_codes = dbg_codes;
  p.dbg_sx = dbg_sx;
  p.dbg_acc = dbg_acc;
  p.signs = a.signs;
  p.n_rht = a.signs ? a.n_rht : 1;
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.r = a.r;
  p.b = a.had_block;
  p.C = a.K / kSlice;
  p.scale_mul = (float)(1.0 / (7.0 * pow(sqrt((double)a.had_block), (double)p.n_rht)));
  // tiles per CTA: spread the channel tiles over the groups the SMs hold,
  // at most kMaxT per CTA
  const int tiles = (a.N + 127) / 128;
  const int groups_max = std::max(1, num_sms() / p.C);
  p.T = std::min(kMaxT, std::max(1, (tiles + groups_max - 1) / groups_max));
  const int groups = (tiles + p.T - 1) / p.T;
  CUtensorMap map_w, map_x, map_l1;
  if (!encode_tiled_2d(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, (uint64_t)(a.K / 2),
                       (uint64_t)a.N, (uint64_t)(a.K / 2), 128u, 128u,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (!encode_tiled_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.X, (uint64_t)a.K,
                       (uint64_t)a.M, (uint64_t)a.K * 2, 64u, (uint32_t)kMT,
                       CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (a.r > 0) {
    if (!encode_tiled_2d(&map_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L1t, (uint64_t)a.K,
                         (uint64_t)a.r, (uint64_t)a.K * 2, 64u, (uint32_t)a.r,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    map_l1 = map_x;  // never read
  }
  using KernelFn = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, DecodeParams);
  const int ri = (a.r == 64 ? 3 : a.r / 16) + (p.n_rht > 1 ? 4 : 0);
  const KernelFn fns[8] = {w4a4_lr_decode_kernel<0, false>, w4a4_lr_decode_kernel<16, false>,
                           w4a4_lr_decode_kernel<32, false>, w4a4_lr_decode_kernel<64, false>,
                           w4a4_lr_decode_kernel<0, true>,  w4a4_lr_decode_kernel<16, true>,
                           w4a4_lr_decode_kernel<32, true>, w4a4_lr_decode_kernel<64, true>};
  const uint32_t allocs[8] = {Sm<0>::kAlloc, Sm<16>::kAlloc, Sm<32>::kAlloc, Sm<64>::kAlloc,
                              Sm<0>::kAlloc, Sm<16>::kAlloc, Sm<32>::kAlloc, Sm<64>::kAlloc};
  const KernelFn fn = fns[ri];
  static uint64_t attr_set[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set[ri] >> dev & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)allocs[ri]);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set[ri] |= uint64_t(1) << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.C, groups, 1);
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = allocs[ri];
  cfg.stream = stream;
  cudaLaunchAttribute attr[3];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = tuning().pdl ? 1 : 0;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = p.C;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  // one CTA of a cluster per SM: the second slot of each SM is meant for
  // the next layer's CTA, not for a second CTA of this layer
  attr[2].id = cudaLaunchAttributeClusterSchedulingPolicyPreference;
  attr[2].val.clusterSchedulingPolicyPreference = cudaClusterSchedulingPolicySpread;
  cfg.attrs = attr;
  cfg.numAttrs = 3;
  return cudaLaunchKernelEx(&cfg, fn, map_w, map_x, map_l1, p);
}

}  // namespace tq
