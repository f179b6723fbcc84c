// tq_gemm_a8.cu -- the W4A4 + low-rank GEMM for many tokens, with the
// activation codes stored one per byte.
//
// tcgen05 has no dense int4 kind, so both operands must reach the tensor core
// as int8.  Expanding both in shared memory costs more shared-memory
// bandwidth per k-block than the MMA has cycles (the packed-activation GEMM
// in tq_gemm.cu is bound by it at large M).  Here:
//
//   * the token codes arrive as int8 (tq_quantize_act_i8), so TMA writes them
//     straight into the MMA's B operand layout (128-byte swizzle, K-major);
//   * the packed int4 weights are expanded in registers and written to tensor
//     memory with tcgen05.st: the MMA reads its A operand from TMEM, so the
//     expanded weights never touch shared memory.  A nibble becomes the byte
//     16*q, the codes stay q, so the INT32 accumulator holds 16 * sum(qx qw)
//     exactly (|acc| <= 16*49*K < 2^31); the epilogue shifts it back.
//
// Tile: 128 channels (MMA M = TMEM lanes) x 192 tokens (MMA N).  TMEM:
// INT32 accumulator [192] | four 32-column A buffers | fp32 low-rank [192].
// Persistent CTAs walk the tiles; a 3-stage TMA ring carries two k-blocks of
// tokens and weights per stage, then the low-rank chunks (64 columns of
// bf16(XL1) and L2^T per stage, kind::f16 into the low-rank accumulator).
//
// Schedule.  Where the tiles fill whole waves of the CTAs well (or without
// scratch in the workspace) CTA c takes tiles c, c + G, ...  Otherwise (stream-K) the
// tiles x stages of k-blocks are dealt out in tile order as equal ranges of
// stages, so no CTA idles through a last partial wave: a tile split between
// CTAs is finished by the CTA holding its first stage (which also runs the
// low-rank stages and the epilogue); each other CTA holding part of it (its
// range starts inside that tile, so the part is the first thing it computes)
// stores its INT32 partial sums in the workspace and raises one flag per
// epilogue warp.  INT32 addition is exact, so Y does not depend on the split.
//
// Warp 0: TMA producer.  Warp 1: TMEM allocation and MMA issue.  Warps 2-9:
// weight expansion into TMEM, then the epilogue of the tile (warp w owns
// lanes 32*(w%4)..: channel rows; warps w and w+4 split the k-blocks and the
// epilogue's token chunks).  No TMA multicast.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

namespace {

constexpr int kCh = 128;           // channels per tile (MMA M)
constexpr int kTkMax = 192;        // tokens per tile (MMA N)
constexpr int kKb = 128;           // codes per k-block
constexpr int kNS = 3;             // stages
// warps 2-9 expand the weights and run the epilogue, two per TMEM lane
// quarter: warps 2-5 take the first k-block of each stage, warps 6-9 the
// second, and the two halves split the epilogue's token chunks
constexpr int kConvWarpsA8 = 8;
constexpr int kConvThreadsA8 = kConvWarpsA8 * 32;
constexpr int kThreadsA8 = 64 + kConvThreadsA8;
constexpr int kQuarterThreads = 128;  // one warp per lane quarter: the writers of a k-block
constexpr uint32_t kColAcc = 0;    // INT32 accumulator, TK columns
// TMEM (512 columns): INT32 accumulator [TK] | A operand buffers, 32 columns
// each (one int8 weight k-block) | fp32 low-rank accumulator [TK]; a narrower
// token tile leaves room for more weight buffers in flight.
template <int TK>
struct A8Tmem {
  static constexpr int kNA = (512 - 2 * TK) / 32;  // 4, 6 or 8
  static constexpr uint32_t kColA = TK;
  static constexpr uint32_t kColLr = TK + 32 * kNA;
  static_assert(kColLr + TK <= 512, "TMEM columns");
};

struct A8Params {
  const float* s_x;    // [M]
  const float* s_w;    // [N]
  __nv_bfloat16* Y;    // [M][N]
  uint32_t* status;
  int M, N, K, r;
  int kb_total, n_st, n_lr;  // k-blocks, k-block stages, low-rank stages per tile
  int tiles_m, tiles;        // token tiles, all tiles
  int swiglu;                // Y[t][c] = silu(y[t][2c]) * y[t][2c+1], Y is [M][N/2]
  const float* z_x;          // asymmetric codes (code - 8): [M] zero-points, or null
  const int32_t* wsum;       //   [N] sums of each channel's weight codes
  const float* s_xl1;        // INT4 low-rank branch: [M] scales of the requantized X L1
  const float* s_l2;         //   and [N] of L2; the low-rank accumulator holds integers
  int sk;                    // stream-K schedule
  long long w_st;            //   tiles * n_st stages, dealt out as equal ranges
  int32_t* part;             //   [gridDim.x][128][TK] INT32 partial sums
  uint32_t* flags;           //   [gridDim.x][8] partial ready (one per epilogue warp)
};

// The segments of a CTA: (tile, stages [st0, st1) of its n_st).
struct SegIter {
  long long u, u_end;  // stream-K: this CTA's range of stages
  int tile;            // otherwise: next tile
  __device__ explicit SegIter(const A8Params& p) {
    u = (long long)blockIdx.x * p.w_st / gridDim.x;
    u_end = (long long)(blockIdx.x + 1) * p.w_st / gridDim.x;
    tile = blockIdx.x;
  }
  __device__ bool next(const A8Params& p, int& t, int& st0, int& st1) {
    if (p.sk) {
      if (u >= u_end) return false;
      t = (int)(u / p.n_st);
      st0 = (int)(u - (long long)t * p.n_st);
      st1 = (int)min((long long)p.n_st, (long long)st0 + (u_end - u));
      u += st1 - st0;
      return true;
    }
    if (tile >= p.tiles) return false;
    t = tile;
    st0 = 0;
    st1 = p.n_st;
    tile += gridDim.x;
    return true;
  }
};

// First stage of CTA c's stream-K range.
__device__ __forceinline__ long long sk_begin(const A8Params& p, int c) {
  return (long long)c * p.w_st / gridDim.x;
}

// Shared memory (offsets from the 1024-aligned base).  Stage s: tokens
// [2 k-blocks][TK rows][128 B] then packed weights [128 rows][128 B]
// (2 k-blocks).  A low-rank stage holds bf16(XL1) [TK][64] in the first token
// sub-tile and L2^T [128][64] in the weight part.
template <int TK>
struct A8Smem {
  static constexpr uint32_t kTokSub = TK * 128;             // 24 KB at TK = 192
  static constexpr uint32_t kWBytes = kCh * 128;            // 16 KB
  static constexpr uint32_t kStage = 2 * kTokSub + kWBytes;  // 64 KB
  // epilogue buffers per converter warp: a [32 tokens][40 bf16] transpose
  // buffer (SwiGLU), or two [32 tokens][32 bf16] tiles in the 64-byte
  // swizzle of the Y tensor map (the TMA store's source, alternating)
  static constexpr uint32_t kYRow = 80;
  static constexpr uint32_t kYTile = 2048;
  static constexpr uint32_t kYWarp = 2 * kYTile;
  static constexpr uint32_t kYBuf = kNS * kStage;
  static constexpr uint32_t kBar = kYBuf + kConvWarpsA8 * kYWarp;
  // full[kNS], empty[kNS], a_full[kNA], a_empty[kNA], acc_full, acc_empty
  static constexpr uint32_t kNumBars = 2 * kNS + 2 * A8Tmem<TK>::kNA + 2;
  static constexpr uint32_t kMisc = kBar + kNumBars * 8;
  static constexpr uint32_t kBytes = kMisc + 16;
  static constexpr uint32_t kAlloc = kBytes + 1024;
};
static_assert(A8Smem<kTkMax>::kAlloc <= 227 * 1024, "a8 GEMM shared memory");
static_assert(A8Smem<kTkMax>::kYBuf % 1024 == 0 && A8Smem<kTkMax>::kYWarp >= 32 * A8Smem<kTkMax>::kYRow,
              "Y tiles 1024-B aligned; the SwiGLU transpose buffer fits a warp's share");

// (float) n for |n| < 2^22, exactly, on the FMA pipe: n added to the bit
// pattern of 1.5 * 2^23 is the float 1.5 * 2^23 + n (the spacing there is
// 1), and the subtraction is exact.
__device__ __forceinline__ float int22_to_float(int n) {
  return __int_as_float(n + 0x4B400000) - 12582912.f;
}

__device__ __forceinline__ uint4 ld_shared_v4_a8(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// Epilogue variants, one instantiation each (the plain one carries no code
// or registers of the others)
enum { kEpiPlain = 0, kEpiSwiglu = 1, kEpiAsym = 2, kEpiQlr = 3 };

template <int TK, int EPI>
__global__ void __launch_bounds__(kThreadsA8, 1)
    w4a4_lr_gemm_a8_kernel(const __grid_constant__ CUtensorMap map_t,   // tokens int8 [M][K]
                           const __grid_constant__ CUtensorMap map_w,   // weights [N][K/2]
                           const __grid_constant__ CUtensorMap map_xb,  // bf16(XL1) [M][r]
                           const __grid_constant__ CUtensorMap map_l2,  // L2^T [N][r]
                           const __grid_constant__ CUtensorMap map_y,   // Y [M][N] (not SwiGLU)
                           const A8Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  using L = A8Smem<TK>;
  constexpr int kNA = A8Tmem<TK>::kNA;
  constexpr uint32_t kColA = A8Tmem<TK>::kColA;
  constexpr uint32_t kColLr = A8Tmem<TK>::kColLr;
  static_assert(TK % 32 == 0 && TK >= 128 && TK <= kTkMax, "token tile (the epilogue takes 32 tokens at a time)");
  static_assert(L::kTokSub % 1024 == 0 && L::kStage % 1024 == 0, "1024-B aligned atoms");

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kNS;
  uint64_t* a_full = bars + 2 * kNS;
  uint64_t* a_empty = a_full + kNA;
  uint64_t* acc_full = a_full + 2 * kNA;
  uint64_t* acc_empty = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::kMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::kMisc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kNS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kNA; ++i) {
      mbar_init(&a_full[i], kQuarterThreads);
      mbar_init(&a_empty[i], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, kConvThreadsA8);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_t);
    tma_prefetch_desc(&map_w);
    if (EPI != kEpiSwiglu) tma_prefetch_desc(&map_y);
    if (p.r > 0) {
      tma_prefetch_desc(&map_xb);
      tma_prefetch_desc(&map_l2);
    }
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ======================================================== TMA producer
    if (lane == 0) {
      const uint64_t pol_w = policy_evict_first();  // weights: streamed once per token tile
      const uint64_t pol_t = policy_evict_last();   // tokens: reused by every channel tile
      bool waited = false;                          // the weights need no predecessor
      int it = 0;
      SegIter seg(p);
      int tile, st0, st1;
      while (!*abort_flag && seg.next(p, tile, st0, st1)) {
        const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
        const int n_lr = st0 == 0 ? p.n_lr : 0;  // the finishing CTA runs the low-rank stages
        for (int j = 0; j < st1 - st0 + n_lr; ++j, ++it) {
          const int s = it % kNS;
          if (!mbar_wait(&empty[s], ((uint32_t)(it / kNS) & 1u) ^ 1u, p.status, abort_flag)) break;
          uint8_t* sp = smem + (uint32_t)s * L::kStage;
          if (j < st1 - st0) {
            const int st = st0 + j;
            const int kb = 2 * st;
            const bool two = kb + 1 < p.kb_total;
            mbar_arrive_expect_tx(&full[s], L::kWBytes + (two ? 2u : 1u) * L::kTokSub);
            tma_load_2d(sp + 2 * L::kTokSub, &map_w, &full[s], st * 128, tn * kCh, pol_w);
            if (!waited) {
              pdl_wait();  // token codes come from the preceding kernel
              waited = true;
            }
            tma_load_2d(sp, &map_t, &full[s], kb * kKb, tm * TK, pol_t);
            if (two) tma_load_2d(sp + L::kTokSub, &map_t, &full[s], (kb + 1) * kKb, tm * TK, pol_t);
          } else {
            const int c = j - (st1 - st0);  // 64-column low-rank chunk
            mbar_arrive_expect_tx(&full[s], L::kWBytes + L::kTokSub);
            if (!waited) {
              pdl_wait();
              waited = true;
            }
            tma_load_2d(sp + 2 * L::kTokSub, &map_l2, &full[s], c * 64, tn * kCh, pol_w);
            tma_load_2d(sp, &map_xb, &full[s], c * 64, tm * TK, pol_t);
          }
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ========================================================== MMA issuer
    const uint32_t id_i8 = idesc_i8_s32(TK);
    const uint32_t id_bf = idesc_bf16_f32(TK);
    int it = 0, ab = 0, tcount = 0;
    bool alive = true;
    SegIter seg(p);
    int tile, st0, st1;
    for (; alive && !*abort_flag && seg.next(p, tile, st0, st1); ++tcount) {
      const int n_lr = st0 == 0 ? p.n_lr : 0;
      // the epilogue has drained the accumulators of the previous segment
      if (!mbar_wait(acc_empty, ((uint32_t)tcount & 1u) ^ 1u, p.status, abort_flag)) break;
      tc_fence_after();
      for (int j = 0; j < st1 - st0 + n_lr && alive; ++j, ++it) {
        const int s = it % kNS;
        if (!mbar_wait(&full[s], (uint32_t)(it / kNS) & 1u, p.status, abort_flag)) {
          alive = false;
          break;
        }
        const uint32_t sp = base + (uint32_t)s * L::kStage;
        if (j < st1 - st0) {
          const int st = st0 + j;
          for (int sub = 0; sub < 2 && 2 * st + sub < p.kb_total; ++sub, ++ab) {
            const int u = ab % kNA;
            if (!mbar_wait(&a_full[u], (uint32_t)(ab / kNA) & 1u, p.status, abort_flag)) {
              alive = false;
              break;
            }
            tc_fence_after();
            if (lane == 0) {
              const uint64_t db = sdesc_sw128(sp + (uint32_t)sub * L::kTokSub);
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)  // K = 32 int8 = 8 TMEM columns per step
                mma_i8_tmem_a(tmem + kColAcc, tmem + kColA + 32u * (uint32_t)u + 8u * (uint32_t)kk,
                              db + 2 * kk, id_i8, (st > st0 || sub > 0 || kk > 0) ? 1u : 0u);
              mma_commit(&a_empty[u]);
            }
            __syncwarp();
          }
        } else {
          tc_fence_after();
          if (lane == 0) {
            const int c = j - (st1 - st0);
            const uint64_t da = sdesc_sw128(sp + 2 * L::kTokSub);  // L2^T chunk [128][64]
            const uint64_t db = sdesc_sw128(sp);                    // bf16(XL1) chunk [192][64]
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // K = 16 bf16 = 32 B per step
              mma_bf16(tmem + kColLr, da + 2 * kk, db + 2 * kk, id_bf, (c > 0 || kk > 0) ? 1u : 0u);
          }
          __syncwarp();
        }
        if (lane == 0) mma_commit(&empty[s]);
        __syncwarp();
      }
      if (lane == 0) mma_commit(acc_full);
      __syncwarp();
    }
  } else {
    // =============================== weight expansion into TMEM, epilogue
    const int q = warp & 3;                          // TMEM lane quarter
    const int half = (warp - 2) >> 2;                // which k-block of a stage
    const int row = q * 32 + lane;                   // channel row of the tile
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    const uint32_t x7 = (uint32_t)row & 7u;
    // every variant but SwiGLU reads the accumulators in the 16x256b
    // fragment layout and stores Y through stmatrix (no shuffles)
    constexpr bool kFrag = EPI != kEpiSwiglu;
    pdl_wait();  // s_x comes from the preceding kernel
    int it = 0, ab = 0, tcount = 0, n_ystores = 0;
    bool alive = true;
    SegIter seg(p);
    int tile, st0, st1;
    for (; alive && !*abort_flag && seg.next(p, tile, st0, st1); ++tcount) {
      const int tm = tile % p.tiles_m, tn = tile / p.tiles_m;
      const int gc = tn * kCh + row;
      const float sw = (!kFrag && gc < p.N) ? __ldg(p.s_w + gc) : 0.f;  // SwiGLU's row scale
      // the epilogue's scales, requested now so that their latency hides
      // behind the main loop.  Fragment epilogue (every variant but SwiGLU):
      // this thread's tokens 8g + 2 (lane % 4) + {0, 1} of each of its 32-token
      // chunks (s_x, and z_x or s_xl1) and channels 16h + lane / 4 + 8s of the
      // warp's 32 (s_w, and wsum or s_L2), f = 2h + s.  SwiGLU: the token lane
      // of each chunk (entry 0).
      constexpr int kChunks = TK / 64;
      float sx_pre[kChunks][8], zx_pre[kChunks][8];
#pragma unroll
      for (int i = 0; i < kChunks; ++i) {
        const int tb = tm * TK + 32 * (half + 2 * i);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int t = kFrag ? tb + 8 * (e >> 1) + 2 * (lane & 3) + (e & 1) : tb + lane;
          const bool in = st0 == 0 && t < p.M && (kFrag || e == 0);
          sx_pre[i][e] = in ? __ldg(p.s_x + t) : 0.f;
          zx_pre[i][e] = (EPI == kEpiAsym && in) ? __ldg(p.z_x + t)
                         : (EPI == kEpiQlr && p.r > 0 && in) ? __ldg(p.s_xl1 + t)
                                                             : 0.f;
        }
      }
      float sw_f[4], sl2_f[4];
      int ws_f[4];
#pragma unroll
      for (int f = 0; f < 4; ++f) {
        const int c = tn * kCh + q * 32 + 16 * (f >> 1) + (lane >> 2) + 8 * (f & 1);
        const bool in = kFrag && st0 == 0 && c < p.N;
        sw_f[f] = in ? __ldg(p.s_w + c) : 0.f;
        ws_f[f] = (EPI == kEpiAsym && in) ? __ldg(p.wsum + c) : 0;
        sl2_f[f] = (EPI == kEpiQlr && p.r > 0 && in) ? __ldg(p.s_l2 + c) : 0.f;
      }
      // int4 -> int8 (16 * code) for this thread's channel row, one k-block
      // (32 TMEM columns) at a time; inside each 16-byte packed chunk the low
      // nibbles are codes 0-15 and the high nibbles codes 16-31 of the group
      for (int st = st0; st < st1 && alive; ++st, ++it) {
        const int s = it % kNS;
        if (!mbar_wait(&full[s], (uint32_t)(it / kNS) & 1u, p.status, abort_flag)) {
          alive = false;
          break;
        }
        const uint32_t wrow = base + (uint32_t)s * L::kStage + 2 * L::kTokSub + (uint32_t)row * 128u;
        const int nsub = (2 * st + 1 < p.kb_total) ? 2 : 1;
        const bool mine = half < nsub;  // this half's k-block exists in the stage
        uint4 w[4];
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4)
          if (mine) w[c4] = ld_shared_v4_a8(wrow + ((((uint32_t)(half * 4 + c4)) ^ x7) << 4));
        bool ok = true;
        if (mine) {
          uint32_t v[32];
#pragma unroll
          for (int c4 = 0; c4 < 4; ++c4) {
            const uint32_t ww[4] = {w[c4].x, w[c4].y, w[c4].z, w[c4].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              v[8 * c4 + e] = (ww[e] << 4) & 0xF0F0F0F0u;
              v[8 * c4 + 4 + e] = ww[e] & 0xF0F0F0F0u;
            }
          }
          const int u = (ab + half) % kNA;
          ok = __all_sync(0xffffffffu, mbar_wait(&a_empty[u],
                                                 ((uint32_t)((ab + half) / kNA) & 1u) ^ 1u,
                                                 p.status, abort_flag));
          if (ok) {
            tc_fence_after();
            tmem_st32(tmem + kColA + 32u * (uint32_t)u + lane_off, v);
          }
        }
        if (!ok) {
          alive = false;
          break;
        }
        tmem_st_wait();
        tc_fence_before();
        if (mine) mbar_arrive(&a_full[(ab + half) % kNA]);
        ab += nsub;
      }
      it += st0 == 0 ? p.n_lr : 0;  // low-rank stages go to the MMA only
      if (!alive) break;
      // ---- epilogue: Y[t][c] = s_x[t] s_w[c] (acc >> 4) + lr, bf16.  Each
      //      warp owns 32 channels; per 32 tokens it transposes its block
      //      through shared memory and stores whole 64-byte row segments.
      if (!__all_sync(0xffffffffu, mbar_wait(acc_full, (uint32_t)tcount & 1u, p.status, abort_flag)))
        break;
      tc_fence_after();
      const int ew = warp - 2;  // epilogue warp: its rows and token chunks are the same in every CTA
      if (st0 > 0) {
        // part of a tile another CTA finishes: this warp's INT32 sums to the
        // workspace, then its flag
        // (slot layout [chunk][8 x 16 bytes][row] in the layout of the
        // finishing CTA's loads: a warp's store of one 16-byte piece covers
        // 512 contiguous bytes)
        uint4* dst = reinterpret_cast<uint4*>(p.part + (size_t)blockIdx.x * kCh * TK);
        if constexpr (kFrag) {
          uint32_t a[kChunks][2][16];
#pragma unroll
          for (int i = 0; i < kChunks; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
              tmem_ld16x256_x4(tmem + kColAcc + (uint32_t)(32 * (half + 2 * i)) + lane_off +
                                   ((uint32_t)(16 * h) << 16), a[i][h]);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(acc_empty);  // the next segment's MMAs may start
#pragma unroll
          for (int i = 0; i < kChunks; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int k = 0; k < 4; ++k)
                dst[(((half + 2 * i) * 2 + h) * 4 + k) * kCh + q * 32 + lane] =
                    make_uint4(a[i][h][4 * k], a[i][h][4 * k + 1], a[i][h][4 * k + 2],
                               a[i][h][4 * k + 3]);
        } else {
          uint32_t a[kChunks][32];
#pragma unroll
          for (int i = 0; i < kChunks; ++i)
            tmem_ld32(tmem + kColAcc + (uint32_t)(32 * (half + 2 * i)) + lane_off, a[i]);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(acc_empty);  // the next segment's MMAs may start
#pragma unroll
          for (int i = 0; i < kChunks; ++i)
#pragma unroll
            for (int v = 0; v < 8; ++v)
              dst[((half + 2 * i) * 8 + v) * kCh + row] =
                  make_uint4(a[i][4 * v], a[i][4 * v + 1], a[i][4 * v + 2], a[i][4 * v + 3]);
        }
        __syncwarp();
        if (lane == 0) {
          __threadfence();
          st_release_gpu(p.flags + (size_t)blockIdx.x * kConvWarpsA8 + ew, 1u);
        }
        __syncwarp();
        continue;
      }
      // the CTAs whose ranges start inside this tile: their partials
      int c_lo = blockIdx.x + 1, c_hi = c_lo;
      if (st1 < p.n_st) {
        const long long tile_end = (long long)(tile + 1) * p.n_st;
        while (c_hi < (int)gridDim.x && sk_begin(p, c_hi) < tile_end) ++c_hi;
        bool ok = true;
        for (int c = c_lo; c < c_hi && ok; ++c)
          ok = flag_wait(p.flags + (size_t)c * kConvWarpsA8 + ew, 1u, p.status, abort_flag);
        if (!__all_sync(0xffffffffu, ok)) break;
      }
      const uint32_t ybuf = base + L::kYBuf + (uint32_t)(warp - 2) * L::kYWarp;
      const int gc0 = tn * kCh + q * 32;  // first channel of this warp
      if constexpr (kFrag) {
        const bool small_k = p.K <= 85504;  // 49 K < 2^22
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
          const int j = half + 2 * i;
          // this warp's tile buffers alternate over all its stores: the
          // store before the last one (same buffer) has read it
          const uint32_t ytile = base + L::kYBuf + (uint32_t)(warp - 2) * L::kYWarp +
                                 (uint32_t)(n_ystores & 1) * L::kYTile;
          if (lane == 0) bulk_wait_read_but1();
          __syncwarp();
          // a[h] / l[h]: lanes 16h .. 16h + 15 of the warp's quarter, 32 tokens
          uint32_t a[2][16], l[2][16];
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t lo = lane_off + ((uint32_t)(16 * h) << 16) + (uint32_t)(32 * j);
            tmem_ld16x256_x4(tmem + kColAcc + lo, a[h]);
            if (p.r > 0) tmem_ld16x256_x4(tmem + kColLr + lo, l[h]);
          }
          tmem_ld_wait();
          for (int c = c_lo; c < c_hi; ++c) {
            const uint4* src = reinterpret_cast<const uint4*>(p.part + (size_t)c * kCh * TK);
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const uint4 x = ld_cg_v4(src + ((j * 2 + h) * 4 + k) * kCh + q * 32 + lane);
                a[h][4 * k] += x.x;
                a[h][4 * k + 1] += x.y;
                a[h][4 * k + 2] += x.z;
                a[h][4 * k + 3] += x.w;
              }
          }
          const int t0 = tm * TK + 32 * j;
          // per group of 8 tokens, four 8x8 blocks (channels 8f .. 8f + 7 of
          // the warp's 32): this thread's two tokens of one channel each, the
          // stmatrix fragment of the channel x token block, stored transposed
          // as token rows of 8 channels
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            uint32_t P[4];
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              const int h = f >> 1, sb = f & 1;
              float y[2];
#pragma unroll
              for (int u = 0; u < 2; ++u) {
                const int rg = 4 * g + 2 * sb + u;  // register of (channel, token 8g + 2(lane%4) + u)
                const int acc = ((int)a[h][rg]) >> 4;
                // |acc| <= 49 K for symmetric codes
                const float facc = (EPI != kEpiAsym && small_k) ? int22_to_float(acc) : (float)acc;
                const float sx = sx_pre[i][2 * g + u];
                float v;
                // y = s_x s_w acc; asymmetric codes c = q - 8 with zero-point
                // z: sum q qw = acc + 8 wsum (exact), y = s_w (s_x (acc + 8
                // wsum) + z wsum); then the low-rank term: fp32 (bf16 branch),
                // or s_xl1 s_L2 times the exact integer sum of the INT4 branch
                if constexpr (EPI == kEpiAsym)
                  v = sw_f[f] * (sx * (float)(acc + 8 * ws_f[f]) + zx_pre[i][2 * g + u] * (float)ws_f[f]);
                else
                  v = sx * sw_f[f] * facc;
                if constexpr (EPI == kEpiQlr) {
                  if (p.r > 0) v += zx_pre[i][2 * g + u] * sl2_f[f] * __uint_as_float(l[h][rg]);
                } else {
                  if (p.r > 0) v += __uint_as_float(l[h][rg]);
                }
                y[u] = v;
              }
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(y[0], y[1]);
              P[f] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            // row 8g + lane % 8 (a token), 16-byte chunk lane / 8 (8
            // channels), in the 64-byte swizzle: chunk ^ ((row / 2) % 4)
            const uint32_t yr = (uint32_t)(8 * g + (lane & 7));
            stmatrix_x4_trans(ytile + yr * 64u + ((((uint32_t)(lane >> 3)) ^ ((yr >> 1) & 3u)) << 4),
                              P[0], P[1], P[2], P[3]);
          }
          fence_proxy_async_smem();  // the tile is read by the TMA store
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&map_y, ytile, gc0, t0);
            bulk_commit_group();
          }
          ++n_ystores;
        }
      } else {
        // SwiGLU: rows alternate gate (even lane) and up (odd lane)
#pragma unroll
        for (int i = 0; i < kChunks; ++i) {
          const int j = half + 2 * i;
          uint32_t a[32], l[32];
          tmem_ld32(tmem + kColAcc + (uint32_t)(32 * j) + lane_off, a);
          if (p.r > 0) tmem_ld32(tmem + kColLr + (uint32_t)(32 * j) + lane_off, l);
          const int t0 = tm * TK + 32 * j;
          const float sx_l = sx_pre[i][0];
          tmem_ld_wait();
          for (int c = c_lo; c < c_hi; ++c) {
            const uint4* src = reinterpret_cast<const uint4*>(p.part + (size_t)c * kCh * TK);
#pragma unroll
            for (int v = 0; v < 8; ++v) {
              const uint4 x = ld_cg_v4(src + (j * 8 + v) * kCh + row);
              a[4 * v] += x.x;
              a[4 * v + 1] += x.y;
              a[4 * v + 2] += x.z;
              a[4 * v + 3] += x.w;
            }
          }
          // y = s_x s_w acc + bf16(X L1) L2^T per element, then for each pair
          // of tokens (2i, 2i+1) one shuffle gives the even lane (g, u) of
          // token 2i and the odd lane those of token 2i+1, so every lane
          // computes 16 of the warp's 16 x 32 outputs; silu(g) = g / (1 +
          // e^-g) with the fast exponential and division (relative error
          // ~1e-6, far below the bf16 output's 2^-9)
          float y[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float sx = __shfl_sync(0xffffffffu, sx_l, e);
            y[e] = sx * sw * (float)(((int)a[e]) >> 4);
            if (p.r > 0) y[e] += __uint_as_float(l[e]);
          }
          const bool odd = lane & 1;
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            const float other = __shfl_xor_sync(0xffffffffu, odd ? y[2 * i2] : y[2 * i2 + 1], 1);
            const float g = odd ? other : y[2 * i2];
            const float u = odd ? y[2 * i2 + 1] : other;
            const __nv_bfloat16 h = __float2bfloat16_rn(__fdividef(g, 1.f + __expf(-g)) * u);
            const int e = 2 * i2 + (odd ? 1 : 0);  // this lane's token
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(ybuf + (uint32_t)e * L::kYRow + (uint32_t)(lane & ~1)),
                         "h"(*reinterpret_cast<const unsigned short*>(&h))
                         : "memory");
          }
          __syncwarp();
          const int n_out = p.N / 2;
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const int idx = lane + 32 * k;      // 32 token rows x 2 16-byte parts
            const int e = idx >> 1, part = idx & 1;
            const uint4 v = ld_shared_v4_a8(ybuf + (uint32_t)e * L::kYRow + (uint32_t)part * 16u);
            const int t = t0 + e, c = gc0 / 2 + part * 8;
            if (t < p.M && c < n_out)
              *reinterpret_cast<uint4*>(p.Y + (size_t)t * n_out + c) = v;
          }
          __syncwarp();
        }
      }
      // the partials are consumed: clear their flags for the next launch
      if (lane == 0)
        for (int c = c_lo; c < c_hi; ++c) p.flags[(size_t)c * kConvWarpsA8 + ew] = 0u;
      tc_fence_before();
      mbar_arrive(acc_empty);
    }
  }

  if (EPI != kEpiSwiglu && warp >= 2 && lane == 0) bulk_wait_all();  // Y tiles written
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

namespace {

// stream-K scratch: [kSkMaxCtas][8] flags, then [kSkMaxCtas][128][192] INT32
constexpr int kSkMaxCtas = 160;
constexpr size_t kSkFlagBytes = (size_t)kSkMaxCtas * kConvWarpsA8 * 4;
constexpr size_t kSkPartBytes = (size_t)kSkMaxCtas * kCh * kTkMax * 4;
static_assert(kSkFlagBytes % 256 == 0, "partials 256-byte aligned");

template <int TK, int EPI>
cudaError_t launch_gemm_a8_tk(const GemmA8Args& a, A8Params p, cudaStream_t stream) {
  p.tiles_m = (a.M + TK - 1) / TK;
  p.tiles = p.tiles_m * ((a.N + kCh - 1) / kCh);
  CUtensorMap map_t, map_w, map_xb, map_l2;
  if (!encode_tiled_2d(&map_t, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Xq8, (uint64_t)a.K, (uint64_t)a.M,
                       (uint64_t)a.K, 128, TK, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tiled_2d(&map_w, CU_TENSOR_MAP_DATA_TYPE_UINT8, a.Wq, (uint64_t)(a.K / 2),
                       (uint64_t)a.N, (uint64_t)(a.K / 2), 128, kCh, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (a.r > 0) {
    if (!encode_tiled_2d(&map_xb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.XL1b, (uint64_t)a.r,
                         (uint64_t)a.M, (uint64_t)a.r * 2, 64, TK, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_tiled_2d(&map_l2, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.L2t, (uint64_t)a.r,
                         (uint64_t)a.N, (uint64_t)a.r * 2, 64, kCh, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    map_xb = map_t;  // never read
    map_l2 = map_t;
  }
  CUtensorMap map_y = map_t;  // SwiGLU stores Y itself
  if (EPI != kEpiSwiglu &&
      !encode_tiled_2d(&map_y, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a.Y, (uint64_t)a.N, (uint64_t)a.M,
                       (uint64_t)a.N * 2, 32, 32, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  // stream-K (see the schedule note at the top) where tile-by-tile CTAs
  // would leave much of their last wave idle: the waves' useful fraction
  // tiles / (G ceil(tiles / G)) below 0.85.  Above it the tile schedule was
  // measured faster (2048 x 4096 x 14336: 0.92, equal; 4096^3: 0.95, 3 %
  // faster; 2048 x 14336 x 4096: 0.79, stream-K 11 % faster).  One CTA per
  // SM, all resident at once.
  const int sms = num_sms();
  p.w_st = (long long)p.tiles * p.n_st;
  const int waves = (p.tiles + sms - 1) / sms;
  const bool uneven = (double)p.tiles < 0.85 * (double)waves * (double)sms;
  p.sk = (a.sk != nullptr && sms <= kSkMaxCtas && uneven && p.w_st >= sms) ? 1 : 0;
  p.flags = p.sk ? static_cast<uint32_t*>(a.sk) : nullptr;
  p.part = p.sk ? reinterpret_cast<int32_t*>(static_cast<uint8_t*>(a.sk) + kSkFlagBytes) : nullptr;
  static uint64_t attr_set = 0;
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set >> dev & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(w4a4_lr_gemm_a8_kernel<TK, EPI>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)A8Smem<TK>::kAlloc);
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(p.sk ? sms : std::min(p.tiles, sms), 1, 1);
  cfg.blockDim = dim3(kThreadsA8, 1, 1);
  cfg.dynamicSmemBytes = A8Smem<TK>::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = tuning().pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, w4a4_lr_gemm_a8_kernel<TK, EPI>, map_t, map_w, map_xb, map_l2, map_y,
                            p);
}

}  // namespace

size_t gemm_a8_sk_bytes() { return kSkFlagBytes + kSkPartBytes; }

cudaError_t launch_gemm_a8(const GemmA8Args& a, cudaStream_t stream) {
  A8Params p{};
  p.s_x = a.s_x;
  p.s_w = a.s_w;
  p.Y = reinterpret_cast<__nv_bfloat16*>(a.Y);
  p.status = reinterpret_cast<uint32_t*>(a.ws);
  p.M = a.M;
  p.N = a.N;
  p.K = a.K;
  p.r = a.r;
  p.kb_total = a.K / kKb;
  p.n_st = (p.kb_total + 1) / 2;
  p.n_lr = (a.r + 63) / 64;
  p.swiglu = a.swiglu;
  p.z_x = a.z_x;
  p.wsum = a.wsum;
  p.s_xl1 = a.s_xl1;
  p.s_l2 = a.s_l2;
  // 128 x 192 tiles: narrower token tiles (160, 128; more TMEM left for
  // weight buffers) were measured slower on every prefill shape but one,
  // where they won by under 1 %
  if (a.swiglu) return launch_gemm_a8_tk<kTkMax, kEpiSwiglu>(a, p, stream);
  if (a.z_x) return launch_gemm_a8_tk<kTkMax, kEpiAsym>(a, p, stream);
  if (a.s_xl1) return launch_gemm_a8_tk<kTkMax, kEpiQlr>(a, p, stream);
  return launch_gemm_a8_tk<kTkMax, kEpiPlain>(a, p, stream);
}

}  // namespace tq
