// tq_act_tc.cu -- the activation stage for many tokens on 5th-generation
// tensor cores.
//
// For a tile of 128 tokens the rotation of one 128-column block of X is a
// dense product with the block-diagonal Sylvester matrix,
//
//   Xh[t][j] = sum_k X[t][k] Hd[k][j],   Hd = diag(H_b, ..., H_b) (b <= 128),
//
// so it runs as tcgen05.mma kind::f16 (bf16 X, +-1 entries, fp32 TMEM
// accumulator) instead of warp shuffles, whose throughput bounds the
// butterfly kernel when M is large.  The products are exact; only the fp32
// summation order differs from the butterflies.  X.L1 is a second MMA on the
// same staged X tiles.  A cluster of C CTAs splits K:
//
//   pass 1  rotation of each block -> TMEM -> per-token partial absmax,
//           pushed to every CTA of the cluster (distributed shared memory)
//   pass 2  X tiles again (now from L2), rotation -> codes, packed into the
//           ABI layout and stored; X.L1 accumulated in TMEM over the slice
//   then    X.L1 partial rows pushed to the CTA that owns the row, summed in
//           cluster-rank order (deterministic) and stored.
//
// Warp 0: TMA producer.  Warp 1: TMEM allocation and MMA issue.  Warps 2-9:
// TMEM readers, two per lane quarter (warp w reads lanes 32*(w%4)..: token
// rows of the tile; warps 2-5 columns 0-63 of each block, warps 6-9 64-127).
// With a randomized Hadamard mask (x D H, the TORQUE page's RHT abstract: signs
// first, then the Hadamard), warps 10-13 negate the masked columns of each
// staged block in shared memory between the TMA's arrival and the MMAs.
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <algorithm>

#include "tq_act_common.cuh"
#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

namespace {

constexpr int kTok = 128;          // tokens per tile (MMA M)
constexpr int kBlk = 128;          // columns per block (MMA N of the rotation, MMA K)
constexpr int kMaxNS = 3;          // X / L1^T stages: three where they fit, else two
constexpr int kRot = 3;            // rotation accumulators in TMEM (128 columns each)
constexpr int kMaxC = 16;          // CTAs per cluster along K (above 8: non-portable size)
constexpr int kMaxRtc = 128;       // X L1 width computed beside the codes
constexpr int kMaxRx = 256;        // X L1 columns of one X-L1-only launch
// Readers: two warps per TMEM lane quarter, each taking half of a block's
// 128 columns (one warp per quarter left the code pass issue-bound).
constexpr int kEpiFirstWarp = 2;
constexpr int kEpiThreadsTc = 256;
constexpr int kThreadsTc = 32 * kEpiFirstWarp + kEpiThreadsTc;
// With a sign mask (randomized Hadamard, x D H): four more warps negate the
// masked columns of each staged block before its MMAs.
constexpr int kFlipFirstWarp = kEpiFirstWarp + kEpiThreadsTc / 32;
constexpr int kFlipThreads = 128;
template <bool kSigned>
constexpr int tc_threads() {
  return kThreadsTc + (kSigned ? kFlipThreads : 0);
}

struct TcParams {
  uint8_t* Xq;       // [M][K/2] packed codes, or null
  int8_t* Xq8;       // [M][K] one code per byte, or null
  float* s_x;        // [M]
  float* XL1;        // [M][r] fp32, or null
  __nv_bfloat16* XL1b;  // [M][r] rounded to bf16, or null
  int M, K, b, r;     // r: X L1 columns of this launch
  int r_ld, r_off;    // row stride of XL1 / XL1b, first column (and L1^T row) of this launch
  int xl1_only;       // X L1 only: no rotation, no codes, no s_x
  float* z_x;         // asymmetric codes: [M] zero-points (row minimum), or null
  float zmul;         // 1 / sqrt(b): the zero-point of the unnormalised transform
  int kb_total, nb;   // 128-column blocks in K, blocks per CTA
  float scale_mul;    // 1 / (7 sqrt(b)); asymmetric: 1 / (15 sqrt(b))
  const uint32_t* signs;  // [K / 32] words: bit k % 32 of word k / 32 negates column k, or null
};

// Shared memory (offsets from the 1024-aligned base).  Atoms are 128-byte
// swizzled K-major tiles of 64 bf16 columns.  A stage holds one X block and,
// when X L1 is computed, the matching L1^T block (2 atoms x r rows); an
// X-L1-only launch has no Hadamard operand.
// full, empty; rot_full, rot_empty; xl1_full; flipped (sign mask applied)
constexpr int kNumBarsTc = 3 * kMaxNS + 2 * kRot + 1;
struct TcLayout {
  uint32_t h, stage0, stage, amax, amin, bar, misc, bytes;
  int ns;  // stages
};
__host__ __device__ inline TcLayout tc_layout_ns(bool xl1_only, int r, int ns) {
  TcLayout L;
  L.ns = ns;
  L.h = 0;                                             // Hd^T: 2 atoms x 128 rows
  L.stage0 = xl1_only ? 0u : 2u * kBlk * 128u;
  L.stage = 2u * kTok * 128u + (uint32_t)r * 256u;     // X block + L1^T block
  L.amax = L.stage0 + (uint32_t)ns * L.stage;          // [C][2 halves][128] fp32: absmax, or max
  L.amin = L.amax + 2u * kMaxC * kTok * 4u;           // [C][2][128] fp32: min (asymmetric)
  L.bar = L.amin + 2u * kMaxC * kTok * 4u;
  L.misc = L.bar + kNumBarsTc * 8u;
  L.bytes = L.misc + 16u;
  return L;
}
// Three stages when they fit (r <= 80 with the rotation; measured 5-8 %
// faster than two at K >= 4096 and many tokens), else two.
constexpr uint32_t kSmemCap = 227u * 1024u;  // dynamic shared memory of one CTA
__host__ __device__ inline TcLayout tc_layout(bool xl1_only, int r) {
  const TcLayout L3 = tc_layout_ns(xl1_only, r, kMaxNS);
  return L3.bytes + 1024u <= kSmemCap ? L3 : tc_layout_ns(xl1_only, r, 2);
}
static_assert(2u * kBlk * 128u + 2u * (2u * kTok * 128u + kMaxRtc * 256u) + 4u * kMaxC * kTok * 4u +
                      kNumBarsTc * 8u + 16u + 1024u <= 227u * 1024u,
              "activation tile shared memory (codes)");
static_assert(2u * (2u * kTok * 128u + kMaxRx * 256u) + 4u * kMaxC * kTok * 4u + kNumBarsTc * 8u +
                      16u + 1024u <= 227u * 1024u,
              "activation tile shared memory (X L1 only)");
static_assert(kRot * kBlk + kMaxRtc <= 512 && kMaxRx <= 512, "tensor memory columns");
// the X L1 receive area [C][128][ceil(r/C)] reuses the stages after pass 2:
// 512 (r + C) bytes <= 2 (32 KB + 256 r) for every C <= 128

__device__ __forceinline__ void st_shared_v4_tc(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(v.x), "r"(v.y),
               "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ float ld_shared_f32_tc(uint32_t addr) {
  float v;
  asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(addr));
  return v;
}
__device__ __forceinline__ void cluster_arrive_rel() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
// 16-byte chunk c (0..15) of row `row` of a two-atom (128 bf16 columns) tile
// with `rows` rows per atom.
__device__ __forceinline__ uint32_t atom_off(uint32_t row, uint32_t c, uint32_t rows) {
  return (c >> 3) * rows * 128u + row * 128u + (((c & 7u) ^ (row & 7u)) << 4);
}

// Two fp32 products in one packed multiply, each rounded to nearest even as
// the scalar one.
__device__ __forceinline__ void mul2_rn(uint32_t& a, uint32_t& b, float s) {
  uint64_t x, sv;
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(a), "r"(b));
  asm("mov.b64 %0, {%1, %1};" : "=l"(sv) : "r"(__float_as_uint(s)));
  asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(x) : "l"(sv));
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(x));
}

// x D on a staged block: negate column k (bit k of the block's 128-bit mask
// m) in every row of a two-atom tile of `rows` rows (rows % 8 == 0).  Chunk
// ch of the tile is 16 bytes at tile + 16 ch: atom ch / (8 rows), row
// (ch / 8) % rows, stored chunk ch % 8, which holds columns 8 (ch % 8 ^ row
// % 8) .. +7 of the atom.  A sign flip is exact, so (x D) H and (x D)(D L1)
// = x L1 lose nothing.
__device__ __forceinline__ uint32_t sign_bits8(uint4 m, uint32_t k0) {
  const uint32_t w = (k0 & 64u) ? ((k0 & 32u) ? m.w : m.z) : ((k0 & 32u) ? m.y : m.x);
  return (w >> (k0 & 31u)) & 0xFFu;
}
__device__ __forceinline__ void flip_columns(uint32_t tile, uint32_t rows, uint4 m, uint32_t t) {
  const uint32_t n = 16u * rows;
  for (uint32_t c0 = t; c0 < n; c0 += 2u * kFlipThreads) {
    uint4 v[2];
    uint32_t bits[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t ch = c0 + (uint32_t)u * kFlipThreads;
      const uint32_t atom = ch >= 8u * rows ? 1u : 0u;
      const uint32_t k0 = 64u * atom + 8u * ((ch & 7u) ^ ((ch >> 3) & 7u));
      bits[u] = ch < n ? sign_bits8(m, k0) : 0u;
      if (ch < n)
        asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(v[u].x), "=r"(v[u].y), "=r"(v[u].z), "=r"(v[u].w)
                     : "r"(tile + 16u * ch));
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const uint32_t ch = c0 + (uint32_t)u * kFlipThreads;
      const uint32_t b = bits[u];
      // element 2e in the low half of word e, 2e + 1 in the high half
      v[u].x ^= ((b & 1u) << 15) | ((b & 2u) << 30);
      v[u].y ^= ((b & 4u) << 13) | ((b & 8u) << 28);
      v[u].z ^= ((b & 16u) << 11) | ((b & 32u) << 26);
      v[u].w ^= ((b & 64u) << 9) | ((b & 128u) << 24);
      if (ch < n) st_shared_v4_tc(tile + 16u * ch, v[u]);
    }
  }
}

template <bool kSigned>
__global__ void __launch_bounds__(tc_threads<kSigned>(), 1)
    quantize_act_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                           const __grid_constant__ CUtensorMap map_l1, const TcParams p) {
  constexpr int kThr = tc_threads<kSigned>();
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_addr = smem_u32(smem_raw);
  const uint32_t base = (raw_addr + 1023u) & ~1023u;
  uint8_t* smem = smem_raw + (base - raw_addr);
  const TcLayout L = tc_layout(p.xl1_only != 0, p.r);
  const bool xo = p.xl1_only != 0;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L.bar);
  uint64_t* full = bars;
  uint64_t* empty = bars + kMaxNS;
  uint64_t* rot_full = bars + 2 * kMaxNS;
  uint64_t* rot_empty = rot_full + kRot;
  uint64_t* xl1_full = rot_full + 2 * kRot;
  uint64_t* flipped = xl1_full + 1;  // [kMaxNS]: the stage's masked columns negated
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L.misc + 4);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const int tile = blockIdx.y;
  const int kb0 = (int)crank * p.nb;
  const int nb = max(0, min(p.nb, p.kb_total - kb0));  // blocks of this CTA
  const int r = p.r;
  const uint32_t l1_bytes = (uint32_t)r * 256u;         // one L1^T block, 2 atoms

  // X (and L1^T) loads: one pass over the slice for X-L1-only launches and
  // for CTAs of at most two blocks (whose rotations stay in the two TMEM
  // buffers until the codes are written), two passes (absmax, then codes)
  // otherwise
  const bool resident = !xo && nb <= 2;
  const int n_loads = (xo || resident) ? nb : 2 * nb;
  auto issue_load = [&](int i, uint64_t pol_x, uint64_t pol_w) {
    const int s = i % L.ns;
    const bool second = xo || resident || i >= nb;
    const int j = i < nb ? i : i - nb;
    const uint32_t st = base + L.stage0 + (uint32_t)s * L.stage;
    const bool with_l1 = second && r > 0;
    mbar_arrive_expect_tx(&full[s], 2u * kTok * 128u + (with_l1 ? l1_bytes : 0u));
    const int x = (kb0 + j) * kBlk;
    tma_load_2d(smem + (st - base), &map_x, &full[s], x, tile * kTok, pol_x);
    tma_load_2d(smem + (st - base) + kTok * 128, &map_x, &full[s], x + 64, tile * kTok, pol_x);
    if (with_l1) {
      const uint32_t l1 = (st - base) + 2u * kTok * 128u;
      tma_load_2d(smem + l1, &map_l1, &full[s], x, p.r_off, pol_w);
      tma_load_2d(smem + l1 + (uint32_t)r * 128u, &map_l1, &full[s], x + 64, p.r_off, pol_w);
    }
  };
  const int n_pre = min(L.ns, n_loads);  // stages requested in the prologue

  // ---------------------------------------------------------------- prologue
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < kMaxNS; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < kRot; ++i) {
      mbar_init(&rot_full[i], 1);
      mbar_init(&rot_empty[i], kEpiThreadsTc);
    }
    mbar_init(xl1_full, 1);
    if (kSigned)
      for (int i = 0; i < kMaxNS; ++i) mbar_init(&flipped[i], kFlipThreads);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&map_x);
    if (r > 0) tma_prefetch_desc(&map_l1);
    pdl_wait();  // X comes from the preceding kernel
    // the first stages go out now, before the operand set-up below (their
    // slots are free: nothing has used them yet)
    for (int i = 0; i < n_pre; ++i) issue_load(i, policy_evict_last(), policy_evict_first());
  }
  // Hd^T as the B operand of the rotation: row j (output column), column k;
  // Hd is symmetric.  +-1 (or 0 off the diagonal blocks), unnormalised.  One
  // 16-byte chunk (k = k0 .. k0+7, k0 % 8 == 0) at a time: for b >= 8 the
  // chunk lies in one block or none, and the parity of j & k splits into
  // that of j & k0 and that of j & e (e = k - k0), read from an 8-entry
  // pattern table indexed by j & 7.
  {
    const int bm = p.b - 1;
    constexpr unsigned long long kParity8 = 0x963C5AF066CCAA00ull;  // byte m: bit e = parity(m & e)
    for (int ch = threadIdx.x - 32; warp > 0 && ch < (xo ? 0 : kBlk * 16); ch += kThr - 32) {
      const int j = ch >> 4, c = ch & 15;
      const int k0 = c * 8;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (bm >= 7) {
        if (((j ^ k0) & ~bm) == 0) {
          const uint32_t flip = (__popc((unsigned)(j & k0 & bm)) & 1) ? 0xFFu : 0u;
          const uint32_t bits = ((uint32_t)(kParity8 >> (8 * (j & 7))) & 0xFFu) ^ flip;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = 0x3F803F80u | (((bits >> (2 * e)) & 1u) << 15) |
                   (((bits >> (2 * e + 1)) & 1u) << 31);
        }
      } else {  // blocks of 1, 2 or 4 columns: element by element
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const int k = k0 + e;
          if (((j ^ k) & ~bm) == 0)
            w[e >> 1] |= ((__popc((unsigned)(j & k & bm)) & 1) ? 0xBF80u : 0x3F80u) << (16 * (e & 1));
        }
      }
      st_shared_v4_tc(base + L.h + atom_off((uint32_t)j, (uint32_t)c, kBlk),
                      make_uint4(w[0], w[1], w[2], w[3]));
    }
  }
  fence_proxy_async_smem();
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  cluster_arrive_relaxed();  // B0: this CTA is running
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tmem_rot = tmem;                           // kRot x 128 columns
  const uint32_t tmem_xl1 = tmem + (xo ? 0u : kRot * kBlk);  // r columns
  pdl_launch_dependents();

  if (warp == 0) {
    // ======================================================== TMA producer
    cluster_wait_acquire();    // B0
    cluster_arrive_rel();      // B1 (nothing to publish)
    if (lane == 0) {
      const uint64_t pol_x = policy_evict_last();    // read again in pass 2
      const uint64_t pol_w = policy_evict_first();
      for (int i = n_pre; i < n_loads; ++i) {
        if (!mbar_wait(&empty[i % L.ns], ((uint32_t)(i / L.ns) & 1u) ^ 1u, nullptr, abort_flag))
          break;
        issue_load(i, pol_x, pol_w);
      }
    }
    __syncwarp();
    cluster_wait_acquire();    // B1
    cluster_arrive_rel();      // B2
    cluster_wait_acquire();
    cluster_arrive_rel();      // B3
    cluster_wait_acquire();
  } else if (warp == 1) {
    // ========================================================== MMA issuer
    cluster_wait_acquire();    // B0
    cluster_arrive_rel();      // B1
    const uint32_t id_rot = idesc_bf16_f32(kBlk);
    const uint32_t id_xl1 = idesc_bf16_f32(r > 0 ? r : 16);
    for (int i = 0; i < n_loads; ++i) {
      const int s = i % L.ns, u = i % kRot;
      const bool second = xo || resident || i >= nb;
      const int j = i < nb ? i : i - nb;
      if (!mbar_wait(kSigned ? &flipped[s] : &full[s], (uint32_t)(i / L.ns) & 1u, nullptr,
                     abort_flag))
        break;
      if (!xo && !mbar_wait(&rot_empty[u], ((uint32_t)(i / kRot) & 1u) ^ 1u, nullptr, abort_flag))
        break;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = base + L.stage0 + (uint32_t)s * L.stage;
#pragma unroll
        for (int kk = 0; kk < kBlk / 16; ++kk) {
          const uint32_t atom = (uint32_t)kk >> 2, ko = ((uint32_t)kk & 3u) * 2u;  // 32 B steps
          const uint64_t da = sdesc_sw128(st + atom * (kTok * 128u)) + ko;
          if (!xo) {
            const uint64_t dh = sdesc_sw128(base + L.h + atom * (kBlk * 128u)) + ko;
            mma_bf16(tmem_rot + (uint32_t)u * kBlk, da, dh, id_rot, kk > 0 ? 1u : 0u);
          }
          if (second && r > 0) {
            const uint64_t dl =
                sdesc_sw128(st + 2u * kTok * 128u + atom * ((uint32_t)r * 128u)) + ko;
            mma_bf16(tmem_xl1, da, dl, id_xl1, (j > 0 || kk > 0) ? 1u : 0u);
          }
        }
        mma_commit(&empty[s]);
        if (!xo) mma_commit(&rot_full[u]);
      }
      __syncwarp();
    }
    if (lane == 0 && r > 0) mma_commit(xl1_full);
    __syncwarp();
    cluster_wait_acquire();    // B1
    cluster_arrive_rel();      // B2
    cluster_wait_acquire();
    cluster_arrive_rel();      // B3
    cluster_wait_acquire();
  } else if (kSigned && warp >= kFlipFirstWarp) {
    // ==================================================== sign mask (x D)
    // every staged X block, and in the code pass its L1^T block, before the
    // MMAs read them (the MMA issuer waits on `flipped` instead of `full`)
    cluster_wait_acquire();    // B0
    cluster_arrive_rel();      // B1
    const uint32_t t = threadIdx.x - kFlipFirstWarp * 32;
    for (int i = 0; i < n_loads; ++i) {
      const int s = i % L.ns;
      const bool second = xo || resident || i >= nb;
      const int j = i < nb ? i : i - nb;
      if (!mbar_wait(&full[s], (uint32_t)(i / L.ns) & 1u, nullptr, abort_flag)) break;
      const uint4 m = __ldg(reinterpret_cast<const uint4*>(p.signs) + (kb0 + j));
      const uint32_t st = base + L.stage0 + (uint32_t)s * L.stage;
      flip_columns(st, kTok, m, t);
      if (second && r > 0) flip_columns(st + 2u * kTok * 128u, (uint32_t)r, m, t);
      fence_proxy_async_smem();  // generic-proxy writes -> the MMAs' reads
      mbar_arrive(&flipped[s]);
    }
    __syncwarp();
    cluster_wait_acquire();    // B1
    cluster_arrive_rel();      // B2
    cluster_wait_acquire();
    cluster_arrive_rel();      // B3
    cluster_wait_acquire();
  } else {
    // ===================================================== TMEM readers
    const int q = warp & 3;                       // TMEM lane quarter
    const int half = (warp - kEpiFirstWarp) >> 2;  // columns [64 half, 64 half + 64) of a block
    const int row = q * 32 + lane;                // token row in the tile
    const int grow = tile * kTok + row;
    const uint32_t lane_off = (uint32_t)(q * 32) << 16;
    cluster_wait_acquire();  // B0: peers are running before they are written to

    // ---- pass 1: partial absmax (asymmetric: min and max) of this token
    //      over the CTA's slice
    const bool asym = p.z_x != nullptr;
    float amax = 0.f, lo = __int_as_float(0x7f800000), hi = -__int_as_float(0x7f800000);
    for (int i = 0; i < (xo ? 0 : nb); ++i) {
      const int u = i % kRot;
      const bool ok = __all_sync(kFull, mbar_wait(&rot_full[u], (uint32_t)(i / kRot) & 1u, nullptr,
                                                  abort_flag));
      tc_fence_after();
      if (ok) {
#pragma unroll
        for (int g = 2 * half; g < 2 * half + 2; ++g) {
          uint32_t v[32];
          tmem_ld32(tmem_rot + (uint32_t)(u * kBlk + 32 * g) + lane_off, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float f = __uint_as_float(v[e]);
            amax = fmaxf(amax, fabsf(f));
            lo = fminf(lo, f);
            hi = fmaxf(hi, f);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&rot_empty[u]);
    }
    if (!xo)
      for (uint32_t z = 0; z < csize; ++z) {
        const uint32_t off = ((crank * 2u + (uint32_t)half) * kTok + (uint32_t)row) * 4u;
        dsmem_st_f32(dsmem_map(base + L.amax + off, z), asym ? hi : amax);
        if (asym) dsmem_st_f32(dsmem_map(base + L.amin + off, z), lo);
      }
    cluster_arrive_rel();  // B1: partial absmax delivered
    cluster_wait_acquire();
    float am = asym ? -__int_as_float(0x7f800000) : 0.f;
    float mn = __int_as_float(0x7f800000);
    for (uint32_t z = 0; z < 2u * csize; ++z) {  // every CTA's two halves
      am = fmaxf(am, ld_shared_f32_tc(base + L.amax + (z * kTok + (uint32_t)row) * 4u));
      if (asym) mn = fminf(mn, ld_shared_f32_tc(base + L.amin + (z * kTok + (uint32_t)row) * 4u));
    }
    // asymmetric: codes of (x - min) over the range max - min, in [0, 15]
    // (stored as code - 8), scale range / 15, zero-point min
    const float range = asym ? am - mn : am;
    if (!xo && crank == 0 && half == 0 && grow < p.M) {
      p.s_x[grow] = range * p.scale_mul;
      if (asym) p.z_x[grow] = mn * p.zmul;
    }
    CodeScale cs = code_scale(range);  // pre (2^64 for a tiny range) and 7 / (range pre)
    if (asym && range > 0.f) cs.inv = 15.f / (range * cs.pre);

    // ---- pass 2: the same rotation again -> codes in the packed layout
    //      (inside each 32-code group byte i = code i | code i+16 << 4)
    for (int i = nb; i < (xo ? nb : 2 * nb); ++i) {
      // resident: block i - nb is still in its buffer from pass 1
      const int u = resident ? i - nb : (i % kRot);
      const bool ok = resident ? !*abort_flag
                               : __all_sync(kFull, mbar_wait(&rot_full[u], (uint32_t)(i / kRot) & 1u,
                                                             nullptr, abort_flag));
      tc_fence_after();
      if (ok) {
        const size_t blk = (size_t)(kb0 + i - nb);
#pragma unroll
        for (int g = 2 * half; g < 2 * half + 2; ++g) {
          uint32_t v[32];
          tmem_ld32(tmem_rot + (uint32_t)(u * kBlk + 32 * g) + lane_off, v);
          tmem_ld_wait();
          uint32_t cb[32];
          if (asym) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              // RoundClip((x - min) / s) to [0, 15] with ties to even, as
              // code - 8 in the byte (one fp32 subtraction, one product)
              const float f = __uint_as_float(v[e]);
              float y = (f * cs.pre - mn * cs.pre) * cs.inv;
              y = fminf(fmaxf(y, 0.f), 15.f);
              cb[e] = __float_as_uint(__fadd_rn(y, 12582912.f)) - 8u;
            }
          } else {
            // code_bits of the values pass 1 took the absmax over (the MMA
            // recomputes them bit for bit, so the clip never acts): the
            // products two per packed multiply, the rounding adds one by one
            // (a packed add after a packed multiply was contracted into one
            // fma, whose single rounding moves exact fp32 ties)
            if (cs.pre != 1.f) {
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * cs.pre);
            }
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              mul2_rn(v[e], v[e + 1], cs.inv);
              cb[e] = __float_as_uint(__fadd_rn(__uint_as_float(v[e]), 12582912.f));
              cb[e + 1] = __float_as_uint(__fadd_rn(__uint_as_float(v[e + 1]), 12582912.f));
            }
          }
          if (p.Xq8 && !asym) {
            // one code per byte: staged per warp (the asymmetric min area,
            // unused here) as [32 rows][64 B], 16-byte chunks swizzled by
            // row, so that the global stores below cover whole sectors
            uint32_t w[8];
#pragma unroll
            for (int h = 0; h < 8; ++h)
              w[h] = low_bytes4(cb[4 * h], cb[4 * h + 1], cb[4 * h + 2], cb[4 * h + 3]);
            const uint32_t sb = base + L.amin + (uint32_t)(warp - kEpiFirstWarp) * 2048u +
                                (uint32_t)lane * 64u;
            const uint32_t sw = ((uint32_t)lane >> 1) & 3u;
            const uint32_t c0 = 2u * (uint32_t)(g - 2 * half);
            st_shared_v4_tc(sb + ((c0 ^ sw) << 4), make_uint4(w[0], w[1], w[2], w[3]));
            st_shared_v4_tc(sb + (((c0 + 1u) ^ sw) << 4), make_uint4(w[4], w[5], w[6], w[7]));
          }
          if (grow < p.M) {
            if (p.Xq8 && asym) {  // one code per byte, in column order
              uint32_t w[8];
#pragma unroll
              for (int h = 0; h < 8; ++h)
                w[h] = low_bytes4(cb[4 * h], cb[4 * h + 1], cb[4 * h + 2], cb[4 * h + 3]);
              int8_t* dst = p.Xq8 + (size_t)grow * (size_t)p.K + blk * kBlk + 32 * g;
              reinterpret_cast<uint4*>(dst)[0] = make_uint4(w[0], w[1], w[2], w[3]);
              reinterpret_cast<uint4*>(dst)[1] = make_uint4(w[4], w[5], w[6], w[7]);
            }
            if (p.Xq) {  // packed (both formats when both are asked for)
              uint32_t w[4];
#pragma unroll
              for (int h = 0; h < 4; ++h)
                w[h] = (low_bytes4(cb[4 * h], cb[4 * h + 1], cb[4 * h + 2], cb[4 * h + 3]) &
                        0x0F0F0F0Fu) |
                       ((low_bytes4(cb[16 + 4 * h], cb[17 + 4 * h], cb[18 + 4 * h], cb[19 + 4 * h])
                         << 4) &
                        0xF0F0F0F0u);
              uint8_t* dst = p.Xq + (size_t)grow * (size_t)(p.K / 2) + blk * 64;
              *reinterpret_cast<uint4*>(dst + 16 * g) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        }
      }
      if (ok && p.Xq8 && !asym) {
        // the warp's 32 rows x 64 B: lane l writes 16-byte part l % 4 of rows
        // l / 4 + 8 i, i.e. 8 whole 64-byte row segments per store
        __syncwarp();
        const size_t blk = (size_t)(kb0 + i - nb);
        const uint32_t sbw = base + L.amin + (uint32_t)(warp - kEpiFirstWarp) * 2048u;
#pragma unroll
        for (int i4 = 0; i4 < 4; ++i4) {
          const int rw = (lane >> 2) + 8 * i4, part = lane & 3;
          const uint32_t src = sbw + (uint32_t)rw * 64u +
                               ((((uint32_t)part) ^ (((uint32_t)rw >> 1) & 3u)) << 4);
          uint4 v4;
          asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
                       : "=r"(v4.x), "=r"(v4.y), "=r"(v4.z), "=r"(v4.w)
                       : "r"(src));
          const int gr = tile * kTok + q * 32 + rw;
          if (gr < p.M)
            *reinterpret_cast<uint4*>(p.Xq8 + (size_t)gr * (size_t)p.K + blk * kBlk + 64 * half +
                                      16 * part) = v4;
        }
        __syncwarp();
      }
      tc_fence_before();
      mbar_arrive(&rot_empty[u]);
    }

    // ---- X L1: partial over the slice -> the row's owner CTA
    bool xl1_ok = true;
    if (r > 0) xl1_ok = __all_sync(kFull, mbar_wait(xl1_full, 0u, nullptr, abort_flag));
    cluster_arrive_rel();  // B2: every CTA is past pass 2 (stages free)
    cluster_wait_acquire();
    // rows of the tile are split among the cluster: CTA o sums rows
    // [o rpo, (o+1) rpo); every CTA sends each row's partial to its owner
    const int rpo = (kTok + (int)csize - 1) / (int)csize;
    const uint32_t recv = base + L.stage0;  // [C senders][rpo][r] fp32
    if (r > 0 && xl1_ok) {
      tc_fence_after();
      const int owner = row / rpo;
      const uint32_t dst = dsmem_map(recv + (uint32_t)(((int)crank * rpo + row - owner * rpo) * r) * 4u,
                                     (uint32_t)owner);
      for (int c0 = 16 * half; c0 < r; c0 += 32) {  // the two halves alternate 16-column chunks
        uint32_t v[16];
        tmem_ld16(tmem_xl1 + (uint32_t)c0 + lane_off, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; e += 4)
          asm volatile("st.shared::cluster.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(dst + (uint32_t)(c0 + e) * 4u),
                       "r"(v[e]), "r"(v[e + 1]), "r"(v[e + 2]), "r"(v[e + 3])
                       : "memory");
      }
    }
    cluster_arrive_rel();  // B3: partials delivered
    cluster_wait_acquire();
    if (r > 0 && !*abort_flag) {
      // this CTA's rows: sum the C partials in cluster-rank order
      const int row0 = (int)crank * rpo;
      const int nrow = min(rpo, kTok - row0);
      const int q4 = r / 4;  // 4-column groups per row
      const int tid = threadIdx.x - kEpiFirstWarp * 32;
      for (int v4 = tid; v4 < nrow * q4; v4 += kEpiThreadsTc) {
        const int rr = v4 / q4, c = (v4 - rr * q4) * 4;
        const int gr = tile * kTok + row0 + rr;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (uint32_t z = 0; z < csize; ++z) {
          float4 t;
          asm volatile("ld.shared.v4.f32 {%0,%1,%2,%3}, [%4];"
                       : "=f"(t.x), "=f"(t.y), "=f"(t.z), "=f"(t.w)
                       : "r"(recv + (uint32_t)((((int)z * rpo + rr) * r + c) * 4)));
          acc.x += t.x;
          acc.y += t.y;
          acc.z += t.z;
          acc.w += t.w;
        }
        if (gr < p.M) {
          const size_t o = (size_t)gr * p.r_ld + p.r_off + c;
          if (p.XL1) *reinterpret_cast<float4*>(p.XL1 + o) = acc;
          if (p.XL1b) {
            __nv_bfloat162 h0 = __floats2bfloat162_rn(acc.x, acc.y);
            __nv_bfloat162 h1 = __floats2bfloat162_rn(acc.z, acc.w);
            uint2 u;
            u.x = *reinterpret_cast<uint32_t*>(&h0);
            u.y = *reinterpret_cast<uint32_t*>(&h1);
            *reinterpret_cast<uint2*>(p.XL1b + o) = u;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

bool act_tc_supported(int M, int K, int had_block, int r) {
  (void)K;
  return M >= 64 && had_block <= kBlk && r <= 2 * kMaxRx;
}

namespace {

// One launch: codes (+ X L1 columns [0, r) when r > 0), or, with xl1_only,
// X L1 columns [r_off, r_off + r) alone.
cudaError_t launch_act_tc_one(const uint16_t* X, int M, int K, int had_block, const uint16_t* L1t,
                              int r_total, int r_off, int r, bool xl1_only, uint8_t* Xq,
                              int8_t* Xq8, float* s_x, float* z_x, float* XL1, uint16_t* XL1b,
                              cudaStream_t stream, const uint32_t* signs) {
  TcParams p{};
  // X L1 alone needs no mask: (x D)(D L1) = x L1
  p.signs = xl1_only ? nullptr : signs;
  const bool sg = p.signs != nullptr;
  auto* kern = sg ? quantize_act_tc_kernel<true> : quantize_act_tc_kernel<false>;
  const int threads = sg ? tc_threads<true>() : tc_threads<false>();
  p.Xq = xl1_only ? nullptr : Xq;
  p.Xq8 = xl1_only ? nullptr : Xq8;
  p.s_x = s_x;
  p.XL1 = r > 0 ? XL1 : nullptr;
  p.XL1b = r > 0 ? reinterpret_cast<__nv_bfloat16*>(XL1b) : nullptr;
  p.M = M;
  p.K = K;
  p.b = had_block;
  p.r = r;
  p.r_ld = r_total;
  p.r_off = r_off;
  p.xl1_only = xl1_only ? 1 : 0;
  p.z_x = xl1_only ? nullptr : z_x;
  p.kb_total = K / kBlk;
  p.scale_mul = (float)(1.0 / ((p.z_x ? 15.0 : 7.0) * sqrt((double)had_block)));
  p.zmul = (float)(1.0 / sqrt((double)had_block));
  const int tiles = (M + kTok - 1) / kTok;
  const uint32_t smem_bytes = tc_layout(xl1_only, r).bytes + 1024u;
  static uint64_t attr_set[2] = {0, 0};  // per kernel variant, a bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set[sg] >> dev & 1u)) {
    // every layout is at most kSmemCap (three stages only where they fit)
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemCap);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set[sg] |= uint64_t(1) << dev;
  }
  // a cluster of C CTAs along K per 128-token tile: about one CTA per SM,
  // and no larger than lets every cluster of the grid be resident at once.
  // Stepping down one size at a time: 16 tiles of 2048 tokens take clusters
  // of 8 (128 CTAs) where 9 do not all fit; halving fell to 4 (64 CTAs) and
  // left more than half of the SMs idle.
  int C = std::max(1, std::min(kMaxC, num_sms() / tiles));
  C = std::min(C, p.kb_total);
  for (;; --C) {
    p.nb = (p.kb_total + C - 1) / C;
    const int Ce = (p.kb_total + p.nb - 1) / p.nb;  // every CTA owns at least one block
    if (C <= 1) {
      C = Ce;
      break;
    }
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(Ce, tiles, 1);
    q.blockDim = dim3(threads, 1, 1);
    q.dynamicSmemBytes = smem_bytes;
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = Ce;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, kern, &q) == cudaSuccess &&
        active >= tiles) {
      C = Ce;
      break;
    }
    cudaGetLastError();
  }
  CUtensorMap map_x, map_l1;
  if (!encode_tiled_2d(&map_x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, (uint64_t)K, (uint64_t)M,
                       (uint64_t)K * 2, 64, kTok, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (r > 0) {
    // all r_total rows of L1^T; a launch reads rows [r_off, r_off + r)
    if (!encode_tiled_2d(&map_l1, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, L1t, (uint64_t)K,
                         (uint64_t)r_total, (uint64_t)K * 2, 64, (uint32_t)r,
                         CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    map_l1 = map_x;  // never read
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, tiles, 1);
  cfg.blockDim = dim3(threads, 1, 1);
  cfg.dynamicSmemBytes = smem_bytes;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map_x, map_l1, p);
}

}  // namespace

// Up to kMaxRtc X L1 columns are computed beside the codes, from the same
// staged X.  Wider ranks (the tensor memory holds the rotation's two buffers
// and 256 accumulator columns) run the codes alone, then X L1 in launches of
// at most kMaxRx columns that skip the rotation.
cudaError_t launch_act_tc(const uint16_t* X, int M, int K, int had_block, const uint16_t* L1t,
                          int r, uint8_t* Xq, int8_t* Xq8, float* s_x, float* XL1, uint16_t* XL1b,
                          cudaStream_t stream, float* z_x, const uint32_t* signs) {
  if (signs && z_x) return cudaErrorInvalidValue;  // the masked codes are symmetric
  if (r <= kMaxRtc)
    return launch_act_tc_one(X, M, K, had_block, L1t, r, 0, r, false, Xq, Xq8, s_x, z_x, XL1,
                             XL1b, stream, signs);
  if (cudaError_t e = launch_act_tc_one(X, M, K, had_block, nullptr, r, 0, 0, false, Xq, Xq8, s_x,
                                        z_x, nullptr, nullptr, stream, signs))
    return e;
  for (int off = 0; off < r; off += kMaxRx) {
    const int w = std::min(kMaxRx, r - off);
    if (cudaError_t e = launch_act_tc_one(X, M, K, had_block, L1t, r, off, w, true, Xq, Xq8, s_x,
                                          nullptr, XL1, XL1b, stream, nullptr))
      return e;
  }
  return cudaSuccess;
}

}  // namespace tq
