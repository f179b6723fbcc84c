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
constexpr int kConvThreads = 128;
constexpr int kThreads = 192;    // 4 converter/epilogue warps + producer + MMA

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
  int32_t* ws_part;               // [tiles][splits][128][BN]
  float* ws_lr;                   // [tiles][128][BN]
  uint32_t* ws_cnt;               // [tiles]
  uint32_t* status;               // device status word
  int use_lr;                     // r > 0 and Y requested
};

template <int BN, int NSTG, int NOPS>
struct SmemLayout {
  static constexpr uint32_t kOpP = kBM * 128;        // int8 / bf16 operand P
  static constexpr uint32_t kOpQ = BN * 128;
  static constexpr uint32_t kOpStage = kOpP + kOpQ;  // multiple of 1024
  static constexpr uint32_t kStgP = kBM * kPackedRow;
  static constexpr uint32_t kStgQ = BN * kPackedRow;
  static constexpr uint32_t kStgStage = kStgP + kStgQ;
  static constexpr uint32_t kOpBase = 0;
  static constexpr uint32_t kStgBase = kOpBase + NOPS * kOpStage;
  static constexpr uint32_t kBarBase = kStgBase + NSTG * kStgStage;
  // barriers: stg_full, stg_empty, op_full, op_empty, acc_full
  static constexpr uint32_t kNumBars = 2 * NSTG + 2 * NOPS + 1;
  static constexpr uint32_t kMiscBase = kBarBase + kNumBars * 8;
  static constexpr uint32_t kBytes = kMiscBase + 32;
  static constexpr uint32_t kAlloc = kBytes + 1024;  // slack for 1024-B alignment
  static_assert(kOpStage % 1024 == 0, "operand stages must keep 1024-B alignment");
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
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int BN, bool SWAP, int NSTG, int NOPS>
__global__ void __launch_bounds__(kThreads, 1)
    w4a4_lr_gemm_kernel(const __grid_constant__ CUtensorMap map_p,
                        const __grid_constant__ CUtensorMap map_q, const GemmParams prm) {
  using L = SmemLayout<BN, NSTG, NOPS>;
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
  volatile int* last_flag = reinterpret_cast<volatile int*>(smem + L::kMiscBase + 8);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile_p = blockIdx.x, tile_q = blockIdx.y, split = blockIdx.z;
  const int kb0 = split * prm.kb_per_split;
  const int n_kb = min(prm.kb_total - kb0, prm.kb_per_split);
  const bool do_lr = prm.use_lr && split == 0;
  const int n_lr = do_lr ? (prm.r + kLrChunk - 1) / kLrChunk : 0;
  const int n_stages = n_kb + n_lr;
  constexpr uint32_t kTmemCols = (2 * BN < 32) ? 32 : 2 * BN;

  if (threadIdx.x == 0) {
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
    *last_flag = 0;
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  if (warp == 4 && lane == 0) {
    tma_prefetch_desc(&map_p);
    tma_prefetch_desc(&map_q);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t tmem_acc = tmem_base;        // INT32, BN columns
  const uint32_t tmem_lr = tmem_base + BN;    // fp32, BN columns

  if (warp == 4) {
    // ------------------------------------------------------ TMA producer
    if (elect_one()) {
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_a = policy_evict_last();
      // Operand order in memory: weights are P when SWAP, else Q.  Weight
      // tiles do not depend on the preceding kernel, so the first NSTG
      // stages of them are issued before waiting on it.
      const int pre = min(n_kb, NSTG);
      for (int i = 0; i < pre; ++i) {
        uint8_t* sp = smem + L::kStgBase + i * L::kStgStage;
        mbar_arrive_expect_tx(&stg_full[i], L::kStgStage);
        const int x = (kb0 + i) * kPackedRow;
        if (SWAP)
          tma_load_2d(sp, &map_p, &stg_full[i], x, tile_p * kBM, pol_w);
        else
          tma_load_2d(sp + L::kStgP, &map_q, &stg_full[i], x, tile_q * BN, pol_w);
      }
      pdl_wait();
      for (int i = 0; i < pre; ++i) {
        uint8_t* sp = smem + L::kStgBase + i * L::kStgStage;
        const int x = (kb0 + i) * kPackedRow;
        if (SWAP)
          tma_load_2d(sp + L::kStgP, &map_q, &stg_full[i], x, tile_q * BN, pol_a);
        else
          tma_load_2d(sp, &map_p, &stg_full[i], x, tile_p * kBM, pol_a);
      }
      for (int i = pre; i < n_kb; ++i) {
        const int s = i % NSTG;
        const uint32_t ph = (uint32_t)(i / NSTG) & 1u;
        if (!mbar_wait(&stg_empty[s], ph ^ 1u, prm.status, abort_flag)) break;
        uint8_t* sp = smem + L::kStgBase + s * L::kStgStage;
        mbar_arrive_expect_tx(&stg_full[s], L::kStgStage);
        const int x = (kb0 + i) * kPackedRow;
        tma_load_2d(sp, &map_p, &stg_full[s], x, tile_p * kBM, SWAP ? pol_w : pol_a);
        tma_load_2d(sp + L::kStgP, &map_q, &stg_full[s], x, tile_q * BN, SWAP ? pol_a : pol_w);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------- MMA issuer
    if (elect_one()) {
      const uint32_t id_i8 = idesc_i8_s32(BN);
      const uint32_t id_bf = idesc_bf16_f32(BN);
      for (int i = 0; i < n_stages; ++i) {
        const int s = i % NOPS;
        const uint32_t ph = (uint32_t)(i / NOPS) & 1u;
        if (!mbar_wait(&op_full[s], ph, prm.status, abort_flag)) break;
        tc_fence_after();
        const uint32_t a_addr = base + L::kOpBase + s * L::kOpStage;
        const uint64_t da = sdesc_sw128(a_addr);
        const uint64_t db = sdesc_sw128(a_addr + L::kOpP);
        if (i < n_kb) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)  // 4 x K=32 int8 per 128-byte row
            mma_i8(tmem_acc, da + 2 * kk, db + 2 * kk, id_i8, (i > 0 || kk > 0) ? 1u : 0u);
        } else {
          const int c = i - n_kb;
          const int nk = min(kLrChunk, prm.r - c * kLrChunk) / 16;
          for (int kk = 0; kk < nk; ++kk)  // K=16 bf16 = 32 bytes per step
            mma_bf16(tmem_lr, da + 2 * kk, db + 2 * kk, id_bf, (c > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&op_empty[s]);
      }
      mma_commit(acc_full);
    }
  } else {
    // ----------------------------------------- converters, then epilogue
    const int tid = threadIdx.x;  // 0..127
    pdl_wait();
    for (int i = 0; i < n_stages; ++i) {
      const int s = i % NOPS;
      const uint32_t ph = (uint32_t)(i / NOPS) & 1u;
      if (!mbar_wait(&op_empty[s], ph ^ 1u, prm.status, abort_flag)) break;
      const uint32_t op_p = base + L::kOpBase + s * L::kOpStage;
      const uint32_t op_q = op_p + L::kOpP;
      if (i < n_kb) {
        const int st = i % NSTG;
        const uint32_t phs = (uint32_t)(i / NSTG) & 1u;
        if (!mbar_wait(&stg_full[st], phs, prm.status, abort_flag)) break;
        const uint32_t sg = base + L::kStgBase + st * L::kStgStage;
        // one 16-byte packed chunk (32 codes) -> two 16-byte int8 chunks
        for (int c = tid; c < (kBM + BN) * 4; c += kConvThreads) {
          const int row = c >> 2, q = c & 3;
          const bool on_p = row < kBM;
          const uint32_t rr = on_p ? row : row - kBM;
          const uint4 w = ld_shared_v4(sg + (uint32_t)c * 16u);
          uint4 lo, hi;
          lo.x = (w.x << 4) & 0xF0F0F0F0u;
          lo.y = (w.y << 4) & 0xF0F0F0F0u;
          lo.z = (w.z << 4) & 0xF0F0F0F0u;
          lo.w = (w.w << 4) & 0xF0F0F0F0u;
          hi.x = w.x & 0xF0F0F0F0u;
          hi.y = w.y & 0xF0F0F0F0u;
          hi.z = w.z & 0xF0F0F0F0u;
          hi.w = w.w & 0xF0F0F0F0u;
          const uint32_t dst = on_p ? op_p : op_q;
          st_shared_v4(dst + sw128_offset(rr, 2 * q), lo);
          st_shared_v4(dst + sw128_offset(rr, 2 * q + 1), hi);
        }
        fence_proxy_async_smem();
        mbar_arrive(&stg_empty[st]);
      } else {
        const int chunk = i - n_kb;
        for (int c = tid; c < (kBM + BN) * 8; c += kConvThreads) {
          const int row = c >> 3, jj = c & 7;
          const bool on_p = row < kBM;
          const int rr = on_p ? row : row - kBM;
          const int g_row = on_p ? tile_p * kBM + rr : tile_q * BN + rr;
          const int g_lim = on_p ? prm.rows_p : prm.rows_q;
          const bool is_f32 = (on_p != SWAP);  // XL1 sits on the token side
          const int col0 = chunk * kLrChunk + jj * 8;
          uint4 out = make_uint4(0u, 0u, 0u, 0u);
          if (g_row < g_lim && col0 < prm.r) {
            if (is_f32) {
              const float4* src =
                  reinterpret_cast<const float4*>(prm.xl1 + (size_t)g_row * prm.r + col0);
              const float4 a = __ldg(src), b = __ldg(src + 1);
              out.x = pack_bf16x2(a.x, a.y);
              out.y = pack_bf16x2(a.z, a.w);
              out.z = pack_bf16x2(b.x, b.y);
              out.w = pack_bf16x2(b.z, b.w);
            } else {
              out = __ldg(reinterpret_cast<const uint4*>(prm.l2t + (size_t)g_row * prm.r + col0));
            }
          }
          st_shared_v4((on_p ? op_p : op_q) + sw128_offset((uint32_t)rr, (uint32_t)jj), out);
        }
        fence_proxy_async_smem();
      }
      mbar_arrive(&op_full[s]);
    }

    // ---------------------------------------------------------- epilogue
    const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full, 0u, prm.status, abort_flag));
    tc_fence_after();
    const int row = warp * 32 + lane;                  // TMEM lane = P row in tile
    const int gp = tile_p * kBM + row;
    const uint32_t t_row = (uint32_t)(warp * 32) << 16;
    const float sp = (!prm.acc_out && gp < prm.rows_p) ? __ldg(prm.s_p + gp) : 0.f;
    const int tile_idx = tile_q * gridDim.x + tile_p;
    if (ok) {
      for (int cb = 0; cb < BN; cb += 16) {
        uint32_t ai[16], af[16];
        tmem_ld16(tmem_acc + t_row + cb, ai);
        if (do_lr) tmem_ld16(tmem_lr + t_row + cb, af);
        tmem_ld_wait();
        if (prm.splits == 1) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int gq = tile_q * BN + cb + j;
            if (gp >= prm.rows_p || gq >= prm.rows_q) continue;
            const int acc = ((int)ai[j]) >> 8;
            const int m = SWAP ? gq : gp, n = SWAP ? gp : gq;
            if (prm.acc_out) {
              prm.acc_out[(size_t)m * prm.ldy + n] = acc;
            } else {
              float y = sp * __ldg(prm.s_q + gq) * (float)acc;
              if (do_lr) y += __uint_as_float(af[j]);
              prm.Y[(size_t)m * prm.ldy + n] = __float2bfloat16_rn(y);
            }
          }
        } else {
          int32_t* dst = prm.ws_part + (((size_t)tile_idx * prm.splits + split) * kBM + row) * BN + cb;
#pragma unroll
          for (int j = 0; j < 16; j += 4)
            *reinterpret_cast<int4*>(dst + j) =
                make_int4((int)ai[j] >> 8, (int)ai[j + 1] >> 8, (int)ai[j + 2] >> 8,
                          (int)ai[j + 3] >> 8);
          if (do_lr) {
            float* dl = prm.ws_lr + ((size_t)tile_idx * kBM + row) * BN + cb;
#pragma unroll
            for (int j = 0; j < 16; j += 4)
              *reinterpret_cast<float4*>(dl + j) =
                  make_float4(__uint_as_float(af[j]), __uint_as_float(af[j + 1]),
                              __uint_as_float(af[j + 2]), __uint_as_float(af[j + 3]));
          }
        }
      }
      if (prm.splits > 1) {
        __threadfence();
        named_bar_sync(1, kConvThreads);
        if (threadIdx.x == 0) {
          const uint32_t prev = atomicAdd(prm.ws_cnt + tile_idx, 1u);
          *last_flag = (prev == (uint32_t)prm.splits - 1u) ? 1 : 0;
        }
        named_bar_sync(1, kConvThreads);
        if (*last_flag) {
          __threadfence();
          const int32_t* part0 = prm.ws_part + ((size_t)tile_idx * prm.splits * kBM + row) * BN;
          const float* lr0 = prm.ws_lr + ((size_t)tile_idx * kBM + row) * BN;
          for (int col = 0; col < BN; ++col) {
            const int gq = tile_q * BN + col;
            if (gp >= prm.rows_p || gq >= prm.rows_q) continue;
            int acc = 0;
            for (int z = 0; z < prm.splits; ++z) acc += __ldcg(part0 + (size_t)z * kBM * BN + col);
            const int m = SWAP ? gq : gp, n = SWAP ? gp : gq;
            if (prm.acc_out) {
              prm.acc_out[(size_t)m * prm.ldy + n] = acc;
            } else {
              float y = sp * __ldg(prm.s_q + gq) * (float)acc;
              if (prm.use_lr) y += __ldcg(lr0 + col);
              prm.Y[(size_t)m * prm.ldy + n] = __float2bfloat16_rn(y);
            }
          }
          if (threadIdx.x == 0) prm.ws_cnt[tile_idx] = 0u;  // leave the counter clean
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
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

// Packed int4 matrix [rows][K/2] bytes, box = 64 bytes x box_rows.
bool make_packed_map(CUtensorMap* m, const uint8_t* ptr, int rows, int K, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)(K / 2), (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(K / 2)};
  cuuint32_t box[2] = {(cuuint32_t)kPackedRow, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(ptr), dims, strides,
                  box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
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

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

Plan make_plan(int M, int N, int K, bool debug) {
  (void)debug;
  Plan p{};
  const int kb = K / kKB;
  if (M <= 128) {
    p.swap = true;
    p.bn = M <= 16 ? 16 : (M <= 32 ? 32 : (M <= 64 ? 64 : 128));
    p.tiles_p = (N + kBM - 1) / kBM;
    p.tiles_q = (M + p.bn - 1) / p.bn;
    int s = tuning().split_k;
    if (s <= 0) {
      const int ctas = p.tiles_p * p.tiles_q;
      s = std::max(1, (num_sms() + ctas - 1) / ctas);
    }
    s = std::min(s, kb);
    p.kb_per_split = (kb + s - 1) / s;
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

template <int BN, bool SWAP, int NSTG, int NOPS>
cudaError_t launch_variant(const GemmArgs& a, const Plan& pl, const GemmParams& prm,
                           cudaStream_t stream) {
  using L = SmemLayout<BN, NSTG, NOPS>;
  CUtensorMap map_p, map_q;
  const uint8_t* P = SWAP ? a.Wq : a.Xq;
  const uint8_t* Q = SWAP ? a.Xq : a.Wq;
  if (!make_packed_map(&map_p, P, prm.rows_p, a.K, kBM)) return cudaErrorInvalidValue;
  if (!make_packed_map(&map_q, Q, prm.rows_q, a.K, BN)) return cudaErrorInvalidValue;
  auto kern = w4a4_lr_gemm_kernel<BN, SWAP, NSTG, NOPS>;
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
  cfg.blockDim = dim3(kThreads, 1, 1);
  cfg.dynamicSmemBytes = L::kAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = tuning().pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map_p, map_q, prm);
}

// workspace: [status 256 B][counters][int32 partials][fp32 low-rank partials]
struct WsLayout {
  size_t cnt_off, part_off, lr_off, total;
};
WsLayout ws_layout(const Plan& pl) {
  WsLayout w{};
  const size_t tiles = (size_t)pl.tiles_p * pl.tiles_q;
  w.cnt_off = 256;
  w.part_off = (w.cnt_off + tiles * 4 + 255) & ~size_t(255);
  const size_t part = (pl.splits > 1) ? tiles * pl.splits * kBM * pl.bn * 4 : 0;
  w.lr_off = (w.part_off + part + 255) & ~size_t(255);
  const size_t lr = (pl.splits > 1) ? tiles * kBM * pl.bn * 4 : 0;
  w.total = w.lr_off + lr;
  return w;
}

}  // namespace

size_t gemm_workspace_bytes(int M, int N, int K, int r) {
  (void)r;
  return ws_layout(make_plan(M, N, K, false)).total;
}

cudaError_t launch_gemm(const GemmArgs& a, cudaStream_t stream) {
  const bool debug = a.acc_out != nullptr;
  const Plan pl = make_plan(a.M, a.N, a.K, debug);
  const WsLayout wl = ws_layout(pl);
  if (a.ws_bytes < wl.total) return cudaErrorInvalidValue;
  uint8_t* ws = static_cast<uint8_t*>(a.ws);
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
  prm.ws_part = reinterpret_cast<int32_t*>(ws + wl.part_off);
  prm.ws_lr = reinterpret_cast<float*>(ws + wl.lr_off);
  prm.ws_cnt = reinterpret_cast<uint32_t*>(ws + wl.cnt_off);
  prm.status = reinterpret_cast<uint32_t*>(ws);
  prm.use_lr = (a.r > 0 && !debug) ? 1 : 0;
  if (!pl.swap) return launch_variant<256, false, 4, 2>(a, pl, prm, stream);
  switch (pl.bn) {
    case 16: return launch_variant<16, true, 8, 2>(a, pl, prm, stream);
    case 32: return launch_variant<32, true, 8, 2>(a, pl, prm, stream);
    case 64: return launch_variant<64, true, 6, 2>(a, pl, prm, stream);
    default: return launch_variant<128, true, 6, 2>(a, pl, prm, stream);
  }
}

}  // namespace tq
