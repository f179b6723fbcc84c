// tq_act.cu -- rotation + symmetric INT4 quantization kernels.
//
//  * quantize_act_kernel: the per-token activation stage.  One thread-block
//    cluster owns 16 tokens; its C CTAs split K.  Each warp owns one token,
//    holds its slice of X in registers, applies the Sylvester fast
//    Walsh-Hadamard transform per block (in-register butterflies, then
//    shuffles), and the cluster combines the per-slice absmax through
//    distributed shared memory before every CTA writes its packed codes.  The
//    same read of X feeds the X.L1 down-projection on tensor cores
//    (mma.sync bf16, fp32 accumulation), reduced across the cluster in a fixed
//    order, so results are deterministic.
//  * pack_weight_kernel: the offline per-output-channel weight stage (one CTA
//    per row of R^T, transform in shared memory).
//
// Quantizer: CoQuant Eq. (1), symmetric, s = max|x| / 7, RoundClip to
// [-7, 7]; rotation: CoQuant Eq. (3) with a Hadamard U.  The transform is
// computed unnormalised; the 1/sqrt(b) factor cancels in the codes and is
// folded into the stored scale.
#include <cuda_bf16.h>

#include <algorithm>

#include "tq_act_common.cuh"
#include "tq_internal.h"
#include "tq_ptx.cuh"

namespace tq {

namespace {

constexpr int kActRows = 16;       // tokens per cluster
constexpr int kActWarps = 8;       // warp w handles tokens w and w + 8
constexpr int kActThreads = 32 * kActWarps;

struct ActParams {
  const __nv_bfloat16* X;
  const __nv_bfloat16* L1t;
  uint8_t* Xq;              // packed codes [M][K/2], or
  int8_t* Xq8;              //   one code per byte [M][K] (when non-null)
  float* s_x;
  float* XL1;               // fp32 X L1 [M][r], or
  __nv_bfloat16* XL1b;      //   bf16(X L1) (when non-null)
  const uint32_t* signs;  // randomized Hadamard sign masks [n_rht][K / 32], or null
  int n_rht;              // composed transforms (masks)
  int M, K, b, r;
  int passes_per_cta;  // P: warp passes of W = 32E columns in this CTA's slice
  int total_passes;    // K / W
  int kc;              // L1 k-chunk (columns) staged per step
  int l1_bufs;         // staged chunk buffers (all chunks, or 2)
  int kparts;          // warps sharing one 8-column tile of r split its k steps
  float scale_mul;     // 1 / (7 sqrt(b))
};

// Shared-memory carve-up of quantize_act_kernel.
//   xs     X tile [16][slice + 8] bf16
//   l1s    staged L1^T chunks [nbuf][r][kc + 8] bf16
//   partk  X L1 partials per k-part [KP][16][r] fp32
//   recv   X L1 partials received from the cluster [C][16][ceil(r/C)] fp32
//   amax   per-CTA absmax received from the cluster [C][16], row absmax [16]
template <int E>
struct ActSmem {
  static constexpr int W = 32 * E;
  int xs_stride;   // bf16 elements per X row (slice + 8 pad)
  int l1_stride;   // bf16 elements per staged L1^T row (kc + 8 pad)
  int cols_max;    // X L1 columns owned per CTA in the cluster reduction
  size_t off_l1, off_part, off_recv, off_amax, total;
  __host__ __device__ ActSmem(int P, int r, int kc, int nbuf, int kp, int C) {
    xs_stride = P * W + 8;
    l1_stride = kc + 8;
    cols_max = (r + C - 1) / C;
    size_t xs_bytes = (size_t)kActRows * xs_stride * 2;
    off_l1 = (xs_bytes + 127) & ~size_t(127);
    size_t l1_bytes = (size_t)nbuf * r * l1_stride * 2;
    off_part = (off_l1 + l1_bytes + 127) & ~size_t(127);
    size_t part_bytes = (size_t)kp * kActRows * r * 4;
    off_recv = (off_part + part_bytes + 127) & ~size_t(127);
    size_t recv_bytes = (size_t)C * kActRows * cols_max * 4;
    off_amax = (off_recv + recv_bytes + 127) & ~size_t(127);
    total = off_amax + (size_t)(C + 1) * kActRows * 4;
  }
};
// Staged L1^T chunks: all of the slice at once when they fit in this budget
// (one round trip to memory), else a double buffer.  Kept small so that
// several CTAs share an SM and hide each other's latencies.
constexpr size_t kL1AllBudget = 40 * 1024;
// Dynamic shared memory the kernel is allowed (every supported shape fits).
constexpr size_t kActSmemMax = 200 * 1024;

// One cluster of C CTAs owns 16 tokens; CTA c owns columns
// [c*P*W, (c+1)*P*W) of K.  Warp w handles tokens w and w+8.  The transform
// is computed twice from the shared-memory copy of X -- once for the absmax,
// once for the codes after the cluster has combined the absmax -- so no
// rotated values have to be kept.  Both passes run the same butterflies in
// the same order, so they give the same bits.
template <int E>
__global__ void __launch_bounds__(kActThreads) quantize_act_kernel(const ActParams p) {
  constexpr int W = 32 * E;
  extern __shared__ __align__(128) uint8_t smem[];

  pdl_launch_dependents();  // let the GEMM start streaming its weights
  // announce this CTA to the cluster; remote stores wait for every peer
  cluster_arrive_relaxed();
  pdl_wait();

  const int P = p.passes_per_cta;
  const uint32_t crank = cluster_ctarank();
  const uint32_t csize = cluster_nctarank();
  const ActSmem<E> L(P, p.r, p.kc, p.l1_bufs, p.kparts, (int)csize);
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* l1s = reinterpret_cast<__nv_bfloat16*>(smem + L.off_l1);
  float* partk = reinterpret_cast<float*>(smem + L.off_part);
  float* recv = reinterpret_cast<float*>(smem + L.off_recv);
  float* amax_all = reinterpret_cast<float*>(smem + L.off_amax);  // [C][16]
  float* amax_row = amax_all + csize * kActRows;

  const int pass0 = (int)crank * P;
  const int np = min(P, p.total_passes - pass0);
  const int slice = np * W;
  const int kbase = pass0 * W;
  const int row0 = blockIdx.y * kActRows;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;

  // ---- stage X[row0:row0+16][kbase:kbase+slice] (zero rows past M)
  {
    const int chunks_per_row = slice / 8;  // 16-byte chunks
    for (int c = tid; c < kActRows * chunks_per_row; c += kActThreads) {
      const int rr = c / chunks_per_row, cc = c % chunks_per_row;
      const int gm = row0 + rr;
      const bool ok = gm < p.M;
      const __nv_bfloat16* src = p.X + (size_t)(ok ? gm : 0) * p.K + kbase + cc * 8;
      cp_async16(xs + (size_t)rr * L.xs_stride + cc * 8, src, ok);
    }
    cp_async_commit();
  }
  // ---- L1^T chunks of this slice: all of them up front when they fit,
  //      otherwise the first of a double buffer
  const int nchunks = (p.r > 0) ? slice / p.kc : 0;
  const bool all_l1 = nchunks > 0 && p.l1_bufs >= nchunks;
  auto stage_l1 = [&](int ci, int buf) {
    const int cpr = p.kc / 8;
    __nv_bfloat16* dst = l1s + (size_t)buf * p.r * L.l1_stride;
    for (int c = tid; c < p.r * cpr; c += kActThreads) {
      const int j = c / cpr, cc = c % cpr;
      const __nv_bfloat16* src = p.L1t + (size_t)j * p.K + kbase + ci * p.kc + cc * 8;
      cp_async16(dst + (size_t)j * L.l1_stride + cc * 8, src, true);
    }
    cp_async_commit();
  };
  if (all_l1) {
    for (int ci = 0; ci < nchunks; ++ci) stage_l1(ci, ci);
  } else if (nchunks > 0) {
    stage_l1(0, 0);
  }
  // X is the oldest group: wait for it alone when L1 is double-buffered
  if (nchunks == 0 || all_l1) cp_async_wait<0>();
  else cp_async_wait<1>();
  __syncthreads();

  // ---- pass 1: transform, absmax of tokens warp and warp + 8
  float amax[2] = {0.f, 0.f};
  for (int t = 0; t < 2; ++t) {
    const int rr = warp + 8 * t;
    for (int ps = 0; ps < np; ++ps) {
      float v[E];
      load_row_values<E>(xs + (size_t)rr * L.xs_stride + ps * W + lane * E, v);
      rotate_signed<E>(v, p.signs, p.n_rht, p.K / 32, kbase + ps * W + lane * E, p.b);
#pragma unroll
      for (int i = 0; i < E; ++i) amax[t] = fmaxf(amax[t], fabsf(v[i]));
    }
    amax[t] = warp_max(amax[t]);
  }
  cluster_wait_acquire();  // every peer is running before it is written to
  // every CTA of the cluster gets this CTA's partial absmax of both tokens
  if (lane < (int)csize) {
    dsmem_st_f32(dsmem_map(smem_u32(&amax_all[crank * kActRows + warp]), (uint32_t)lane), amax[0]);
    dsmem_st_f32(dsmem_map(smem_u32(&amax_all[crank * kActRows + warp + 8]), (uint32_t)lane),
                 amax[1]);
  }

  // ---- X L1 partial over this CTA's slice: warp w owns 8-column tiles
  //      (w % NT8) + 8j of r and k-part w / NT8 of every staged chunk; two
  //      accumulator chains per tile (even / odd k steps)
  if (nchunks > 0) {
    const int ntiles = p.r / 8;
    const int nt8 = min(ntiles, kActWarps);
    const int KP = p.kparts;
    const int kp = warp / nt8;
    const bool active = warp < nt8 * KP;
    constexpr int kMaxTilesPerWarp = 8;  // r <= 512
    float acc[kMaxTilesPerWarp][2][4];
#pragma unroll
    for (int t = 0; t < kMaxTilesPerWarp; ++t)
#pragma unroll
      for (int h = 0; h < 2; ++h) acc[t][h][0] = acc[t][h][1] = acc[t][h][2] = acc[t][h][3] = 0.f;
    const uint32_t xs_base = smem_u32(xs);
    const int ksteps = p.kc / 16;
    const int ks0 = kp * ksteps / KP, ks1 = (kp + 1) * ksteps / KP;
    for (int ci = 0; ci < nchunks; ++ci) {
      if (!all_l1) {
        if (ci + 1 < nchunks) {
          stage_l1(ci + 1, (ci + 1) & 1);
          cp_async_wait<1>();
        } else {
          cp_async_wait<0>();
        }
        __syncthreads();
      }
      const int buf = all_l1 ? ci : (ci & 1);
      const uint32_t l1_base = smem_u32(l1s + (size_t)buf * p.r * L.l1_stride);
      if (active) {
        for (int ks = ks0; ks < ks1; ++ks) {
          const int kk = ks * 16;
          const int h = ks & 1;
          uint32_t a[4];
          {
            const int mat = lane >> 3, rin = lane & 7;
            const int rr = rin + (mat & 1) * 8;
            const int cc = ci * p.kc + kk + (mat >> 1) * 8;
            ldmatrix_x4(a, xs_base + (uint32_t)((rr * L.xs_stride + cc) * 2));
          }
#pragma unroll
          for (int t = 0; t < kMaxTilesPerWarp; ++t) {
            const int tile = (warp % nt8) + kActWarps * t;
            if (tile < ntiles) {
              uint32_t bb[2];
              const int l = lane & 15;
              const int jr = tile * 8 + (l & 7);
              const int cc = kk + (l >> 3) * 8;
              ldmatrix_x2(bb, l1_base + (uint32_t)((jr * L.l1_stride + cc) * 2));
              if (h == 0) mma_16816(acc[t][0], a, bb);
              else mma_16816(acc[t][1], a, bb);
            }
          }
        }
      }
      if (!all_l1) __syncthreads();  // buffer (ci & 1) is refilled two chunks later
    }
    // C fragment: rows lane/4 and lane/4 + 8, columns 2*(lane%4) + {0, 1}
    if (active) {
      float* pk = partk + (size_t)kp * kActRows * p.r;
#pragma unroll
      for (int t = 0; t < kMaxTilesPerWarp; ++t) {
        const int tile = (warp % nt8) + kActWarps * t;
        if (tile < ntiles) {
          const int rr = lane >> 2, cc = tile * 8 + 2 * (lane & 3);
          pk[rr * p.r + cc] = acc[t][0][0] + acc[t][1][0];
          pk[rr * p.r + cc + 1] = acc[t][0][1] + acc[t][1][1];
          pk[(rr + 8) * p.r + cc] = acc[t][0][2] + acc[t][1][2];
          pk[(rr + 8) * p.r + cc + 1] = acc[t][0][3] + acc[t][1][3];
        }
      }
    }
    __syncthreads();
    // this CTA's partial (k-parts summed in order) -> the column's owner CTA
    for (int idx = tid; idx < kActRows * p.r; idx += kActThreads) {
      const int rr = idx / p.r, col = idx - rr * p.r;
      float v = 0.f;
      for (int k = 0; k < KP; ++k) v += partk[(size_t)k * kActRows * p.r + idx];
      const int owner = col * (int)csize / p.r;
      const int lo = (owner * p.r + (int)csize - 1) / (int)csize;
      const uint32_t dst = smem_u32(&recv[((int)crank * kActRows + rr) * L.cols_max + (col - lo)]);
      dsmem_st_f32(dsmem_map(dst, (uint32_t)owner), v);
    }
  }

  cluster_sync();  // every partial absmax and X L1 has been delivered

  if (tid < kActRows) {
    float m = 0.f;
    for (uint32_t c = 0; c < csize; ++c) m = fmaxf(m, amax_all[c * kActRows + tid]);
    amax_row[tid] = m;
  }
  __syncthreads();

  // ---- pass 2: the same transform again, then codes of this CTA's slice
  for (int t = 0; t < 2; ++t) {
    const int rr = warp + 8 * t;
    const int my_row = row0 + rr;
    if (my_row >= p.M) continue;  // warp-uniform
    const float am = amax_row[rr];
    const CodeScale cs = code_scale(am);
    uint8_t* xrow = p.Xq8 ? nullptr : p.Xq + (size_t)my_row * (p.K / 2);
    int8_t* xrow8 = p.Xq8 ? p.Xq8 + (size_t)my_row * p.K : nullptr;
    for (int ps = 0; ps < np; ++ps) {
      float v[E];
      load_row_values<E>(xs + (size_t)rr * L.xs_stride + ps * W + lane * E, v);
      rotate_signed<E>(v, p.signs, p.n_rht, p.K / 32, kbase + ps * W + lane * E, p.b);
      if (cs.pre != 1.f) {
#pragma unroll
        for (int i = 0; i < E; ++i) v[i] *= cs.pre;
      }
      uint32_t cb[E];
#pragma unroll
      for (int i = 0; i < E; ++i) cb[i] = code_bits(v[i], cs.inv);
      if (xrow8) {
        // E consecutive codes, byte i the low byte of cb[i]
        int8_t* dst = xrow8 + kbase + ps * W + lane * E;
        if constexpr (E == 4) {
          *reinterpret_cast<uint32_t*>(dst) = low_bytes4(cb[0], cb[1], cb[2], cb[3]);
        } else {
#pragma unroll
          for (int i = 0; i < E; i += 8)
            *reinterpret_cast<uint2*>(dst + i) =
                make_uint2(low_bytes4(cb[i], cb[i + 1], cb[i + 2], cb[i + 3]),
                           low_bytes4(cb[i + 4], cb[i + 5], cb[i + 6], cb[i + 7]));
        }
      } else {
        store_packed<E>(cb, xrow + (kbase + ps * W) / 2);
      }
    }
    if (crank == 0 && lane == 0) p.s_x[my_row] = am * p.scale_mul;
  }

  // ---- X L1 of the columns this CTA owns: sum over the cluster in rank order
  if (p.r > 0) {
    const int lo = ((int)crank * p.r + (int)csize - 1) / (int)csize;
    const int hi = (((int)crank + 1) * p.r + (int)csize - 1) / (int)csize;
    const int ncol = hi - lo;
    for (int idx = tid; idx < kActRows * ncol; idx += kActThreads) {
      const int rr = idx / ncol, cc = idx - rr * ncol;
      if (row0 + rr >= p.M) continue;
      float v = 0.f;
      for (uint32_t c = 0; c < csize; ++c) v += recv[((int)c * kActRows + rr) * L.cols_max + cc];
      if (p.XL1b)
        p.XL1b[(size_t)(row0 + rr) * p.r + lo + cc] = __float2bfloat16_rn(v);
      else
        p.XL1[(size_t)(row0 + rr) * p.r + lo + cc] = v;
    }
  }
}

// ------------------------------------------------------------ weight pack

constexpr int kPackThreads = 256;

// Rows of fp32 R^T (the residual), or of bf16 L1^T (the low-rank down
// projection, quantized per column of H^T L1 for the INT4 low-rank branch).
__device__ __forceinline__ float4 load4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xFFFF0000u));
}

// kBytes: codes one per byte ([N][K] int8) instead of packed ([N][K/2]).
template <typename T, bool kBytes = false>
__global__ void __launch_bounds__(kPackThreads) pack_weight_kernel(const T* __restrict__ Rt,
                                                                   int K, int b, float scale_mul,
                                                                   uint8_t* __restrict__ Wq,
                                                                   float* __restrict__ s_w,
                                                                   const uint32_t* signs,
                                                                   int n_rht) {
  extern __shared__ __align__(16) float row[];
  __shared__ float red[kPackThreads / 32];
  const int n = blockIdx.x;
  const T* src = Rt + (size_t)n * K;
  for (int k = threadIdx.x * 4; k < K; k += kPackThreads * 4) {
    float4 f = load4(src + k);
    if (signs) {  // randomized Hadamard: row n of R^T D H
      float v[4] = {f.x, f.y, f.z, f.w};
      apply_signs<4>(v, signs, k);
      f = make_float4(v[0], v[1], v[2], v[3]);
    }
    *reinterpret_cast<float4*>(row + k) = f;
  }
  __syncthreads();
  // in-place Sylvester butterflies, level by level (pairs never cross
  // blocks); composed randomized transforms: the next mask, then again
  for (int pass = 0; pass < (signs ? n_rht : 1); ++pass) {
    if (pass > 0) {
      for (int k = threadIdx.x * 4; k < K; k += kPackThreads * 4) {
        float v[4] = {row[k], row[k + 1], row[k + 2], row[k + 3]};
        apply_signs<4>(v, signs + (size_t)pass * (K / 32), k);
        row[k] = v[0];
        row[k + 1] = v[1];
        row[k + 2] = v[2];
        row[k + 3] = v[3];
      }
      __syncthreads();
    }
    for (int h = 1; h < b; h <<= 1) {
      for (int t = threadIdx.x; t < K / 2; t += kPackThreads) {
        const int i = (t / h) * 2 * h + (t % h);
        const float a = row[i], c = row[i + h];
        row[i] = a + c;
        row[i + h] = a - c;
      }
      __syncthreads();
    }
  }
  float m = 0.f;
  for (int k = threadIdx.x; k < K; k += kPackThreads) m = fmaxf(m, fabsf(row[k]));
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    float mm = threadIdx.x < kPackThreads / 32 ? red[threadIdx.x] : 0.f;
    mm = warp_max(mm);
    if (threadIdx.x == 0) red[0] = mm;
  }
  __syncthreads();
  const float amax = red[0];
  const float inv = amax > 0.f ? 7.f / amax : 0.f;
  if constexpr (kBytes) {
    int8_t* dst8 = reinterpret_cast<int8_t*>(Wq) + (size_t)n * K;
    for (int k = threadIdx.x; k < K; k += kPackThreads) dst8[k] = (int8_t)quant_code(row[k], inv);
    if (threadIdx.x == 0) s_w[n] = amax * scale_mul;
    // the layer kernels read packed weights before they wait on the
    // preceding kernel: make these stores visible before the block exits
    __threadfence();
    return;
  }
  uint8_t* dst = Wq + (size_t)n * (K / 2);
  for (int byte = threadIdx.x; byte < K / 2; byte += kPackThreads) {
    const int g = byte / 16, i = byte % 16;
    const int lo = quant_code(row[g * 32 + i], inv);
    const int hi = quant_code(row[g * 32 + 16 + i], inv);
    dst[byte] = (uint8_t)((lo & 0xF) | ((hi & 0xF) << 4));
  }
  if (threadIdx.x == 0) s_w[n] = amax * scale_mul;
  // the layer kernels read packed weights before they wait on the preceding
  // kernel: make these stores visible before the block exits
  __threadfence();
}

template <int E>
cudaError_t launch_act_e(const ActParams& prm_in, int max_cluster, cudaStream_t stream) {
  constexpr int W = 32 * E;
  constexpr int PMAX = 2048 / W;  // X tile of at most 2048 columns per CTA
  ActParams prm = prm_in;
  const int tp = prm.K / W;
  int P = (tp + max_cluster - 1) / max_cluster;
  if (P > PMAX) P = (tp + 15) / 16;
  if (P > PMAX) return cudaErrorInvalidValue;
  const int C = (tp + P - 1) / P;
  prm.passes_per_cta = P;
  prm.total_passes = tp;
  prm.kc = prm.r > 256 ? 32 : (prm.r > 128 ? 64 : 128);
  if (prm.kc > W) prm.kc = W;
  const int nchunks_max = (P * W) / prm.kc;
  const size_t all_bytes = (size_t)nchunks_max * prm.r * (prm.kc + 8) * 2;
  prm.l1_bufs = (all_bytes <= kL1AllBudget) ? nchunks_max : 2;
  const int ntiles = prm.r / 8;
  prm.kparts = (ntiles == 0)
                   ? 1
                   : std::max(1, std::min(kActWarps / std::min(ntiles, kActWarps), prm.kc / 16));
  const ActSmem<E> L(P, prm.r, prm.kc, prm.l1_bufs, prm.kparts, C);
  auto kern = quantize_act_kernel<E>;
  static uint64_t attr_set = 0;  // one bit per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (!(attr_set >> dev & 1u)) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kActSmemMax);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
    attr_set |= uint64_t(1) << dev;
  }
  if (L.total > kActSmemMax) return cudaErrorInvalidValue;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, (prm.M + kActRows - 1) / kActRows, 1);
  cfg.blockDim = dim3(kActThreads, 1, 1);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, prm);
}

// Symmetric per-row INT4 codes of r values, written as bf16 integers (exact:
// |code| <= 7), one warp per row: either rows of bf16 L2^T (offline, the
// low-rank up projection per output channel), or the dequantized INT32
// X L1 of the INT4 low-rank branch, xl1[t][j] = s_x[t] s_L1[j] acc[t][j]
// (per token).  Scale = absmax / 7, codes RoundClip(v * 7 / absmax) with ties
// to even; an all-zero row gets scale 0 and codes 0.
__global__ void lowrank_codes_kernel(const __nv_bfloat16* __restrict__ src_bf16,
                                     const int32_t* __restrict__ acc,
                                     const float* __restrict__ s_x, const float* __restrict__ s_L1,
                                     int rows, int r, __nv_bfloat16* __restrict__ codes,
                                     float* __restrict__ scale) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  constexpr int kMaxPerLane = 16;  // r <= 512
  float v[kMaxPerLane];
  float amax = 0.f;
  const float sx = acc ? __ldg(s_x + row) : 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int j = lane + 32 * i;
    v[i] = 0.f;
    if (j < r) {
      if (acc)
        v[i] = sx * __ldg(s_L1 + j) * (float)__ldg(acc + (size_t)row * r + j);
      else
        v[i] = __bfloat162float(src_bf16[(size_t)row * r + j]);
      amax = fmaxf(amax, fabsf(v[i]));
    }
  }
  amax = warp_max(amax);
  const float inv = amax > 0.f ? 7.f / amax : 0.f;
#pragma unroll
  for (int i = 0; i < kMaxPerLane; ++i) {
    const int j = lane + 32 * i;
    if (j < r) codes[(size_t)row * r + j] = __float2bfloat16_rn((float)quant_code(v[i], inv));
  }
  if (lane == 0) scale[row] = amax / 7.f;
}

// Sum of each channel's weight codes (offline; the zero-point term of
// asymmetric activation codes): one warp per row of Wq, signed nibbles.
__global__ void weight_code_sums_kernel(const uint8_t* __restrict__ Wq, int N, int K,
                                        int32_t* __restrict__ wsum) {
  const int row = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(Wq + (size_t)row * (K / 2));
  int sum = 0;
  for (int i = lane; i < K / 8; i += 32) {
    const uint32_t v = __ldg(w + i);
#pragma unroll
    for (int n = 0; n < 8; ++n) sum += (int)(v << (28 - 4 * n)) >> 28;  // sign-extended nibble n
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) wsum[row] = sum;
}

// Gate / up pair as one layer (offline): row 2i of the pair is gate channel
// i, row 2i+1 up channel i (packed codes and scales); the low-rank factors
// stack along r, L1^T as [gate; up] (two copies) and L2^T block-diagonally:
// row 2i = [gate L2^T row i, 0], row 2i+1 = [0, up L2^T row i].  One CTA per
// row of the pair.
__global__ void pack_gate_up_kernel(const uint8_t* __restrict__ Wq_g, const float* __restrict__ s_w_g,
                                    const uint16_t* __restrict__ L2t_g,
                                    const uint8_t* __restrict__ Wq_u, const float* __restrict__ s_w_u,
                                    const uint16_t* __restrict__ L2t_u, int K, int r,
                                    uint8_t* __restrict__ Wq2, float* __restrict__ s_w2,
                                    uint16_t* __restrict__ L2t2) {
  const int o = blockIdx.x, i = o >> 1;
  const bool up = o & 1;
  const uint4* src = reinterpret_cast<const uint4*>((up ? Wq_u : Wq_g) + (size_t)i * (K / 2));
  uint4* dst = reinterpret_cast<uint4*>(Wq2 + (size_t)o * (K / 2));
  for (int c = threadIdx.x; c < K / 32; c += blockDim.x) dst[c] = src[c];
  if (threadIdx.x == 0) s_w2[o] = (up ? s_w_u : s_w_g)[i];
  if (r > 0) {
    const uint4* l2 = reinterpret_cast<const uint4*>((up ? L2t_u : L2t_g) + (size_t)i * r);
    uint4* d2 = reinterpret_cast<uint4*>(L2t2 + (size_t)o * 2 * r);
    for (int c = threadIdx.x; c < r / 4; c += blockDim.x) {  // 2r bf16 = r/4 chunks
      const bool mine = up ? c >= r / 8 : c < r / 8;
      d2[c] = mine ? l2[up ? c - r / 8 : c] : make_uint4(0u, 0u, 0u, 0u);
    }
  }
}

}  // namespace

// 1 / (7 sqrt(b)^n): the codes' scale after n unnormalised transforms
static float scale_after(int had_block, int n) {
  return (float)(1.0 / (7.0 * pow(sqrt((double)had_block), (double)n)));
}

cudaError_t launch_quantize_act(const uint16_t* X, int M, int K, int had_block,
                                const uint16_t* L1t, int r, uint8_t* Xq, float* s_x, float* XL1,
                                cudaStream_t stream, const uint32_t* signs, int n_rht) {
  ActParams prm{};
  prm.X = reinterpret_cast<const __nv_bfloat16*>(X);
  prm.L1t = reinterpret_cast<const __nv_bfloat16*>(L1t);
  prm.Xq = Xq;
  prm.s_x = s_x;
  prm.XL1 = XL1;
  prm.M = M;
  prm.K = K;
  prm.b = had_block;
  prm.r = r;
  prm.signs = signs;
  prm.n_rht = signs ? n_rht : 1;
  prm.scale_mul = scale_after(had_block, prm.n_rht);
  // Many tokens: 128-token tiles, rotation and X L1 on the tensor cores, with
  // at most one sign mask (negated in shared memory before the rotation);
  // composed transforms take the butterfly kernel below.
  if ((!signs || prm.n_rht == 1) && act_tc_supported(M, K, had_block, r))
    return launch_act_tc(X, M, K, had_block, L1t, r, Xq, nullptr, s_x, XL1, nullptr, stream,
                         nullptr, signs);
  // Few token groups (decode): spread K over up to 16 CTAs of 256 columns.
  const int groups = (M + kActRows - 1) / kActRows;
  if (groups <= 8 && K % 256 == 0 && K / 256 <= 16) return launch_act_e<8>(prm, 16, stream);
  if (K % 512 == 0) return launch_act_e<16>(prm, 8, stream);
  if (K % 256 == 0) return launch_act_e<8>(prm, 8, stream);
  if (had_block <= 128) return launch_act_e<4>(prm, 8, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_act_bf_i8(const uint16_t* X, int M, int K, int had_block,
                                      const uint16_t* L1t, int r, int8_t* Xq8, float* s_x,
                                      uint16_t* XL1b, cudaStream_t stream, const uint32_t* signs,
                                      int n_rht) {
  ActParams prm{};
  prm.X = reinterpret_cast<const __nv_bfloat16*>(X);
  prm.L1t = reinterpret_cast<const __nv_bfloat16*>(L1t);
  prm.Xq8 = Xq8;
  prm.s_x = s_x;
  prm.XL1b = reinterpret_cast<__nv_bfloat16*>(XL1b);
  prm.M = M;
  prm.K = K;
  prm.b = had_block;
  prm.r = r;
  prm.signs = signs;
  prm.n_rht = signs ? n_rht : 1;
  prm.scale_mul = scale_after(had_block, prm.n_rht);
  const int groups = (M + kActRows - 1) / kActRows;
  if (groups <= 8 && K % 256 == 0 && K / 256 <= 16) return launch_act_e<8>(prm, 16, stream);
  if (K % 512 == 0) return launch_act_e<16>(prm, 8, stream);
  if (K % 256 == 0) return launch_act_e<8>(prm, 8, stream);
  if (had_block <= 128) return launch_act_e<4>(prm, 8, stream);
  return cudaErrorInvalidValue;
}

cudaError_t launch_pack_weight(const float* Rt, int N, int K, int had_block, uint8_t* Wq,
                               float* s_w, cudaStream_t stream, const uint32_t* signs, int n_rht) {
  const size_t smem = (size_t)K * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(pack_weight_kernel<float>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int n = signs ? n_rht : 1;
  pack_weight_kernel<float><<<N, kPackThreads, smem, stream>>>(Rt, K, had_block,
                                                                scale_after(had_block, n), Wq, s_w,
                                                                signs, n);
  return cudaGetLastError();
}

cudaError_t launch_pack_lowrank_q4(const uint16_t* L1t, const uint16_t* L2t, int N, int K, int r,
                                   int had_block, int8_t* qL1, float* s_L1, uint16_t* qL2,
                                   float* s_L2, cudaStream_t stream) {
  const size_t smem = (size_t)K * sizeof(float);
  auto pack = pack_weight_kernel<__nv_bfloat16, true>;
  cudaError_t e = cudaFuncSetAttribute(pack, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const float scale_mul = (float)(1.0 / (7.0 * sqrt((double)had_block)));
  pack<<<r, kPackThreads, smem, stream>>>(reinterpret_cast<const __nv_bfloat16*>(L1t), K, had_block,
                                          scale_mul, reinterpret_cast<uint8_t*>(qL1), s_L1,
                                          nullptr, 1);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lowrank_codes_kernel<<<(N + 7) / 8, 256, 0, stream>>>(
      reinterpret_cast<const __nv_bfloat16*>(L2t), nullptr, nullptr, nullptr, N, r,
      reinterpret_cast<__nv_bfloat16*>(qL2), s_L2);
  return cudaGetLastError();
}

cudaError_t launch_requant_xl1(const int32_t* acc, const float* s_x, const float* s_L1, int M,
                               int r, uint16_t* XL1q, float* s_xl1, cudaStream_t stream) {
  lowrank_codes_kernel<<<(M + 7) / 8, 256, 0, stream>>>(
      nullptr, acc, s_x, s_L1, M, r, reinterpret_cast<__nv_bfloat16*>(XL1q), s_xl1);
  return cudaGetLastError();
}

cudaError_t launch_weight_code_sums(const uint8_t* Wq, int N, int K, int32_t* wsum,
                                     cudaStream_t stream) {
  weight_code_sums_kernel<<<(N + 7) / 8, 256, 0, stream>>>(Wq, N, K, wsum);
  return cudaGetLastError();
}

cudaError_t launch_pack_gate_up(const uint8_t* Wq_g, const float* s_w_g, const uint16_t* L1t_g,
                                const uint16_t* L2t_g, const uint8_t* Wq_u, const float* s_w_u,
                                const uint16_t* L1t_u, const uint16_t* L2t_u, int N, int K, int r,
                                uint8_t* Wq2, float* s_w2, uint16_t* L1t2, uint16_t* L2t2,
                                cudaStream_t stream) {
  if (r > 0) {
    const size_t bytes = (size_t)r * K * 2;
    if (cudaError_t e = cudaMemcpyAsync(L1t2, L1t_g, bytes, cudaMemcpyDeviceToDevice, stream))
      return e;
    if (cudaError_t e = cudaMemcpyAsync(L1t2 + (size_t)r * K, L1t_u, bytes,
                                        cudaMemcpyDeviceToDevice, stream))
      return e;
  }
  pack_gate_up_kernel<<<2 * N, 128, 0, stream>>>(Wq_g, s_w_g, L2t_g, Wq_u, s_w_u, L2t_u, K, r, Wq2,
                                                  s_w2, L2t2);
  return cudaGetLastError();
}

}  // namespace tq
