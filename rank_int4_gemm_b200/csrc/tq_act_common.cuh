// tq_act_common.cuh -- device helpers shared by the activation kernel and the
// fused decode layer: the warp-level Sylvester transform, the RoundClip code,
// the packed-code store, and mma.sync / ldmatrix / DSMEM wrappers.  Both
// kernels use these same functions, so a token's codes do not depend on which
// kernel computed them.
#pragma once
#include <cuda_bf16.h>

#include <cstdint>

#include "tq_ptx.cuh"

namespace tq {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v = fmaxf(v, __shfl_xor_sync(kFull, v, o));
  return v;
}

// Unnormalised Sylvester transform over blocks of b consecutive values; a lane
// holds E consecutive values, so a block spans b/E lanes when b > E.
template <int E>
__device__ __forceinline__ void fwht_warp(float (&v)[E], int b) {
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
    if (h < b) {
#pragma unroll
      for (int i = 0; i < E; ++i) {
        if ((i & h) == 0) {
          const float a = v[i], c = v[i + h];
          v[i] = a + c;
          v[i + h] = a - c;
        }
      }
    }
  }
  const uint32_t lane = threadIdx.x & 31u;
  for (int s = 1; s * E < b; s <<= 1) {
    const bool upper = (lane & (uint32_t)s) != 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(kFull, v[i], s);
      v[i] = upper ? (o - v[i]) : (v[i] + o);
    }
  }
}

// RoundClip(v * inv) with ties to even.
__device__ __forceinline__ int quant_code(float v, float inv) {
  float t = rintf(v * inv);
  t = fminf(fmaxf(t, -7.f), 7.f);
  return (int)t;
}

// Writes the E codes of this lane into the packed layout: inside a 32-code
// group byte i = code i | code (i+16) << 4.  The lanes holding codes i and
// i+16 of a group exchange nibbles and each writes half of their bytes.
// `row_bytes` points at the byte of the row where this warp pass starts.
template <int E>
__device__ __forceinline__ void store_packed(const int (&q)[E], uint8_t* row_bytes) {
  constexpr int G = 32 / E;  // lanes per 32-code group
  constexpr int H = G / 2;   // lanes holding the low nibbles
  uint64_t mine = 0;
#pragma unroll
  for (int i = 0; i < E; ++i) mine |= (uint64_t)(q[i] & 0xF) << (4 * i);
  const int lane = (int)(threadIdx.x & 31u);
  const uint64_t other = __shfl_xor_sync(kFull, mine, H);
  const int a = lane % G;
  const bool low_side = a < H;
  const uint64_t lo = low_side ? mine : other;
  const uint64_t hi = low_side ? other : mine;
  const int nib0 = low_side ? 0 : E / 2;
  uint64_t out = 0;
#pragma unroll
  for (int i = 0; i < E / 2; ++i) {
    const uint64_t l = (lo >> (4 * (nib0 + i))) & 0xFull;
    const uint64_t h = (hi >> (4 * (nib0 + i))) & 0xFull;
    out |= (l | (h << 4)) << (8 * i);
  }
  uint8_t* dst = row_bytes + (lane / G) * 16 + (a % H) * E + nib0;
  if constexpr (E == 16) {
    *reinterpret_cast<uint64_t*>(dst) = out;
  } else if constexpr (E == 8) {
    *reinterpret_cast<uint32_t*>(dst) = (uint32_t)out;
  } else {
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)out;
  }
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldmatrix_x2(uint32_t (&r)[2], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];"
               : "=r"(r[0]), "=r"(r[1])
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&d)[4], const uint32_t (&a)[4],
                                          const uint32_t (&b)[2]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

__device__ __forceinline__ void dsmem_st_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// Loads E consecutive bf16 values of a row from shared memory as fp32.
template <int E>
__device__ __forceinline__ void load_row_values(const __nv_bfloat16* src, float (&v)[E]) {
  if constexpr (E >= 8) {
#pragma unroll
    for (int i = 0; i < E; i += 8) {  // 16-byte aligned: lane * E * 2 bytes
      const uint4 u = *reinterpret_cast<const uint4*>(src + i);
      const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 f = __bfloat1622float2(h2[j]);
        v[i + 2 * j] = f.x;
        v[i + 2 * j + 1] = f.y;
      }
    }
  } else {  // E == 4: one 8-byte load
    const uint2 u = *reinterpret_cast<const uint2*>(src);
    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const float2 f = __bfloat1622float2(h2[j]);
      v[2 * j] = f.x;
      v[2 * j + 1] = f.y;
    }
  }
}


}  // namespace tq
