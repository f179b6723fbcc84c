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
  // across lanes: the upper partner keeps o - v, the lower v + o; both are
  // one correctly rounded fma with a +-1 multiplier
  const uint32_t lane = threadIdx.x & 31u;
  for (int s = 1; s * E < b; s <<= 1) {
    const float sgn = (lane & (uint32_t)s) ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(kFull, v[i], s);
      v[i] = fmaf(sgn, v[i], o);
    }
  }
}

// Randomized Hadamard transform: x D H with D = diag(d), d_k = -1 where
// bit (k % 32) of word k / 32 of `signs` is set.  Negates (sign-bit flip,
// exact) the E values of columns col0 .. col0 + E - 1 held by this thread
// before the butterflies; col0 is a multiple of E and E divides 32.
template <int E>
__device__ __forceinline__ void apply_signs(float (&v)[E], const uint32_t* signs, int col0) {
  if (!signs) return;
  const uint32_t w = __ldg(signs + (col0 >> 5)) >> (col0 & 31);
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] = __uint_as_float(__float_as_uint(v[i]) ^ (((w >> i) & 1u) << 31));
}

// x D_1 H D_2 H ... D_n H on this lane's E values (n_rht composed randomized
// Hadamard transforms, masks of `words` words each, the first first), or x H
// without masks.  n_rht is warp-uniform (the butterflies shuffle).
template <int E>
__device__ __forceinline__ void rotate_signed(float (&v)[E], const uint32_t* signs, int n_rht,
                                              int words, int col0, int b) {
  if (!signs) {
    fwht_warp<E>(v, b);
    return;
  }
  for (int i = 0; i < n_rht; ++i) {
    apply_signs<E>(v, signs + (size_t)i * words, col0);
    fwht_warp<E>(v, b);
  }
}

// RoundClip(v * inv) with ties to even, for any v and inv (weights).
__device__ __forceinline__ int quant_code(float v, float inv) {
  float t = rintf(v * inv);
  t = fminf(fmaxf(t, -7.f), 7.f);
  return (int)t;
}

// Activation codes of a row with absmax `am` (over the same fp32 values that
// are quantized).  With inv = 7 / am and |v| <= am the product y = v * inv
// has |y| <= 7 (1 + 2^-23), so RoundClip's clip never acts, and adding
// 1.5 * 2^23 rounds y to an integer with ties to even (the sum lies in
// [2^23, 2^24), where the float spacing is 1), leaving the integer in two's
// complement in the low mantissa bits: the low byte of the sum's bit pattern
// is the code as an int8.  A row with a tiny absmax is first scaled by 2^64
// (exact) so that 7 / am stays finite.
struct CodeScale {
  float pre;  // 1, or 2^64 for a tiny row
  float inv;  // 7 / (am * pre), or 0 for an all-zero row
};
__device__ __forceinline__ CodeScale code_scale(float am) {
  CodeScale c{1.f, 0.f};
  if (am > 0.f) {
    if (am < 1e-30f) c.pre = 0x1p64f;
    c.inv = 7.f / (am * c.pre);
  }
  return c;
}
__device__ __forceinline__ uint32_t code_bits(float v, float inv) {
  return __float_as_uint(__fadd_rn(__fmul_rn(v, inv), 12582912.f));
}
// Byte j of the result is the low byte of the j-th argument.
__device__ __forceinline__ uint32_t low_bytes4(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}
// Eight int8 codes (two words, code j in byte j % 4) -> eight nibbles, code j
// in bits 4j..4j+3.
__device__ __forceinline__ uint32_t nibbles8(uint32_t w0, uint32_t w1) {
  w0 &= 0x0F0F0F0Fu;
  w1 &= 0x0F0F0F0Fu;
  w0 |= w0 >> 4;
  w1 |= w1 >> 4;
  return __byte_perm(w0, w1, 0x6420);
}
// Nibbles 4h..4h+3 of x, one per byte (low nibble) of the result.
__device__ __forceinline__ uint32_t spread4(uint32_t x, int h) {
  const uint32_t e = __byte_perm(x, 0u, h ? 0x3322 : 0x1100);
  return (e & 0x000F000Fu) | ((e >> 4) & 0x0F000F00u);
}

// Writes the E codes of this lane into the packed layout: inside a 32-code
// group byte i = code i | code (i+16) << 4.  The lanes holding codes i and
// i+16 of a group exchange nibbles and each writes half of their bytes.
// `row_bytes` points at the byte of the row where this warp pass starts.
template <int E>
__device__ __forceinline__ void store_packed(const uint32_t (&cb)[E], uint8_t* row_bytes) {
  constexpr int G = 32 / E;  // lanes per 32-code group
  constexpr int H = G / 2;   // lanes holding the low nibbles
  // this lane's codes as nibbles, code i in bits 4i..4i+3
  uint32_t mine[2] = {0u, 0u};
  if constexpr (E == 4) {
    mine[0] = nibbles8(low_bytes4(cb[0], cb[1], cb[2], cb[3]), 0u) & 0xFFFFu;
  } else {
#pragma unroll
    for (int h = 0; h < E / 8; ++h)
      mine[h] = nibbles8(low_bytes4(cb[8 * h], cb[8 * h + 1], cb[8 * h + 2], cb[8 * h + 3]),
                         low_bytes4(cb[8 * h + 4], cb[8 * h + 5], cb[8 * h + 6], cb[8 * h + 7]));
  }
  const int lane = (int)(threadIdx.x & 31u);
  const int a = lane % G;
  const bool low_side = a < H;
  // each lane writes E/2 bytes, codes nib0 .. nib0 + E/2 - 1 of its lane
  // pair; the partner holds the other nibble of each of those bytes
  const int nib0 = low_side ? 0 : E / 2;
  uint8_t* dst = row_bytes + (lane / G) * 16 + (a % H) * E + nib0;
  if constexpr (E == 16) {
    const uint32_t got = __shfl_xor_sync(kFull, low_side ? mine[1] : mine[0], H);
    const uint32_t lo = low_side ? mine[0] : got;
    const uint32_t hi = low_side ? got : mine[1];
    uint2 out;
    out.x = spread4(lo, 0) | (spread4(hi, 0) << 4);
    out.y = spread4(lo, 1) | (spread4(hi, 1) << 4);
    *reinterpret_cast<uint2*>(dst) = out;
  } else if constexpr (E == 8) {
    uint32_t other[1] = {__shfl_xor_sync(kFull, mine[0], H)};
    const uint32_t lo = (low_side ? mine[0] : other[0]) >> (4 * nib0);
    const uint32_t hi = (low_side ? other[0] : mine[0]) >> (4 * nib0);
    *reinterpret_cast<uint32_t*>(dst) = spread4(lo, 0) | (spread4(hi, 0) << 4);
  } else {
    uint32_t other[1] = {__shfl_xor_sync(kFull, mine[0], H)};
    const uint32_t lo = (low_side ? mine[0] : other[0]) >> (4 * nib0);
    const uint32_t hi = (low_side ? other[0] : mine[0]) >> (4 * nib0);
    *reinterpret_cast<uint16_t*>(dst) = (uint16_t)(spread4(lo, 0) | (spread4(hi, 0) << 4));
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
