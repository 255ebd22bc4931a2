// Dequantizers of the tensor-core GEMM regime: packed words (plus group scale,
// bias or zero) -> 16-byte chunks of the A operand (bf16, fp16 or int8), for the
// MLX affine layout (2/4/8-bit), the GPTQ int4 layout and symmetric int4.
// Shared by the per-tile kernel (k_gemm_tc.cu) and the persistent kernel
// (k_gemm_tc2.cu).
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cstdint>

namespace gwb {
namespace dq {

// (a & mask) | magic as a single LOP3.  Written as inline asm with the magic in
// a register: left to itself the compiler splits the two-immediate form into
// two instructions.
template <uint32_t MASK>
__device__ __forceinline__ uint32_t lop_and_or(uint32_t a, uint32_t magic) {
  uint32_t r;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(a), "n"(MASK), "r"(magic));
  return r;
}
__device__ __forceinline__ float bf16_val(uint16_t h) { return __uint_as_float(static_cast<uint32_t>(h) << 16); }

__device__ __forceinline__ uint32_t bf162_bits(__nv_bfloat162 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) { return *reinterpret_cast<__nv_bfloat162 *>(&u); }
__device__ __forceinline__ uint32_t h2_bits(__half2 v) { return *reinterpret_cast<uint32_t *>(&v); }
__device__ __forceinline__ __half2 as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// Byte offset of 16-byte chunk `c` of row `r` in a 128-byte-swizzled K-major tile.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

// ---------------------------------------------------------------- dequantizers
// Affine, 4-bit: one word = 8 consecutive k = one 16-byte chunk of bf16.
// Pair p (k = 2p, 2p+1) sits in byte p of the word; PRMT moves the low nibble
// of byte p of w and of w>>4 into the two halves, and OR-ing 0x4300 makes the
// exact bf16 value 128 + code.
__device__ __forceinline__ uint4 dq_affine4(uint32_t w, __nv_bfloat162 s2, __nv_bfloat162 b2) {
  const uint32_t t = w >> 4;
  const __nv_bfloat162 m128 = __floats2bfloat162_rn(128.0f, 128.0f);
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t pr = lop_and_or<0x000F000Fu>(__byte_perm(w, t, p | ((4 + p) << 8)), 0x43004300u);
    o[p] = bf162_bits(__hfma2(__hsub2(as_bf162(pr), m128), s2, b2));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Affine, 2-bit: one word = 16 consecutive k = two chunks.  Pair p (k = 2p,
// 2p+1) is nibble p; its two codes land at bits 0-1 (value 128 + q) and bits
// 2-3 of the high half (value 128 + 4q), so the high half uses scale s/4.
__device__ __forceinline__ void dq_affine2(uint32_t w, __nv_bfloat162 s2q, __nv_bfloat162 b2, uint4 &c0, uint4 &c1) {
  const uint32_t t = w >> 4;
  const __nv_bfloat162 m128 = __floats2bfloat162_rn(128.0f, 128.0f);
  uint32_t o[8];
#pragma unroll
  for (int p = 0; p < 8; p++) {
    const uint32_t idx = (p & 1) ? (4 + (p >> 1)) : (p >> 1);
    const uint32_t pr = lop_and_or<0x000C0003u>(__byte_perm(w, t, idx | (idx << 8)), 0x43004300u);
    o[p] = bf162_bits(__hfma2(__hsub2(as_bf162(pr), m128), s2q, b2));
  }
  c0 = make_uint4(o[0], o[1], o[2], o[3]);
  c1 = make_uint4(o[4], o[5], o[6], o[7]);
}

// Affine, 8-bit: codes above 127 do not fit the bf16 mantissa trick, so each
// byte becomes the fp32 2^23 + code (exact), then fmaf(code, s, b) in fp32 and
// a paired round to bf16.  Two words = one chunk.
__device__ __forceinline__ uint4 dq_affine8(uint32_t w0, uint32_t w1, float s, float b) {
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 2; h++) {
    const uint32_t w = h ? w1 : w0;
#pragma unroll
    for (int p = 0; p < 2; p++) {
      const float lo = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540 | (2 * p))) - 8388608.0f;
      const float hi = __uint_as_float(__byte_perm(w, 0x4B000000u, 0x7540 | (2 * p + 1))) - 8388608.0f;
      o[2 * h + p] = bf162_bits(__floats2bfloat162_rn(fmaf(lo, s, b), fmaf(hi, s, b)));
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// GPTQ: one qweight word = 8 consecutive k of one out-feature = one chunk of
// fp16.  (1024 + q) - (1024 + zero) is exact, and the product with the fp16
// scale is the single rounding gptq_dequant also performs.
__device__ __forceinline__ uint4 dq_gptq(uint32_t w, const uint32_t (&z2)[4], const uint32_t (&s2)[4]) {
  const uint32_t t = w >> 4;
  uint32_t o[4];
#pragma unroll
  for (int p = 0; p < 4; p++) {
    const uint32_t pr = lop_and_or<0x000F000Fu>(__byte_perm(w, t, p | ((4 + p) << 8)), 0x64006400u);
    o[p] = h2_bits(__hmul2(__hsub2(as_h2(pr), as_h2(z2[p])), as_h2(s2[p])));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// Symmetric int4 -> int8: each nibble is placed in the high half of its byte,
// i.e. the byte holds 16 * code as a signed int8; the accumulator is divided
// by 16 (exactly) in the epilogue.  Two words = one 16-byte chunk.
__device__ __forceinline__ uint2 dq_i4(uint32_t w) {
  const uint32_t lo = (w << 4) & 0xF0F0F0F0u;  // codes 0,2,4,6
  const uint32_t hi = w & 0xF0F0F0F0u;         // codes 1,3,5,7
  return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

}  // namespace dq
}  // namespace gwb
