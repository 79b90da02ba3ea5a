// kvq_decode_common.cuh — device helpers shared by the two decode kernels (code unpacking to exact
// fp16, hi/lo fp16 splitting of fp32 operands, base-2 exponentials).
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace kvq {

__device__ __forceinline__ uint32_t hsub2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Eight exact fp16x2 code pairs from a 2-bit word, pair k of the word in element k.
__device__ __forceinline__ void unpack_word2(uint32_t x, uint32_t (&h)[8]) {
  const uint32_t y = x >> 10;
  h[0] = hsub2((x & 0x00030003u) | 0x64006400u, 0x64006400u);  // 1024 + c
  h[1] = hsub2((x & 0x000C000Cu) | 0x5C005C00u, 0x5C005C00u);  // 256 + c
  h[2] = hsub2((x & 0x00300030u) | 0x54005400u, 0x54005400u);  // 64 + c
  h[3] = hsub2((x & 0x00C000C0u) | 0x4C004C00u, 0x4C004C00u);  // 16 + c
  h[4] = hsub2((x & 0x03000300u) | 0x44004400u, 0x44004400u);  // 4 + c
  h[5] = hsub2((y & 0x00030003u) | 0x64006400u, 0x64006400u);
  h[6] = hsub2((y & 0x000C000Cu) | 0x5C005C00u, 0x5C005C00u);
  h[7] = hsub2((y & 0x00300030u) | 0x54005400u, 0x54005400u);
}

// Four exact fp16x2 code pairs from a 4-bit word.
__device__ __forceinline__ void unpack_word4(uint32_t x, uint32_t (&h)[4]) {
  const uint32_t y = x >> 8;
  h[0] = hsub2((x & 0x000F000Fu) | 0x64006400u, 0x64006400u);  // 1024 + c
  h[1] = hsub2((x & 0x00F000F0u) | 0x54005400u, 0x54005400u);  // 64 + c
  h[2] = hsub2((y & 0x000F000Fu) | 0x64006400u, 0x64006400u);
  h[3] = hsub2((y & 0x00F000F0u) | 0x54005400u, 0x54005400u);
}

// Value codes are used centered, c - (2^b - 1)/2, so that sum_t p_t * sv * code does not carry the
// group minimum's large offset (the offset moves into the group midpoint, see below). With 2-bit
// codes the centered value is exact in fp16 after one subtraction of (2^(10-2k) + 1.5), except at
// the pair positions whose constant is 1024 (spacing 1), which subtract 1024 and then 1.5.
__device__ __forceinline__ void unpack_word2_centered(uint32_t x, uint32_t (&h)[8]) {
  const uint32_t y = x >> 10;
  h[0] = hsub2(hsub2((x & 0x00030003u) | 0x64006400u, 0x64006400u), 0x3E003E00u);  // c - 1.5
  h[1] = hsub2((x & 0x000C000Cu) | 0x5C005C00u, 0x5C065C06u);                      // 256 + c - 257.5
  h[2] = hsub2((x & 0x00300030u) | 0x54005400u, 0x54185418u);                      // 64 + c - 65.5
  h[3] = hsub2((x & 0x00C000C0u) | 0x4C004C00u, 0x4C604C60u);                      // 16 + c - 17.5
  h[4] = hsub2((x & 0x03000300u) | 0x44004400u, 0x45804580u);                      // 4 + c - 5.5
  h[5] = hsub2(hsub2((y & 0x00030003u) | 0x64006400u, 0x64006400u), 0x3E003E00u);
  h[6] = hsub2((y & 0x000C000Cu) | 0x5C005C00u, 0x5C065C06u);
  h[7] = hsub2((y & 0x00300030u) | 0x54005400u, 0x54185418u);
}

// 4-bit codes centered at 7.5.
__device__ __forceinline__ void unpack_word4_centered(uint32_t x, uint32_t (&h)[4]) {
  const uint32_t y = x >> 8;
  h[0] = hsub2(hsub2((x & 0x000F000Fu) | 0x64006400u, 0x64006400u), 0x47804780u);  // c - 7.5
  h[1] = hsub2((x & 0x00F000F0u) | 0x54005400u, 0x54785478u);                      // 64 + c - 71.5
  h[2] = hsub2(hsub2((y & 0x000F000Fu) | 0x64006400u, 0x64006400u), 0x47804780u);
  h[3] = hsub2((y & 0x00F000F0u) | 0x54005400u, 0x54785478u);
}

// Subnormal unpacking (the mma.sync decode). A code AND-ed out in place at bit offset o of a 16-bit half
// reads, as an fp16 with a zero exponent field, as the subnormal code * 2^(o - 24): exact, one AND with
// an immediate per code pair, and no constant to OR in or subtract. Each position's power of two is
// taken out again around the tensor-core product (on the other operand and on the result rows).
//
// 2-bit: pairs 0..3 of the word from bits 0, 2, 4, 6 and pairs 4..7 from bits 8 .. 14 shifted down to
// the same offsets, so element k of each group of four carries 2^(2k - 24).
__device__ __forceinline__ void unpack_word2_sub(uint32_t x, uint32_t (&h)[8]) {
  const uint32_t y = x >> 8;
  h[0] = x & 0x00030003u;
  h[1] = x & 0x000C000Cu;
  h[2] = x & 0x00300030u;
  h[3] = x & 0x00C000C0u;
  h[4] = y & 0x00030003u;
  h[5] = y & 0x000C000Cu;
  h[6] = y & 0x00300030u;
  h[7] = y & 0x00C000C0u;
}

// 4-bit: elements 0, 2 carry 2^-24 and elements 1, 3 carry 2^-20.
__device__ __forceinline__ void unpack_word4_sub(uint32_t x, uint32_t (&h)[4]) {
  const uint32_t y = x >> 8;
  h[0] = x & 0x000F000Fu;
  h[1] = x & 0x00F000F0u;
  h[2] = y & 0x000F000Fu;
  h[3] = y & 0x00F000F0u;
}

// Centered value codes as subnormals: the code is taken one bit higher (2c), and the odd integer
// 2c - (2^b - 1) = 2 (c - cbar) stays exact after one subnormal subtraction (fixed-point, no rounding).
// Scales per element as in unpack_word2_sub / unpack_word4_sub.
__device__ __forceinline__ void unpack_word2_centered_sub(uint32_t x, uint32_t (&h)[8]) {
  const uint32_t z = x << 1, y = x >> 7;
  h[0] = hsub2(z & 0x00060006u, 0x00030003u);  // (2c - 3) 2^-24
  h[1] = hsub2(z & 0x00180018u, 0x000C000Cu);  // (2c - 3) 2^-22
  h[2] = hsub2(z & 0x00600060u, 0x00300030u);  // (2c - 3) 2^-20
  h[3] = hsub2(z & 0x01800180u, 0x00C000C0u);  // (2c - 3) 2^-18
  h[4] = hsub2(y & 0x00060006u, 0x00030003u);
  h[5] = hsub2(y & 0x00180018u, 0x000C000Cu);
  h[6] = hsub2(y & 0x00600060u, 0x00300030u);
  h[7] = hsub2(y & 0x01800180u, 0x00C000C0u);
}

__device__ __forceinline__ void unpack_word4_centered_sub(uint32_t x, uint32_t (&h)[4]) {
  const uint32_t z = x << 1, y = x >> 7;
  h[0] = hsub2(z & 0x001E001Eu, 0x000F000Fu);  // (2c - 15) 2^-24
  h[1] = hsub2(z & 0x01E001E0u, 0x00F000F0u);  // (2c - 15) 2^-20
  h[2] = hsub2(y & 0x001E001Eu, 0x000F000Fu);
  h[3] = hsub2(y & 0x01E001E0u, 0x00F000F0u);
}

// hi keeps the leading 11 significant bits of x (exact in fp16 when x is in fp16's normal range),
// lo = x - hi exactly; each fp16 column gets one of them.
__device__ __forceinline__ float split_part(float x, bool lo) {
  const float hi = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
  return lo ? __fsub_rn(x, hi) : hi;
}
__device__ __forceinline__ uint32_t pack_h2(float a, float b) {
  const __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}
__device__ __forceinline__ float pow2i(int e) { return __int_as_float((127 + e) << 23); }

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

}  // namespace kvq
