// kvq_common.cuh — device helpers shared by the libkvq kernels (sm_100a).
//
// Codec (every kernel that writes codes uses exactly these steps, in IEEE fp32 with explicit
// round-to-nearest intrinsics so nothing is contracted into an FMA):
//   group min mn / max mx under the IEEE total order (-0 below +0);
//   s32 = (f32(mx) - f32(mn)) / (2^b - 1);  s16 = fp16_rn(s32);  zero = mn;
//   s16 == 0 -> code 0; else code = clamp(rint_even((f32(x) - f32(mn)) * (1 / f32(s16))), 0, 2^b-1).
// The uniform min/max grid at 2 or 4 bits with per-channel key groups and per-token value groups is
// the KIVI-style recipe (KVQuant review, Method and Comparison; KV cache quantization wiki page,
// KIVI notes). The exact fp32 formula is this library's fixed reading.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

#include "kvq.h"

namespace kvq {

constexpr int kHeadDim = 128;
constexpr int kTile = 16;  // tokens per packed tile

__host__ __device__ inline int64_t quantized_len(int64_t T, int R, int G) {
  const int64_t over = T - R;
  return over > 0 ? (over / G) * G : 0;
}

// Words per unit-tile and per-unit buffer extents.
__host__ __device__ inline int64_t tile_words(int bits) { return 64 * bits; }

// --- fp16 total order (-0 < +0) on raw bits -------------------------------------------------------
__device__ __forceinline__ uint32_t order_key(uint32_t h) {
  return (h & 0x8000u) ? (~h & 0xffffu) : (h | 0x8000u);
}
__device__ __forceinline__ uint16_t key_to_half(uint32_t k) {
  return static_cast<uint16_t>((k & 0x8000u) ? (k & 0x7fffu) : (~k & 0xffffu));
}

struct QuantParams {
  float zf;      // f32(mn)
  float inv;     // 1 / f32(s16)
  uint16_t s16;  // scale bits
  uint16_t z16;  // zero bits (= mn)
  bool zero_scale;
};

__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }

// Scale / zero of a group from its min and max keys (order_key values).
__device__ __forceinline__ QuantParams make_params(uint32_t kmin, uint32_t kmax, int bits) {
  QuantParams p;
  p.z16 = key_to_half(kmin);
  const uint16_t mx = key_to_half(kmax);
  p.zf = h2f(p.z16);
  const float range = __fsub_rn(h2f(mx), p.zf);
  const float s32 = __fdiv_rn(range, static_cast<float>((1 << bits) - 1));
  p.s16 = __half_as_ushort(__float2half_rn(s32));
  p.zero_scale = (p.s16 & 0x7fffu) == 0;
  p.inv = p.zero_scale ? 0.0f : __fdiv_rn(1.0f, h2f(p.s16));
  return p;
}

// --- tile v1 layout ----------------------------------------------------------------------------------
// Word index `widx` of a tile (0 .. 64*bits-1) -> (lane, logical word w).
__device__ __forceinline__ void widx_to_lane_word(int widx, int* lane, int* w) {
  const int slab = widx >> 7, rem = widx & 127;
  *lane = rem >> 2;
  *w = slab * 4 + (rem & 3);
}
// Pair slot p of lane -> (token in tile, channel) of the pair's first code (e = 0), and the offset
// of the second code (e = 1): keys step one channel, values step one token.
__device__ __forceinline__ void key_slot(int lane, int p, int* i, int* c) {
  const int m = p >> 2, u = p & 1, hh = (p >> 1) & 1, r = lane >> 2, qd = lane & 3;
  *i = r + 8 * u;
  *c = 16 * m + 2 * qd + 8 * hh;
}
__device__ __forceinline__ void value_slot(int lane, int p, int* i, int* c) {
  const int m = p >> 2, u = p & 1, hh = (p >> 1) & 1, r = lane >> 2, qd = lane & 3;
  *i = 2 * qd + 8 * hh;
  *c = 16 * m + r + 8 * u;
}
// Position of channel c inside a key group's 128 scale / zero entries.
__device__ __forceinline__ int key_param_pos(int c) {
  const int m = c >> 4, within = c & 15;
  const int hh = within >> 3, qd = (within & 7) >> 1, e = within & 1;
  return 32 * qd + 4 * m + 2 * hh + e;
}

// --- dense-and-sparse outliers ------------------------------------------------------------------------
// KVQuant review, Method: a small share of the entries stays in fp16, chosen per vector. For each of
// the n staged rows (stride `stride` halves), the entry of largest magnitude, ties to the lowest
// channel: fp16 magnitudes order like the integers of their low 15 bits, so the wanted entry has the
// largest (|x| bits << 7) | (127 - channel). One warp per row (nwarps warps take part); the lane holding
// the entry records its channel in och[i] (0xff: none, which is row 0 when `sink_first`) and the word
// channel | fp16 value << 16 in out[i] (0xffff: none). With `replace` the entry is then overwritten
// with its neighbour ch ^ 1, which lies in the same value group (G is even), so that group's min / max
// become those of its other entries.
__device__ __forceinline__ void select_outliers(uint16_t* rows, int stride, int n, uint32_t* out, uint8_t* och,
                                                bool sink_first, bool replace, int nwarps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < n; i += nwarps) {
    const uint2 x = *reinterpret_cast<const uint2*>(rows + i * stride + 4 * lane);
    const uint32_t h[4] = {x.x & 0xffffu, x.x >> 16, x.y & 0xffffu, x.y >> 16};
    uint32_t key = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) key = max(key, ((h[e] & 0x7fffu) << 7) | (127u - (4 * lane + e)));
    key = __reduce_max_sync(0xffffffffu, key);
    const int ch = 127 - static_cast<int>(key & 127u);
    if (lane == (ch >> 2)) {
      const bool none = sink_first && i == 0;
      const int e = ch & 3;
      const uint32_t val = e == 0 ? h[0] : e == 1 ? h[1] : e == 2 ? h[2] : h[3];
      const uint32_t nbr = e == 0 ? h[1] : e == 1 ? h[0] : e == 2 ? h[3] : h[2];
      och[i] = none ? 0xffu : static_cast<uint8_t>(ch);
      out[i] = none ? 0xffffu : (static_cast<uint32_t>(ch) | (val << 16));
      if (replace && !none) rows[i * stride + ch] = static_cast<uint16_t>(nbr);
    }
  }
}

// --- 128-point Walsh-Hadamard rotation ----------------------------------------------------------------
// Sylvester-ordered butterflies with strides 1, 2, ..., 64 (pair (i, i+h) -> (a+b, a-b)) in fp32,
// then one multiply by fp32(1/sqrt(128)) (bit pattern 0x3DB504F3). The framework page (In practice)
// fuses this rotation into the kernels; the Dual-QK abstract notes the query must get the same
// orthogonal transform. Every butterfly is the same IEEE operation whichever thread evaluates it,
// so the result is independent of the thread mapping.
__device__ __forceinline__ float inv_sqrt128() { return __uint_as_float(0x3DB504F3u); }

// Rotate 128 values held 8 per thread by 16 consecutive lanes (lane & 15 owns elements
// 8*(lane&15) .. +7). All 32 lanes of the warp must call it (two rows per warp).
__device__ __forceinline__ void wht128_16lanes(float x[8]) {
#pragma unroll
  for (int h = 1; h < 8; h <<= 1) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if ((i & h) == 0) {
        const float a = x[i], b = x[i + h];
        x[i] = __fadd_rn(a, b);
        x[i + h] = __fsub_rn(a, b);
      }
  }
  const int sub = threadIdx.x & 15;
#pragma unroll
  for (int d = 1; d < 16; d <<= 1) {  // element stride 8*d
    // lower lane holds a (first of the pair) and makes a + b; upper lane holds b and makes a - b.
    // fma(+-1, x, other) rounds the exact sum once, the same as the IEEE add / subtract (signed
    // zeros included), in one instruction.
    const float sgn = (sub & d) != 0 ? -1.f : 1.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float other = __shfl_xor_sync(0xffffffffu, x[i], d);
      x[i] = __fmaf_rn(sgn, x[i], other);
    }
  }
  const float s = inv_sqrt128();
#pragma unroll
  for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(x[i], s);
}

}  // namespace kvq
