// kvq_decode.cu — split-K decode attention that reads the packed cache directly, plus the split
// combine.
//
// Decode is bandwidth-bound: every step reads the whole cache once (NOVA-KV abstract on the
// thelatestinai listing), and the compressed cache is consumed by custom kernels without being
// expanded in memory (KVQuant review, Method). The grouped (quantized) part and the FP16 residual
// part both enter the same softmax (KV cache quantization wiki page, KIVI notes on combining the
// grouped and residual parts when computing the scores).
//
// Work split. The grid is (split, unit) with unit = (sequence, KV head). A CTA of 4 warps owns one
// token range of split_len tokens; each warp owns a contiguous run of 16-token tiles of it (so a key
// group's query fold is built once per group per warp) and round-robin the FP16 residual tokens.
// Tiles stream through a per-warp 4-stage cp.async ring (codes, value scale/zero and, at a group
// boundary, the group's key scale/zero) so about 4 tiles per warp are in flight.
//
// Arithmetic (per 16-token tile; scores in base-2 units, q already multiplied by sm_scale*log2 e):
//   QK: s_t = 2^e * (sum_c code[t][c] * (q^[c] * sk[g][c]) + sum_c q^[c] * zk[g][c]), q^ = q * 2^-e.
//       The code sum runs on the tensor cores (mma m16n8k16, tokens on M, channels on K); A = exact
//       fp16 codes unpacked straight from the packed words, B = q^ * sk split into hi + lo fp16
//       parts in separate N columns (columns 2h, 2h+1 = head h hi / lo), so the products keep ~22
//       significant bits; the zero-point term is an fp32 dot per group.
//   PV: o[c] = sum_t (p_t * sv[t][j]) * (code[t][c] - cbar) + sum_t p_t * mid[t][j], j = c / G, with
//       cbar = (2^b - 1) / 2 and mid = zv + cbar * sv the midpoint of the token's value group. The
//       first sum is an mma with channels on M, tokens on K, A = the centered codes (exact in fp16),
//       B = p * sv (hi + lo per head); the second is an fp32 accumulator per (head, channel group).
//       Centering keeps both sums the size of the result: with the zero-point (the group minimum)
//       left in, each sum would be ~|min| / |o| times larger than the output and the fp32
//       accumulation error of a million-token sum would be amplified by that cancellation.
//   Online softmax keeps a running max per head; accumulators are rescaled only when some head's
//   max moves.
// Codes -> fp16: a 2-bit code at bit 2k of a 16-bit half is OR-ed into the mantissa of the fp16
// constant 2^(10-2k) (so the half reads 2^(10-2k) + code) and the constant is subtracted again: two
// ALU instructions per pair of codes, exact. 4-bit codes use 2^(10-4k) the same way.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kStages = 4;
constexpr unsigned kFull = 0xffffffffu;

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

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
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

// Load 2*VPT consecutive fp16 (aligned to 4*VPT bytes) as floats.
template <int VPT>
__device__ __forceinline__ void load_halves(const uint8_t* p, float (&out)[2 * VPT]) {
  uint32_t w[VPT];
  if constexpr (VPT == 1) {
    w[0] = *reinterpret_cast<const uint32_t*>(p);
  } else if constexpr (VPT == 2) {
    const uint2 v = *reinterpret_cast<const uint2*>(p);
    w[0] = v.x;
    w[1] = v.y;
  } else {
#pragma unroll
    for (int i = 0; i < VPT / 4; ++i) {
      const uint4 v = reinterpret_cast<const uint4*>(p)[i];
      w[4 * i] = v.x;
      w[4 * i + 1] = v.y;
      w[4 * i + 2] = v.z;
      w[4 * i + 3] = v.w;
    }
  }
#pragma unroll
  for (int i = 0; i < VPT; ++i) {
    out[2 * i] = h2f(static_cast<uint16_t>(w[i] & 0xffffu));
    out[2 * i + 1] = h2f(static_cast<uint16_t>(w[i] >> 16));
  }
}

template <int KB, int VB, int VPT>
struct Stage {
  static constexpr int kKC = 256 * KB;  // key codes of one tile
  static constexpr int kVC = 256 * VB;  // value codes of one tile
  static constexpr int kVS = 32 * VPT;  // value scale (or zero) of 16 tokens
  static constexpr int kKP = 512;       // key scale[128] + zero[128] of one group
  static constexpr int oKC = 0;
  static constexpr int oVC = oKC + kKC;
  static constexpr int oVS = oVC + kVC;
  static constexpr int oVZ = oVS + kVS;
  static constexpr int oKP = oVZ + kVS;
  static constexpr int kBytes = oKP + kKP;
};

// Shared memory: query [4][128] f32, exponents [4] i32 (16 B), warp partials [W][4][130] f32,
// zero sums [W][4][8] f32, then the per-warp stage rings.
constexpr int kSmemQ = 4 * 128 * 4;
constexpr int kSmemE = 16;
constexpr int kSmemCM = kDecodeWarps * 4 * kPartFloats * 4;
constexpr int kSmemZB = kDecodeWarps * 4 * 8 * 4;
constexpr int kSmemFixed = kSmemQ + kSmemE + kSmemCM + kSmemZB;
static_assert(kSmemFixed % 16 == 0, "stage ring must start 16-byte aligned");

template <int KB, int VB, int VPT>
constexpr int decode_smem_bytes() {
  return kSmemFixed + kDecodeWarps * kStages * Stage<KB, VB, VPT>::kBytes;
}

template <int KB, int VB, int VPT>
__global__ void __launch_bounds__(128, 3) decode_split_kernel(const DecodeArgs a) {
  using S = Stage<KB, VB, VPT>;
  constexpr int G = 128 / VPT;
  extern __shared__ __align__(16) uint8_t smem[];
  float* sq = reinterpret_cast<float*>(smem);
  int* se = reinterpret_cast<int*>(smem + kSmemQ);
  float* cm = reinterpret_cast<float*>(smem + kSmemQ + kSmemE);
  float* zb = reinterpret_cast<float*>(smem + kSmemQ + kSmemE + kSmemCM);
  uint8_t* rings = smem + kSmemFixed;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int split = blockIdx.x;
  const int64_t unit = blockIdx.y;
  const int64_t b = unit / a.num_kv_heads;
  const int kvh = static_cast<int>(unit % a.num_kv_heads);
  const int gq = a.gqa;
  const int64_t T = a.seq_len[b];
  const int64_t start = static_cast<int64_t>(split) * a.split_len;
  if (start >= T) return;
  const int64_t end = min(start + static_cast<int64_t>(a.split_len), T);
  const int64_t Q = quantized_len(T, a.R, G);
  const int64_t qend = min(end, Q);

  // ---- query: optional Hadamard rotation, scale to base-2 logits, per-head power-of-two exponent.
  {
    float x[4] = {0.f, 0.f, 0.f, 0.f};
    if (warp < gq) {
      const uint2 raw = *reinterpret_cast<const uint2*>(
          a.q + (b * a.num_q_heads + static_cast<int64_t>(kvh) * gq + warp) * kHeadDim + 4 * lane);
      x[0] = h2f(static_cast<uint16_t>(raw.x & 0xffffu));
      x[1] = h2f(static_cast<uint16_t>(raw.x >> 16));
      x[2] = h2f(static_cast<uint16_t>(raw.y & 0xffffu));
      x[3] = h2f(static_cast<uint16_t>(raw.y >> 16));
      if (a.hadamard) {
        const float t0 = x[0] + x[1], t1 = x[0] - x[1], t2 = x[2] + x[3], t3 = x[2] - x[3];
        x[0] = t0 + t2;
        x[2] = t0 - t2;
        x[1] = t1 + t3;
        x[3] = t1 - t3;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const bool upper = (lane & d) != 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float o = __shfl_xor_sync(kFull, x[i], d);
            x[i] = upper ? o - x[i] : x[i] + o;
          }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] *= inv_sqrt128();
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] *= a.qscale;
    }
    float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, d));
    const int e = mx > 0.f ? ((__float_as_int(mx) >> 23) & 0xff) - 126 : 0;
    *reinterpret_cast<float4*>(sq + warp * kHeadDim + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
    if (lane == 0) se[warp] = e;
  }
  __syncthreads();

  const int qd = lane & 3, r = lane >> 2;
  const int hb = r >> 1;              // head of this lane's B-fragment column (lane >> 2 = column n)
  const bool lo_half = (r & 1) != 0;  // column n = 2*head + (0: hi, 1: lo)
  float qn[32];                       // q^ of head hb at channel 16m + 2qd + 8hh + e, index 4m + 2hh + e
  {
    const float inv = pow2i(-se[hb]);
#pragma unroll
    for (int m = 0; m < 8; ++m)
#pragma unroll
      for (int k = 0; k < 4; ++k) qn[4 * m + k] = sq[hb * kHeadDim + 16 * m + 2 * qd + 8 * (k >> 1) + (k & 1)] * inv;
  }
  const float p2e_d = pow2i(se[qd]);  // scale of this lane's D-fragment head (head qd)

  // ---- this warp's quantized tiles
  const int64_t ntiles = qend > start ? (qend - start) / kTile : 0;
  const int64_t per = (ntiles + kDecodeWarps - 1) / kDecodeWarps;
  const int64_t tb = min(ntiles, per * warp);
  const int nt = static_cast<int>(min(ntiles, per * (warp + 1)) - tb);
  uint8_t* ring = rings + warp * kStages * S::kBytes;
  const int64_t first_token = start + tb * kTile;

  float m_run = -CUDART_INF_F, l_run = 0.f;
  float O[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m) O[m][0] = O[m][1] = O[m][2] = O[m][3] = 0.f;
  float zacc[VPT];
#pragma unroll
  for (int j = 0; j < VPT; ++j) zacc[j] = 0.f;
  uint32_t bq[8][2];
#pragma unroll
  for (int m = 0; m < 8; ++m) bq[m][0] = bq[m][1] = 0u;
  float bias_d = 0.f;

  const uint8_t* kc_base = reinterpret_cast<const uint8_t*>(a.k_codes + unit * a.tiles * (64 * KB));
  const uint8_t* vc_base = reinterpret_cast<const uint8_t*>(a.v_codes + unit * a.tiles * (64 * VB));
  const uint8_t* vs_base = reinterpret_cast<const uint8_t*>(a.v_scale + unit * a.capacity * VPT);
  const uint8_t* vz_base = reinterpret_cast<const uint8_t*>(a.v_zero + unit * a.capacity * VPT);
  const uint16_t* ks_base = a.k_scale + unit * a.groups * kHeadDim;
  const uint16_t* kz_base = a.k_zero + unit * a.groups * kHeadDim;

  auto issue = [&](int i) {
    uint8_t* st = ring + (i % kStages) * S::kBytes;
    const int64_t t = first_token + static_cast<int64_t>(i) * kTile;
    const int64_t tile = t / kTile;
#pragma unroll
    for (int c = lane; c < S::kKC / 16; c += 32) cp_async16(st + S::oKC + 16 * c, kc_base + tile * S::kKC + 16 * c);
#pragma unroll
    for (int c = lane; c < S::kVC / 16; c += 32) cp_async16(st + S::oVC + 16 * c, vc_base + tile * S::kVC + 16 * c);
    if (lane < S::kVS / 16) {
      cp_async16(st + S::oVS + 16 * lane, vs_base + t * (2 * VPT) + 16 * lane);
      cp_async16(st + S::oVZ + 16 * lane, vz_base + t * (2 * VPT) + 16 * lane);
    }
    if (i == 0 || (t % G) == 0) {
      const int64_t g = t / G;
      const uint16_t* src = lane < 16 ? ks_base + g * kHeadDim + 8 * lane : kz_base + g * kHeadDim + 8 * (lane - 16);
      cp_async16(st + S::oKP + 16 * lane, src);
    }
  };

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < nt) issue(i);
    cp_async_commit();
  }

  for (int i = 0; i < nt; ++i) {
    if (i + kStages - 1 < nt) issue(i + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint8_t* st = ring + (i % kStages) * S::kBytes;
    const int64_t t = first_token + static_cast<int64_t>(i) * kTile;

    // -- new key group: fold its scale into the query (hi/lo fp16) and its zero into a bias
    if (i == 0 || (t % G) == 0) {
      const uint4* sp = reinterpret_cast<const uint4*>(st + S::oKP + 64 * qd);
      const uint4* zp = reinterpret_cast<const uint4*>(st + S::oKP + 256 + 64 * qd);
      float bias = 0.f;
#pragma unroll
      for (int v4 = 0; v4 < 4; ++v4) {
        const uint4 s4 = sp[v4], z4 = zp[v4];
        const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
        const uint32_t zw[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int idx = 8 * v4 + 2 * k;  // = 4m + 2hh
          const float s0 = h2f(static_cast<uint16_t>(sw[k] & 0xffffu)), s1 = h2f(static_cast<uint16_t>(sw[k] >> 16));
          const float z0 = h2f(static_cast<uint16_t>(zw[k] & 0xffffu)), z1 = h2f(static_cast<uint16_t>(zw[k] >> 16));
          const float x0 = qn[idx] * s0, x1 = qn[idx + 1] * s1;
          bq[idx >> 2][(idx >> 1) & 1] = pack_h2(split_part(x0, lo_half), split_part(x1, lo_half));
          bias = fmaf(qn[idx], z0, bias);
          bias = fmaf(qn[idx + 1], z1, bias);
        }
      }
      bias += __shfl_xor_sync(kFull, bias, 1);
      bias += __shfl_xor_sync(kFull, bias, 2);
      bias_d = __shfl_sync(kFull, bias, 8 * qd);  // lanes with column n = 2qd hold head qd
    }

    // -- scores of the 16 tokens: rows r, r+8; columns (head qd hi, head qd lo)
    float sacc[4] = {0.f, 0.f, 0.f, 0.f};
    if constexpr (KB == 2) {
      const uint4 kw = *reinterpret_cast<const uint4*>(st + S::oKC + 16 * lane);
      const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t h[8];
        unpack_word2(w4[w], h);
        mma16816(sacc, h[0], h[1], h[2], h[3], bq[2 * w][0], bq[2 * w][1]);
        mma16816(sacc, h[4], h[5], h[6], h[7], bq[2 * w + 1][0], bq[2 * w + 1][1]);
      }
    } else {
      const uint4 k0 = *reinterpret_cast<const uint4*>(st + S::oKC + 16 * lane);
      const uint4 k1 = *reinterpret_cast<const uint4*>(st + S::oKC + 512 + 16 * lane);
      const uint32_t w8[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t h[4];
        unpack_word4(w8[w], h);
        mma16816(sacc, h[0], h[1], h[2], h[3], bq[w][0], bq[w][1]);
      }
    }
    const float s_lo = (sacc[0] + sacc[1] + bias_d) * p2e_d;  // token r
    const float s_hi = (sacc[2] + sacc[3] + bias_d) * p2e_d;  // token r + 8

    // -- online softmax for head qd over this tile
    float tmax = fmaxf(s_lo, s_hi);
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 4));
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 8));
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 16));
    const float m_new = fmaxf(m_run, tmax);
    const float alpha = exp2f(m_run - m_new);
    const float p_lo = exp2f(s_lo - m_new), p_hi = exp2f(s_hi - m_new);
    l_run = l_run * alpha + p_lo + p_hi;
    if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        O[m][0] *= alpha;
        O[m][1] *= alpha;
        O[m][2] *= alpha;
        O[m][3] *= alpha;
      }
      const float az = __shfl_sync(kFull, alpha, hb);  // lane hb holds head hb's factor
#pragma unroll
      for (int j = 0; j < VPT; ++j) zacc[j] *= az;
    }
    m_run = m_new;

    // -- P.V: B = p * sv (hi/lo) for tokens 2qd, 2qd+1, 2qd+8, 2qd+9 of head hb
    const int la = 8 * qd + hb;
    const float pa = __shfl_sync(kFull, p_lo, la), pb = __shfl_sync(kFull, p_lo, la + 4);
    const float pc = __shfl_sync(kFull, p_hi, la), pd = __shfl_sync(kFull, p_hi, la + 4);
    float sv01[2 * VPT], sv89[2 * VPT], zv01[2 * VPT], zv89[2 * VPT];
    load_halves<VPT>(st + S::oVS + 4 * VPT * qd, sv01);
    load_halves<VPT>(st + S::oVS + 4 * VPT * qd + 16 * VPT, sv89);
    load_halves<VPT>(st + S::oVZ + 4 * VPT * qd, zv01);
    load_halves<VPT>(st + S::oVZ + 4 * VPT * qd + 16 * VPT, zv89);
    // v^ = code * sv + zv = (code - cbar) * sv + mid with mid = zv + cbar * sv, the group midpoint
    constexpr float kCbar = VB == 2 ? 1.5f : 7.5f;
    uint32_t bp[VPT][2];
#pragma unroll
    for (int j = 0; j < VPT; ++j) {
      bp[j][0] = pack_h2(split_part(pa * sv01[j], lo_half), split_part(pb * sv01[VPT + j], lo_half));
      bp[j][1] = pack_h2(split_part(pc * sv89[j], lo_half), split_part(pd * sv89[VPT + j], lo_half));
      float z = zacc[j];
      z = fmaf(pa, fmaf(kCbar, sv01[j], zv01[j]), z);
      z = fmaf(pb, fmaf(kCbar, sv01[VPT + j], zv01[VPT + j]), z);
      z = fmaf(pc, fmaf(kCbar, sv89[j], zv89[j]), z);
      z = fmaf(pd, fmaf(kCbar, sv89[VPT + j], zv89[VPT + j]), z);
      zacc[j] = z;
    }
    if constexpr (VB == 2) {
      const uint4 vw = *reinterpret_cast<const uint4*>(st + S::oVC + 16 * lane);
      const uint32_t w4[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t h[8];
        unpack_word2_centered(w4[w], h);
        constexpr int kMPerJ = 8 / VPT;  // 16-channel blocks per value group
        mma16816(O[2 * w], h[0], h[1], h[2], h[3], bp[(2 * w) / kMPerJ][0], bp[(2 * w) / kMPerJ][1]);
        mma16816(O[2 * w + 1], h[4], h[5], h[6], h[7], bp[(2 * w + 1) / kMPerJ][0], bp[(2 * w + 1) / kMPerJ][1]);
      }
    } else {
      const uint4 v0 = *reinterpret_cast<const uint4*>(st + S::oVC + 16 * lane);
      const uint4 v1 = *reinterpret_cast<const uint4*>(st + S::oVC + 512 + 16 * lane);
      const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        uint32_t h[4];
        unpack_word4_centered(w8[w], h);
        constexpr int kMPerJ = 8 / VPT;
        mma16816(O[w], h[0], h[1], h[2], h[3], bp[w / kMPerJ][0], bp[w / kMPerJ][1]);
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  __syncwarp();

  // ---- FP16 residual tokens (CUDA cores): lane (r, qd) covers channels 16m + r, 16m + r + 8 of head qd
  const int64_t rbeg = max(start, Q);
  if (rbeg + warp < end) {
    float qr[16];
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      qr[2 * m] = sq[qd * kHeadDim + 16 * m + r];
      qr[2 * m + 1] = sq[qd * kHeadDim + 16 * m + r + 8];
    }
    uint16_t* kbuf = reinterpret_cast<uint16_t*>(ring);
    uint16_t* vbuf = kbuf + kHeadDim;
    for (int64_t t = rbeg + warp; t < end; t += kDecodeWarps) {
      const int64_t slot = (unit * a.ring + t % a.ring) * kHeadDim;
      reinterpret_cast<uint2*>(kbuf)[lane] = reinterpret_cast<const uint2*>(a.k_res + slot)[lane];
      reinterpret_cast<uint2*>(vbuf)[lane] = reinterpret_cast<const uint2*>(a.v_res + slot)[lane];
      __syncwarp();
      float dot = 0.f;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        dot = fmaf(qr[2 * m], h2f(kbuf[16 * m + r]), dot);
        dot = fmaf(qr[2 * m + 1], h2f(kbuf[16 * m + r + 8]), dot);
      }
      dot += __shfl_xor_sync(kFull, dot, 4);
      dot += __shfl_xor_sync(kFull, dot, 8);
      dot += __shfl_xor_sync(kFull, dot, 16);
      const float m_new = fmaxf(m_run, dot);
      const float alpha = exp2f(m_run - m_new);
      const float p = exp2f(dot - m_new);
      l_run = l_run * alpha + (r == 0 ? p : 0.f);
      if (__any_sync(kFull, alpha != 1.f)) {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          O[m][0] *= alpha;
          O[m][1] *= alpha;
          O[m][2] *= alpha;
          O[m][3] *= alpha;
        }
        const float az = __shfl_sync(kFull, alpha, hb);
#pragma unroll
        for (int j = 0; j < VPT; ++j) zacc[j] *= az;
      }
      m_run = m_new;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        O[m][0] = fmaf(p, h2f(vbuf[16 * m + r]), O[m][0]);
        O[m][2] = fmaf(p, h2f(vbuf[16 * m + r + 8]), O[m][2]);
      }
      __syncwarp();
    }
  }

  // ---- warp partial -> shared memory
  l_run += __shfl_xor_sync(kFull, l_run, 4);
  l_run += __shfl_xor_sync(kFull, l_run, 8);
  l_run += __shfl_xor_sync(kFull, l_run, 16);
#pragma unroll
  for (int j = 0; j < VPT; ++j) {
    zacc[j] += __shfl_xor_sync(kFull, zacc[j], 1);
    zacc[j] += __shfl_xor_sync(kFull, zacc[j], 2);
  }
  float* cw = cm + warp * 4 * kPartFloats;
  if (qd < gq) {
    float* o = cw + qd * kPartFloats + 2;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      o[16 * m + r] = O[m][0] + O[m][1];
      o[16 * m + r + 8] = O[m][2] + O[m][3];
    }
    if (r == 0) {
      cw[qd * kPartFloats] = m_run;
      cw[qd * kPartFloats + 1] = l_run;
    }
  }
  if (qd == 0 && !lo_half && hb < gq) {
#pragma unroll
    for (int j = 0; j < VPT; ++j) zb[(warp * 4 + hb) * 8 + j] = zacc[j];
  }
  __syncwarp();
  for (int idx = lane; idx < gq * kHeadDim; idx += 32) {
    const int h = idx >> 7, c = idx & 127;
    cw[h * kPartFloats + 2 + c] += zb[(warp * 4 + h) * 8 + c / G];
  }
  __syncthreads();

  // ---- CTA partial (merge the warps) -> workspace
  float* part = a.part + ((unit * a.nsplit + split) * gq) * kPartFloats;
  for (int idx = threadIdx.x; idx < gq * kHeadDim; idx += blockDim.x) {
    const int h = idx >> 7, c = idx & 127;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, cm[(w * 4 + h) * kPartFloats]);
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float* pw = cm + (w * 4 + h) * kPartFloats;
      const float f = exp2f(pw[0] - M);
      o = fmaf(f, pw[2 + c], o);
      l = fmaf(f, pw[1], l);
    }
    part[h * kPartFloats + 2 + c] = o;
    if (c == 0) {
      part[h * kPartFloats] = M;
      part[h * kPartFloats + 1] = l;
    }
  }
}

// out[b][hq] = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the splits that hold tokens.
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeArgs a) {
  const int64_t row = blockIdx.x;
  const int64_t b = row / a.num_q_heads;
  const int hq = static_cast<int>(row % a.num_q_heads);
  const int64_t unit = b * a.num_kv_heads + hq / a.gqa;
  const int h = hq % a.gqa;
  const int64_t T = a.seq_len[b];
  const int c = threadIdx.x;
  uint16_t* out = a.out + row * kHeadDim;
  if (T <= 0) {
    out[c] = 0;
    return;
  }
  const int ns = static_cast<int>((T + a.split_len - 1) / a.split_len);
  const int64_t stride = static_cast<int64_t>(a.gqa) * kPartFloats;
  const float* base = a.part + (unit * a.nsplit * a.gqa + h) * kPartFloats;
  float M = -CUDART_INF_F;
  for (int s = 0; s < ns; ++s) M = fmaxf(M, base[s * stride]);
  float l = 0.f, acc = 0.f;
  for (int s = 0; s < ns; ++s) {
    const float* p = base + s * stride;
    const float f = exp2f(p[0] - M);
    l = fmaf(f, p[1], l);
    acc = fmaf(f, p[2 + c], acc);
  }
  out[c] = __half_as_ushort(__float2half_rn(acc / l));
}

template <int KB, int VB, int VPT>
cudaError_t launch_split(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int smem = decode_smem_bytes<KB, VB, VPT>();
  cudaError_t e = cudaFuncSetAttribute(decode_split_kernel<KB, VB, VPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(static_cast<int64_t>(a.batch) * a.num_kv_heads));
  decode_split_kernel<KB, VB, VPT><<<grid, 32 * kDecodeWarps, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int KB, int VB, int VPT>
int occupancy() {
  constexpr int smem = decode_smem_bytes<KB, VB, VPT>();
  if (cudaFuncSetAttribute(decode_split_kernel<KB, VB, VPT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return 1;
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_split_kernel<KB, VB, VPT>, 32 * kDecodeWarps, smem) != cudaSuccess)
    return 1;
  return n > 0 ? n : 1;
}

template <int KB, int VB>
cudaError_t dispatch_vpt(const DecodeArgs& a, cudaStream_t s) {
  switch (a.G) {
    case 128: return launch_split<KB, VB, 1>(a, s);
    case 64: return launch_split<KB, VB, 2>(a, s);
    case 32: return launch_split<KB, VB, 4>(a, s);
    default: return launch_split<KB, VB, 8>(a, s);
  }
}

template <int KB, int VB>
int occupancy_vpt(int G) {
  switch (G) {
    case 128: return occupancy<KB, VB, 1>();
    case 64: return occupancy<KB, VB, 2>();
    case 32: return occupancy<KB, VB, 4>();
    default: return occupancy<KB, VB, 8>();
  }
}

}  // namespace

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e;
  if (a.key_bits == 2)
    e = a.value_bits == 2 ? dispatch_vpt<2, 2>(a, stream) : dispatch_vpt<2, 4>(a, stream);
  else
    e = a.value_bits == 2 ? dispatch_vpt<4, 2>(a, stream) : dispatch_vpt<4, 4>(a, stream);
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<static_cast<unsigned>(static_cast<int64_t>(a.batch) * a.num_q_heads), kHeadDim, 0, stream>>>(a);
  return cudaGetLastError();
}

int decode_ctas_per_sm(int key_bits, int value_bits, int G) {
  if (key_bits == 2) return value_bits == 2 ? occupancy_vpt<2, 2>(G) : occupancy_vpt<2, 4>(G);
  return value_bits == 2 ? occupancy_vpt<4, 2>(G) : occupancy_vpt<4, 4>(G);
}

}  // namespace kvq
