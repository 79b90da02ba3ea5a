// kvq_quantize.cu — streaming append and group flush.
//
// Append writes one token per sequence into the FP16 ring of R + G slots (framework page, In practice)
// and, once the window holds a whole group beyond R, quantizes that group and appends it along the
// token axis (KV cache quantization wiki page, KIVI notes): keys per channel over the G tokens, values
// per token over G channels (KVQuant review, Method), 2- or 4-bit codes with fp16 scale / zero. The
// bulk prefill lives in kvq_prefill.cu.
//
// One CTA flushes one (sequence, KV head) for keys (blockIdx.y == 0) or values (blockIdx.y == 1): the
// group is gathered from the ring into shared memory, reduced to min/max, coded and packed word by word
// in the cache layout.
#include <cuda_runtime.h>

#include "kvq_common.cuh"
#include "kvq_internal.h"

namespace kvq {

// Shared memory of one chunk: fp16 rows [G][128], then per-chunk parameters: keys use (f32(zero),
// 1/f32(scale)) per channel [128] plus per-quarter min/max keys [4][128] x 2; values use
// (f32(zero), 1/f32(scale)) per (token, channel group) [G][128/G] = 128 entries. Then the outlier
// channel of each row [G] u8 (0xff: none).
constexpr int kChunkParamBytes = 128 * 8 + 2 * 4 * 128 * 4;
static size_t chunk_smem_bytes(int G) { return static_cast<size_t>(G) * kHeadDim * 2 + kChunkParamBytes + 128; }

// Code of x on the grid (zf, inv): rint_even((f32(x) - zf) * inv) clamped to [0, 2^bits - 1].
// inv == 0 encodes a zero scale and yields code 0 (x - zf is finite). v = (x - zf) * inv is >= 0
// because x >= zf; clamping before rounding gives the same code as rounding then clamping. The
// round-half-even to an integer is an IEEE add of 1.5 * 2^23 (exact for 0 <= v < 2^22): the sum's low
// mantissa bits are the rounded integer.
__device__ __forceinline__ uint32_t code_with(uint16_t x, float zf, float inv, int top) {
  const float v = fminf(__fmul_rn(__fsub_rn(h2f(x), zf), inv), static_cast<float>(top));
  return __float_as_uint(__fadd_rn(v, 12582912.0f)) & 0xffu;
}

// Quantize G staged key rows (tokens t0 .. t0+G-1 of a unit, stored in slot `slot` from in-slot token
// ts0 on: the unit and t0, or with paged storage the pool page and t0 mod page_tokens) and write their
// key group.
// All 256 threads work in every phase: min/max over token quarters for channel pairs, parameters per
// channel, then one packed word per thread-iteration built straight from the fp16 rows.
// With the outliers on, och[i] is row i's outlier channel: that entry stays out of its channel's
// min / max, a channel whose entries are all outliers gets scale and zero 0, and the entry is then
// overwritten with its channel's zero (code 0).
__device__ void quantize_keys_chunk(const QuantizeArgs& a, int64_t slot, int64_t ts0, int64_t t0, const uint16_t* rows,
                                    uint8_t* pbuf, const uint8_t* och) {
  const int G = a.G, bits = a.key_bits, top = (1 << bits) - 1;
  float2* prm = reinterpret_cast<float2*>(pbuf);                  // [128] (zf, inv)
  uint32_t* pmin = reinterpret_cast<uint32_t*>(pbuf + 128 * 8);   // [4][128]
  uint32_t* pmax = pmin + 4 * 128;                                // [4][128]
  const int64_t g = ts0 / G;  // key group within the slot
  const bool sink0 = a.sink && t0 == 0;  // token 0 stays out of group 0 (min/max and codes)
  {
    const int cp = threadIdx.x & 63, tq = threadIdx.x >> 6;
    const int n = G / 4;
    uint32_t mn0 = 0xffffffffu, mx0 = 0u, mn1 = 0xffffffffu, mx1 = 0u;
    for (int i = tq * n + ((sink0 && tq == 0) ? 1 : 0); i < (tq + 1) * n; ++i) {
      const uint32_t w = *reinterpret_cast<const uint32_t*>(rows + i * kHeadDim + 2 * cp);
      const uint32_t k0 = order_key(w & 0xffffu), k1 = order_key(w >> 16);
      const int o = a.outliers ? och[i] : 0xff;
      if (o != 2 * cp) {
        mn0 = min(mn0, k0);
        mx0 = max(mx0, k0);
      }
      if (o != 2 * cp + 1) {
        mn1 = min(mn1, k1);
        mx1 = max(mx1, k1);
      }
    }
    pmin[tq * 128 + 2 * cp] = mn0;
    pmin[tq * 128 + 2 * cp + 1] = mn1;
    pmax[tq * 128 + 2 * cp] = mx0;
    pmax[tq * 128 + 2 * cp + 1] = mx1;
  }
  __syncthreads();
  if (threadIdx.x < kHeadDim) {
    const int c = threadIdx.x;
    const uint32_t kmin = min(min(pmin[c], pmin[128 + c]), min(pmin[256 + c], pmin[384 + c]));
    const uint32_t kmax = max(max(pmax[c], pmax[128 + c]), max(pmax[256 + c], pmax[384 + c]));
    // no entry outside the outliers: scale and zero 0
    const QuantParams p = kmin == 0xffffffffu ? QuantParams{0.f, 0.f, 0, 0, true} : make_params(kmin, kmax, bits);
    const int pos = a.layout == KVQ_LAYOUT_ROWS_V2 ? c : key_param_pos(c);  // rows v2: natural channel order
    const int64_t pidx = (slot * a.groups + g) * kHeadDim + pos;
    a.k_scale[pidx] = p.s16;
    a.k_zero[pidx] = p.z16;
    prm[c] = make_float2(p.zf, p.inv);
    if (sink0) const_cast<uint16_t*>(rows)[c] = p.z16;  // codes to 0: x - zf = 0
  }
  __syncthreads();
  if (a.outliers) {  // outlier entries -> their channel's zero (f32(zero) converts back exactly)
    if (threadIdx.x < G && och[threadIdx.x] != 0xff) {
      const int o = och[threadIdx.x];
      const_cast<uint16_t*>(rows)[threadIdx.x * kHeadDim + o] = __half_as_ushort(__float2half_rn(prm[o].x));
    }
    __syncthreads();
  }
  const int words = 64 * bits;
  const int P = 16 / bits;
  if (a.layout == KVQ_LAYOUT_ROWS_V2) {
    // one row of 4*bits words per token: pair j = P*w + k holds channels 2j, 2j + 1
    const int wpt = 4 * bits;
    uint32_t* dst2 = a.k_codes + (slot * a.slot_tokens + ts0) * wpt;
    for (int idx = threadIdx.x; idx < G * wpt; idx += blockDim.x) {
      const int i = idx / wpt, w = idx % wpt;
      uint32_t word = 0;
      for (int k = 0; k < P; ++k) {
        const int c = 2 * (P * w + k);
        const uint32_t x = *reinterpret_cast<const uint32_t*>(rows + i * kHeadDim + c);
        const float4 pp = *reinterpret_cast<const float4*>(prm + c);
        word |= code_with(static_cast<uint16_t>(x & 0xffffu), pp.x, pp.y, top) << (bits * k);
        word |= code_with(static_cast<uint16_t>(x >> 16), pp.z, pp.w, top) << (16 + bits * k);
      }
      dst2[idx] = word;
    }
    return;
  }
  uint32_t* dst = a.k_codes + (slot * a.tiles + ts0 / kTile) * words;
  for (int idx = threadIdx.x; idx < (G / kTile) * words; idx += blockDim.x) {
    const int tile = idx / words, widx = idx % words;
    int lane, w;
    widx_to_lane_word(widx, &lane, &w);
    uint32_t word = 0;
    for (int j = 0; j < P; ++j) {
      int i, c;
      key_slot(lane, w * P + j, &i, &c);  // c is even: the pair is channels c, c + 1 of token i
      const uint32_t x = *reinterpret_cast<const uint32_t*>(rows + (tile * kTile + i) * kHeadDim + c);
      const float4 pp = *reinterpret_cast<const float4*>(prm + c);  // (zf, inv) of c and c + 1
      word |= code_with(static_cast<uint16_t>(x & 0xffffu), pp.x, pp.y, top) << (bits * j);
      word |= code_with(static_cast<uint16_t>(x >> 16), pp.z, pp.w, top) << (16 + bits * j);
    }
    dst[static_cast<int64_t>(tile) * words + widx] = word;
  }
}

// Quantize G staged value rows (per token, channel groups of G) and write their codes. With the
// outliers on, each row's outlier entry has been replaced by its neighbour before (so the min / max
// leave it out) and becomes its group's zero (code 0) once the parameters are known.
__device__ void quantize_values_chunk(const QuantizeArgs& a, int64_t slot, int64_t ts0, int64_t t0, const uint16_t* rows,
                                      uint8_t* pbuf, const uint8_t* och) {
  const int G = a.G, bits = a.value_bits, top = (1 << bits) - 1;
  const int vpt = kHeadDim / G;
  float2* prm = reinterpret_cast<float2*>(pbuf);  // [G][vpt] (zf, inv)
  {
    // item (token i, group j) = threadIdx.x / 2; each of the two threads scans half of the G channels
    const int item = threadIdx.x >> 1, half = threadIdx.x & 1;
    const int i = item / vpt, j = item % vpt;
    const uint16_t* x = rows + i * kHeadDim + j * G + half * (G / 2);
    uint32_t kmin = 0xffffffffu, kmax = 0u;
    for (int c8 = 0; c8 < G / 2; c8 += 8) {
      const uint4 v = *reinterpret_cast<const uint4*>(x + c8);
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t k0 = order_key(wv[q] & 0xffffu), k1 = order_key(wv[q] >> 16);
        kmin = min(kmin, min(k0, k1));
        kmax = max(kmax, max(k0, k1));
      }
    }
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, 1));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, 1));
    if (half == 0) {
      QuantParams p = make_params(kmin, kmax, bits);
      if (a.sink && t0 + i == 0) p = QuantParams{0.f, 0.f, 0, 0, true};  // the sink token: all zero
      const int64_t pidx = (slot * a.slot_tokens + ts0 + i) * vpt + j;
      a.v_scale[pidx] = p.s16;
      a.v_zero[pidx] = p.z16;
      prm[i * vpt + j] = make_float2(p.zf, p.inv);
      if (a.outliers && och[i] != 0xff && och[i] / G == j) const_cast<uint16_t*>(rows)[i * kHeadDim + och[i]] = p.z16;
    }
  }
  __syncthreads();
  const int words = 64 * bits;
  const int P = 16 / bits;
  if (a.layout == KVQ_LAYOUT_ROWS_V2) {
    // the chunk lies inside one 128-token block; channel c's row of that block gets G / (2P) words
    const int wpr = 4 * bits, wpc = G / (2 * P);
    const int64_t block = ts0 / 128;
    const int ib = static_cast<int>(ts0 % 128);
    uint32_t* dst2 = a.v_codes + slot * a.vwords + block * 128 * wpr + (ib / 2) / P;
    for (int idx = threadIdx.x; idx < kHeadDim * wpc; idx += blockDim.x) {
      const int c = idx / wpc, w = idx % wpc;
      uint32_t word = 0;
      for (int k = 0; k < P; ++k) {
        const int i0 = 2 * (P * w + k);  // chunk-relative token pair i0, i0 + 1
        const float2 p0 = prm[i0 * vpt + c / G], p1 = prm[(i0 + 1) * vpt + c / G];
        word |= code_with(rows[i0 * kHeadDim + c], p0.x, p0.y, top) << (bits * k);
        word |= code_with(rows[(i0 + 1) * kHeadDim + c], p1.x, p1.y, top) << (16 + bits * k);
      }
      dst2[c * wpr + w] = word;
    }
    return;
  }
  uint32_t* dst = a.v_codes + (slot * a.tiles + ts0 / kTile) * words;
  for (int idx = threadIdx.x; idx < (G / kTile) * words; idx += blockDim.x) {
    const int tile = idx / words, widx = idx % words;
    int lane, w;
    widx_to_lane_word(widx, &lane, &w);
    uint32_t word = 0;
    for (int j = 0; j < P; ++j) {
      int i, c;
      value_slot(lane, w * P + j, &i, &c);  // the pair is tokens i, i + 1 of channel c
      const int ti = tile * kTile + i;
      const float2 p0 = prm[ti * vpt + c / G], p1 = prm[(ti + 1) * vpt + c / G];
      word |= code_with(rows[ti * kHeadDim + c], p0.x, p0.y, top) << (bits * j);
      word |= code_with(rows[(ti + 1) * kHeadDim + c], p1.x, p1.y, top) << (16 + bits * j);
    }
    dst[static_cast<int64_t>(tile) * words + widx] = word;
  }
}

// Append one token to every (sequence, KV head) of the chunk's sequences and flush a full group out
// of the window. Each CTA takes its sequence's old length from the by-value chunk, so no CTA reads
// the device mirror, and the key CTA of KV head 0 stores the new length there: one launch per chunk.
__global__ void __launch_bounds__(256) append_kernel(QuantizeArgs a, const LenChunk lens, const uint16_t* __restrict__ k_new,
                                                     const uint16_t* __restrict__ v_new) {
  extern __shared__ __align__(16) uint8_t smem[];
  const int64_t unit = lens.base * a.num_kv_heads + blockIdx.x;
  const bool is_key = blockIdx.y == 0;
  const int64_t b = unit / a.num_kv_heads;
  const int G = a.G;
  const int64_t t = lens.len[blockIdx.x / a.num_kv_heads];
  if (is_key && threadIdx.x == 0 && blockIdx.x % a.num_kv_heads == 0) a.seq_len[b] = t + 1;
  const int64_t Q_old = quantized_len(t, a.R, G);
  const int64_t Q_new = quantized_len(t + 1, a.R, G);
  uint16_t* rows = reinterpret_cast<uint16_t*>(smem);
  uint8_t* pbuf = smem + static_cast<size_t>(G) * kHeadDim * 2;
  uint16_t* ring = (is_key ? a.k_res : a.v_res) + unit * a.res_rows * kHeadDim;
  const uint16_t* src = (is_key ? k_new : v_new) + unit * kHeadDim;
  // New token -> ring slot t mod (R + G), rotated first for keys when enabled (warp 0, 16 lanes).
  if (threadIdx.x < 32) {
    float x[8];
    const uint4 raw = (threadIdx.x < 16) ? __ldg(reinterpret_cast<const uint4*>(src) + threadIdx.x) : make_uint4(0, 0, 0, 0);
    const uint16_t* hv = reinterpret_cast<const uint16_t*>(&raw);
#pragma unroll
    for (int i = 0; i < 8; ++i) x[i] = h2f(hv[i]);
    if (is_key && a.hadamard) wht128_16lanes(x);
    uint16_t o[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] = __half_as_ushort(__float2half_rn(x[i]));
    if (threadIdx.x < 16) {
      const uint4 row = (is_key && a.hadamard) ? *reinterpret_cast<const uint4*>(o) : raw;
      reinterpret_cast<uint4*>(ring + (t % a.ring) * kHeadDim)[threadIdx.x] = row;
      if (a.sink && t == 0) reinterpret_cast<uint4*>(ring + a.ring * kHeadDim)[threadIdx.x] = row;  // sink row
    }
  }
  if (Q_new == Q_old) return;
  __syncthreads();  // the new token is in the ring (it is not part of the flushed group, but keep order simple)
  // Flush tokens [Q_old, Q_old + G): gather from the ring, quantize as one group.
  for (int idx = threadIdx.x; idx < G * 16; idx += blockDim.x) {
    const int i = idx >> 4, part = idx & 15;
    const int64_t slot = (Q_old + i) % a.ring;
    reinterpret_cast<uint4*>(rows + i * kHeadDim)[part] = reinterpret_cast<const uint4*>(ring + slot * kHeadDim)[part];
  }
  __syncthreads();
  // Storage slot of the group: the unit, or with paged storage the pool page of its logical page (a
  // group never crosses a page; the host has checked the entry).
  int64_t slot = unit, ts0 = Q_old;
  if (a.page_tokens > 0) {
    slot = a.page_table[unit * a.pages_per_unit + Q_old / a.page_tokens];
    ts0 = Q_old % a.page_tokens;
  }
  uint8_t* och = pbuf + kChunkParamBytes;
  if (a.outliers) {
    select_outliers(rows, kHeadDim, G, (is_key ? a.k_out : a.v_out) + slot * a.slot_tokens + ts0, och,
                    a.sink && Q_old == 0, !is_key, blockDim.x / 32);
    __syncthreads();
  }
  if (is_key)
    quantize_keys_chunk(a, slot, ts0, Q_old, rows, pbuf, och);
  else
    quantize_values_chunk(a, slot, ts0, Q_old, rows, pbuf, och);
}

__global__ void set_lengths_kernel(int64_t* seq_len, const LenChunk lens) {
  const int i = threadIdx.x;
  if (i < lens.n) seq_len[lens.base + i] = lens.len[i];
}

// ---- host launchers ---------------------------------------------------------------------------------
static LenChunk make_chunk(const int64_t* lens, int batch, int base) {
  LenChunk c;
  c.base = base;
  c.n = batch - base < kLenChunk ? batch - base : kLenChunk;
  c.pad = 0;
  for (int i = 0; i < kLenChunk; ++i) c.len[i] = i < c.n ? lens[base + i] : 0;
  return c;
}

cudaError_t launch_set_lengths(int64_t* seq_len_dev, const int64_t* lens, int batch, cudaStream_t stream) {
  for (int base = 0; base < batch; base += kLenChunk) {
    set_lengths_kernel<<<1, kLenChunk, 0, stream>>>(seq_len_dev, make_chunk(lens, batch, base));
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_append(const QuantizeArgs& a, const int64_t* old_lens, const uint16_t* k_new, const uint16_t* v_new,
                          cudaStream_t stream) {
  const size_t smem = chunk_smem_bytes(a.G);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  for (int base = 0; base < a.batch; base += kLenChunk) {
    const LenChunk c = make_chunk(old_lens, a.batch, base);
    const dim3 grid(static_cast<unsigned>(static_cast<int64_t>(c.n) * a.num_kv_heads), 2);
    append_kernel<<<grid, 256, smem, stream>>>(a, c, k_new, v_new);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace kvq
