// kvq_decode_rope.cu — split-K decode attention over pre-RoPE keys (rows-v2 layout): QK on CUDA
// cores, P.V on the tensor cores (2-bit values).
//
// Keys can be cached before RoPE and rotated only after dequantization (KVQuant review, Method and
// Key idea: RoPE mixes channel pairs and smears the key outlier channels, so the quantizer runs
// before the rotation and a fused kernel applies RoPE to the dequantized keys). Token t's key is
// turned pair by pair, channels (i, i + 64), by the angle t * theta^(-i/64); the query arrives already
// rotated at its own position.
//
// A rotation per token defeats the shared-B tensor-core formulation of QK in the other decode kernels
// (the effective query would change with every key row), so QK runs on CUDA cores:
//   * QK, lane = token. <q, R_t k> = <R_-t0 q, R_j k> with t = t0 + j and t0 the warp step's first
//     token (a multiple of 32): the query is turned once per step to R_-t0 q (cooperatively, into
//     shared memory) and each lane turns its dequantized key by its in-step offset j only, from a
//     padded shared table of (cos, sin) (j w_i) for two channel pairs per 16-byte entry. The
//     dequantization, rotation and dot products run in packed f32x2 arithmetic.
//   * Codes are read as fp16 subnormals (one AND per code pair, the position's power of two folded
//     into the staged scales), as in the tile-v1 kernel.
//   * P.V is untouched by the rotation: with 2-bit values it is an mma.sync (channels on M, tokens on
//     K, A = the centered value codes, B = p * sv as hi / lo fp16 per value group and head), and the
//     next step's value words and value / key parameters are staged with cp.async. With 4-bit values
//     (and in the CUDA-core control instance, ROT = false) P.V runs on CUDA cores, lane = 4 channels:
//     o = sum_t (p_t sv_t) c_t + sum_t p_t zv_t per value group.
// The angle tables are built once per call in fp64 (cos / sin of 32 s w_i and of j w_i) into the
// decode workspace behind the split partials; partials have the layout the split-combine kernel
// reads.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kvq_common.cuh"
#include "kvq_decode_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kRW = 4;         // warps per CTA
constexpr int kRStep = 32;     // tokens per warp step
constexpr unsigned kAll = 0xffffffffu;
constexpr int kOffStride = 33;  // padded row (float4) of the in-step table: 8 lanes, 8 bank groups
constexpr int kRPart = 132;    // shared partial stride (floats): m, l, 2 pad, o[128]

// (cos, sin) of 32 s w_i for s < nbase and of j w_i for j < 32, w_i = theta^(-i/64), in fp64.
__global__ void rope_table_kernel(float2* base, float2* off, int nbase, float theta) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  const int i = idx & 63, s = idx >> 6;
  const double w = pow(static_cast<double>(theta), -static_cast<double>(i) / 64.0);
  double sn, cs;
  if (s < nbase) {
    sincos(static_cast<double>(kRStep) * static_cast<double>(s) * w, &sn, &cs);
    base[idx] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
  if (s < kRStep) {
    sincos(static_cast<double>(s) * w, &sn, &cs);
    off[idx] = make_float2(static_cast<float>(cs), static_cast<float>(sn));
  }
}

// Shared memory layout (bytes). TC: the tensor-core P.V instance, which also stages the next
// step's value words, value scale / zero and key scale / zero with cp.async.
template <int GQ, int G, bool TC>
struct RopeSmem {
  static constexpr int VPT = kHeadDim / G;
  static constexpr int NG = G >= kRStep ? 1 : kRStep / G;       // key groups per step
  static constexpr int oQ = 0;                                  // q~ [GQ][128] f32 (base-2 logits)
  static constexpr int oOff = oQ + GQ * 128 * 4;                // (cos, cos, sin, sin) (j w_i), pairs 2p, 2p + 1: [32][33] float4
  static constexpr int oWarp = oOff + kRStep * kOffStride * 16;  // per-warp areas
  // per warp: turned query [GQ][64] float4 (q_i, q_{i+1}, q_{i+64}, q_{i+65}) for even i -> [GQ][32]
  // float4; key scale / zero of the step's groups [NG][2][32] float4 (low / high channel pairs);
  // value scale / zero (f32) of the step's tokens [32][VPT] x 2
  static constexpr int wQ = 0;
  static constexpr int wKP = wQ + GQ * 32 * 16;
  static constexpr int wVS = wKP + NG * 2 * 32 * 16;
  static constexpr int wVZ = wVS + kRStep * VPT * 4;
  static constexpr int wP = wVZ + kRStep * VPT * 4;                      // p of the step's tokens [32][GQ] f32
  static constexpr int wVC = wP + (TC ? kRStep * GQ * 4 : 0);            // value words [2 stages][128 rows] x 8 bytes
  static constexpr int kVR = 2 * kRStep * VPT * 2;                       // fp16 value scale | zero of one step
  static constexpr int wVR = wVC + (TC ? 2 * 128 * 8 : 0);               // [2 stages][kVR]
  static constexpr int wKR = wVR + (TC ? 2 * kVR : 0);                   // fp16 key scale | zero: [2][NG][512]
  static constexpr int kWarpBytes = wKR + (TC ? 2 * NG * 512 : 0);
  static constexpr int kLoop = oWarp + kRW * kWarpBytes;
  static constexpr int kEpi = oWarp + kRW * GQ * kRPart * 4;  // warp partials reuse the per-warp areas
  static constexpr int kBytes = kLoop > kEpi ? kLoop : kEpi;
  static_assert(wVC % 16 == 0 && wVR % 16 == 0 && wKR % 16 == 0 && kWarpBytes % 16 == 0, "cp.async alignment");
};

__device__ __forceinline__ void rope_cp8(uint32_t saddr, const void* g) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(saddr), "l"(g));
}
__device__ __forceinline__ void rope_cp16(uint32_t saddr, const void* g) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(saddr), "l"(g));
}
__device__ __forceinline__ void rope_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void rope_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Two codes of a word as the fp16 subnormals code * 2^(bit - 24), converted to fp32. Only bits 0..9
// of a half are mantissa, so a code at bit offset o >= 8 of its half is first shifted down by 8:
// codes are read at offset o & 7 and carry 2^((o & 7) - 24).
__device__ __forceinline__ float2 sub2f(uint32_t x) {
  return __half22float2(*reinterpret_cast<const __half2*>(&x));
}
__device__ __forceinline__ void mma16816_rope(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Centered 2-bit value codes of one token pair of a rows-v2 value word (channel row), as the fp16
// subnormal pair (2c - 3) 2^-24 of the pair's two tokens. x is the word moved so that the pair's codes
// sit at bits 1..2 (even token) and 17..18 (odd token), i.e. the codes doubled; the odd integer 2c - 3
// comes from one exact subnormal subtraction. Pair slot k sits at bits 2k and 16 + 2k of the word:
// slots 0..3 are read from (word << 1) >> 2k, slots 4..7 from word >> (2k - 1), so that no code bit
// is shifted out.
__device__ __forceinline__ uint32_t vpair_centered(uint32_t x) {
  return hsub2(x & 0x00060006u, 0x00030003u);
}

template <int BITS>
__device__ __forceinline__ float2 code_pair(uint32_t word, int slot) {  // slot: compile-time after unrolling
  const int o = BITS * slot;
  const uint32_t m = ((1u << BITS) - 1u) << (o & 7);
  return sub2f((o >= 8 ? word >> 8 : word) & (m | (m << 16)));
}

// ROT = false: the same kernel with every rotation left out (keys used as cached, no angle tables): a
// CUDA-core decode of the rows-v2 cache, kept as the control against which the tensor-core kernels'
// gain is measured (selected with KVQ_DECODE_CUDA_CORES=1, see launch_decode_cuda_cores).
template <int KB, int VB, int G, int GQ, bool ROT = true>
__global__ void __launch_bounds__(kRW * 32, (ROT && VB == 2) ? ((GQ == 4 || (KB == 4 && GQ == 2)) ? 4 : 5) : 1) decode_rope_kernel(const DecodeArgs a, const float2* __restrict__ rbase,
                                                               const float2* __restrict__ roff) {
  // P.V on the tensor cores (mma.sync, channels on M, tokens on K) for 2-bit values with the
  // rotations on; the CUDA-core control (ROT = false) and 4-bit values keep the CUDA-core P.V.
  constexpr bool TCPV = ROT && VB == 2;
  using SM = RopeSmem<GQ, G, TCPV>;
  constexpr int VPT = kHeadDim / G;
  constexpr int VGB = 4 / GQ, NBV = (VPT + VGB - 1) / VGB;  // value groups per n-block, n-blocks
  static_assert(GQ == 1 || GQ == 2 || GQ == 4, "an n-block holds 4 / GQ value groups of GQ heads");
  static_assert(G >= 16, "a 16-channel m-tile lies in one value group");
  constexpr int KW = 4 * KB;       // key words per token
  constexpr int KP = 16 / KB;      // code pairs per key word
  constexpr int VW = 4 * VB;       // value words per channel row of a 128-token block
  constexpr int VP = 16 / VB;      // token pairs per value word
  extern __shared__ __align__(16) uint8_t smem[];
  float* sq = reinterpret_cast<float*>(smem + SM::oQ);
  float4* soff = reinterpret_cast<float4*>(smem + SM::oOff);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  uint8_t* wsm = smem + SM::oWarp + warp * SM::kWarpBytes;
  float4* wq = reinterpret_cast<float4*>(wsm + SM::wQ);    // [GQ][32]
  float4* wkp = reinterpret_cast<float4*>(wsm + SM::wKP);  // [2 groups][2 halves][32]
  float* wvs = reinterpret_cast<float*>(wsm + SM::wVS);    // [32][VPT]
  float* wvz = reinterpret_cast<float*>(wsm + SM::wVZ);

  const int split = blockIdx.x;
  const int64_t unit = blockIdx.y;
  const int64_t b = unit / a.num_kv_heads;
  const int kvh = static_cast<int>(unit % a.num_kv_heads);
  const int gq = a.gqa;
  const int T = static_cast<int>(a.seq_len[b]);
  const int L = a.split_len;
  const int start = split * L;
  if (start >= T) return;
  const int end = min(start + L, T);
  const int Q = static_cast<int>(quantized_len(T, a.R, G));
  const int qend = min(end, Q);

  // ---- query (scaled to base-2 logits) and the in-step angle tables
  for (int idx = threadIdx.x; idx < GQ * kHeadDim; idx += kRW * 32) {
    const int h = idx >> 7, c = idx & 127;
    sq[idx] = h < gq ? h2f(a.q[(b * a.num_q_heads + static_cast<int64_t>(kvh) * gq + h) * kHeadDim + c]) * a.qscale : 0.f;
  }
  if constexpr (ROT) {
    for (int idx = threadIdx.x; idx < kRStep * 32; idx += kRW * 32) {
      const int j = idx >> 5, p = idx & 31;
      const float2 c0 = roff[j * 64 + 2 * p], c1 = roff[j * 64 + 2 * p + 1];
      soff[j * kOffStride + p] = make_float4(c0.x, c1.x, c0.y, c1.y);
    }
  }
  __syncthreads();

  // ---- this warp's quantized steps (contiguous runs of 32 tokens)
  const int nsteps = qend > start ? (qend - start + kRStep - 1) / kRStep : 0;
  const int per = (nsteps + kRW - 1) / kRW;
  const int sb = min(nsteps, per * warp);
  const int nst = min(nsteps, per * (warp + 1)) - sb;

  float m_run[GQ], l_run[GQ], o[GQ][4], zacc[GQ];
#pragma unroll
  for (int h = 0; h < GQ; ++h) {
    m_run[h] = -CUDART_INF_F;
    l_run[h] = 0.f;
    zacc[h] = 0.f;
    o[h][0] = o[h][1] = o[h][2] = o[h][3] = 0.f;
  }
  // TCPV roles (the m16n8k16 fragments): lane (r, qd); B column n = r holds (value group offset
  // col_off, head col_head, hi / lo part); D columns 2qd, 2qd + 1 belong to head h_d.
  const int qd = lane & 3, r = lane >> 2;
  const int col_off = r / (2 * GQ), col_head = (r >> 1) % GQ, h_d = qd % GQ;
  const bool lo_half = (r & 1) != 0;
  float O[8][4], zt[NBV];
#pragma unroll
  for (int m = 0; m < 8; ++m) O[m][0] = O[m][1] = O[m][2] = O[m][3] = 0.f;
#pragma unroll
  for (int j = 0; j < NBV; ++j) zt[j] = 0.f;
  float* wp = reinterpret_cast<float*>(wsm + SM::wP);  // TCPV: p of the step's tokens [32][GQ]
  const int c0 = 4 * lane;    // PV: this lane's channels c0 .. c0 + 3
  const int jv = c0 / G;      // their value group
  int kp_group = -1;          // first key group staged in wkp

  // Codes of step i (this lane's key row and its channels' value words), loaded one step ahead so that
  // the global loads of the next step overlap this step's arithmetic.
  constexpr int NWV = kRStep / (2 * VP);  // value words per step per channel
  uint32_t kw_next[KW], vw_next[4][NWV];
  auto load_codes = [&](int ii) {
    const int tn = start + (sb + ii) * kRStep;
    const int tl = tn + lane;
    const uint4* src = reinterpret_cast<const uint4*>(a.k_codes + (unit * a.capacity + (tl < qend ? tl : 0)) * KW);
#pragma unroll
    for (int v = 0; v < KW / 4; ++v) {
      const uint4 x = src[v];
      kw_next[4 * v] = x.x;
      kw_next[4 * v + 1] = x.y;
      kw_next[4 * v + 2] = x.z;
      kw_next[4 * v + 3] = x.w;
    }
    if constexpr (!TCPV) {
      const int64_t blk = tn / 128;
      const int wv0 = ((tn & 127) >> 1) / VP;  // first value word of the step
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t* row = a.v_codes + (unit * a.capacity + blk * 128 + c0 + e) * VW + wv0;
#pragma unroll
        for (int k = 0; k < NWV; ++k) vw_next[e][k] = row[k];
      }
    }
  };
  if (nst > 0) load_codes(0);
  // TCPV: the step's value words (channel rows 0..127, the two words of its 32 tokens), fp16 value
  // scale / zero and, when the step starts a key group, the fp16 key scale / zero of its groups, copied
  // with cp.async into stage ii & 1 one step ahead
  const uint32_t wsm_s = static_cast<uint32_t>(__cvta_generic_to_shared(wsm));
  auto stage_copy = [&](int ii) {
    const int tn = start + (sb + ii) * kRStep;
    const int stg = ii & 1;
    const uint32_t* vsrc = a.v_codes + (unit * a.capacity + (tn / 128) * 128 + lane) * VW + ((tn & 127) >> 1) / VP;
    const uint32_t vdst = wsm_s + SM::wVC + stg * 1024 + 8 * lane;
#pragma unroll
    for (int k = 0; k < 4; ++k) rope_cp8(vdst + 256 * k, vsrc + 32 * k * VW);  // rows lane + 32 k
    if (lane < 4 * VPT) {  // 64 VPT bytes of scales and as many of zeros: 16 bytes per lane
      const int64_t pb = (unit * a.capacity + tn) * VPT;
      const uint32_t rdst = wsm_s + SM::wVR + stg * SM::kVR + 16 * lane;
      rope_cp16(rdst, reinterpret_cast<const uint8_t*>(a.v_scale + pb) + 16 * lane);
      rope_cp16(rdst + SM::kVR / 2, reinterpret_cast<const uint8_t*>(a.v_zero + pb) + 16 * lane);
    }
    if (ii == 0 || tn / G != (tn - kRStep) / G) {  // lanes 0..15: scales, 16..31: zeros of a group
#pragma unroll
      for (int gg = 0; gg < SM::NG; ++gg) {
        const uint16_t* src =
            (lane < 16 ? a.k_scale : a.k_zero) + (unit * a.groups + tn / G + gg) * kHeadDim + 8 * (lane & 15);
        rope_cp16(wsm_s + SM::wKR + (stg * SM::NG + gg) * 512 + 16 * lane, src);
      }
    }
    rope_commit();
  };
  if constexpr (TCPV) {
    if (nst > 0) stage_copy(0);
  }

  for (int i = 0; i < nst; ++i) {
    const int t0 = start + (sb + i) * kRStep;
    const int t = t0 + lane;
    const bool valid = t < qend && !(a.sink && t == 0);
    uint32_t kw[KW], vw[4][NWV];
#pragma unroll
    for (int k = 0; k < KW; ++k) kw[k] = kw_next[k];
#pragma unroll
    for (int e = 0; e < 4; ++e)
#pragma unroll
      for (int k = 0; k < NWV; ++k) vw[e][k] = vw_next[e][k];
    if (i + 1 < nst) load_codes(i + 1);
    if constexpr (TCPV) {  // the next step's copies in flight, this step's landed (every lane's)
      if (i + 1 < nst) stage_copy(i + 1);
      else rope_commit();
      rope_wait<1>();
      __syncwarp();
    }
    // key scale / zero of the step's groups: wkp[g][half][p] = (s, s, z, z) of channels 2p, 2p + 1
    // (half 0) or 64 + 2p, 65 + 2p (half 1), fp16 scales pre-multiplied by 2^(24 - (bit & 7)) of
    // their code position (code_pair reads a code at bit & 7) so that the subnormal code times the
    // scale is code * s
    const int g0 = t0 / G;
    if (g0 != kp_group) {
      kp_group = g0;
      constexpr int NG = G >= kRStep ? 1 : kRStep / G;
#pragma unroll
      for (int gg = 0; gg < NG; ++gg) {
        const int64_t gidx = (unit * a.groups + g0 + gg) * kHeadDim;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int c = 64 * hf + 2 * lane;
          uint32_t sv, zv;
          if constexpr (TCPV) {  // staged by cp.async
            const uint8_t* kr = wsm + SM::wKR + ((i & 1) * SM::NG + gg) * 512;
            sv = *reinterpret_cast<const uint32_t*>(kr + 2 * c);
            zv = *reinterpret_cast<const uint32_t*>(kr + 256 + 2 * c);
          } else {
            sv = *reinterpret_cast<const uint32_t*>(a.k_scale + gidx + c);
            zv = *reinterpret_cast<const uint32_t*>(a.k_zero + gidx + c);
          }
          // channel c sits in key word c / (2 KP) at pair slot (c % (2 KP)) / 2, bit KB * slot
          const int slot = (c % (2 * KP)) / 2;
          const float sc = pow2i(24 - ((KB * slot) & 7));
          wkp[(gg * 2 + hf) * 32 + lane] = make_float4(h2f(static_cast<uint16_t>(sv & 0xffffu)) * sc,
                                                       h2f(static_cast<uint16_t>(sv >> 16)) * sc,
                                                       h2f(static_cast<uint16_t>(zv & 0xffffu)),
                                                       h2f(static_cast<uint16_t>(zv >> 16)));
        }
      }
    }
    // value scale / zero of the step's tokens: wvs pre-multiplied by 2^(24 - (bit & 7)) of the
    // token's position in its value word (token pair slot (t % 128 / 2) % VP, bit VB * slot)
    for (int idx = lane; idx < kRStep * VPT; idx += 32) {
      const int jj = idx / VPT, g = idx % VPT;
      const int tt = t0 + jj;
      const bool ok = tt < qend;
      const int64_t pidx = (unit * a.capacity + (ok ? tt : 0)) * VPT + g;
      const int slot = ((tt & 127) >> 1) % VP;
      if constexpr (TCPV) {  // the scale and the group midpoint zero + 1.5 scale (centered codes)
        const uint16_t* vr = reinterpret_cast<const uint16_t*>(wsm + SM::wVR + (i & 1) * SM::kVR);
        const float sv = ok ? h2f(vr[idx]) : 0.f;
        wvs[jj * VPT + g] = sv;
        wvz[jj * VPT + g] = ok ? fmaf(1.5f, sv, h2f(vr[kRStep * VPT + idx])) : 0.f;
      } else {
        wvs[jj * VPT + g] = ok ? h2f(a.v_scale[pidx]) * pow2i(24 - ((VB * slot) & 7)) : 0.f;
        wvz[jj * VPT + g] = ok ? h2f(a.v_zero[pidx]) : 0.f;
      }
    }
    // the query turned back to the step start: R_-t0 q, pair (i, i + 64) by -t0 w_i
    if constexpr (!ROT) {
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        const float* qh = sq + h * kHeadDim;
        wq[h * 32 + lane] = make_float4(qh[2 * lane], qh[2 * lane + 1], qh[64 + 2 * lane], qh[65 + 2 * lane]);
      }
    } else {
      const float2* bt = rbase + static_cast<int64_t>(t0 / kRStep) * 64;
      const float2 cs0 = bt[2 * lane], cs1 = bt[2 * lane + 1];  // pairs 2 lane, 2 lane + 1
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        const float* qh = sq + h * kHeadDim;
        const float a0 = qh[2 * lane], a1 = qh[2 * lane + 1], b0 = qh[64 + 2 * lane], b1 = qh[65 + 2 * lane];
        // R_-x (a, b) = (a cos + b sin, b cos - a sin)
        wq[h * 32 + lane] = make_float4(fmaf(a0, cs0.x, b0 * cs0.y), fmaf(a1, cs1.x, b1 * cs1.y),
                                        fmaf(b0, cs0.x, -a0 * cs0.y), fmaf(b1, cs1.x, -a1 * cs1.y));
      }
    }
    __syncwarp();

    // -- QK: lane = token t, offset j = lane from the step start
    // Packed fp32 (f32x2) arithmetic on the channel pairs (c, c + 1) and (c + 64, c + 65): half the
    // instructions of the scalar form for the same operations.
    float s[GQ];
    {
      float2 s2[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) s2[h] = make_float2(0.f, 0.f);
      const int gl = G >= kRStep ? 0 : lane / G;  // this token's group among the staged ones
      const float4* oj = soff + lane * kOffStride;
#pragma unroll
      for (int p = 0; p < 32; ++p) {  // channel pairs 2p, 2p + 1 (low) and 64 + 2p, 65 + 2p (high)
        const int c = 2 * p, w = c / (2 * KP), slot = (c % (2 * KP)) / 2;
        const float2 lo = code_pair<KB>(kw[w], slot);           // codes of c, c + 1
        const float2 hi = code_pair<KB>(kw[w + KW / 2], slot);  // codes of c + 64, c + 65
        const float4 kl = wkp[(gl * 2 + 0) * 32 + p];           // (s_c, s_c+1, z_c, z_c+1)
        const float4 kh = wkp[(gl * 2 + 1) * 32 + p];
        const float2 x = __ffma2_rn(lo, make_float2(kl.x, kl.y), make_float2(kl.z, kl.w));  // k_c, k_c+1
        const float2 y = __ffma2_rn(hi, make_float2(kh.x, kh.y), make_float2(kh.z, kh.w));  // k_c+64, k_c+65
        // R_j on pairs (c, c + 64) and (c + 1, c + 65): r = x cos - y sin, u = x sin + y cos
        float2 r = x, u = y;
        if constexpr (ROT) {
          const float4 csn = oj[p];  // (cos_c, cos_c+1, sin_c, sin_c+1)
          const float2 cs = make_float2(csn.x, csn.y), sn = make_float2(csn.z, csn.w);
          r = __ffma2_rn(make_float2(-y.x, -y.y), sn, __fmul2_rn(x, cs));
          u = __ffma2_rn(x, sn, __fmul2_rn(y, cs));
        }
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          const float4 qv = wq[h * 32 + p];
          s2[h] = __ffma2_rn(make_float2(qv.x, qv.y), r, s2[h]);
          s2[h] = __ffma2_rn(make_float2(qv.z, qv.w), u, s2[h]);
        }
      }
#pragma unroll
      for (int h = 0; h < GQ; ++h) s[h] = s2[h].x + s2[h].y;
    }

    // -- online softmax per head over the step
    float p[GQ], alph[GQ];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
      const float sh = valid && h < gq ? s[h] : -CUDART_INF_F;
      float mx = sh;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, d));
      const float m_new = fmaxf(m_run[h], mx);
      const float alpha = m_new == -CUDART_INF_F ? 1.f : fast_exp2(m_run[h] - m_new);
      alph[h] = alpha;
      p[h] = sh == -CUDART_INF_F ? 0.f : fast_exp2(sh - m_new);
      l_run[h] = fmaf(l_run[h], alpha, p[h]);
      if constexpr (!TCPV) {
        zacc[h] *= alpha;
        o[h][0] *= alpha;
        o[h][1] *= alpha;
        o[h][2] *= alpha;
        o[h][3] *= alpha;
      }
      m_run[h] = m_new;
    }
    if constexpr (TCPV) {
      // rescale the fragments of head h_d (D) and of col_head (the midpoint sums) when a maximum moved
      bool moved = false;
#pragma unroll
      for (int h = 0; h < GQ; ++h) moved |= alph[h] != 1.f;  // warp-uniform
      if (moved) {
        float ad = alph[0], ac = alph[0];
#pragma unroll
        for (int h = 1; h < GQ; ++h) {
          ad = h_d == h ? alph[h] : ad;
          ac = col_head == h ? alph[h] : ac;
        }
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          O[m][0] *= ad;
          O[m][1] *= ad;
          O[m][2] *= ad;
          O[m][3] *= ad;
        }
#pragma unroll
        for (int j = 0; j < NBV; ++j) zt[j] *= ac;
      }
    }

    if constexpr (TCPV) {
      // -- PV on the tensor cores. p of the step's tokens goes through shared memory to the B
      //    fragments: B = p * sv of head col_head, value group nb * VGB + col_off, for tokens 2qd,
      //    2qd + 1 (b0) and 2qd + 8, 2qd + 9 (b1) of each 16-token k-block, as hi / lo fp16 parts (the
      //    hi lane of a column makes both parts of its two tokens and passes the lo lane its part, and
      //    the other way round); A = the centered value codes (channels on M).
#pragma unroll
      for (int h = 0; h < GQ; ++h) wp[lane * GQ + h] = p[h];
      __syncwarp();
      const int sh_lo = 2 * qd, sh_hi = 7 + 2 * qd;  // pairs qd (from word << 1) and 4 + qd (from word)
      uint32_t bp[2][NBV][2];
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const int tb = 16 * kb + 2 * qd + (lo_half ? 8 : 0);  // this lane's first token in the step
        const float pe = wp[tb * GQ + col_head], po = wp[(tb + 1) * GQ + col_head];
#pragma unroll
        for (int nb = 0; nb < NBV; ++nb) {
          const int j = nb * VGB + col_off;
          uint32_t hpk = 0u, lpk = 0u;
          if (VPT % VGB == 0 || j < VPT) {
            const float se = wvs[tb * VPT + j], so = wvs[(tb + 1) * VPT + j];
            const float xe = pe * se, xo = po * so;
            const float he = __uint_as_float(__float_as_uint(xe) & 0xFFFFE000u);
            const float ho = __uint_as_float(__float_as_uint(xo) & 0xFFFFE000u);
            hpk = pack_h2(he, ho);
            lpk = pack_h2(__fsub_rn(xe, he), __fsub_rn(xo, ho));
            zt[nb] = fmaf(pe, wvz[tb * VPT + j], fmaf(po, wvz[(tb + 1) * VPT + j], zt[nb]));
          }
          const uint32_t recv = __shfl_xor_sync(kAll, lo_half ? hpk : lpk, 4);
          bp[kb][nb][0] = lo_half ? recv : hpk;
          bp[kb][nb][1] = lo_half ? lpk : recv;
        }
      }
      // A: the staged value words of channel rows 16m + r and 16m + r + 8 (word x: tokens 0..15 of
      // the step, k-block 0; word y: tokens 16..31, k-block 1)
      const uint2* vc = reinterpret_cast<const uint2*>(wsm + SM::wVC + (i & 1) * 1024);
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        const uint2 wl = vc[16 * m + r], wh = vc[16 * m + 8 + r];
        const int nb = ((16 * m) / G) / VGB;
        mma16816_rope(O[m], vpair_centered((wl.x << 1) >> sh_lo), vpair_centered((wh.x << 1) >> sh_lo),
                      vpair_centered(wl.x >> sh_hi), vpair_centered(wh.x >> sh_hi), bp[0][nb][0], bp[0][nb][1]);
        mma16816_rope(O[m], vpair_centered((wl.y << 1) >> sh_lo), vpair_centered((wh.y << 1) >> sh_lo),
                      vpair_centered(wl.y >> sh_hi), vpair_centered(wh.y >> sh_hi), bp[1][nb][0], bp[1][nb][1]);
      }
    } else {
    // -- PV: lane = channels c0 .. c0 + 3; token pairs of the channel rows of this 128-token block
#pragma unroll
      for (int jp = 0; jp < kRStep / 2; ++jp) {  // token pair (2 jp, 2 jp + 1) of the step
        const int k = jp / VP, slot = jp % VP;
        float pe[GQ], po[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          pe[h] = __shfl_sync(kAll, p[h], 2 * jp);
          po[h] = __shfl_sync(kAll, p[h], 2 * jp + 1);
        }
        const float se = wvs[(2 * jp) * VPT + jv], so = wvs[(2 * jp + 1) * VPT + jv];
        const float ze = wvz[(2 * jp) * VPT + jv], zo = wvz[(2 * jp + 1) * VPT + jv];
        float pse[GQ], pso[GQ];
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          pse[h] = pe[h] * se;
          pso[h] = po[h] * so;
          zacc[h] = fmaf(pe[h], ze, fmaf(po[h], zo, zacc[h]));
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 cc = code_pair<VB>(vw[e][k], slot);  // codes of tokens 2 jp, 2 jp + 1
#pragma unroll
          for (int h = 0; h < GQ; ++h) o[h][e] = fmaf(pse[h], cc.x, fmaf(pso[h], cc.y, o[h][e]));
        }
      }
    }
    __syncwarp();  // the per-warp staging is rewritten by the next step
  }

  // ---- warp partials -> shared memory (l summed over lanes; the zero-point term per value group)
  if constexpr (TCPV) rope_wait<0>();  // no copy in flight into the per-warp areas
  __syncthreads();  // the per-warp areas become the partials
  float* cw = reinterpret_cast<float*>(smem + SM::oWarp) + warp * GQ * kRPart;
#pragma unroll
  for (int h = 0; h < GQ; ++h) {
    float l = l_run[h];
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) l += __shfl_xor_sync(kAll, l, d);
    float* ph = cw + h * kRPart;
    if (lane == 0) {
      ph[0] = m_run[h];
      ph[1] = l;
    }
    if constexpr (!TCPV)
      *reinterpret_cast<float4*>(ph + 4 + c0) =
          make_float4(o[h][0] + zacc[h], o[h][1] + zacc[h], o[h][2] + zacc[h], o[h][3] + zacc[h]);
  }
  if constexpr (TCPV) {
    // midpoint sums over the 8 lanes of a column pair (lanes 8 cp .. 8 cp + 7, pair cp = off GQ + head);
    // channel rows 16m + r and 16m + r + 8 of head h_d come from the column pair of their value group
    // jm = 16m / G, held by the lanes with qd / GQ = jm mod VGB; the centered codes carry 2^-24 and
    // the factor 1/2 of (2c - 3) / 2, hence 2^23
#pragma unroll
    for (int j = 0; j < NBV; ++j) {
      zt[j] += __shfl_xor_sync(kAll, zt[j], 1);
      zt[j] += __shfl_xor_sync(kAll, zt[j], 2);
      zt[j] += __shfl_xor_sync(kAll, zt[j], 4);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int jm = (16 * m) / G;
      const float z = __shfl_sync(kAll, zt[jm / VGB], 8 * ((jm % VGB) * GQ + h_d));
      if (qd / GQ == jm % VGB) {
        float* ph = cw + h_d * kRPart + 4 + 16 * m + r;
        ph[0] = fmaf(O[m][0] + O[m][1], 0x1p23f, z);
        ph[8] = fmaf(O[m][2] + O[m][3], 0x1p23f, z);
      }
    }
  }
  __syncwarp();

  // ---- FP16 window (and the sink row): tokens W0 + split + k ns, warp w the k = w (mod 4); RoPE at
  //      each token's position. Lane l holds channels 2l, 2l + 1, 64 + 2l, 65 + 2l.
  {
    const int ns = (T + L - 1) / L;
    const int W0 = (a.sink && Q > 0) ? Q - 1 : Q;
    const uint16_t* kres = a.k_res + unit * a.res_rows * kHeadDim;
    const uint16_t* vres = a.v_res + unit * a.res_rows * kHeadDim;
    for (int k0 = warp; W0 + split + k0 * ns < T; k0 += kRW) {
      const int tt = W0 + split + k0 * ns;
      const int pos = tt < Q ? 0 : tt;  // the sink row is token 0
      const int slot = tt < Q ? static_cast<int>(a.ring) : tt % static_cast<int>(a.ring);
      const uint16_t* kr = kres + static_cast<int64_t>(slot) * kHeadDim;
      const uint16_t* vr = vres + static_cast<int64_t>(slot) * kHeadDim;
      const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(kr + 2 * lane));
      const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(kr + 64 + 2 * lane));
      float r[4] = {lo.x, lo.y, hi.x, hi.y};
      if constexpr (ROT) {
      const float2* bt = rbase + static_cast<int64_t>(pos / kRStep) * 64;
      const int j = pos % kRStep;
      const float4 oj = soff[j * kOffStride + lane];  // in-step (cos, sin) of pairs 2 lane, 2 lane + 1
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int i = 2 * lane + e;
        const float2 cb = bt[i];
        const float co = e ? oj.y : oj.x, so = e ? oj.w : oj.z;
        const float cs = fmaf(cb.x, co, -cb.y * so);
        const float sn = fmaf(cb.y, co, cb.x * so);
        const float x = e ? lo.y : lo.x, y = e ? hi.y : hi.x;
        r[e] = fmaf(x, cs, -y * sn);      // channel i
        r[2 + e] = fmaf(x, sn, y * cs);   // channel i + 64
      }
      }
      const float2 v_lo = __half22float2(*reinterpret_cast<const __half2*>(vr + 2 * lane));
      const float2 v_hi = __half22float2(*reinterpret_cast<const __half2*>(vr + 64 + 2 * lane));
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        if (h >= gq) break;
        const float* qh = sq + h * kHeadDim;
        float d = qh[2 * lane] * r[0];
        d = fmaf(qh[2 * lane + 1], r[1], d);
        d = fmaf(qh[64 + 2 * lane], r[2], d);
        d = fmaf(qh[65 + 2 * lane], r[3], d);
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) d += __shfl_xor_sync(kAll, d, x);
        float* ph = cw + h * kRPart;
        const float m_old = ph[0];
        const float m_new = fmaxf(m_old, d);
        const float f_old = m_old == -CUDART_INF_F ? 0.f : fast_exp2(m_old - m_new);
        const float pj = fast_exp2(d - m_new);
        __syncwarp();
        float* oo = ph + 4;
        oo[2 * lane] = fmaf(oo[2 * lane], f_old, pj * v_lo.x);
        oo[2 * lane + 1] = fmaf(oo[2 * lane + 1], f_old, pj * v_lo.y);
        oo[64 + 2 * lane] = fmaf(oo[64 + 2 * lane], f_old, pj * v_hi.x);
        oo[65 + 2 * lane] = fmaf(oo[65 + 2 * lane], f_old, pj * v_hi.y);
        __syncwarp();
        if (lane == 0) {
          ph[0] = m_new;
          ph[1] = fmaf(ph[1], f_old, pj);
        }
        __syncwarp();
      }
    }
  }
  __syncthreads();

  // ---- CTA partial (merge the warps) -> workspace, the split-combine kernel's layout
  float* part = a.part + ((unit * a.nsplit + split) * gq) * kPartFloats;
  const float* allw = reinterpret_cast<const float*>(smem + SM::oWarp);
  for (int idx = threadIdx.x; idx < gq * kHeadDim; idx += kRW * 32) {
    const int h = idx >> 7, c = idx & 127;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kRW; ++w) M = fmaxf(M, allw[(w * GQ + h) * kRPart]);
    const bool empty = M == -CUDART_INF_F;
    float ov = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kRW; ++w) {
      const float* pw = allw + (w * GQ + h) * kRPart;
      const float f = empty || pw[0] == -CUDART_INF_F ? 0.f : fast_exp2(pw[0] - M);
      ov = fmaf(f, pw[4 + c], ov);
      l = fmaf(f, pw[1], l);
    }
    part[h * kPartFloats + 2 + c] = ov;
    if (c == 0) {
      part[h * kPartFloats] = M;
      part[h * kPartFloats + 1] = l;
    }
  }
}

template <int KB, int VB, int G, int GQ, bool ROT>
cudaError_t launch_rope_kernel(const DecodeArgs& a, cudaStream_t stream) {
  using SM = RopeSmem<GQ, G, ROT && VB == 2>;
  static DeviceMemo attr;
  const int ok = attr.get([] {
    return cudaFuncSetAttribute(decode_rope_kernel<KB, VB, G, GQ, ROT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                SM::kBytes) == cudaSuccess ? 1 : -1;
  });
  if (ok < 0) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(static_cast<int64_t>(a.batch) * a.num_kv_heads));
  decode_rope_kernel<KB, VB, G, GQ, ROT><<<grid, kRW * 32, SM::kBytes, stream>>>(a, a.rope_base, a.rope_off);
  return cudaGetLastError();
}

template <int KB, int VB, int G, bool ROT>
cudaError_t rope_gq(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.gqa) {
    case 1: return launch_rope_kernel<KB, VB, G, 1, ROT>(a, stream);
    case 2: return launch_rope_kernel<KB, VB, G, 2, ROT>(a, stream);
    case 3:
    case 4: return launch_rope_kernel<KB, VB, G, 4, ROT>(a, stream);
  }
  return cudaErrorInvalidValue;
}

template <int KB, int VB, bool ROT>
cudaError_t rope_g(const DecodeArgs& a, cudaStream_t stream) {
  switch (a.G) {
    case 16: return rope_gq<KB, VB, 16, ROT>(a, stream);
    case 32: return rope_gq<KB, VB, 32, ROT>(a, stream);
    case 64: return rope_gq<KB, VB, 64, ROT>(a, stream);
    case 128: return rope_gq<KB, VB, 128, ROT>(a, stream);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

int64_t rope_table_floats(int64_t capacity) {
  return ((capacity + kRStep - 1) / kRStep) * 64 * 2 + kRStep * 64 * 2;
}

cudaError_t launch_decode_rope(const DecodeArgs& a, cudaStream_t stream) {
  const int nbase = static_cast<int>((a.capacity + kRStep - 1) / kRStep);
  const int n = (nbase > kRStep ? nbase : kRStep) * 64;
  rope_table_kernel<<<(n + 255) / 256, 256, 0, stream>>>(a.rope_base, a.rope_off, nbase, a.rope_theta);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (a.key_bits == 2) return a.value_bits == 2 ? rope_g<2, 2, true>(a, stream) : rope_g<2, 4, true>(a, stream);
  return a.value_bits == 2 ? rope_g<4, 2, true>(a, stream) : rope_g<4, 4, true>(a, stream);
}

cudaError_t launch_decode_cuda_cores(const DecodeArgs& a, cudaStream_t stream) {
  if (a.key_bits == 2) return a.value_bits == 2 ? rope_g<2, 2, false>(a, stream) : rope_g<2, 4, false>(a, stream);
  return a.value_bits == 2 ? rope_g<4, 2, false>(a, stream) : rope_g<4, 4, false>(a, stream);
}

namespace {
// CTAs per SM of the instance a launch uses (its registers and shared memory depend on the
// template arguments, GQ above all).
template <int KB, int VB, int G, int GQ, bool ROT>
int rope_occupancy() {
  static DeviceMemo occ;
  return occ.get([] {
    using SM = RopeSmem<GQ, G, ROT && VB == 2>;
    if (cudaFuncSetAttribute(decode_rope_kernel<KB, VB, G, GQ, ROT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             SM::kBytes) != cudaSuccess)
      return 1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_rope_kernel<KB, VB, G, GQ, ROT>, kRW * 32, SM::kBytes) !=
        cudaSuccess)
      return 1;
    return n > 0 ? n : 1;
  });
}
template <int KB, int VB, int G, bool ROT>
int rope_occ_gq(int gqa) {
  switch (gqa) {
    case 1: return rope_occupancy<KB, VB, G, 1, ROT>();
    case 2: return rope_occupancy<KB, VB, G, 2, ROT>();
    default: return rope_occupancy<KB, VB, G, 4, ROT>();
  }
}
template <int KB, int VB, bool ROT>
int rope_occ_g(int G, int gqa) {
  switch (G) {
    case 16: return rope_occ_gq<KB, VB, 16, ROT>(gqa);
    case 32: return rope_occ_gq<KB, VB, 32, ROT>(gqa);
    case 64: return rope_occ_gq<KB, VB, 64, ROT>(gqa);
    default: return rope_occ_gq<KB, VB, 128, ROT>(gqa);
  }
}
template <bool ROT>
int rope_occ(int key_bits, int value_bits, int G, int gqa) {
  if (key_bits == 2) return value_bits == 2 ? rope_occ_g<2, 2, ROT>(G, gqa) : rope_occ_g<2, 4, ROT>(G, gqa);
  return value_bits == 2 ? rope_occ_g<4, 2, ROT>(G, gqa) : rope_occ_g<4, 4, ROT>(G, gqa);
}
}  // namespace

int decode_rope_ctas_per_sm(int key_bits, int value_bits, int G, int gqa) {
  return rope_occ<true>(key_bits, value_bits, G, gqa);
}
int decode_cuda_cores_ctas_per_sm(int key_bits, int value_bits, int G, int gqa) {
  return rope_occ<false>(key_bits, value_bits, G, gqa);
}

}  // namespace kvq
