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
// Tiles stream through a per-warp cp.async ring (codes, value scale/zero and, at a key-block
// boundary, the block's key scale/zero): 3 stages of steps of 1 or 2 tiles, or 2 stages of 4-tile
// steps for 2-bit caches with G >= 64, so up to 6 or 8 tiles per warp are in flight.
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
// Codes -> fp16: a code AND-ed out in place at bit offset o of a 16-bit half is the fp16 subnormal
// code * 2^(o - 24), exact, one AND per code pair (value codes are taken one bit higher and centered
// with one exact subnormal subtraction). The m16n8k16 A fragment of one word holds element k at
// 2^(2k - 24) (2-bit) or 2^(-24), 2^(-20), 2^(-24), 2^(-20) (4-bit). Elements 0 and 1 (2 and 3)
// share the K columns 2qd, 2qd+1 (2qd+8, 2qd+9) and elements 0, 2 (1, 3) the M row r (r + 8), so
// the scale factors into a per-K-half factor, put on the B operand (2-bit: 2^-4 on the upper
// K half), and a per-row factor taken off the fp32 result (row r: 2^24, row r + 8: 2^22 for 2-bit,
// 2^20 for 4-bit; value rows carry one more factor 1/2 from the doubled centered code).
#include <cuda_runtime.h>
#include <math_constants.h>

#include <cstdlib>

#include "kvq_common.cuh"
#include "kvq_decode_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// cp.async of 16 bytes to a shared-space address with compile-time offsets folded into the
// instruction's address operands (no per-copy address arithmetic).
template <int SOFF, int GOFF>
__device__ __forceinline__ void cp_async16_at(uint32_t saddr, const void* gmem) {
  asm volatile("cp.async.cg.shared.global [%0+%2], [%1+%3], 16;\n" ::"r"(saddr), "l"(gmem), "n"(SOFF), "n"(GOFF));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Per-warp pipeline: a ring of kStages stages, each holding one step of TS 16-token tiles (codes
// and value scale/zero), plus a ring of KP slots holding the key scale and zero of the KGB key groups
// of one key block. A key block spans kBlockSteps steps; its parameters are read only when the
// block's first step is consumed. Step j is issued at the top of iteration j - (kStages - 1) (j - 2,
// or j - 1 with two stages), so a new block's parameters may land in the slot of the block two back
// only once that block's first step has been consumed: with kBlockSteps >= 2 this holds for two
// slots (a partial first block plus a full block lie in between); one-step blocks use four slots
// (three blocks lie in between). With OUT a stage also holds the key and value outlier words of the
// step's tokens.
template <int KB, int VB, int VPT, int KGB, int TS, bool OUT>
struct Stage {
  // 3 stages of steps of 1 or 2 tiles, or 2 stages of 4-tile steps (the same 8 tiles in flight in less
  // shared memory, so that 4 CTAs still fit an SM)
  static constexpr int kStages = TS >= 4 ? 2 : 3;
  static constexpr int kKC = 256 * KB * TS;  // key codes of the step's tiles
  static constexpr int kVC = 256 * VB * TS;  // value codes
  static constexpr int kVS = 32 * VPT * TS;  // value scale (or zero) of the step's tokens
  static constexpr int oKC = 0;
  static constexpr int oVC = oKC + kKC;
  static constexpr int oVS = oVC + kVC;
  static constexpr int oVZ = oVS + kVS;
  static constexpr int kKO = OUT ? 64 * TS : 0;  // key (or value) outlier words of the step's tokens
  static constexpr int oKO = oVZ + kVS;
  static constexpr int oVO = oKO + kKO;
  static constexpr int kBytes = oVO + kKO;
  static constexpr int kKP = 512 * KGB;  // key scale[128] + zero[128] per group of the block
  static constexpr int kBlockSteps = (128 / VPT) * KGB / (16 * TS);
  // one-step blocks: with two stages the next block's parameters land while the current one is read
  // (two slots); with three, two later blocks may be in flight (four slots, a power of two)
  static constexpr int kKPSlots = kBlockSteps >= 2 ? 2 : (kStages == 2 ? 2 : 4);
  static constexpr int kWarpBytes = kStages * kBytes + kKPSlots * kKP;
};

// Shared memory: q~ [GQ][128] f32 (base-2 logit units), q^ = q~ * 2^-e [GQ][128] f32, then the
// per-warp rings (GQ: the query heads per KV head the instance serves, 1, 2 or 4). The per-head
// exponents [4] i32 sit at the start of the ring area until every warp has read them (a CTA barrier
// separates that from the first copy into the rings). After the main loops the ring area holds the
// warp partials [W][4][130] f32 and the zero-point sums [W][4][8] f32.
template <int GQ>
constexpr int smem_q() { return 2 * GQ * 128 * 4; }
template <int GQ>
constexpr int smem_fixed() { return smem_q<GQ>(); }
constexpr int kCm = 132;   // shared-memory partial stride (floats): m, l, 2 pad, o[128] 16-byte aligned
constexpr int kCmO = 4;    // offset of o[] within a shared-memory partial
constexpr int kSmemEpilogue = kDecodeWarps * 4 * kCm * 4 + kDecodeWarps * 4 * 8 * 4;
static_assert(smem_fixed<1>() % 16 == 0 && smem_fixed<2>() % 16 == 0 && smem_fixed<4>() % 16 == 0,
              "stage ring must start 16-byte aligned");

template <int KB, int VB, int VPT, int GQ, bool OUT>
struct Shape {
  static constexpr int KGB = 4 / GQ;                     // key groups per QK B block
  // P.V B operand: with every column of an n-block in use (VPT a multiple of 8 / GQ), one fp16 column
  // per (value group, head), 8 / GQ value groups per n-block (PV1); else hi / lo fp16 column pairs,
  // 4 / GQ value groups per n-block
  static constexpr bool PV1 = VPT % (8 / GQ) == 0;
  static constexpr int VGB = PV1 ? 8 / GQ : 4 / GQ;      // value groups per PV n-block
  static constexpr int NBV = (VPT + VGB - 1) / VGB;      // PV n-blocks
  static constexpr int G = 128 / VPT;
  // tiles per step: 4 for 2-bit keys and values with G >= 64 (a step never spans two key groups),
  // which halves the per-step pipeline and softmax bookkeeping per tile
  static constexpr int TS = (KB == 2 && VB == 2 && G >= 64) ? 4 : (G >= 32 ? 2 : 1);
  using S = Stage<KB, VB, VPT, KGB, TS, OUT>;
};

// With OUT, the per-warp outlier corrections of the value sum [W][GQ][128] f32 follow the ring /
// epilogue area (they live through both).
template <int GQ>
constexpr int smem_corr() { return kDecodeWarps * GQ * 128 * 4; }
template <int KB, int VB, int VPT, int GQ, bool OUT>
constexpr int decode_corr_offset() {
  using S = typename Shape<KB, VB, VPT, GQ, OUT>::S;
  constexpr int ring = kDecodeWarps * S::kWarpBytes;
  return smem_fixed<GQ>() + (ring > kSmemEpilogue ? ring : kSmemEpilogue);
}
template <int KB, int VB, int VPT, int GQ, bool OUT>
constexpr int decode_smem_bytes() {
  return decode_corr_offset<KB, VB, VPT, GQ, OUT>() + (OUT ? smem_corr<GQ>() : 0);
}

// cp.async of 16 bytes that writes zeros (and reads nothing) when `valid` is false.
__device__ __forceinline__ void cp_async16_zfill(void* smem, const void* gmem, bool valid) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n));
}

// QK of one 16-token tile: scores (base-2 units) of tokens r and r + 8 for this lane's column pair
// (2 independent accumulator chains over the 8 channel blocks).
template <int KB>
__device__ __forceinline__ void tile_scores(const uint8_t* kc, int lane, const uint32_t (&bq)[8][2], float bias,
                                            float p2e, float& s_lo, float& s_hi) {
  float acc[2][4];
#pragma unroll
  for (int c = 0; c < 2; ++c) acc[c][0] = acc[c][1] = acc[c][2] = acc[c][3] = 0.f;
  if constexpr (KB == 2) {
    const uint4 kw = *reinterpret_cast<const uint4*>(kc + 16 * lane);
    const uint32_t w4[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t h[8];
      unpack_word2_sub(w4[w], h);
      mma16816(acc[0], h[0], h[1], h[2], h[3], bq[2 * w][0], bq[2 * w][1]);
      mma16816(acc[1], h[4], h[5], h[6], h[7], bq[2 * w + 1][0], bq[2 * w + 1][1]);
    }
  } else {
    const uint4 k0 = *reinterpret_cast<const uint4*>(kc + 16 * lane);
    const uint4 k1 = *reinterpret_cast<const uint4*>(kc + 512 + 16 * lane);
    const uint32_t w8[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t h[4];
      unpack_word4_sub(w8[w], h);
      mma16816(acc[w & 1], h[0], h[1], h[2], h[3], bq[w][0], bq[w][1]);
    }
  }
  // hi + lo columns; the subnormal row scales come off here
  constexpr float kRowLo = 16777216.0f, kRowHi = KB == 2 ? 4194304.0f : 1048576.0f;  // 2^24, 2^22 / 2^20
  s_lo = fmaf((acc[0][0] + acc[1][0]) + (acc[0][1] + acc[1][1]), kRowLo, bias) * p2e;  // token r
  s_hi = fmaf((acc[0][2] + acc[1][2]) + (acc[0][3] + acc[1][3]), kRowHi, bias) * p2e;  // token r + 8
}

// N columns of the tensor-core tiles. GQ (1, 2 or 4) query heads share one KV head; the 8 columns of
// an m16n8k16 B operand hold (group offset, head, hi/lo) for 4/GQ key (or value) groups:
//   column n -> group offset n / (2 GQ), head (n / 2) % GQ, part n % 2 (0 = hi, 1 = lo).
// With GQ = 4 every column is a (head, part) of one group; with GQ = 1 one B fragment covers 4 key
// groups (QK) or 4 value groups (PV), so the per-group B rebuild is shared by 4 groups.
// A lane (r, qd) of a D fragment holds columns 2qd, 2qd + 1, i.e. (group offset qd / GQ, head qd % GQ).
//
// OUT: dense-and-sparse outliers (KVQuant review, Method). Each quantized token's key and value keep
// one fp16 entry (channel, value); its code is 0, so the packed path dequantizes it to the group's
// zero. The score of the token gets q~[ch] * (k_out - zk[g][ch]) added before the softmax, and the
// value sum gets p * (v_out - zv[t][ch / G]) at channel ch, gathered per warp in shared memory
// (rescaled with the running max like the accumulators) and added to the warp partial at the end.
template <int KB, int VB, int VPT, int GQ, bool OUT>
__global__ void __launch_bounds__(128, 4) decode_split_kernel(const DecodeArgs a) {
  using SH = Shape<KB, VB, VPT, GQ, OUT>;
  using S = typename SH::S;
  constexpr int KGB = SH::KGB, VGB = SH::VGB, NBV = SH::NBV, G = SH::G, TS = SH::TS;
  constexpr bool PV1 = SH::PV1;
  constexpr int kBlockTokens = G * KGB;
  constexpr int kStepTokens = 16 * TS;
  extern __shared__ __align__(16) uint8_t smem[];
  float* sq = reinterpret_cast<float*>(smem);
  uint8_t* rings = smem + smem_fixed<GQ>();
  int* se = reinterpret_cast<int*>(rings);  // until the barrier after the exponents are read
  float* cm = reinterpret_cast<float*>(rings);        // epilogue: [W][4][kCm] (m, l, -, -, o[128])
  float* zb = cm + kDecodeWarps * 4 * kCm;            // epilogue: [W][4][8]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
  float* corr = reinterpret_cast<float*>(smem + decode_corr_offset<KB, VB, VPT, GQ, OUT>()) + warp * GQ * kHeadDim;
  if constexpr (OUT) {
#pragma unroll
    for (int h = 0; h < GQ; ++h) *reinterpret_cast<float4*>(corr + h * kHeadDim + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
    __syncwarp();
  }

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
    if (warp < GQ) {  // the instance holds GQ heads (gq <= GQ; the heads past gq get zeros)
      *reinterpret_cast<float4*>(sq + warp * kHeadDim + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
      const float inv = pow2i(-e);
      *reinterpret_cast<float4*>(sq + GQ * kHeadDim + warp * kHeadDim + 4 * lane) =
          make_float4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
    }
    if (lane == 0) se[warp] = e;
  }
  __syncthreads();

  const int qd = lane & 3, r = lane >> 2;
  // B-fragment role (column n = r): group offset, head, hi/lo part.
  const int col_off = r / (2 * GQ);
  const int col_head = (r >> 1) % GQ;
  const bool lo_half = (r & 1) != 0;
  // P.V B-fragment role (column n = r): value group offset and head (PV1: one column each; else the
  // QK roles, hi / lo pairs)
  const int pv_off = PV1 ? r / GQ : col_off;
  const int pv_head = PV1 ? r % GQ : col_head;
  // D-fragment role: this lane's head for the softmax.
  const int h_d = qd % GQ;
  const float* qn_row = sq + GQ * kHeadDim + col_head * kHeadDim + 2 * qd;  // q^ of head col_head
  const float p2e_d = pow2i(se[h_d]);
  __syncthreads();  // every warp has its exponent: the ring area may be written

  // ---- this warp's quantized steps (contiguous)
  const int nsteps = qend > start ? (qend - start) / kStepTokens : 0;
  const int per = (nsteps + kDecodeWarps - 1) / kDecodeWarps;
  const int sb = min(nsteps, per * warp);
  const int nst = min(nsteps, per * (warp + 1)) - sb;
  uint8_t* ring = rings + warp * S::kWarpBytes;
  constexpr int kStages = S::kStages;
  uint8_t* kp_ring = ring + kStages * S::kBytes;
  const int first_token = start + sb * kStepTokens;
  const int q_groups = Q / G;

  float m_run = -CUDART_INF_F, l_run = 0.f;
  float O[8][4];
#pragma unroll
  for (int m = 0; m < 8; ++m) O[m][0] = O[m][1] = O[m][2] = O[m][3] = 0.f;
  float zacc[NBV];
#pragma unroll
  for (int j = 0; j < NBV; ++j) zacc[j] = 0.f;
  uint32_t bq[8][2];
#pragma unroll
  for (int m = 0; m < 8; ++m) bq[m][0] = bq[m][1] = 0u;
  float bias_col = 0.f;

  // Lane pointers of the step at token t: its storage slot (the unit, or with paged storage the pool
  // page of its logical page) and in-slot token. A step never crosses a page (a page is a whole number
  // of 128-token blocks), so with paged storage the pointers are re-based at every page start; the
  // host has checked every table entry of the quantized part.
  const uint8_t* kc_ptr = nullptr;
  const uint8_t* vc_ptr = nullptr;
  const uint8_t* vs_ptr = nullptr;
  const uint8_t* vz_ptr = nullptr;
  const uint8_t* ko_ptr = nullptr;
  const uint8_t* vo_ptr = nullptr;
  int64_t page_slot = unit;  // storage slot of the page of the steps being issued
  auto rebase = [&](int t) {
    int64_t slot = unit, ts = t;
    if (a.page_tokens > 0) {
      slot = a.page_table[unit * a.pages_per_unit + t / a.page_tokens];
      ts = t % a.page_tokens;
    }
    page_slot = slot;
    kc_ptr = reinterpret_cast<const uint8_t*>(a.k_codes + slot * a.tiles * (64 * KB)) + (ts / kTile) * (256 * KB) + 16 * lane;
    vc_ptr = reinterpret_cast<const uint8_t*>(a.v_codes + slot * a.tiles * (64 * VB)) + (ts / kTile) * (256 * VB) + 16 * lane;
    vs_ptr = reinterpret_cast<const uint8_t*>(a.v_scale + (slot * a.slot_tokens + ts) * VPT) + 16 * lane;
    vz_ptr = reinterpret_cast<const uint8_t*>(a.v_zero + (slot * a.slot_tokens + ts) * VPT) + 16 * lane;
    if constexpr (OUT) {
      ko_ptr = reinterpret_cast<const uint8_t*>(a.k_out + slot * a.slot_tokens + ts) + 16 * lane;
      vo_ptr = reinterpret_cast<const uint8_t*>(a.v_out + slot * a.slot_tokens + ts) + 16 * lane;
    }
  };
  if (nst > 0) rebase(first_token);
  // Key scale / zero row of key group g (g < q_groups) for this lane's 16-byte part.
  const uint16_t* kp_base = (lane < 16 ? a.k_scale : a.k_zero) + 8 * (lane & 15);
  // A key block (at most 128 tokens) never crosses a page, so its groups live in the page of the
  // step that issues them (rebased just before): no second table lookup.
  auto kp_row = [&](int g) -> const uint16_t* {
    int64_t slot = unit, gs = g;
    if (a.page_tokens > 0) {
      slot = page_slot;
      gs = ((g * G) % a.page_tokens) / G;
    }
    return kp_base + (slot * a.groups + gs) * kHeadDim;
  };

  // issue(i): step i of this warp into stage i % kStages (tracked by stage_in); the lane pointers
  // advance one step per call
  static_assert(S::kKC % 512 == 0 && S::kKC / 512 <= 4 && S::kVC % 512 == 0 && S::kVC / 512 <= 4, "stage copies");
  const uint32_t ring_s = static_cast<uint32_t>(__cvta_generic_to_shared(ring)) + 16 * lane;
  int stage_in = 0;
  auto issue = [&](int i) {
    if (a.page_tokens > 0 && i > 0 && (first_token + i * kStepTokens) % a.page_tokens == 0)
      rebase(first_token + i * kStepTokens);  // the step starts a new page
    const uint32_t st = ring_s + stage_in * S::kBytes;
    stage_in = stage_in == kStages - 1 ? 0 : stage_in + 1;
    cp_async16_at<S::oKC, 0>(st, kc_ptr);
    if constexpr (S::kKC / 512 > 1) cp_async16_at<S::oKC + 512, 512>(st, kc_ptr);
    if constexpr (S::kKC / 512 > 2) cp_async16_at<S::oKC + 1024, 1024>(st, kc_ptr);
    if constexpr (S::kKC / 512 > 3) cp_async16_at<S::oKC + 1536, 1536>(st, kc_ptr);
    cp_async16_at<S::oVC, 0>(st, vc_ptr);
    if constexpr (S::kVC / 512 > 1) cp_async16_at<S::oVC + 512, 512>(st, vc_ptr);
    if constexpr (S::kVC / 512 > 2) cp_async16_at<S::oVC + 1024, 1024>(st, vc_ptr);
    if constexpr (S::kVC / 512 > 3) cp_async16_at<S::oVC + 1536, 1536>(st, vc_ptr);
    if (lane < S::kVS / 16) {
      cp_async16_at<S::oVS, 0>(st, vs_ptr);
      cp_async16_at<S::oVZ, 0>(st, vz_ptr);
    }
    if constexpr (OUT) {
      if (lane < S::kKO / 16) {
        cp_async16_at<S::oKO, 0>(st, ko_ptr);
        cp_async16_at<S::oVO, 0>(st, vo_ptr);
      }
      ko_ptr += S::kKO;
      vo_ptr += S::kKO;
    }
    const int t = first_token + i * kStepTokens;
    if (i == 0 || (t % kBlockTokens) == 0) {
      const int blk = t / kBlockTokens;
      uint8_t* kp = kp_ring + (blk % S::kKPSlots) * S::kKP + 16 * lane;
#pragma unroll
      for (int kg = 0; kg < KGB; ++kg) {
        const int g = blk * KGB + kg;
        const bool valid = g < q_groups;
        cp_async16_zfill(kp + 512 * kg, valid ? kp_row(g) : kp_base, valid);  // nothing is read when invalid
      }
    }
    kc_ptr += S::kKC;
    vc_ptr += S::kVC;
    vs_ptr += S::kVS;
    vz_ptr += S::kVS;
  };

#pragma unroll
  for (int i = 0; i < kStages - 1; ++i) {
    if (i < nst) issue(i);
    cp_async_commit();
  }

  int stage_out = 0;  // i % kStages for the consumed step
  for (int i = 0; i < nst; ++i) {
    if (i + kStages - 1 < nst) issue(i + kStages - 1);
    cp_async_commit();
    cp_async_wait<kStages - 1>();
    __syncwarp();
    const uint8_t* st = ring + stage_out * S::kBytes;
    stage_out = stage_out == kStages - 1 ? 0 : stage_out + 1;
    const int t = first_token + i * kStepTokens;

    // -- new key block: fold the scales of its KGB groups into the query (hi/lo fp16) and the
    //    zero-points into per-column biases
    if (i == 0 || (t % kBlockTokens) == 0) {
      const uint8_t* kp = kp_ring + ((t / kBlockTokens) % S::kKPSlots) * S::kKP + 512 * col_off;
      const uint4* sp = reinterpret_cast<const uint4*>(kp + 64 * qd);
      const uint4* zp = reinterpret_cast<const uint4*>(kp + 256 + 64 * qd);
      // The hi and lo lanes of a column (r, r ^ 1: lanes L, L ^ 4) share the products q^ * sk: the hi
      // lane makes both parts for m-blocks 0..3, the lo lane for 4..7, and each passes the other the
      // parts it needs.
      const int vb = lo_half ? 2 : 0;
      float bias = 0.f;
      uint32_t hpk[4][2], lpk[4][2];  // hi / lo packs of this lane's m-blocks (local index mm)
#pragma unroll
      for (int vv = 0; vv < 2; ++vv) {
        const int v4 = vb + vv;
        const uint4 s4 = sp[v4], z4 = zp[v4];
        const uint32_t sw[4] = {s4.x, s4.y, s4.z, s4.w};
        const uint32_t zw[4] = {z4.x, z4.y, z4.z, z4.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int hh = k & 1, mm = 2 * vv + (k >> 1);  // m = 4 lo_half + mm
          const float2 qq = *reinterpret_cast<const float2*>(qn_row + 16 * (2 * v4 + (k >> 1)) + 8 * hh);
          const float s0 = h2f(static_cast<uint16_t>(sw[k] & 0xffffu)), s1 = h2f(static_cast<uint16_t>(sw[k] >> 16));
          const float z0 = h2f(static_cast<uint16_t>(zw[k] & 0xffffu)), z1 = h2f(static_cast<uint16_t>(zw[k] >> 16));
          // 2-bit: the upper K half (channels 16m + 8 ..) carries 2^-4 against the subnormal codes
          const float kf = (KB == 2 && hh) ? 0.0625f : 1.f;
          const float x0 = qq.x * s0 * kf, x1 = qq.y * s1 * kf;
          const float h0 = split_part(x0, false), h1 = split_part(x1, false);
          hpk[mm][hh] = pack_h2(h0, h1);
          lpk[mm][hh] = pack_h2(__fsub_rn(x0, h0), __fsub_rn(x1, h1));
          bias = fmaf(qq.x, z0, bias);
          bias = fmaf(qq.y, z1, bias);
        }
      }
#pragma unroll
      for (int mm = 0; mm < 4; ++mm)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const uint32_t recv = __shfl_xor_sync(kFull, lo_half ? hpk[mm][hh] : lpk[mm][hh], 4);
          bq[mm][hh] = lo_half ? recv : hpk[mm][hh];
          bq[4 + mm][hh] = lo_half ? lpk[mm][hh] : recv;
        }
      bias += __shfl_xor_sync(kFull, bias, 4);  // the two halves of the channels
      bias += __shfl_xor_sync(kFull, bias, 1);
      bias += __shfl_xor_sync(kFull, bias, 2);
      bias_col = __shfl_sync(kFull, bias, 8 * qd);  // lanes of column 2qd hold its bias
    }

    // -- scores of the step's tokens (TS tiles). With GQ < 4 the tile's key group offset selects the
    //    lane whose column pair holds its score.
    float s[TS][2];
#pragma unroll
    for (int u = 0; u < TS; ++u) tile_scores<KB>(st + S::oKC + u * 256 * KB, lane, bq, bias_col, p2e_d, s[u][0], s[u][1]);
    if constexpr (GQ < 4) {
      const int src = 4 * r + ((t / G) % KGB) * GQ + h_d;  // one key group per step (G >= step)
#pragma unroll
      for (int u = 0; u < TS; ++u) {
        s[u][0] = __shfl_sync(kFull, s[u][0], src);
        s[u][1] = __shfl_sync(kFull, s[u][1], src);
      }
    }
    if constexpr (OUT) {  // key outliers: q~[ch] * (k_out - zk[g][ch]) for this lane's tokens and head h_d
      const uint32_t* kos = reinterpret_cast<const uint32_t*>(st + S::oKO);
      const uint16_t* kz = reinterpret_cast<const uint16_t*>(kp_ring + ((t / kBlockTokens) % S::kKPSlots) * S::kKP +
                                                             512 * ((t / G) % KGB) + 256);
      const float* qh = sq + h_d * kHeadDim;
#pragma unroll
      for (int u = 0; u < TS; ++u)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const uint32_t ko = kos[16 * u + r + 8 * e];
          const uint32_t ch = ko & 0xffffu;
          if (ch < 128u)
            s[u][e] = fmaf(qh[ch], h2f(static_cast<uint16_t>(ko >> 16)) - h2f(kz[key_param_pos(static_cast<int>(ch))]), s[u][e]);
        }
    }
    if (a.sink && t == 0 && r == 0) s[0][0] = -CUDART_INF_F;  // the sink token is read from its fp16 row

    // -- online softmax for head h_d over the step
    float tmax = fmaxf(s[0][0], s[0][1]);
#pragma unroll
    for (int u = 1; u < TS; ++u) tmax = fmaxf(tmax, fmaxf(s[u][0], s[u][1]));
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 4));
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 8));
    tmax = fmaxf(tmax, __shfl_xor_sync(kFull, tmax, 16));
    const float m_new = fmaxf(m_run, tmax);
    const float alpha = fast_exp2(m_run - m_new);
    float p[TS][2];
    float lsum = 0.f;
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      p[u][0] = fast_exp2(s[u][0] - m_new);
      p[u][1] = fast_exp2(s[u][1] - m_new);
      lsum += p[u][0] + p[u][1];
    }
    l_run = fmaf(l_run, alpha, lsum);
    if (__any_sync(kFull, alpha != 1.f)) {
      if constexpr (PV1) {  // D columns 2qd, 2qd + 1: heads (2qd) % GQ and (2qd + 1) % GQ
        const float a0 = __shfl_sync(kFull, alpha, (2 * qd) % GQ);  // lane h has h_d == h
        const float a1 = __shfl_sync(kFull, alpha, (2 * qd + 1) % GQ);
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          O[m][0] *= a0;
          O[m][1] *= a1;
          O[m][2] *= a0;
          O[m][3] *= a1;
        }
      } else {
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          O[m][0] *= alpha;
          O[m][1] *= alpha;
          O[m][2] *= alpha;
          O[m][3] *= alpha;
        }
      }
      const float az = __shfl_sync(kFull, alpha, pv_head);  // lane pv_head has h_d == pv_head
#pragma unroll
      for (int j = 0; j < NBV; ++j) zacc[j] *= az;
      if constexpr (OUT) {
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          const float ah = __shfl_sync(kFull, alpha, h);  // lane h has h_d == h
          float4* c4 = reinterpret_cast<float4*>(corr + h * kHeadDim + 4 * lane);
          float4 v = *c4;
          v.x *= ah;
          v.y *= ah;
          v.z *= ah;
          v.w *= ah;
          *c4 = v;
        }
      }
    }
    m_run = m_new;
    if constexpr (OUT) {  // value outliers: p * (v_out - zv[t][ch / G]) at channel ch, one lane per (token, head)
      __syncwarp();
      if (qd < GQ) {
        const uint32_t* vos = reinterpret_cast<const uint32_t*>(st + S::oVO);
        const uint16_t* vz = reinterpret_cast<const uint16_t*>(st + S::oVZ);
#pragma unroll
        for (int u = 0; u < TS; ++u)
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int tk = 16 * u + r + 8 * e;
            const uint32_t vo = vos[tk];
            const uint32_t ch = vo & 0xffffu;
            if (ch < 128u)
              atomicAdd(corr + h_d * kHeadDim + ch,
                        p[u][e] * (h2f(static_cast<uint16_t>(vo >> 16)) - h2f(vz[tk * VPT + ch / G])));
          }
      }
    }

    // -- P.V per tile: B = p * sv (hi/lo) of head col_head for tokens 2qd, 2qd+1, 2qd+8, 2qd+9 and
    //    the value group of this lane's column in each n-block; A = centered value codes
    const int la = 8 * qd + pv_head;
    constexpr float kCbar = VB == 2 ? 1.5f : 7.5f;
#pragma unroll
    for (int u = 0; u < TS; ++u) {
      const float pa = __shfl_sync(kFull, p[u][0], la), pb = __shfl_sync(kFull, p[u][0], la + 4);
      const float pc = __shfl_sync(kFull, p[u][1], la), pd = __shfl_sync(kFull, p[u][1], la + 4);
      // 2-bit: tokens 2qd + 8, + 9 (the upper K half) carry 2^-4 against the subnormal codes
      constexpr float kTf = VB == 2 ? 0.0625f : 1.f;
      const uint16_t* vsh = reinterpret_cast<const uint16_t*>(st + S::oVS) + u * 16 * VPT;
      const uint16_t* vzh = reinterpret_cast<const uint16_t*>(st + S::oVZ) + u * 16 * VPT;
      uint32_t bp[NBV][2];
      if constexpr (PV1) {
        // one fp16 column per (value group, head): this lane makes all four products of its column,
        // tokens 2qd, 2qd + 1 (b0) and 2qd + 8, 2qd + 9 (b1). The products keep fp16's 11 significant
        // bits: a relative error of at most 2^-12 per term of the output sum, far inside the output
        // tolerance (QK keeps hi / lo, where an error is exponentiated).
        const float pcs = pc * kTf, pds = pd * kTf;
#pragma unroll
        for (int nb = 0; nb < NBV; ++nb) {
          const int j = nb * VGB + pv_off;  // < VPT: every column is in use
          const int te = 2 * qd * VPT + j;
          const float s0 = h2f(vsh[te]), s1 = h2f(vsh[te + VPT]);
          const float s8 = h2f(vsh[te + 8 * VPT]), s9 = h2f(vsh[te + 9 * VPT]);
          const float z0 = h2f(vzh[te]), z1 = h2f(vzh[te + VPT]);
          const float z8 = h2f(vzh[te + 8 * VPT]), z9 = h2f(vzh[te + 9 * VPT]);
          bp[nb][0] = pack_h2(pa * s0, pb * s1);
          bp[nb][1] = pack_h2(pcs * s8, pds * s9);
          float z = zacc[nb];
          z = fmaf(pa, fmaf(kCbar, s0, z0), z);
          z = fmaf(pb, fmaf(kCbar, s1, z1), z);
          z = fmaf(pc, fmaf(kCbar, s8, z8), z);
          z = fmaf(pd, fmaf(kCbar, s9, z9), z);
          zacc[nb] = z;
        }
      } else {
        // The hi lane of a column (r even) takes tokens 2qd, 2qd + 1 (the lower K half of the B
        // fragment), the lo lane (r odd) tokens 2qd + 8, 2qd + 9; each makes both parts of its products
        // and passes the partner lane (L ^ 4) the part that lane needs.
        const float pe = lo_half ? pc : pa, po = lo_half ? pd : pb;  // probabilities of this lane's tokens
        const float pes = lo_half ? pc * kTf : pa, pos = lo_half ? pd * kTf : pb;
#pragma unroll
        for (int nb = 0; nb < NBV; ++nb) {
          const int j = nb * VGB + col_off;
          uint32_t hpk = 0u, lpk = 0u;  // both parts of this lane's two products (0 past the groups)
          if (VPT % VGB == 0 || j < VPT) {
            const int te = 2 * qd * VPT + j + (lo_half ? 8 * VPT : 0);  // this lane's first token
            const float se = h2f(vsh[te]), so = h2f(vsh[te + VPT]);
            const float ze = h2f(vzh[te]), zo = h2f(vzh[te + VPT]);
            const float xe = pes * se, xo = pos * so;
            const float he = split_part(xe, false), ho = split_part(xo, false);
            hpk = pack_h2(he, ho);
            lpk = pack_h2(__fsub_rn(xe, he), __fsub_rn(xo, ho));
            float z = zacc[nb];
            z = fmaf(pe, fmaf(kCbar, se, ze), z);
            z = fmaf(po, fmaf(kCbar, so, zo), z);
            zacc[nb] = z;
          }
          const uint32_t recv = __shfl_xor_sync(kFull, lo_half ? hpk : lpk, 4);
          bp[nb][0] = lo_half ? recv : hpk;  // tokens 2qd, 2qd + 1: hi part here (hi lane), lo part from it
          bp[nb][1] = lo_half ? lpk : recv;  // tokens 2qd + 8, + 9: lo part here (lo lane), hi part from it
        }
      }
      // m-block m (channels 16m .. 16m+15) lies in value group (16m) / G, held by n-block group / VGB
      const uint8_t* vc = st + S::oVC + u * 256 * VB;
      if constexpr (VB == 2) {
        const uint4 vw = *reinterpret_cast<const uint4*>(vc + 16 * lane);
        const uint32_t w4[4] = {vw.x, vw.y, vw.z, vw.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t h[8];
          unpack_word2_centered_sub(w4[w], h);
          const int nb0 = (2 * w * VPT / 8) / VGB;
          const int nb1 = ((2 * w + 1) * VPT / 8) / VGB;
          mma16816(O[2 * w], h[0], h[1], h[2], h[3], bp[nb0][0], bp[nb0][1]);
          mma16816(O[2 * w + 1], h[4], h[5], h[6], h[7], bp[nb1][0], bp[nb1][1]);
        }
      } else {
        const uint4 v0 = *reinterpret_cast<const uint4*>(vc + 16 * lane);
        const uint4 v1 = *reinterpret_cast<const uint4*>(vc + 512 + 16 * lane);
        const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int w = 0; w < 8; ++w) {
          uint32_t h[4];
          unpack_word4_centered_sub(w8[w], h);
          const int nb = (w * VPT / 8) / VGB;
          mma16816(O[w], h[0], h[1], h[2], h[3], bp[nb][0], bp[nb][1]);
        }
      }
    }
    __syncwarp();  // every lane is done with this stage before it is refilled
  }
  cp_async_wait<0>();
  __syncthreads();  // the ring area becomes the epilogue area below

  // ---- warp partial of the quantized tokens -> shared memory
  l_run += __shfl_xor_sync(kFull, l_run, 4);
  l_run += __shfl_xor_sync(kFull, l_run, 8);
  l_run += __shfl_xor_sync(kFull, l_run, 16);
#pragma unroll
  for (int j = 0; j < NBV; ++j) {
    if constexpr (!PV1) zacc[j] += __shfl_xor_sync(kFull, zacc[j], 4);  // the hi and lo lanes' tokens
    zacc[j] += __shfl_xor_sync(kFull, zacc[j], 1);
    zacc[j] += __shfl_xor_sync(kFull, zacc[j], 2);
  }
  float* cw = cm + warp * 4 * kCm;
  // row scales of the subnormal centered codes (2 (c - cbar) 2^-24 on row r)
  constexpr float kORowLo = 8388608.0f, kORowHi = VB == 2 ? 2097152.0f : 524288.0f;  // 2^23, 2^21 / 2^19
  if constexpr (PV1) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int jm = (16 * m) / G;
#pragma unroll
      for (int e = 0; e < 2; ++e) {  // D column 2qd + e: value group offset (2qd + e) / GQ, head (2qd + e) % GQ
        const int he = (2 * qd + e) % GQ;
        if ((2 * qd + e) / GQ == jm % VGB && he < gq) {
          float* o = cw + he * kCm + kCmO;
          o[16 * m + r] = O[m][e] * kORowLo;
          o[16 * m + r + 8] = O[m][2 + e] * kORowHi;
        }
      }
    }
  } else if (h_d < gq) {
    float* o = cw + h_d * kCm + kCmO;
#pragma unroll
    for (int m = 0; m < 8; ++m) {
      const int jm = (16 * m) / G;
      if (qd / GQ == jm % VGB) {  // this lane owns the columns of m-block m's value group
        o[16 * m + r] = (O[m][0] + O[m][1]) * kORowLo;
        o[16 * m + r + 8] = (O[m][2] + O[m][3]) * kORowHi;
      }
    }
  }
  if (h_d < gq && r == 0 && qd < GQ) {
    cw[h_d * kCm] = m_run;
    cw[h_d * kCm + 1] = l_run;
  }
  if (qd == 0 && (PV1 || !lo_half) && pv_head < gq) {
#pragma unroll
    for (int nb = 0; nb < NBV; ++nb) {
      const int j = nb * VGB + pv_off;
      if (j < VPT) zb[(warp * 4 + pv_head) * 8 + j] = zacc[nb];
    }
  }
  __syncwarp();
  for (int idx = lane; idx < gq * kHeadDim; idx += 32) {
    const int h = idx >> 7, c = idx & 127;
    cw[h * kCm + kCmO + c] += zb[(warp * 4 + h) * 8 + c / G] + (OUT ? corr[h * kHeadDim + c] : 0.f);
  }
  __syncwarp();

  // ---- FP16 window tokens [Q, T), spread over all splits of the unit: this CTA takes tokens
  //      Q + split + k * ns (ns = splits holding tokens), warp w the k = w (mod 4); batches of 8 with
  //      all loads issued first. Lane l holds channels 4l .. 4l + 3; the batch's partial is merged
  //      into the warp partial in shared memory. With the sink on and Q > 0 the list starts one
  //      earlier, at Q - 1, which stands for the sink token's row R + G.
  {
    const int W0 = (a.sink && Q > 0) ? Q - 1 : Q;
    const int ns = (T + L - 1) / L;
    float qr[GQ][4];
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
      const float4 v = *reinterpret_cast<const float4*>(sq + h * kHeadDim + 4 * lane);
      qr[h][0] = v.x;
      qr[h][1] = v.y;
      qr[h][2] = v.z;
      qr[h][3] = v.w;
    }
    const uint2* kres = reinterpret_cast<const uint2*>(a.k_res + unit * a.res_rows * kHeadDim) + lane;
    const uint2* vres = reinterpret_cast<const uint2*>(a.v_res + unit * a.res_rows * kHeadDim) + lane;
    for (int k0 = warp; W0 + split + k0 * ns < T; k0 += 4 * 8) {
      uint2 kk[8], vv[8];
      bool valid[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int tt = W0 + split + (k0 + 4 * j) * ns;
        valid[j] = tt < T;
        const int slot = !valid[j] ? 0 : tt < Q ? static_cast<int>(a.ring) : static_cast<int>(tt % a.ring);
        kk[j] = kres[slot * (kHeadDim / 4)];
        vv[j] = vres[slot * (kHeadDim / 4)];
      }
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        if (h >= gq) break;
        float sc[8];
        float mb = -CUDART_INF_F;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float d = qr[h][0] * h2f(static_cast<uint16_t>(kk[j].x & 0xffffu));
          d = fmaf(qr[h][1], h2f(static_cast<uint16_t>(kk[j].x >> 16)), d);
          d = fmaf(qr[h][2], h2f(static_cast<uint16_t>(kk[j].y & 0xffffu)), d);
          d = fmaf(qr[h][3], h2f(static_cast<uint16_t>(kk[j].y >> 16)), d);
#pragma unroll
          for (int x = 16; x > 0; x >>= 1) d += __shfl_xor_sync(kFull, d, x);
          sc[j] = valid[j] ? d : -CUDART_INF_F;
          mb = fmaxf(mb, sc[j]);
        }
        // merge this batch into the warp partial of head h (channels 4 lane .. 4 lane + 3)
        float* ph = cw + h * kCm;
        const float m_old = ph[0];
        const float m_new = fmaxf(m_old, mb);
        const float f_old = fast_exp2(m_old - m_new);
        float o4[4] = {0.f, 0.f, 0.f, 0.f};
        float lb = 0.f;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float pj = fast_exp2(sc[j] - m_new);
          lb += pj;
          o4[0] = fmaf(pj, h2f(static_cast<uint16_t>(vv[j].x & 0xffffu)), o4[0]);
          o4[1] = fmaf(pj, h2f(static_cast<uint16_t>(vv[j].x >> 16)), o4[1]);
          o4[2] = fmaf(pj, h2f(static_cast<uint16_t>(vv[j].y & 0xffffu)), o4[2]);
          o4[3] = fmaf(pj, h2f(static_cast<uint16_t>(vv[j].y >> 16)), o4[3]);
        }
        float4 cur = *reinterpret_cast<float4*>(ph + kCmO + 4 * lane);
        cur.x = fmaf(cur.x, f_old, o4[0]);
        cur.y = fmaf(cur.y, f_old, o4[1]);
        cur.z = fmaf(cur.z, f_old, o4[2]);
        cur.w = fmaf(cur.w, f_old, o4[3]);
        *reinterpret_cast<float4*>(ph + kCmO + 4 * lane) = cur;
        __syncwarp();
        if (lane == 0) {
          ph[0] = m_new;
          ph[1] = fmaf(ph[1], f_old, lb);
        }
        __syncwarp();
      }
    }
  }
  __syncthreads();

  // ---- CTA partial (merge the warps) -> workspace
  float* part = a.part + ((unit * a.nsplit + split) * gq) * kPartFloats;
  for (int idx = threadIdx.x; idx < gq * kHeadDim; idx += blockDim.x) {
    const int h = idx >> 7, c = idx & 127;
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) M = fmaxf(M, cm[(w * 4 + h) * kCm]);
    // A split can hold no token at all (its range lies in the FP16 window and the window tokens went
    // to other splits): its partial is (m = -inf, l = 0, o = 0), which the combine weighs by 0.
    const bool empty = M == -CUDART_INF_F;
    float o = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < kDecodeWarps; ++w) {
      const float* pw = cm + (w * 4 + h) * kCm;
      const float f = empty ? 0.f : fast_exp2(pw[0] - M);
      o = fmaf(f, pw[kCmO + c], o);
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
    if (c == 0) a.status[row] = 0u;
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
    const float f = fast_exp2(p[0] - M);
    l = fmaf(f, p[1], l);
    acc = fmaf(f, p[2 + c], acc);
  }
  out[c] = __half_as_ushort(__float2half_rn(acc / l));
  // l is NaN only where a split kernel gave up a bounded wait and wrote a NaN partial (finite inputs)
  if (c == 0) a.status[row] = l != l ? 1u : 0u;
}

template <int KB, int VB, int VPT, int GQ, bool OUT>
cudaError_t launch_split(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int smem = decode_smem_bytes<KB, VB, VPT, GQ, OUT>();
  static DeviceMemo attr;
  const int ok = attr.get([] {
    return cudaFuncSetAttribute(decode_split_kernel<KB, VB, VPT, GQ, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess ? 1 : -1;
  });
  if (ok < 0) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(static_cast<int64_t>(a.batch) * a.num_kv_heads));
  decode_split_kernel<KB, VB, VPT, GQ, OUT><<<grid, 32 * kDecodeWarps, smem, stream>>>(a);
  return cudaGetLastError();
}

template <int KB, int VB, int VPT, int GQ, bool OUT>
int occupancy() {
  static DeviceMemo memo;
  return memo.get([] {
    constexpr int smem = decode_smem_bytes<KB, VB, VPT, GQ, OUT>();
    if (cudaFuncSetAttribute(decode_split_kernel<KB, VB, VPT, GQ, OUT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return 1;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, decode_split_kernel<KB, VB, VPT, GQ, OUT>, 32 * kDecodeWarps, smem) != cudaSuccess)
      return 1;
    return n > 0 ? n : 1;
  });
}

// GQ template: the smallest of 1, 2, 4 that holds the query heads of one KV head.
inline int gq_class(int gqa) { return gqa <= 1 ? 1 : (gqa <= 2 ? 2 : 4); }

template <int KB, int VB, int VPT, bool OUT>
cudaError_t dispatch_gq_out(const DecodeArgs& a, cudaStream_t s) {
  switch (gq_class(a.gqa)) {
    case 1: return launch_split<KB, VB, VPT, 1, OUT>(a, s);
    case 2: return launch_split<KB, VB, VPT, 2, OUT>(a, s);
    default: return launch_split<KB, VB, VPT, 4, OUT>(a, s);
  }
}

template <int KB, int VB, int VPT>
cudaError_t dispatch_gq(const DecodeArgs& a, cudaStream_t s) {
  return a.outliers ? dispatch_gq_out<KB, VB, VPT, true>(a, s) : dispatch_gq_out<KB, VB, VPT, false>(a, s);
}

template <int KB, int VB, int VPT, bool OUT>
int occupancy_gq_out(int gqa) {
  switch (gq_class(gqa)) {
    case 1: return occupancy<KB, VB, VPT, 1, OUT>();
    case 2: return occupancy<KB, VB, VPT, 2, OUT>();
    default: return occupancy<KB, VB, VPT, 4, OUT>();
  }
}

template <int KB, int VB, int VPT>
int occupancy_gq(int gqa, int outliers) {
  return outliers ? occupancy_gq_out<KB, VB, VPT, true>(gqa) : occupancy_gq_out<KB, VB, VPT, false>(gqa);
}

template <int KB, int VB>
cudaError_t dispatch_vpt(const DecodeArgs& a, cudaStream_t s) {
  switch (a.G) {
    case 128: return dispatch_gq<KB, VB, 1>(a, s);
    case 64: return dispatch_gq<KB, VB, 2>(a, s);
    case 32: return dispatch_gq<KB, VB, 4>(a, s);
    default: return dispatch_gq<KB, VB, 8>(a, s);
  }
}

template <int KB, int VB>
int occupancy_vpt(int G, int gqa, int outliers) {
  switch (G) {
    case 128: return occupancy_gq<KB, VB, 1>(gqa, outliers);
    case 64: return occupancy_gq<KB, VB, 2>(gqa, outliers);
    case 32: return occupancy_gq<KB, VB, 4>(gqa, outliers);
    default: return occupancy_gq<KB, VB, 8>(gqa, outliers);
  }
}

}  // namespace

bool cuda_core_control_requested(int layout, float rope_theta, int hadamard) {
  if (layout != KVQ_LAYOUT_ROWS_V2 || rope_theta > 0.f || hadamard) return false;
  const char* v = std::getenv("KVQ_DECODE_CUDA_CORES");
  return v != nullptr && v[0] == '1';
}

bool stall_test_requested() {
  const char* v = std::getenv("KVQ_TEST_STALL_TC");
  return v != nullptr && v[0] == '1';
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  cudaError_t e;
  if (a.rope_theta > 0.f)
    e = launch_decode_rope(a, stream);
  else if (cuda_core_control_requested(a.layout, a.rope_theta, a.hadamard))
    e = launch_decode_cuda_cores(a, stream);
  else if (a.layout == KVQ_LAYOUT_ROWS_V2)
    e = launch_decode_tc(a, stream);
  else if (a.key_bits == 2)
    e = a.value_bits == 2 ? dispatch_vpt<2, 2>(a, stream) : dispatch_vpt<2, 4>(a, stream);
  else
    e = a.value_bits == 2 ? dispatch_vpt<4, 2>(a, stream) : dispatch_vpt<4, 4>(a, stream);
  if (e != cudaSuccess) return e;
  decode_combine_kernel<<<static_cast<unsigned>(static_cast<int64_t>(a.batch) * a.num_q_heads), kHeadDim, 0, stream>>>(a);
  return cudaGetLastError();
}

int decode_ctas_per_sm(int key_bits, int value_bits, int G, int gqa, int outliers) {
  if (key_bits == 2) return value_bits == 2 ? occupancy_vpt<2, 2>(G, gqa, outliers) : occupancy_vpt<2, 4>(G, gqa, outliers);
  return value_bits == 2 ? occupancy_vpt<4, 2>(G, gqa, outliers) : occupancy_vpt<4, 4>(G, gqa, outliers);
}

}  // namespace kvq
