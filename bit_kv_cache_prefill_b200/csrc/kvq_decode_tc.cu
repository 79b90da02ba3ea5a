// kvq_decode_tc.cu — split-K decode attention on the rows-v2 layout with the 5th-generation tensor
// cores (tcgen05, sm_100a).
//
// What is computed is the same as the tile-v1 kernel: the grouped (quantized) tokens and the FP16
// window enter one softmax (KV cache quantization wiki page, KIVI notes on combining the grouped and
// residual parts), the packed cache is consumed in place (KVQuant review, Method), and every split
// writes a (max, sum, output) partial that the combine kernel merges.
//
// Work split. The grid is (split, unit) with unit = (sequence, KV head); a CTA of 8 warps owns one
// token range of split_len tokens (a multiple of 128) and walks it in 128-token steps. Thread roles:
// warps 0-3 ("token warps") own TMEM lanes 0..127 as the step's tokens, warps 4-7 ("channel warps")
// own the same lanes as channels.
//
// Per step i (scores in base-2 units; q~ = q * sm_scale * log2 e, q^ = q~ * 2^-e per head):
//   QK(i):  S[t][n] = sum_c codeK[t][c] * B_QK[c][n] on the tensor cores, A = the step's key codes
//           as exact fp16 in TMEM (lane = token), B = q^[h][c] * sk[g][c] split into hi + lo fp16
//           columns n = (group offset, head, part) in shared memory. A token reads the two columns of
//           its own group: s_t = 2^e (S_hi + S_lo) + sum_c q~[h][c] zk[g][c].
//   PV(i):  O[c][n] += sum_t (codeV[t][c] - cbar) * B_PV[t][n], A = centered value codes in TMEM
//           (lane = channel), B = p_t * sv[t][j] split hi + lo, n = (value group j, head, part). The
//           accumulator O lives in TMEM for the whole split; the midpoint term
//           sum_t p_t (zv + cbar sv) is an fp32 register sum per token slot (the tile-v1 kernel
//           explains why the codes are centered).
//   Online softmax: one running max per head for the CTA; O, l and the midpoint sums are rescaled
//   only in a step where some score exceeds it (a CTA vote), so p <= 1 always.
// Pipeline: one elected thread streams each step's key rows, value block, value scale / zero and
// key scale / zero with bulk async copies into a 4-8 stage ring (one mbarrier per stage) and issues
// the MMAs; each MMA batch signals an mbarrier through tcgen05.commit. The key side runs two steps
// ahead: A_K, B_QK and S are double-buffered, so in iteration i the token warps read S(i) (issued two
// iterations earlier), write B_PV(i) and unpack the keys of step i + 2, while the channel warps build
// B_QK(i + 2) and unpack the values of step i. One CTA barrier per step carries the vote on a new
// maximum; only a step that raises it takes a second barrier (rescale and redo its probabilities).
// Configs whose columns fit 256 TMEM columns run two CTAs per SM, the others one CTA with 512.
// Every wait is bounded; a CTA that gives up on a wait marks its partial (l = NaN), so the affected
// outputs read NaN instead of the kernel hanging.
#include <cuda_runtime.h>
#include <math_constants.h>

#include "kvq_common.cuh"
#include "kvq_decode_common.cuh"
#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kThreads = 256;
constexpr int kStep = 128;  // tokens per step
constexpr uint32_t kWaitSliceNs = 1000000;  // 1 ms
constexpr int kWaitSlices = 2000;
constexpr int kPartStride = 132;  // shared-memory partial: m, l, 2 pad, o[128] (16-byte aligned)
constexpr int kPartO = 4;
constexpr unsigned kAll = 0xffffffffu;

// ---- PTX wrappers -----------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
// try_wait with a suspend-time hint: the thread sleeps until the phase completes or about
// kWaitSliceNs elapse, instead of spinning on the barrier.
__device__ __forceinline__ bool mbar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(kWaitSliceNs)
      : "memory");
  return ok != 0;
}
// Bounded wait on an mbarrier phase: at most kWaitSlices sleeps of up to kWaitSliceNs each (about 2 s
// in all). Gives up (and raises the CTA's abort flag) after that, or at once when another thread of
// the CTA has already given up.
__device__ __forceinline__ void mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
  for (int it = 0; it < kWaitSlices; ++it) {
    if (mbar_try(bar, parity)) return;
    if (*abort_flag) return;
  }
  *abort_flag = 1;
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)), "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(cols) : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem], kind::f16, fp32 accumulate, one CTA.
__device__ __forceinline__ void mma_f16_ts(uint32_t d, uint32_t a, uint64_t bdesc, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(bdesc), "r"(idesc), "r"(acc)
      : "memory");
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// Shared-memory descriptor of a B operand stored MN-major without swizzle: core matrices of 8 K-rows x
// 8 N-values (16 bytes per row), K-adjacent core matrices 128 bytes apart (leading byte offset),
// N-adjacent ones 2048 bytes apart (stride byte offset; 16 core matrices cover K = 128).
__device__ __forceinline__ uint64_t b_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(128u >> 4) << 16;
  d |= static_cast<uint64_t>(2048u >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;  // descriptor version of sm_100
  return d;
}
// Instruction descriptor, kind::f16: fp16 A and B, fp32 D, A K-major, B MN-major, M = 128.
__host__ __device__ constexpr uint32_t idesc_f16(int n) {
  return (1u << 4) | (1u << 16) | (static_cast<uint32_t>(n >> 3) << 17) | (static_cast<uint32_t>(128 >> 4) << 24);
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,"
      "%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// tcgen05.ld of N consecutive 32-bit columns of the warp's 32 lanes (N = 2, 4, 8 or 16).
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]);
template <>
__device__ __forceinline__ void tmem_ld<2>(uint32_t taddr, uint32_t (&r)[2]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(taddr) : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<4>(uint32_t taddr, uint32_t (&r)[4]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr)
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<8>(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
}
template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// ---- shared-memory and TMEM plan -----------------------------------------------------------------------
template <int KB, int VB, int VPT, int GQ>
struct TcPlan {
  static constexpr int G = 128 / VPT;
  static constexpr int kUsedCols = VPT * GQ * 2;  // B columns in use, QK and PV alike (128/G = VPT groups per step)
  static constexpr int kN = kUsedCols < 16 ? 16 : kUsedCols;
  static constexpr int kChunks = (kUsedCols + 7) / 8;  // 16-byte chunks per B row written
  // TMEM columns: A_K double-buffered (steps of even / odd index), A_V, S double-buffered, O.
  static constexpr uint32_t kColAK = 0, kColAV = 128, kColS = 192, kColO = 192 + 2 * kN;
  static constexpr uint32_t kTmemCols = kColO + kN <= 256 ? 256 : 512;
  static constexpr int kCtasPerSm = 512 / kTmemCols;
  // One stage: everything a step reads from the cache.
  static constexpr int kKC = kStep * 16 * KB;  // key rows of 128 tokens
  static constexpr int kVC = 128 * 16 * VB;    // value rows of 128 channels (one 128-token block)
  static constexpr int kVS = kStep * VPT * 2;  // value scale of 128 tokens (value zero: same)
  static constexpr int kKS = VPT * 256;        // key scale of the step's groups (key zero: same)
  static constexpr int oKC = 0, oVC = oKC + kKC, oVS = oVC + kVC, oVZ = oVS + kVS, oKS = oVZ + kVS, oKZ = oKS + kKS;
  static constexpr int kStageBytes = oKZ + kKS;
  static constexpr int kStageBudget = kCtasPerSm == 2 ? 64 * 1024 : 144 * 1024;
  static constexpr int kStagesRaw = kStageBudget / kStageBytes;
  static constexpr int kStages = kStagesRaw < 4 ? 4 : (kStagesRaw > 8 ? 8 : kStagesRaw);
  static constexpr int kB = 128 * kN * 2;  // one B operand
  static constexpr int oBQK = kStages * kStageBytes;  // [2] (by step parity)
  static constexpr int oBPV = oBQK + 2 * kB;
  static constexpr int oQ = oBPV + kB;                   // q~ [GQ][128] f32
  static constexpr int oQH = oQ + GQ * 512;              // q^ [GQ][128] f32
  static constexpr int oBias = oQH + GQ * 512;           // [4][VPT * GQ] f32, by step index mod 4
  static constexpr int oRed = oBias + 4 * VPT * GQ * 4;  // [4][GQ] f32 warp maxima
  static constexpr int oE = oRed + 4 * GQ * 4;           // [4] i32 per-head exponents
  static constexpr int oBar = oE + 16;                   // mbarriers: QK[2], PV, stage[kStages]
  static constexpr int kBarQK = 0, kBarPV = 2, kBarStage = 3;
  static constexpr int oTmem = oBar + 8 * (3 + kStages);
  static constexpr int oFlag = oTmem + 4;
  static constexpr int kUsed = oFlag + 4;
  // Two CTAs per SM (256 TMEM columns each) need at least 78 KB each so that a third never fits;
  // one CTA per SM (512 columns) needs more than half of the SM's shared memory.
  static constexpr int kFloor = kCtasPerSm == 2 ? 78 * 1024 : 116 * 1024;
  static constexpr int kSmem = kUsed > kFloor ? kUsed : kFloor;
  // Epilogue (in the stage area): quantized partial [GQ], window partials [8][GQ], sums [4][GQ*(1+VPT)].
  static constexpr int kEpiFloats = 9 * GQ * kPartStride + 4 * GQ * (1 + VPT);
  static_assert(kEpiFloats * 4 <= kStages * kStageBytes, "epilogue does not fit the stage area");
  static_assert(oBar % 8 == 0 && oBQK % 16 == 0 && oBPV % 16 == 0, "alignment");
  static_assert(kColO + kN <= kTmemCols, "TMEM plan");
  static_assert(kSmem <= 227 * 1024, "shared memory");
};

template <int N>
__device__ __forceinline__ void load_u16s(const uint16_t* p, float (&out)[N]) {
  if constexpr (N == 1) {
    out[0] = h2f(p[0]);
  } else if constexpr (N == 2) {
    const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
    out[0] = h2f(static_cast<uint16_t>(w & 0xffffu));
    out[1] = h2f(static_cast<uint16_t>(w >> 16));
  } else {
#pragma unroll
    for (int i = 0; i < N / 4; ++i) {
      const uint2 w = reinterpret_cast<const uint2*>(p)[i];
      out[4 * i] = h2f(static_cast<uint16_t>(w.x & 0xffffu));
      out[4 * i + 1] = h2f(static_cast<uint16_t>(w.x >> 16));
      out[4 * i + 2] = h2f(static_cast<uint16_t>(w.y & 0xffffu));
      out[4 * i + 3] = h2f(static_cast<uint16_t>(w.y >> 16));
    }
  }
}

// One 32-column half (64 fp16 pairs) of a row of codes -> exact fp16 pairs in TMEM columns
// [col, col + 32). `src` holds 16 * bits bytes: pair k of word w is TMEM column (16/bits) w + k.
template <int BITS, bool CENTER>
__device__ __forceinline__ void unpack_row_half(const uint8_t* src, uint32_t taddr) {
  uint32_t r[32];
  if constexpr (BITS == 2) {
    const uint4 v = *reinterpret_cast<const uint4*>(src);
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t h[8];
      if constexpr (CENTER)
        unpack_word2_centered(w4[w], h);
      else
        unpack_word2(w4[w], h);
#pragma unroll
      for (int k = 0; k < 8; ++k) r[8 * w + k] = h[k];
    }
  } else {
    const uint4 v0 = reinterpret_cast<const uint4*>(src)[0];
    const uint4 v1 = reinterpret_cast<const uint4*>(src)[1];
    const uint32_t w8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t h[4];
      if constexpr (CENTER)
        unpack_word4_centered(w8[w], h);
      else
        unpack_word4(w8[w], h);
#pragma unroll
      for (int k = 0; k < 4; ++k) r[4 * w + k] = h[k];
    }
  }
  tmem_st32(taddr, r);
}

template <int KB, int VB, int VPT, int GQ>
__global__ void __launch_bounds__(kThreads, TcPlan<KB, VB, VPT, GQ>::kCtasPerSm) decode_tc_kernel(const DecodeArgs a) {
  using P = TcPlan<KB, VB, VPT, GQ>;
  constexpr int G = P::G, S = P::kStages, NC = P::kUsedCols;
  constexpr float kCbar = VB == 2 ? 1.5f : 7.5f;
  extern __shared__ __align__(1024) uint8_t smem[];
  float* sq = reinterpret_cast<float*>(smem + P::oQ);
  float* sqh = reinterpret_cast<float*>(smem + P::oQH);
  float* sbias = reinterpret_cast<float*>(smem + P::oBias);
  float* sred = reinterpret_cast<float*>(smem + P::oRed);
  int* se = reinterpret_cast<int*>(smem + P::oE);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P::oBar);
  uint32_t* stmem = reinterpret_cast<uint32_t*>(smem + P::oTmem);
  volatile int* sflag = reinterpret_cast<volatile int*>(smem + P::oFlag);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool token_warp = warp < 4;
  const int wq = warp & 3, row = 32 * wq + lane;  // TMEM lane: token (token warps) / channel (channel warps)
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
  // a.stall_test: no quantized step is issued (nothing lands in shared memory, no MMA runs), and one
  // thread waits below on a barrier phase that nothing completes
  const int nsteps = qend > start && !a.stall_test ? (qend - start + kStep - 1) / kStep : 0;

  // Bulk copies of step j into stage j % S (one thread).
  const uint8_t* kc_base = reinterpret_cast<const uint8_t*>(a.k_codes) + (unit * a.capacity + start) * (16 * KB);
  const uint8_t* vc_base = reinterpret_cast<const uint8_t*>(a.v_codes) + (unit * a.capacity + start) * (16 * VB);
  const uint8_t* vs_base = reinterpret_cast<const uint8_t*>(a.v_scale) + (unit * a.capacity + start) * (2 * VPT);
  const uint8_t* vz_base = reinterpret_cast<const uint8_t*>(a.v_zero) + (unit * a.capacity + start) * (2 * VPT);
  const uint8_t* ks_base = reinterpret_cast<const uint8_t*>(a.k_scale) + (unit * a.groups + start / G) * 256;
  const uint8_t* kz_base = reinterpret_cast<const uint8_t*>(a.k_zero) + (unit * a.groups + start / G) * 256;
  auto issue = [&](int j) {
    uint8_t* st = smem + (j % S) * P::kStageBytes;
    uint64_t* bar = &bars[P::kBarStage + j % S];
    const int64_t t0 = static_cast<int64_t>(j) * kStep;
    mbar_expect_tx(bar, P::kStageBytes);
    bulk_g2s(st + P::oKC, kc_base + t0 * (16 * KB), P::kKC, bar);
    bulk_g2s(st + P::oVC, vc_base + t0 * (16 * VB), P::kVC, bar);
    bulk_g2s(st + P::oVS, vs_base + t0 * (2 * VPT), P::kVS, bar);
    bulk_g2s(st + P::oVZ, vz_base + t0 * (2 * VPT), P::kVS, bar);
    bulk_g2s(st + P::oKS, ks_base + (t0 / G) * 256, P::kKS, bar);
    bulk_g2s(st + P::oKZ, kz_base + (t0 / G) * 256, P::kKS, bar);
  };
  auto wait_stage = [&](int j) { mbar_wait(&bars[P::kBarStage + j % S], (j / S) & 1, sflag); };

  if (warp == 0) tmem_alloc(stmem, P::kTmemCols);
  if (tid == 32) {
    for (int i = 0; i < 3 + S; ++i) mbar_init(&bars[i], 1);
    *sflag = 0;
    fence_mbar_init();
    fence_proxy_async();
    for (int j = 0; j < S && j < nsteps; ++j) issue(j);
  }

  // ---- query: optional Hadamard rotation, scale to base-2 logits, per-head power-of-two exponent
  if (warp < gq) {
    float x[4];
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
          const float o = __shfl_xor_sync(kAll, x[i], d);
          x[i] = upper ? o - x[i] : x[i] + o;
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) x[i] *= inv_sqrt128();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] *= a.qscale;
    float mx = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, d));
    const int e = mx > 0.f ? ((__float_as_int(mx) >> 23) & 0xff) - 126 : 0;
    *reinterpret_cast<float4*>(sq + warp * kHeadDim + 4 * lane) = make_float4(x[0], x[1], x[2], x[3]);
    const float inv = pow2i(-e);
    *reinterpret_cast<float4*>(sqh + warp * kHeadDim + 4 * lane) = make_float4(x[0] * inv, x[1] * inv, x[2] * inv, x[3] * inv);
    if (lane == 0) se[warp] = e;
  } else if (warp < GQ) {  // heads of the template beyond gqa: zero query
    *reinterpret_cast<float4*>(sq + warp * kHeadDim + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
    *reinterpret_cast<float4*>(sqh + warp * kHeadDim + 4 * lane) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0) se[warp] = 0;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *stmem;
  const uint32_t lane_base = static_cast<uint32_t>(32 * wq) << 16;

  // per-role constants
  float qh[GQ];   // channel warps: q^[h][row]
  float qz[4];    // channel warps: q~[h_w][4 lane .. 4 lane + 3], h_w = wq % GQ (bias dots)
  float p2e[GQ];  // token warps: 2^e per head
#pragma unroll
  for (int h = 0; h < GQ; ++h) {
    qh[h] = sqh[h * kHeadDim + row];
    p2e[h] = pow2i(se[h]);
  }
  {
    const float4 v = *reinterpret_cast<const float4*>(sq + (wq % GQ) * kHeadDim + 4 * lane);
    qz[0] = v.x;
    qz[1] = v.y;
    qz[2] = v.z;
    qz[3] = v.w;
  }

  // Channel warps: B_QK of step j (row = channel) into buffer j % 2, and the step's zero-point biases
  // into slot j % 4 (one warp-wide dot per (group, head); warp wq takes the pairs d = wq (mod 4), whose
  // head is wq % GQ).
  auto build_qk = [&](int j) {
    const uint8_t* st = smem + (j % S) * P::kStageBytes;
    const uint16_t* ks = reinterpret_cast<const uint16_t*>(st + P::oKS);
    uint32_t w[P::kChunks * 4];
#pragma unroll
    for (int i = 0; i < P::kChunks * 4; ++i) w[i] = 0u;
#pragma unroll
    for (int gl = 0; gl < VPT; ++gl) {
      const float s = h2f(ks[gl * 128 + row]);
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        const float x = qh[h] * s;
        w[gl * GQ + h] = pack_h2(split_part(x, false), split_part(x, true));
      }
    }
    uint8_t* dst = smem + P::oBQK + (j & 1) * P::kB + row * 16;
#pragma unroll
    for (int c = 0; c < P::kChunks; ++c)
      *reinterpret_cast<uint4*>(dst + c * 2048) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    const uint16_t* kz = reinterpret_cast<const uint16_t*>(st + P::oKZ);
    float* bias = sbias + (j & 3) * (VPT * GQ);
#pragma unroll
    for (int d0 = 0; d0 < VPT * GQ; d0 += 4) {
      const int d = d0 + wq;
      if (d < VPT * GQ) {
        const uint2 zz = *reinterpret_cast<const uint2*>(kz + (d / GQ) * 128 + 4 * lane);
        float dot = qz[0] * h2f(static_cast<uint16_t>(zz.x & 0xffffu));
        dot = fmaf(qz[1], h2f(static_cast<uint16_t>(zz.x >> 16)), dot);
        dot = fmaf(qz[2], h2f(static_cast<uint16_t>(zz.y & 0xffffu)), dot);
        dot = fmaf(qz[3], h2f(static_cast<uint16_t>(zz.y >> 16)), dot);
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) dot += __shfl_xor_sync(kAll, dot, x);
        if (lane == 0) bias[d] = dot;
      }
    }
  };
  // Token warps: key rows of step j -> A_K buffer j % 2 (row = token).
  auto unpack_keys = [&](int j) {
    const uint8_t* src = smem + (j % S) * P::kStageBytes + P::oKC + row * (16 * KB);
    const uint32_t col = P::kColAK + 64 * (j & 1);
    unpack_row_half<KB, false>(src, tmem + lane_base + col);
    unpack_row_half<KB, false>(src + 8 * KB, tmem + lane_base + col + 32);
  };
  // Channel warps: value rows of step j -> A_V (row = channel), centered.
  auto unpack_values = [&](int j) {
    const uint8_t* src = smem + (j % S) * P::kStageBytes + P::oVC + row * (16 * VB);
    unpack_row_half<VB, true>(src, tmem + lane_base + P::kColAV);
    unpack_row_half<VB, true>(src + 8 * VB, tmem + lane_base + P::kColAV + 32);
  };

  constexpr uint32_t kIdesc = idesc_f16(P::kN);
  const uint32_t bqk_addr = smem_u32(smem + P::oBQK), bpv_addr = smem_u32(smem + P::oBPV);
  // One thread: QK(j) = S[j % 2] from A_K[j % 2] and B_QK[j % 2], signalled on the QK barrier j % 2.
  auto issue_qk = [&](int j) {
    const uint32_t d = tmem + P::kColS + P::kN * (j & 1), acol = tmem + P::kColAK + 64 * (j & 1);
    const uint32_t baddr = bqk_addr + (j & 1) * P::kB;
#pragma unroll
    for (int s2 = 0; s2 < 8; ++s2) mma_f16_ts(d, acol + 8 * s2, b_desc(baddr + 256 * s2), kIdesc, s2 > 0);
    mma_commit(&bars[P::kBarQK + (j & 1)]);
  };

  // token-warp softmax state (m_ref is CTA-uniform and kept by every thread)
  float m_ref[GQ], l_run[GQ], zacc[GQ][VPT];
#pragma unroll
  for (int h = 0; h < GQ; ++h) {
    m_ref[h] = -CUDART_INF_F;
    l_run[h] = 0.f;
#pragma unroll
    for (int j = 0; j < VPT; ++j) zacc[h][j] = 0.f;
  }

  // ---- prologue: key operands of steps 0 and 1, then QK(0) and QK(1)
  const int npro = nsteps < 2 ? nsteps : 2;
  for (int j = 0; j < npro; ++j) {
    wait_stage(j);
    if (token_warp)
      unpack_keys(j);
    else
      build_qk(j);
  }
  fence_proxy_async();
  tc_wait_st();
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && npro > 0) {
    tc_fence_after();
    for (int j = 0; j < npro; ++j) issue_qk(j);
  }

  // ---- main loop. Iteration i: softmax and PV operands of step i, key operands of step i + 2; one
  //      barrier (with the new-maximum vote) in the common case; then PV(i) and QK(i + 2) are issued.
  for (int i = 0; i < nsteps; ++i) {
    const int t_step = start + i * kStep;
    const bool ahead = i + 2 < nsteps;
    const uint8_t* st = smem + (i % S) * P::kStageBytes;
    mbar_wait(&bars[P::kBarQK + (i & 1)], (i >> 1) & 1, sflag);  // QK(i): S(i) readable; A_K, B_QK buffer i % 2 free
    tc_fence_after();

    float s[GQ], p[GQ], sv[VPT], zv[VPT];
    bool exceed = false;
    const bool valid = t_step + row < qend && t_step + row >= a.sink;  // the sink token: fp16 row instead
#pragma unroll
    for (int h = 0; h < GQ; ++h) s[h] = p[h] = 0.f;
    // B_PV row of this token from p: hi/lo of p * sv per (value group, head); zero for masked tokens.
    auto write_bpv = [&]() {
      uint32_t w[P::kChunks * 4];
#pragma unroll
      for (int k = 0; k < P::kChunks * 4; ++k) w[k] = 0u;
#pragma unroll
      for (int j = 0; j < VPT; ++j)
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          const float x = valid ? p[h] * sv[j] : 0.f;
          w[j * GQ + h] = pack_h2(split_part(x, false), split_part(x, true));
        }
      uint8_t* dst = smem + P::oBPV + row * 16;
#pragma unroll
      for (int c = 0; c < P::kChunks; ++c)
        *reinterpret_cast<uint4*>(dst + c * 2048) = make_uint4(w[4 * c], w[4 * c + 1], w[4 * c + 2], w[4 * c + 3]);
    };
    if (token_warp) {
      constexpr int kGpw = G >= 32 ? 1 : 32 / G;  // groups per warp
      constexpr int kCols = kGpw * 2 * GQ;
      uint32_t d[kCols];
      const int gl0 = (32 * wq) / G;
      tmem_ld<kCols>(tmem + lane_base + P::kColS + P::kN * (i & 1) + gl0 * 2 * GQ, d);
      tc_wait_ld();
      const int gsel = kGpw > 1 ? (lane * kGpw) / 32 : 0;  // this token's group within the warp's columns
      const float* bias = sbias + (i & 3) * (VPT * GQ) + (row / G) * GQ;
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        float hi = __uint_as_float(d[2 * h]), lo = __uint_as_float(d[2 * h + 1]);
        if constexpr (kGpw > 1) {
#pragma unroll
          for (int g = 1; g < kGpw; ++g)
            if (gsel == g) {
              hi = __uint_as_float(d[g * 2 * GQ + 2 * h]);
              lo = __uint_as_float(d[g * 2 * GQ + 2 * h + 1]);
            }
        }
        s[h] = valid ? fmaf(hi + lo, p2e[h], bias[h]) : -CUDART_INF_F;
        exceed |= (h < gq) && (s[h] > m_ref[h]);
        float mx = s[h];
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) mx = fmaxf(mx, __shfl_xor_sync(kAll, mx, x));
        if (lane == 0) sred[wq * GQ + h] = mx;
      }
      load_u16s<VPT>(reinterpret_cast<const uint16_t*>(st + P::oVS) + row * VPT, sv);
      load_u16s<VPT>(reinterpret_cast<const uint16_t*>(st + P::oVZ) + row * VPT, zv);
#pragma unroll
      for (int h = 0; h < GQ; ++h) p[h] = valid ? fast_exp2(s[h] - m_ref[h]) : 0.f;
      if (i > 0) mbar_wait(&bars[P::kBarPV], (i - 1) & 1, sflag);  // PV(i-1): B_PV and O free
      tc_fence_after();
      write_bpv();  // rewritten below if the vote finds a new maximum
      if (ahead) {
        wait_stage(i + 2);
        unpack_keys(i + 2);
      }
    } else {
      if (ahead) {
        wait_stage(i + 2);
        build_qk(i + 2);
      }
      if (i > 0) mbar_wait(&bars[P::kBarPV], (i - 1) & 1, sflag);  // PV(i-1): A_V free
      tc_fence_after();
      unpack_values(i);
    }
    fence_proxy_async();
    tc_wait_st();
    tc_fence_before();
    if (__syncthreads_or(exceed)) {
      // A score above the running maximum: move the maximum to the step's, rescale l, the midpoint
      // sums and O (held in TMEM), and redo this step's probabilities.
      tc_fence_after();
      float alpha[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) {
        float mn = m_ref[h];
#pragma unroll
        for (int w = 0; w < 4; ++w) mn = fmaxf(mn, sred[w * GQ + h]);
        alpha[h] = mn == -CUDART_INF_F ? 1.f : fast_exp2(m_ref[h] - mn);
        m_ref[h] = mn;
      }
      if (token_warp) {
#pragma unroll
        for (int h = 0; h < GQ; ++h) {
          l_run[h] *= alpha[h];
#pragma unroll
          for (int j = 0; j < VPT; ++j) zacc[h][j] *= alpha[h];
          p[h] = valid ? fast_exp2(s[h] - m_ref[h]) : 0.f;
        }
        if (i > 0) {
#pragma unroll
          for (int c0 = 0; c0 < P::kN; c0 += 16) {
            uint32_t o[16];
            tmem_ld<16>(tmem + lane_base + P::kColO + c0, o);
            tc_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) o[c] = __float_as_uint(__uint_as_float(o[c]) * alpha[((c0 + c) >> 1) % GQ]);
            tmem_st16(tmem + lane_base + P::kColO + c0, o);
          }
        }
        write_bpv();
      }
      fence_proxy_async();
      tc_wait_st();
      tc_fence_before();
      __syncthreads();
    }
    if (token_warp) {
#pragma unroll
      for (int h = 0; h < GQ; ++h) l_run[h] += p[h];
      if (valid) {
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
          const float mid = fmaf(kCbar, sv[j], zv[j]);
#pragma unroll
          for (int h = 0; h < GQ; ++h) zacc[h][j] = fmaf(p[h], mid, zacc[h][j]);
        }
      }
    }
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int s2 = 0; s2 < 8; ++s2)
        mma_f16_ts(tmem + P::kColO, tmem + P::kColAV + 8 * s2, b_desc(bpv_addr + 256 * s2), kIdesc,
                   (i > 0 || s2 > 0) ? 1u : 0u);
      mma_commit(&bars[P::kBarPV]);
      if (ahead) issue_qk(i + 2);
      if (i + S < nsteps) issue(i + S);  // stage i % S is consumed
    }
  }
  if (nsteps > 0) mbar_wait(&bars[P::kBarPV], (nsteps - 1) & 1, sflag);
  tc_fence_after();

  // ---- epilogue: quantized partial of the CTA -> shared memory (stage area)
  float* qp = reinterpret_cast<float*>(smem);      // [GQ][kPartStride]
  float* wp = qp + GQ * kPartStride;               // [8][GQ][kPartStride]
  float* red = wp + 8 * GQ * kPartStride;          // [4][GQ * (1 + VPT)]
  if (token_warp) {
#pragma unroll
    for (int h = 0; h < GQ; ++h) {
      float l = l_run[h];
#pragma unroll
      for (int x = 16; x > 0; x >>= 1) l += __shfl_xor_sync(kAll, l, x);
      if (lane == 0) red[wq * GQ * (1 + VPT) + h] = l;
#pragma unroll
      for (int j = 0; j < VPT; ++j) {
        float z = zacc[h][j];
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) z += __shfl_xor_sync(kAll, z, x);
        if (lane == 0) red[wq * GQ * (1 + VPT) + GQ + h * VPT + j] = z;
      }
    }
    if (nsteps > 0) {
      // row = channel c; its value group j = c / G; O columns (j GQ + h) * 2 + {0, 1}
      float o[GQ];
#pragma unroll
      for (int h = 0; h < GQ; ++h) o[h] = 0.f;
#pragma unroll
      for (int c0 = 0; c0 < NC; c0 += 16) {
        uint32_t d[16];
        tmem_ld<16>(tmem + lane_base + P::kColO + c0, d);
        tc_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int n = c0 + c;
          if (n < NC && (n >> 1) / GQ == row / G) o[(n >> 1) % GQ] += __uint_as_float(d[c]);
        }
      }
#pragma unroll
      for (int h = 0; h < GQ; ++h) qp[h * kPartStride + kPartO + row] = o[h];
    }
  }
  // empty window partials
  for (int idx = tid; idx < 8 * GQ * kPartStride; idx += kThreads) {
    const int f = idx % kPartStride;
    wp[idx] = f == 0 ? -CUDART_INF_F : 0.f;
  }
  tc_fence_before();
  __syncthreads();
  for (int idx = tid; idx < GQ * kHeadDim; idx += kThreads) {
    const int h = idx >> 7, c = idx & 127;
    float z = 0.f, l = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      z += red[w * GQ * (1 + VPT) + GQ + h * VPT + c / G];
      l += red[w * GQ * (1 + VPT) + h];
    }
    float* ph = qp + h * kPartStride;
    ph[kPartO + c] = nsteps > 0 ? ph[kPartO + c] + z : 0.f;
    if (c == 0) {
      ph[0] = nsteps > 0 ? m_ref[h] : -CUDART_INF_F;
      ph[1] = nsteps > 0 ? l : 0.f;
    }
  }
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, P::kTmemCols);
  }

  // ---- FP16 window tokens [Q, T), spread over all splits of the unit: this CTA takes tokens
  //      Q + split + k * ns (ns = splits holding tokens), warp w the k = w (mod 8), in batches of 8
  //      with all loads issued first. Lane l holds channels 4l .. 4l + 3. With the sink on and Q > 0
  //      the list starts at Q - 1, which stands for the sink token's row R + G.
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
    float* cw = wp + warp * GQ * kPartStride;
    const uint2* kres = reinterpret_cast<const uint2*>(a.k_res + unit * a.res_rows * kHeadDim) + lane;
    const uint2* vres = reinterpret_cast<const uint2*>(a.v_res + unit * a.res_rows * kHeadDim) + lane;
    for (int k0 = warp; W0 + split + k0 * ns < T; k0 += 8 * 8) {
      uint2 kk[8], vv[8];
      bool valid[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int tt = W0 + split + (k0 + 8 * j) * ns;
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
          for (int x = 16; x > 0; x >>= 1) d += __shfl_xor_sync(kAll, d, x);
          sc[j] = valid[j] ? d : -CUDART_INF_F;
          mb = fmaxf(mb, sc[j]);
        }
        float* ph = cw + h * kPartStride;
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
        float4 cur = *reinterpret_cast<float4*>(ph + kPartO + 4 * lane);
        cur.x = fmaf(cur.x, f_old, o4[0]);
        cur.y = fmaf(cur.y, f_old, o4[1]);
        cur.z = fmaf(cur.z, f_old, o4[2]);
        cur.w = fmaf(cur.w, f_old, o4[3]);
        *reinterpret_cast<float4*>(ph + kPartO + 4 * lane) = cur;
        __syncwarp();
        if (lane == 0) {
          ph[0] = m_new;
          ph[1] = fmaf(ph[1], f_old, lb);
        }
        __syncwarp();
      }
    }
  }
  if (a.stall_test && tid == 0) mbar_wait(&bars[P::kBarPV], 0, sflag);  // gives up after about 2 s
  const bool gave_up = __syncthreads_or(*sflag != 0);

  // ---- CTA partial: merge the quantized partial and the 8 window partials -> workspace
  float* part = a.part + ((unit * a.nsplit + split) * gq) * kPartFloats;
  for (int idx = tid; idx < gq * kHeadDim; idx += kThreads) {
    const int h = idx >> 7, c = idx & 127;
    float M = qp[h * kPartStride];
#pragma unroll
    for (int w = 0; w < 8; ++w) M = fmaxf(M, wp[(w * GQ + h) * kPartStride]);
    // a split can hold no token at all: (m = -inf, l = 0, o = 0), weighed 0 by the combine
    const bool empty = M == -CUDART_INF_F;
    float f = empty ? 0.f : fast_exp2(qp[h * kPartStride] - M);
    float o = f * qp[h * kPartStride + kPartO + c];
    float l = f * qp[h * kPartStride + 1];
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      const float* pw = wp + (w * GQ + h) * kPartStride;
      f = empty ? 0.f : fast_exp2(pw[0] - M);
      o = fmaf(f, pw[kPartO + c], o);
      l = fmaf(f, pw[1], l);
    }
    part[h * kPartFloats + 2 + c] = o;
    if (c == 0) {
      part[h * kPartFloats] = M;
      part[h * kPartFloats + 1] = gave_up ? __int_as_float(0x7fc00000) : l;
    }
  }
}

template <int KB, int VB, int VPT, int GQ>
cudaError_t launch_tc(const DecodeArgs& a, cudaStream_t stream) {
  constexpr int smem = TcPlan<KB, VB, VPT, GQ>::kSmem;
  static DeviceMemo attr;
  const int ok = attr.get([] {
    return cudaFuncSetAttribute(decode_tc_kernel<KB, VB, VPT, GQ>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) == cudaSuccess ? 1 : -1;
  });
  if (ok < 0) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(a.nsplit), static_cast<unsigned>(static_cast<int64_t>(a.batch) * a.num_kv_heads));
  decode_tc_kernel<KB, VB, VPT, GQ><<<grid, kThreads, smem, stream>>>(a);
  return cudaGetLastError();
}

inline int gq_class_tc(int gqa) { return gqa <= 1 ? 1 : (gqa <= 2 ? 2 : 4); }

template <int KB, int VB, int VPT>
cudaError_t dispatch_tc_gq(const DecodeArgs& a, cudaStream_t s) {
  switch (gq_class_tc(a.gqa)) {
    case 1: return launch_tc<KB, VB, VPT, 1>(a, s);
    case 2: return launch_tc<KB, VB, VPT, 2>(a, s);
    default: return launch_tc<KB, VB, VPT, 4>(a, s);
  }
}

template <int KB, int VB>
cudaError_t dispatch_tc_vpt(const DecodeArgs& a, cudaStream_t s) {
  switch (a.G) {
    case 128: return dispatch_tc_gq<KB, VB, 1>(a, s);
    case 64: return dispatch_tc_gq<KB, VB, 2>(a, s);
    case 32: return dispatch_tc_gq<KB, VB, 4>(a, s);
    default: return dispatch_tc_gq<KB, VB, 8>(a, s);
  }
}

template <int KB, int VB, int VPT>
int ctas_tc_gq(int gqa) {
  switch (gq_class_tc(gqa)) {
    case 1: return TcPlan<KB, VB, VPT, 1>::kCtasPerSm;
    case 2: return TcPlan<KB, VB, VPT, 2>::kCtasPerSm;
    default: return TcPlan<KB, VB, VPT, 4>::kCtasPerSm;
  }
}

}  // namespace

int decode_tc_ctas_per_sm(int G, int gqa) {
  // TMEM columns depend on G and gqa only (bits do not enter the plan's column count)
  switch (G) {
    case 128: return ctas_tc_gq<2, 2, 1>(gqa);
    case 64: return ctas_tc_gq<2, 2, 2>(gqa);
    case 32: return ctas_tc_gq<2, 2, 4>(gqa);
    default: return ctas_tc_gq<2, 2, 8>(gqa);
  }
}

cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream) {
  if (a.key_bits == 2) return a.value_bits == 2 ? dispatch_tc_vpt<2, 2>(a, stream) : dispatch_tc_vpt<2, 4>(a, stream);
  return a.value_bits == 2 ? dispatch_tc_vpt<4, 2>(a, stream) : dispatch_tc_vpt<4, 4>(a, stream);
}

}  // namespace kvq
