// kvq_internal.h — argument blocks passed from the C-ABI host code to the kernels (not installed).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace kvq {

struct QuantizeArgs {
  const uint16_t* k;  // prefill input fp16 [b][t][h][d] (strided); unused by append
  const uint16_t* v;
  int64_t stride_b, stride_t, stride_h;
  int64_t* seq_len;  // device mirror [batch]
  uint32_t* k_codes;
  uint32_t* v_codes;
  uint16_t* k_scale;
  uint16_t* k_zero;
  uint16_t* v_scale;
  uint16_t* v_zero;
  uint16_t* k_res;
  uint16_t* v_res;
  int batch, num_kv_heads, G, R, key_bits, value_bits, hadamard;
  int64_t capacity, tiles, groups, ring;  // per unit: capacity tokens, capacity/16 tiles, capacity/G groups, R+G slots
  int layout;                             // KVQ_LAYOUT_TILE_V1 or KVQ_LAYOUT_ROWS_V2
  int64_t vwords;                         // value code words per unit
  int sink;                               // 1: token 0 stays in fp16 in ring row R+G
  int64_t res_rows;                       // rows of k_res / v_res per unit: R + G + sink
  int outliers;                           // 1: each quantized token's largest entry stays fp16
  uint32_t* k_out;                        // [slots][slot_tokens]: channel | fp16 value << 16 (0xffff: none)
  uint32_t* v_out;
  // Storage slots: one per unit (contiguous) or one per pool page (paged). tiles, groups and vwords
  // above count per slot; token t of a unit lives in slot page_table[unit][t / page_tokens] at
  // t mod page_tokens (paged), else in slot `unit` at t.
  int64_t slot_tokens;                    // capacity, or page_tokens when paged
  int page_tokens;                        // 0: contiguous
  int64_t pages_per_unit;                 // capacity / page_tokens
  const int32_t* page_table;              // device [units][pages_per_unit]
};

struct DecodeArgs {
  const uint32_t* k_codes;
  const uint32_t* v_codes;
  const uint16_t* k_scale;
  const uint16_t* k_zero;
  const uint16_t* v_scale;
  const uint16_t* v_zero;
  const uint16_t* k_res;
  const uint16_t* v_res;
  const int64_t* seq_len;  // device mirror [batch]
  const uint16_t* q;       // fp16 [batch][Hq][128]
  uint16_t* out;           // fp16 [batch][Hq][128]
  float* part;             // split partials [units][nsplit][g][2 + 128]
  uint32_t* status;        // [batch][Hq]: 1 where the output is NaN from a bounded wait that gave up
  int batch, num_q_heads, num_kv_heads, gqa, G, R, key_bits, value_bits, hadamard;
  int64_t capacity, tiles, groups, ring;
  int sink;          // 1: token 0 is read from ring row R+G (fp16) and masked in the quantized part
  int64_t res_rows;  // rows of k_res / v_res per unit: R + G + sink
  int outliers;             // 1: add each quantized token's fp16 key / value outlier (tile v1 only)
  const uint32_t* k_out;    // [slots][slot_tokens]: channel | fp16 value << 16 (0xffff: none)
  const uint32_t* v_out;
  int64_t slot_tokens;      // storage slot extent (tiles, groups count per slot): capacity, or page_tokens
  int page_tokens;          // 0: contiguous; else token t of a unit lives in slot page_table[unit][t / page_tokens]
  int64_t pages_per_unit;
  const int32_t* page_table;  // device [units][pages_per_unit]
  int layout;     // KVQ_LAYOUT_TILE_V1 or KVQ_LAYOUT_ROWS_V2
  int split_len;  // tokens per split (multiple of 64; rows v2: multiple of 128)
  int nsplit;     // splits per unit in the grid
  float qscale;   // sm_scale * log2(e): scores are kept in base-2 units
  float rope_theta;  // > 0: keys are cached before RoPE; decode rotates them (rows v2 only)
  float2* rope_base;  // workspace: (cos, sin)(32 s w_i), [ceil(capacity / 32)][64]
  float2* rope_off;   // workspace: (cos, sin)(j w_i), [32][64]
  int stall_test;     // 1: the tcgen05 kernel runs no quantized step and waits on a barrier that nothing
                      // completes, so its bounded wait gives up (a test of the give-up path; KVQ_TEST_STALL_TC=1)
};

// Sequence lengths of up to kLenChunk consecutive sequences [base, base + n), passed to a kernel by
// value. The host never hands the device a pointer to its length array: a queued copy from caller
// memory that the library rewrites on the next call could otherwise read the later value.
constexpr int kLenChunk = 256;
struct LenChunk {
  int64_t base;
  int32_t n;
  int32_t pad;
  int64_t len[kLenChunk];
};

// The 128-token blocks of up to kLenChunk consecutive sequences [b0, b0 + n), numbered in sequence
// order: sequence b0 + i owns blocks cum[i] .. cum[i + 1] - 1. Passed by value to a prefill launch
// whose grid enumerates only the blocks that exist (ragged batches); n = 0 selects the plain grid.
struct BlockMap {
  int32_t b0;
  int32_t n;
  int32_t cum[kLenChunk + 1];
};

// Write lens[0 .. batch) into the device mirror (one small launch per kLenChunk sequences).
cudaError_t launch_set_lengths(int64_t* seq_len_dev, const int64_t* lens, int batch, cudaStream_t stream);
cudaError_t launch_prefill(const QuantizeArgs& a, const int64_t* lens, cudaStream_t stream);  // lens: host [batch]
// Append one token to every sequence; old_lens[b] is sequence b's length before the append (the host
// mirror). The launch also writes the new lengths into the device mirror.
cudaError_t launch_append(const QuantizeArgs& a, const int64_t* old_lens, const uint16_t* k_new, const uint16_t* v_new,
                          cudaStream_t stream);
cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);     // split + combine, either layout
cudaError_t launch_decode_tc(const DecodeArgs& a, cudaStream_t stream);  // rows-v2 split kernel only
cudaError_t launch_decode_rope(const DecodeArgs& a, cudaStream_t stream);  // pre-RoPE keys: tables + split kernel
int decode_rope_ctas_per_sm(int key_bits, int value_bits, int G, int gqa);  // pre-RoPE kernel
// The CUDA-core control: the pre-RoPE kernel without its rotations, on a rows-v2 cache without
// rotations (rope_theta = 0, hadamard = 0), for measuring the tensor-core kernels' gain. It runs in
// place of the tcgen05 kernel when the environment sets KVQ_DECODE_CUDA_CORES=1.
cudaError_t launch_decode_cuda_cores(const DecodeArgs& a, cudaStream_t stream);
int decode_cuda_cores_ctas_per_sm(int key_bits, int value_bits, int G, int gqa);
bool cuda_core_control_requested(int layout, float rope_theta, int hadamard);
// KVQ_TEST_STALL_TC=1: the tcgen05 decode gives up a bounded wait on purpose (no copy or MMA in flight).
bool stall_test_requested();
int64_t rope_table_floats(int64_t capacity);  // floats of the two RoPE tables in the workspace
int decode_ctas_per_sm(int key_bits, int value_bits, int G, int gqa, int outliers);  // tile-v1 kernel
int decode_tc_ctas_per_sm(int G, int gqa);                              // rows-v2 kernel (1 or 2)

// Per-device memo of a small non-negative value (a function attribute already set, an occupancy, an
// SM count), so that the launch path does not repeat runtime queries on every call. Concurrent first
// calls may both compute the value; they store the same result.
constexpr int kMaxDevices = 64;
struct DeviceMemo {
  std::atomic<int> v[kMaxDevices];
  DeviceMemo() {
    for (auto& x : v) x.store(-1, std::memory_order_relaxed);
  }
  // Value for the current device, computing it with fn() (returning < 0 on failure) the first time.
  template <typename F>
  int get(F&& fn) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return fn();
    int x = v[dev].load(std::memory_order_acquire);
    if (x >= 0) return x;
    x = fn();
    if (x >= 0) v[dev].store(x, std::memory_order_release);
    return x;
  }
};

constexpr int kDecodeWarps = 4;
constexpr int kPartFloats = 2 + 128;  // m, l, o[128]

}  // namespace kvq
