// kvq_api.cu — host side of the libkvq C ABI: argument validation, split planning and launches.
// The entry points, their arguments and error behaviour are documented in include/kvq.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "kvq.h"
#include "kvq_common.cuh"
#include "kvq_internal.h"

using kvq::DecodeArgs;
using kvq::QuantizeArgs;

namespace {

constexpr int kMaxResidual = 4096;
constexpr int64_t kTargetCtas = 2048;  // split budget used to bound the decode workspace
constexpr int kSplitQuantum = 64;      // tile v1: split lengths are multiples of 4 warps x 16-token tiles
constexpr int kSplitQuantumTc = 128;   // rows v2: whole 128-token steps

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

kvq_status check_config(const kvq_config* c) {
  if (c == nullptr) return KVQ_ERR_INVALID_ARG;
  if (c->layout != KVQ_LAYOUT_TILE_V1 && c->layout != KVQ_LAYOUT_ROWS_V2) return KVQ_ERR_UNSUPPORTED;
  if (c->head_dim != 128) return KVQ_ERR_UNSUPPORTED;
  if (c->batch < 1 || c->num_kv_heads < 1 || c->num_q_heads < 1) return KVQ_ERR_INVALID_ARG;
  if (c->num_q_heads % c->num_kv_heads != 0) return KVQ_ERR_INVALID_ARG;
  if (c->num_q_heads / c->num_kv_heads > 4) return KVQ_ERR_UNSUPPORTED;
  if ((c->key_bits != 2 && c->key_bits != 4) || (c->value_bits != 2 && c->value_bits != 4)) return KVQ_ERR_INVALID_ARG;
  const int G = c->group_size;
  if (G != 16 && G != 32 && G != 64 && G != 128) return KVQ_ERR_INVALID_ARG;
  if (c->residual < 0 || c->residual > kMaxResidual) return KVQ_ERR_INVALID_ARG;
  if (c->hadamard != 0 && c->hadamard != 1) return KVQ_ERR_INVALID_ARG;
  if (c->sink != 0 && c->sink != 1) return KVQ_ERR_INVALID_ARG;
  if (!(c->rope_theta >= 0.f) || !std::isfinite(c->rope_theta)) return KVQ_ERR_INVALID_ARG;
  if (c->rope_theta > 0.f && c->hadamard) return KVQ_ERR_INVALID_ARG;                 // the two exclude each other
  if (c->rope_theta > 0.f && c->layout != KVQ_LAYOUT_ROWS_V2) return KVQ_ERR_UNSUPPORTED;  // token-row keys only
  if (c->outliers != 0 && c->outliers != 1) return KVQ_ERR_INVALID_ARG;
  if (c->outliers && (c->layout != KVQ_LAYOUT_TILE_V1 || c->rope_theta > 0.f)) return KVQ_ERR_UNSUPPORTED;
  if (c->page_tokens < 0) return KVQ_ERR_INVALID_ARG;
  if (c->page_tokens > 0) {
    if (c->page_tokens % 128 != 0 || c->capacity % c->page_tokens != 0 || c->num_pages < 1) return KVQ_ERR_INVALID_ARG;
    if (c->layout != KVQ_LAYOUT_TILE_V1 || c->rope_theta > 0.f) return KVQ_ERR_UNSUPPORTED;
  }
  if (c->capacity < 0 || c->capacity % G != 0) return KVQ_ERR_INVALID_ARG;
  if (c->capacity >= (int64_t(1) << 31)) return KVQ_ERR_INVALID_ARG;  // token indices are 32-bit on the device
  if (c->layout == KVQ_LAYOUT_ROWS_V2 && c->capacity % 128 != 0) return KVQ_ERR_INVALID_ARG;  // whole value blocks
  if (static_cast<int64_t>(c->batch) * c->num_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;  // grid.y
  return KVQ_OK;
}

// Storage slots of the per-token buffers and tokens per slot: one slot of capacity tokens per unit,
// or (paged) one slot of page_tokens tokens per pool page.
size_t storage_slots(const kvq_config* c) {
  return c->page_tokens > 0 ? static_cast<size_t>(c->num_pages) : static_cast<size_t>(c->batch) * c->num_kv_heads;
}
int64_t slot_tokens(const kvq_config* c) { return c->page_tokens > 0 ? c->page_tokens : c->capacity; }

void buffer_bytes(const kvq_config* c, size_t out[KVQ_NUM_BUFFERS]) {
  const size_t units = static_cast<size_t>(c->batch) * c->num_kv_heads;
  const size_t slots = storage_slots(c);
  const size_t cap = static_cast<size_t>(slot_tokens(c));
  const size_t G = static_cast<size_t>(c->group_size);
  out[KVQ_BUF_K_CODES] = slots * (cap / 16) * 64 * c->key_bits * 4;
  const size_t vcap = c->layout == KVQ_LAYOUT_ROWS_V2 ? (cap + 127) / 128 * 128 : cap;
  out[KVQ_BUF_V_CODES] = slots * (vcap / 16) * 64 * c->value_bits * 4;
  out[KVQ_BUF_K_SCALE] = slots * (cap / G) * 128 * 2;
  out[KVQ_BUF_K_ZERO] = out[KVQ_BUF_K_SCALE];
  out[KVQ_BUF_V_SCALE] = slots * cap * (128 / G) * 2;
  out[KVQ_BUF_V_ZERO] = out[KVQ_BUF_V_SCALE];
  out[KVQ_BUF_K_RES] = units * (static_cast<size_t>(c->residual) + G + c->sink) * 128 * 2;
  out[KVQ_BUF_V_RES] = out[KVQ_BUF_K_RES];
}

kvq_status check_cache(const kvq_config* c, const kvq_cache* k) {
  if (k == nullptr || k->seq_len_host == nullptr || k->seq_len_dev == nullptr) return KVQ_ERR_INVALID_ARG;
  size_t sz[KVQ_NUM_BUFFERS];
  buffer_bytes(c, sz);
  const void* p[KVQ_NUM_BUFFERS] = {k->k_codes, k->v_codes, k->k_scale, k->k_zero, k->v_scale, k->v_zero, k->k_res, k->v_res};
  for (int i = 0; i < KVQ_NUM_BUFFERS; ++i) {
    if (sz[i] == 0) continue;
    if (p[i] == nullptr || !aligned(p[i], 16)) return KVQ_ERR_INVALID_ARG;
  }
  if (!aligned(k->seq_len_dev, 8)) return KVQ_ERR_INVALID_ARG;
  if (c->outliers && (k->k_out == nullptr || k->v_out == nullptr || !aligned(k->k_out, 16) || !aligned(k->v_out, 16)))
    return KVQ_ERR_INVALID_ARG;
  if (c->page_tokens > 0 && (k->page_table_host == nullptr || k->page_table_dev == nullptr || !aligned(k->page_table_dev, 16)))
    return KVQ_ERR_INVALID_ARG;
  return KVQ_OK;
}

int64_t pages_per_unit(const kvq_config* c) { return c->page_tokens > 0 ? c->capacity / c->page_tokens : 0; }

// Paged storage: every page that holds quantized tokens of a sequence of lens[b] tokens must map to a
// page of the pool (the kernels read exactly those table entries).
kvq_status check_pages(const kvq_config* c, const kvq_cache* k, const int64_t* lens) {
  if (c->page_tokens <= 0) return KVQ_OK;
  const int64_t M = pages_per_unit(c);
  for (int b = 0; b < c->batch; ++b) {
    const int64_t Q = kvq::quantized_len(lens[b], c->residual, c->group_size);
    const int64_t used = (Q + c->page_tokens - 1) / c->page_tokens;
    for (int h = 0; h < c->num_kv_heads; ++h) {
      const int32_t* row = k->page_table_host + (static_cast<int64_t>(b) * c->num_kv_heads + h) * M;
      for (int64_t j = 0; j < used; ++j)
        if (row[j] < 0 || row[j] >= c->num_pages) return KVQ_ERR_INVALID_ARG;
    }
  }
  return KVQ_OK;
}

// Copy the whole page table to its device mirror on the stream.
cudaError_t upload_pages(const kvq_config* c, const kvq_cache* k, cudaStream_t stream) {
  const size_t bytes = static_cast<size_t>(c->batch) * c->num_kv_heads * pages_per_unit(c) * sizeof(int32_t);
  return cudaMemcpyAsync(k->page_table_dev, k->page_table_host, bytes, cudaMemcpyHostToDevice, stream);
}

QuantizeArgs quantize_args(const kvq_config* c, kvq_cache* k) {
  QuantizeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.seq_len = k->seq_len_dev;
  a.k_codes = static_cast<uint32_t*>(k->k_codes);
  a.v_codes = static_cast<uint32_t*>(k->v_codes);
  a.k_scale = static_cast<uint16_t*>(k->k_scale);
  a.k_zero = static_cast<uint16_t*>(k->k_zero);
  a.v_scale = static_cast<uint16_t*>(k->v_scale);
  a.v_zero = static_cast<uint16_t*>(k->v_zero);
  a.k_res = static_cast<uint16_t*>(k->k_res);
  a.v_res = static_cast<uint16_t*>(k->v_res);
  a.batch = c->batch;
  a.num_kv_heads = c->num_kv_heads;
  a.G = c->group_size;
  a.R = c->residual;
  a.key_bits = c->key_bits;
  a.value_bits = c->value_bits;
  a.hadamard = c->hadamard;
  a.capacity = c->capacity;
  a.slot_tokens = slot_tokens(c);
  a.tiles = a.slot_tokens / kvq::kTile;
  a.groups = a.slot_tokens / c->group_size;
  a.ring = static_cast<int64_t>(c->residual) + c->group_size;
  a.layout = c->layout;
  a.page_tokens = c->page_tokens;
  a.pages_per_unit = pages_per_unit(c);
  a.page_table = k->page_table_dev;
  a.sink = c->sink;
  a.res_rows = a.ring + c->sink;
  a.outliers = c->outliers;
  a.k_out = static_cast<uint32_t*>(k->k_out);
  a.v_out = static_cast<uint32_t*>(k->v_out);
  a.vwords = (c->layout == KVQ_LAYOUT_ROWS_V2 ? (a.slot_tokens + 127) / 128 * 128 : a.slot_tokens) * 4 * c->value_bits;
  return a;
}

int64_t max_splits(const kvq_config* c);

// Decode workspace: split partials, then (pre-RoPE keys) the angle tables, then one status record per
// (sequence, query head); each part starts 256-byte aligned.
struct WorkspaceLayout {
  size_t rope, status, total;
};
WorkspaceLayout workspace_layout(const kvq_config* c) {
  const int64_t units = static_cast<int64_t>(c->batch) * c->num_kv_heads;
  const int64_t g = c->num_q_heads / c->num_kv_heads;
  const size_t part = static_cast<size_t>(units * max_splits(c) * g * kvq::kPartFloats) * sizeof(float);
  WorkspaceLayout w;
  w.rope = (part + 255) / 256 * 256;
  size_t end = part;
  if (c->rope_theta > 0.f) end = w.rope + static_cast<size_t>(kvq::rope_table_floats(c->capacity)) * 4;
  w.status = (end + 255) / 256 * 256;
  w.total = w.status + static_cast<size_t>(c->batch) * c->num_q_heads * 4;
  return w;
}

int64_t max_splits(const kvq_config* c) {
  const int64_t units = static_cast<int64_t>(c->batch) * c->num_kv_heads;
  return std::max<int64_t>(1, (2 * kTargetCtas + units - 1) / units);
}

// Choose the split length: among n = 1 .. max_splits splits of the longest sequence, minimise
// (waves of CTAs) x (tokens per CTA + a fixed per-CTA overhead), counting only CTAs that hold
// tokens. Returns the split length; *nsplit = ceil(Tmax / L).
int plan_splits(const kvq_config* c, const int64_t* lens, int slots, int* nsplit) {
  int64_t tmax = 0;
  for (int b = 0; b < c->batch; ++b) tmax = std::max(tmax, lens[b]);
  const bool tc = c->layout == KVQ_LAYOUT_ROWS_V2;
  const int64_t quantum = tc ? kSplitQuantumTc : kSplitQuantum;
  if (tmax <= 0) {
    *nsplit = 1;
    return static_cast<int>(quantum);
  }
  const int64_t smax = max_splits(c);
  const int64_t nmin = 1;
  const double overhead = 256.0;  // tokens' worth of per-CTA fixed cost (query prep, partial write)
  double best = 1e300;
  int64_t best_L = 0;
  for (int64_t n = nmin; n <= smax; ++n) {
    int64_t L = (tmax + n - 1) / n;
    L = (L + quantum - 1) / quantum * quantum;
    if (n > nmin && L == best_L) continue;
    int64_t ctas = 0;
    for (int b = 0; b < c->batch; ++b) ctas += (lens[b] + L - 1) / L;
    ctas *= c->num_kv_heads;
    const double waves = std::ceil(static_cast<double>(ctas) / slots);
    const double cost = waves * (static_cast<double>(L) + overhead);
    if (cost < best) {
      best = cost;
      best_L = L;
    }
  }
  *nsplit = static_cast<int>((tmax + best_L - 1) / best_L);
  return static_cast<int>(best_L);
}

kvq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KVQ_OK : KVQ_ERR_CUDA; }

}  // namespace

extern "C" {

kvq_status kvq_cache_buffer_bytes(const kvq_config* cfg, size_t out_bytes[KVQ_NUM_BUFFERS]) {
  const kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if (out_bytes == nullptr) return KVQ_ERR_INVALID_ARG;
  buffer_bytes(cfg, out_bytes);
  return KVQ_OK;
}

kvq_status kvq_outlier_buffer_bytes(const kvq_config* cfg, size_t out_bytes[2]) {
  const kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if (out_bytes == nullptr) return KVQ_ERR_INVALID_ARG;
  const size_t n = cfg->outliers ? storage_slots(cfg) * static_cast<size_t>(slot_tokens(cfg)) * 4 : 0;
  out_bytes[0] = out_bytes[1] = n;
  return KVQ_OK;
}

kvq_status kvq_quantize_prefill(const kvq_config* cfg, kvq_cache* cache, const void* k, const void* v, int64_t stride_b,
                                int64_t stride_t, int64_t stride_h, const int64_t* seq_lens, void* cuda_stream) {
  kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if ((s = check_cache(cfg, cache)) != KVQ_OK) return s;
  if (seq_lens == nullptr) return KVQ_ERR_INVALID_ARG;
  int64_t tmax = 0;
  for (int b = 0; b < cfg->batch; ++b) {
    if (seq_lens[b] < 0 || seq_lens[b] > cfg->capacity) return KVQ_ERR_CAPACITY;
    tmax = std::max(tmax, seq_lens[b]);
  }
  if (tmax > 0) {
    if (k == nullptr || v == nullptr || !aligned(k, 16) || !aligned(v, 16)) return KVQ_ERR_INVALID_ARG;
    if (stride_b < 0 || stride_t < 0 || stride_h < 0 || stride_b % 8 || stride_t % 8 || stride_h % 8) return KVQ_ERR_INVALID_ARG;
  }
  if ((s = check_pages(cfg, cache, seq_lens)) != KVQ_OK) return s;
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  std::memcpy(cache->seq_len_host, seq_lens, sizeof(int64_t) * cfg->batch);
  // The lengths reach the device by value (kernel arguments), never by a queued copy of host memory
  // that a later call rewrites.
  if (kvq::launch_set_lengths(static_cast<int64_t*>(cache->seq_len_dev), cache->seq_len_host, cfg->batch, stream) !=
      cudaSuccess)
    return KVQ_ERR_CUDA;
  if (cfg->page_tokens > 0 && upload_pages(cfg, cache, stream) != cudaSuccess) return KVQ_ERR_CUDA;
  QuantizeArgs a = quantize_args(cfg, cache);
  a.k = static_cast<const uint16_t*>(k);
  a.v = static_cast<const uint16_t*>(v);
  a.stride_b = stride_b;
  a.stride_t = stride_t;
  a.stride_h = stride_h;
  return cuda_status(kvq::launch_prefill(a, cache->seq_len_host, stream));
}

kvq_status kvq_append_token(const kvq_config* cfg, kvq_cache* cache, const void* k_new, const void* v_new,
                            void* cuda_stream) {
  kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if ((s = check_cache(cfg, cache)) != KVQ_OK) return s;
  if (k_new == nullptr || v_new == nullptr || !aligned(k_new, 16) || !aligned(v_new, 16)) return KVQ_ERR_INVALID_ARG;
  for (int b = 0; b < cfg->batch; ++b)
    if (cache->seq_len_host[b] < 0 || cache->seq_len_host[b] + 1 > cfg->capacity) return KVQ_ERR_CAPACITY;
  if (cfg->page_tokens > 0) {
    // The flush of this append may enter a new page: check the table for the new lengths and, if
    // some unit's quantized part reaches a page it did not reach before, refresh the device mirror.
    std::vector<int64_t> next(cache->seq_len_host, cache->seq_len_host + cfg->batch);
    bool enters = false;
    for (int b = 0; b < cfg->batch; ++b) {
      const int64_t q0 = kvq::quantized_len(next[b], cfg->residual, cfg->group_size);
      const int64_t q1 = kvq::quantized_len(next[b] + 1, cfg->residual, cfg->group_size);
      enters |= (q1 + cfg->page_tokens - 1) / cfg->page_tokens > (q0 + cfg->page_tokens - 1) / cfg->page_tokens;
      next[b] += 1;
    }
    if ((s = check_pages(cfg, cache, next.data())) != KVQ_OK) return s;
    if (enters && upload_pages(cfg, cache, static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return KVQ_ERR_CUDA;
  }
  QuantizeArgs a = quantize_args(cfg, cache);
  const kvq_status r = cuda_status(kvq::launch_append(a, cache->seq_len_host, static_cast<const uint16_t*>(k_new),
                                                      static_cast<const uint16_t*>(v_new),
                                                      static_cast<cudaStream_t>(cuda_stream)));
  if (r == KVQ_OK)
    for (int b = 0; b < cfg->batch; ++b) cache->seq_len_host[b] += 1;
  return r;
}

kvq_status kvq_decode_workspace_bytes(const kvq_config* cfg, size_t* bytes) {
  const kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if (bytes == nullptr) return KVQ_ERR_INVALID_ARG;
  *bytes = workspace_layout(cfg).total;
  return KVQ_OK;
}

kvq_status kvq_decode_status(const kvq_config* cfg, const void* workspace, void* cuda_stream) {
  const kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if (workspace == nullptr || !aligned(workspace, 256)) return KVQ_ERR_INVALID_ARG;
  const WorkspaceLayout w = workspace_layout(cfg);
  const uint32_t* rec = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(workspace) + w.status);
  cudaStream_t stream = static_cast<cudaStream_t>(cuda_stream);
  const int64_t n = static_cast<int64_t>(cfg->batch) * cfg->num_q_heads;
  uint32_t buf[1024];  // the records, a chunk at a time (no host allocation)
  bool gave_up = false;
  for (int64_t i = 0; i < n; i += 1024) {
    const int64_t m = std::min<int64_t>(1024, n - i);
    if (cudaMemcpyAsync(buf, rec + i, static_cast<size_t>(m) * 4, cudaMemcpyDeviceToHost, stream) != cudaSuccess ||
        cudaStreamSynchronize(stream) != cudaSuccess)
      return KVQ_ERR_CUDA;
    for (int64_t j = 0; j < m; ++j) gave_up |= buf[j] != 0;
  }
  return gave_up ? KVQ_ERR_TIMEOUT : KVQ_OK;
}

kvq_status kvq_decode_attention(const kvq_config* cfg, const kvq_cache* cache, const void* q, void* out, float sm_scale,
                                void* workspace, size_t workspace_bytes, void* cuda_stream) {
  kvq_status s = check_config(cfg);
  if (s != KVQ_OK) return s;
  if ((s = check_cache(cfg, cache)) != KVQ_OK) return s;
  if (q == nullptr || out == nullptr || !aligned(q, 16) || !aligned(out, 16)) return KVQ_ERR_INVALID_ARG;
  if (!(sm_scale > 0.f) || !std::isfinite(sm_scale)) return KVQ_ERR_INVALID_ARG;
  size_t need = 0;
  kvq_decode_workspace_bytes(cfg, &need);
  if (workspace == nullptr || workspace_bytes < need || !aligned(workspace, 256)) return KVQ_ERR_WORKSPACE;
  for (int b = 0; b < cfg->batch; ++b)
    if (cache->seq_len_host[b] < 0 || cache->seq_len_host[b] > cfg->capacity) return KVQ_ERR_INVALID_ARG;
  if ((s = check_pages(cfg, cache, cache->seq_len_host)) != KVQ_OK) return s;

  static kvq::DeviceMemo sm_count;
  const int sms = sm_count.get([] {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
    return n;
  });
  if (sms <= 0) return KVQ_ERR_CUDA;
  const int gqa = cfg->num_q_heads / cfg->num_kv_heads;
  const int occ = cfg->rope_theta > 0.f ? kvq::decode_rope_ctas_per_sm(cfg->key_bits, cfg->value_bits, cfg->group_size, gqa)
                  : kvq::cuda_core_control_requested(cfg->layout, cfg->rope_theta, cfg->hadamard)
                      ? kvq::decode_cuda_cores_ctas_per_sm(cfg->key_bits, cfg->value_bits, cfg->group_size, gqa)
                  : cfg->layout == KVQ_LAYOUT_ROWS_V2
                      ? kvq::decode_tc_ctas_per_sm(cfg->group_size, cfg->num_q_heads / cfg->num_kv_heads)
                      : kvq::decode_ctas_per_sm(cfg->key_bits, cfg->value_bits, cfg->group_size,
                                                cfg->num_q_heads / cfg->num_kv_heads, cfg->outliers);
  int nsplit = 1;
  const int L = plan_splits(cfg, cache->seq_len_host, sms * occ, &nsplit);

  DecodeArgs a;
  std::memset(&a, 0, sizeof(a));
  a.k_codes = static_cast<const uint32_t*>(cache->k_codes);
  a.v_codes = static_cast<const uint32_t*>(cache->v_codes);
  a.k_scale = static_cast<const uint16_t*>(cache->k_scale);
  a.k_zero = static_cast<const uint16_t*>(cache->k_zero);
  a.v_scale = static_cast<const uint16_t*>(cache->v_scale);
  a.v_zero = static_cast<const uint16_t*>(cache->v_zero);
  a.k_res = static_cast<const uint16_t*>(cache->k_res);
  a.v_res = static_cast<const uint16_t*>(cache->v_res);
  a.seq_len = cache->seq_len_dev;
  a.q = static_cast<const uint16_t*>(q);
  a.out = static_cast<uint16_t*>(out);
  a.part = static_cast<float*>(workspace);
  a.batch = cfg->batch;
  a.num_q_heads = cfg->num_q_heads;
  a.num_kv_heads = cfg->num_kv_heads;
  a.gqa = cfg->num_q_heads / cfg->num_kv_heads;
  a.G = cfg->group_size;
  a.R = cfg->residual;
  a.key_bits = cfg->key_bits;
  a.value_bits = cfg->value_bits;
  a.hadamard = cfg->hadamard;
  a.capacity = cfg->capacity;
  a.slot_tokens = slot_tokens(cfg);
  a.tiles = a.slot_tokens / kvq::kTile;
  a.groups = a.slot_tokens / cfg->group_size;
  a.page_tokens = cfg->page_tokens;
  a.pages_per_unit = pages_per_unit(cfg);
  a.page_table = cache->page_table_dev;
  a.ring = static_cast<int64_t>(cfg->residual) + cfg->group_size;
  a.sink = cfg->sink;
  a.res_rows = a.ring + cfg->sink;
  a.outliers = cfg->outliers;
  a.k_out = static_cast<const uint32_t*>(cache->k_out);
  a.v_out = static_cast<const uint32_t*>(cache->v_out);
  a.layout = cfg->layout;
  a.split_len = L;
  a.nsplit = nsplit;
  a.qscale = static_cast<float>(static_cast<double>(sm_scale) * 1.4426950408889634);
  const WorkspaceLayout wl = workspace_layout(cfg);
  a.status = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + wl.status);
  a.stall_test = kvq::stall_test_requested() ? 1 : 0;
  if (cfg->rope_theta > 0.f) {
    a.rope_theta = cfg->rope_theta;
    a.rope_base = reinterpret_cast<float2*>(static_cast<uint8_t*>(workspace) + wl.rope);
    a.rope_off = a.rope_base + (cfg->capacity + 31) / 32 * 64;
  }
  return cuda_status(kvq::launch_decode(a, static_cast<cudaStream_t>(cuda_stream)));
}

const char* kvq_status_string(kvq_status status) {
  switch (status) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID_ARG: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_CAPACITY: return "sequence would exceed the cache capacity";
    case KVQ_ERR_WORKSPACE: return "decode workspace missing, misaligned or too small";
    case KVQ_ERR_CUDA: return "CUDA launch or copy failed";
    case KVQ_ERR_TIMEOUT: return "a decode kernel gave up a bounded wait (its outputs are NaN)";
  }
  return "unknown status";
}

}  // extern "C"
