// kvq_static.cu — decode attention for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: a plugin or extension running inside a host framework that
// owns every device allocation through its own pool (a raw cudaMalloc would bypass, fragment or
// exceed that pool), or a latency-critical serving loop whose policy forbids allocation after
// start-up. kvq_decode_attention needs a caller-provided workspace for its split partials; this file
// provides the same computation with that scratch memory held in a fixed file-scope device array
// instead, so such a caller only passes its inputs and outputs.
//
// The array is part of the library's device image: every GPU that loads the library holds
// KVQ_STATIC_SCRATCH_BYTES for it until the process exits. All calls share it, so calls whose GPU
// work overlaps (for instance on two streams at once) race on it and must be serialised by the
// caller. Nothing in it needs to start at zero: every split partial the combine step reads is
// written earlier in the same call.
#include <cuda_runtime.h>

#include <mutex>

#include "kvq.h"

namespace {

constexpr size_t kScratchBytes = static_cast<size_t>(KVQ_STATIC_SCRATCH_BYTES);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_setup_mutex;
void* g_scratch_ptr[kMaxDevices] = {};  // device address of g_decode_scratch, per device

// Set-up, once per device, with that device current: look up the array's device address. In host
// code the symbol names a host-side stand-in, never the device memory itself.
kvq_status scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return KVQ_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return KVQ_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  if (g_scratch_ptr[dev] == nullptr) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_decode_scratch) != cudaSuccess || ptr == nullptr) return KVQ_ERR_CUDA;
    g_scratch_ptr[dev] = ptr;
  }
  *out = g_scratch_ptr[dev];
  return KVQ_OK;
}

}  // namespace

extern "C" kvq_status kvq_decode_attention_noalloc(const kvq_config* cfg, const kvq_cache* cache, const void* q,
                                                   void* out, float sm_scale, void* cuda_stream) {
  size_t need = 0;
  const kvq_status s = kvq_decode_workspace_bytes(cfg, &need);
  if (s != KVQ_OK) return s;
  if (need > kScratchBytes) return KVQ_ERR_WORKSPACE;  // config needs more than the fixed scratch
  void* scratch = nullptr;
  const kvq_status r = scratch_for_current_device(&scratch);
  if (r != KVQ_OK) return r;
  return kvq_decode_attention(cfg, cache, q, out, sm_scale, scratch, kScratchBytes, cuda_stream);
}
