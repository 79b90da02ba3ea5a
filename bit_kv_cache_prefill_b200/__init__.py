"""B200-native asymmetric low-bit KV cache: quantize/pack, streaming append and decode attention.

The compute lives in ``libkvq.so`` (CUDA for sm_100a, C ABI in ``include/kvq.h``); ``_lib`` is a thin
ctypes binding with the same entry-point names. The binding is loaded on first use of any of its
names, and that first use raises ImportError if the library has not been built
(``python -m bit_kv_cache_prefill_b200.build``): there is no fallback implementation.
"""
_BINDING_NAMES = {
    "BUFFER_NAMES", "Cache", "KvqError", "KVQ_ERR_CAPACITY", "KVQ_ERR_CUDA", "KVQ_ERR_INVALID_ARG",
    "KVQ_ERR_UNSUPPORTED", "KVQ_ERR_WORKSPACE", "KVQ_OK", "LIB_PATH", "kvq_append_token", "kvq_cache",
    "kvq_cache_buffer_bytes", "kvq_config", "kvq_decode_attention", "kvq_decode_workspace_bytes",
    "kvq_quantize_prefill", "kvq_status_string", "make_config", "kvq_decode_attention_noalloc",
    "STATIC_SCRATCH_BYTES", "KVQ_LAYOUT_TILE_V1", "KVQ_LAYOUT_ROWS_V2", "kvq_outlier_buffer_bytes",
    "KVQ_ERR_TIMEOUT", "kvq_decode_status",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import _lib

        return getattr(_lib, name)
    raise AttributeError(name)
