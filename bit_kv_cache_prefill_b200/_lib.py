"""ctypes binding of libkvq (include/kvq.h): argument marshalling only.

Every step of the computation runs in the CUDA library; this module converts torch tensors and
Python ints into the C structs and pointers the C ABI takes, and raises ``KvqError`` on a non-OK
status. If ``libkvq.so`` is missing the import fails loudly: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from typing import List, Optional, Sequence

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libkvq.so")

KVQ_OK = 0
KVQ_ERR_INVALID_ARG = -1
KVQ_ERR_UNSUPPORTED = -2
KVQ_ERR_CAPACITY = -3
KVQ_ERR_WORKSPACE = -4
KVQ_ERR_CUDA = -5
KVQ_ERR_TIMEOUT = -6
KVQ_LAYOUT_TILE_V1 = 1
KVQ_LAYOUT_ROWS_V2 = 2
BUFFER_NAMES = ("k_codes", "v_codes", "k_scale", "k_zero", "v_scale", "v_zero", "k_res", "v_res")


class KvqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {kvq_status_string(status)} (status {status})")


class kvq_config(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("key_bits", ctypes.c_int32), ("value_bits", ctypes.c_int32),
        ("group_size", ctypes.c_int32), ("residual", ctypes.c_int32), ("hadamard", ctypes.c_int32),
        ("layout", ctypes.c_int32), ("sink", ctypes.c_int32), ("rope_theta", ctypes.c_float),
        ("outliers", ctypes.c_int32), ("page_tokens", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
    ]


class kvq_cache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in BUFFER_NAMES] + [
        ("seq_len_host", ctypes.POINTER(ctypes.c_int64)), ("seq_len_dev", ctypes.c_void_p),
        ("k_out", ctypes.c_void_p), ("v_out", ctypes.c_void_p),
        ("page_table_host", ctypes.POINTER(ctypes.c_int32)), ("page_table_dev", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libkvq.so is not built ({LIB_PATH}); run python -m bit_kv_cache_prefill_b200.build")
    L = ctypes.CDLL(LIB_PATH)
    C, K, P, I64, S = (ctypes.POINTER(kvq_config), ctypes.POINTER(kvq_cache), ctypes.c_void_p, ctypes.c_int64,
                       ctypes.c_int)
    L.kvq_cache_buffer_bytes.argtypes = [C, ctypes.POINTER(ctypes.c_size_t)]
    L.kvq_cache_buffer_bytes.restype = S
    L.kvq_outlier_buffer_bytes.argtypes = [C, ctypes.POINTER(ctypes.c_size_t)]
    L.kvq_outlier_buffer_bytes.restype = S
    L.kvq_quantize_prefill.argtypes = [C, K, P, P, I64, I64, I64, ctypes.POINTER(ctypes.c_int64), P]
    L.kvq_quantize_prefill.restype = S
    L.kvq_append_token.argtypes = [C, K, P, P, P]
    L.kvq_append_token.restype = S
    L.kvq_decode_workspace_bytes.argtypes = [C, ctypes.POINTER(ctypes.c_size_t)]
    L.kvq_decode_workspace_bytes.restype = S
    L.kvq_decode_attention.argtypes = [C, K, P, P, ctypes.c_float, P, ctypes.c_size_t, P]
    L.kvq_decode_attention.restype = S
    L.kvq_decode_attention_noalloc.argtypes = [C, K, P, P, ctypes.c_float, P]
    L.kvq_decode_attention_noalloc.restype = S
    L.kvq_decode_status.argtypes = [C, P, P]
    L.kvq_decode_status.restype = S
    L.kvq_status_string.argtypes = [S]
    L.kvq_status_string.restype = ctypes.c_char_p
    return L


lib = _load()


def kvq_status_string(status: int) -> str:
    return lib.kvq_status_string(int(status)).decode()


def make_config(batch: int, num_q_heads: int, num_kv_heads: int, key_bits: int, value_bits: int, group_size: int,
                residual: int, hadamard: int, capacity: int, head_dim: int = 128,
                layout: int = KVQ_LAYOUT_TILE_V1, sink: int = 0, rope_theta: float = 0.0,
                outliers: int = 0, page_tokens: int = 0, num_pages: int = 0) -> kvq_config:
    return kvq_config(batch, num_q_heads, num_kv_heads, head_dim, key_bits, value_bits, group_size, residual,
                      hadamard, layout, sink, rope_theta, outliers, page_tokens, num_pages, capacity)


def _check(status: int, where: str) -> None:
    if status != KVQ_OK:
        raise KvqError(status, where)


def _stream_ptr(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def kvq_cache_buffer_bytes(cfg: kvq_config) -> List[int]:
    out = (ctypes.c_size_t * 8)()
    _check(lib.kvq_cache_buffer_bytes(ctypes.byref(cfg), out), "kvq_cache_buffer_bytes")
    return [int(x) for x in out]


def kvq_outlier_buffer_bytes(cfg: kvq_config) -> List[int]:
    out = (ctypes.c_size_t * 2)()
    _check(lib.kvq_outlier_buffer_bytes(ctypes.byref(cfg), out), "kvq_outlier_buffer_bytes")
    return [int(x) for x in out]


class Cache:
    """Device buffers of the packed cache (allocated with torch) plus the host / device length mirrors,
    the two outlier buffers when the config has outliers = 1, and with paged storage the page table
    (``page_table_host``: numpy int32 [B][Hkv][capacity / page_tokens], by default unit u's page j at
    pool page u * (capacity / page_tokens) + j; the caller may edit it in place before a call)."""

    def __init__(self, cfg: kvq_config, device: str = "cuda", page_table: Optional[np.ndarray] = None):
        self.cfg = cfg
        sizes = kvq_cache_buffer_bytes(cfg)
        self.buffers = {n: torch.zeros(max(s, 16), dtype=torch.uint8, device=device) for n, s in zip(BUFFER_NAMES, sizes)}
        self.sizes = dict(zip(BUFFER_NAMES, sizes))
        out_sizes = kvq_outlier_buffer_bytes(cfg)
        for n, s in zip(("k_out", "v_out"), out_sizes):
            if s:
                self.buffers[n] = torch.zeros(s, dtype=torch.uint8, device=device)
                self.sizes[n] = s
        self.seq_len_host = np.zeros(cfg.batch, np.int64)
        self.seq_len_dev = torch.zeros(cfg.batch, dtype=torch.int64, device=device)
        self.page_table_host = None
        self.page_table_dev = None
        if cfg.page_tokens > 0:
            per_unit = cfg.capacity // cfg.page_tokens
            shape = (cfg.batch, cfg.num_kv_heads, per_unit)
            if page_table is None:
                page_table = np.arange(cfg.batch * cfg.num_kv_heads * per_unit, dtype=np.int32).reshape(shape)
            self.page_table_host = np.ascontiguousarray(page_table, np.int32)
            assert self.page_table_host.shape == shape
            self.page_table_dev = torch.full((max(self.page_table_host.size, 4),), -1, dtype=torch.int32, device=device)
        self.c = kvq_cache(*(self.buffers[n].data_ptr() for n in BUFFER_NAMES),
                           self.seq_len_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)),
                           self.seq_len_dev.data_ptr(),
                           self.buffers["k_out"].data_ptr() if "k_out" in self.buffers else None,
                           self.buffers["v_out"].data_ptr() if "v_out" in self.buffers else None,
                           self.page_table_host.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
                           if self.page_table_host is not None else None,
                           self.page_table_dev.data_ptr() if self.page_table_dev is not None else None)

    def view(self, name: str, dtype: torch.dtype) -> torch.Tensor:
        return self.buffers[name][: self.sizes[name]].view(dtype)


def kvq_quantize_prefill(cfg: kvq_config, cache: Cache, k: torch.Tensor, v: torch.Tensor, seq_lens: Sequence[int],
                         stream: Optional[torch.cuda.Stream] = None) -> None:
    """k, v: fp16 CUDA tensors [B][T][Hkv][128] with a contiguous last dim and equal strides."""
    assert k.dtype == torch.float16 and v.dtype == torch.float16 and k.stride() == v.stride() and k.stride(3) == 1
    lens = np.ascontiguousarray(np.asarray(seq_lens, np.int64))
    _check(lib.kvq_quantize_prefill(ctypes.byref(cfg), ctypes.byref(cache.c), k.data_ptr(), v.data_ptr(),
                                    k.stride(0), k.stride(1), k.stride(2),
                                    lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), _stream_ptr(stream)),
           "kvq_quantize_prefill")


def kvq_append_token(cfg: kvq_config, cache: Cache, k_new: torch.Tensor, v_new: torch.Tensor,
                     stream: Optional[torch.cuda.Stream] = None) -> None:
    """k_new, v_new: contiguous fp16 CUDA tensors [B][Hkv][128]."""
    assert k_new.is_contiguous() and v_new.is_contiguous()
    _check(lib.kvq_append_token(ctypes.byref(cfg), ctypes.byref(cache.c), k_new.data_ptr(), v_new.data_ptr(),
                                _stream_ptr(stream)), "kvq_append_token")


def kvq_decode_workspace_bytes(cfg: kvq_config) -> int:
    n = ctypes.c_size_t()
    _check(lib.kvq_decode_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n)), "kvq_decode_workspace_bytes")
    return int(n.value)


def kvq_decode_attention(cfg: kvq_config, cache: Cache, q: torch.Tensor, out: torch.Tensor, sm_scale: float,
                         workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> None:
    """q, out: contiguous fp16 CUDA tensors [B][Hq][128]; workspace: CUDA byte tensor."""
    assert q.is_contiguous() and out.is_contiguous()
    _check(lib.kvq_decode_attention(ctypes.byref(cfg), ctypes.byref(cache.c), q.data_ptr(), out.data_ptr(),
                                    float(sm_scale), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                                    _stream_ptr(stream)), "kvq_decode_attention")


STATIC_SCRATCH_BYTES = 16 << 20


def kvq_decode_attention_noalloc(cfg: kvq_config, cache: Cache, q: torch.Tensor, out: torch.Tensor, sm_scale: float,
                                 stream: Optional[torch.cuda.Stream] = None) -> None:
    """Decode attention for callers that cannot allocate device memory: the split partials live in
    the library's fixed 16 MiB per-GPU scratch array (see include/kvq.h). Calls that overlap on the
    GPU race on that array."""
    assert q.is_contiguous() and out.is_contiguous()
    _check(lib.kvq_decode_attention_noalloc(ctypes.byref(cfg), ctypes.byref(cache.c), q.data_ptr(), out.data_ptr(),
                                            float(sm_scale), _stream_ptr(stream)), "kvq_decode_attention_noalloc")


def kvq_decode_status(cfg: kvq_config, workspace: torch.Tensor, stream: Optional[torch.cuda.Stream] = None) -> int:
    """Status of the last decode that used ``workspace``: KVQ_OK or KVQ_ERR_TIMEOUT (other errors raise).
    Synchronises the stream."""
    st = lib.kvq_decode_status(ctypes.byref(cfg), workspace.data_ptr(), _stream_ptr(stream))
    if st not in (KVQ_OK, KVQ_ERR_TIMEOUT):
        raise KvqError(st, "kvq_decode_status")
    return st
