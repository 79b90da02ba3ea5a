"""CPU oracle for the asymmetric low-bit KV cache — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` may import this
module. The product (``bit_kv_cache_prefill_b200``) never imports, loads or calls it, and it shares no
code with the CUDA library. The arithmetic lives in ``kvq_oracle.cpp`` (plain C++17, fp64 attention,
exact IEEE fp32 codec, built with ``-ffp-contract=off -fno-fast-math``); this file only marshals numpy
arrays through ctypes.

Every function here follows the passages cited in ``kvq_oracle.cpp``: per-channel keys and per-token
values (KVQuant review, Method; KV cache quantization wiki page, KIVI notes), the FP16 recent window
(Asymmetric KV Cache Compression framework page, In practice), grouped/residual split with
token-axis append (wiki page, KIVI notes), and the Hadamard rotation shared by keys and query
(framework page, Method; Dual-QK abstract).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kvq_oracle.cpp")
_SO = os.path.join(_HERE, "libkvq_oracle.so")
CXXFLAGS = ["-O2", "-std=c++17", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-pthread"]


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/libkvq_oracle.so`` (host C++ only)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(["g++", *CXXFLAGS, "-o", tmp, _SRC])
        os.replace(tmp, _SO)
    return _SO


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _declare(_lib)
    return _lib


class _CConfig(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("key_bits", ctypes.c_int32), ("value_bits", ctypes.c_int32),
        ("group_size", ctypes.c_int32), ("residual", ctypes.c_int32), ("hadamard", ctypes.c_int32),
        ("layout", ctypes.c_int32), ("sink", ctypes.c_int32), ("rope_theta", ctypes.c_float),
        ("outliers", ctypes.c_int32), ("page_tokens", ctypes.c_int32), ("num_pages", ctypes.c_int32),
        ("capacity", ctypes.c_int64),
    ]


class _CCache(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("k_codes", "v_codes", "k_scale", "k_zero", "v_scale", "v_zero", "k_res", "v_res", "seq_len",
                 "k_out_ch", "k_out_val", "v_out_ch", "v_out_val", "page_table")]


def _declare(L: ctypes.CDLL) -> None:
    P, I, I64, D = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    C, K = ctypes.POINTER(_CConfig), ctypes.POINTER(_CCache)
    L.kvq_ref_quantize_prefill.argtypes = [C, K, P, P, I64, I64, I64, P, I]
    L.kvq_ref_quantize_prefill.restype = I
    L.kvq_ref_append_token.argtypes = [C, K, P, P]
    L.kvq_ref_append_token.restype = I
    L.kvq_ref_decode.argtypes = [C, K, P, D, P, I]
    L.kvq_ref_decode.restype = I
    L.kvq_ref_f16_to_f32.argtypes = [P, P, I64]
    L.kvq_ref_f32_to_f16.argtypes = [P, P, I64]
    L.kvq_ref_wht128_f32.argtypes = [P]
    L.kvq_ref_wht128_f64.argtypes = [P]
    L.kvq_ref_quantize_group.argtypes = [P, I, I, P, P, P]
    L.kvq_ref_key_word_bit.argtypes = [I, I, I, P, P]
    L.kvq_ref_value_word_bit.argtypes = [I, I, I, P, P]
    L.kvq_ref_key_word_bit_v2.argtypes = [I64, I, I, P, P]
    L.kvq_ref_value_word_bit_v2.argtypes = [I64, I, I, P, P]
    L.kvq_ref_key_param_pos.argtypes = [I]
    L.kvq_ref_key_param_pos.restype = I
    L.kvq_ref_quantized_len.argtypes = [I64, I, I]
    L.kvq_ref_quantized_len.restype = I64
    L.kvq_ref_check_f32_to_f16_range.argtypes = [ctypes.c_uint64, ctypes.c_uint64]
    L.kvq_ref_check_f32_to_f16_range.restype = I64


@dataclass
class Config:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    key_bits: int
    value_bits: int
    group_size: int
    residual: int
    hadamard: int
    capacity: int
    head_dim: int = 128
    layout: int = 1  # 1 = tile v1 (mma fragment order), 2 = rows v2 (token rows of keys, channel rows of values)
    sink: int = 0    # 1: the first token stays in fp16 (an extra row after the ring)
    rope_theta: float = 0.0  # > 0: keys are cached before RoPE and decode applies it (0: off)
    outliers: int = 0  # 1: each quantized token's largest-magnitude key / value entry stays fp16
    page_tokens: int = 0  # > 0: paged storage with pages of this many tokens (a multiple of 128); 0: contiguous
    num_pages: int = 0    # pages in the pool (paged storage only)

    def c(self) -> _CConfig:
        return _CConfig(self.batch, self.num_q_heads, self.num_kv_heads, self.head_dim, self.key_bits,
                        self.value_bits, self.group_size, self.residual, self.hadamard, self.layout, self.sink,
                        self.rope_theta, self.outliers, self.page_tokens, self.num_pages, self.capacity)


class Cache:
    """Host buffers of the packed cache, laid out exactly as the product's device buffers.

    Contiguous storage: every per-token array has one slot of ``capacity`` tokens per unit, shape
    [B][Hkv][...]. Paged storage (``cfg.page_tokens`` = P > 0, reading R13): one slot of P tokens per
    physical page, shape [num_pages][...], and ``page_table`` [B][Hkv][capacity / P] (int32) names the
    physical page of each logical page; by default unit u's page j is u * (capacity / P) + j."""

    def __init__(self, cfg: Config, page_table: np.ndarray | None = None):
        B, H, cap, G = cfg.batch, cfg.num_kv_heads, cfg.capacity, cfg.group_size
        ring = cfg.residual + G + cfg.sink  # ring slots, then the first token's row when the sink is on
        if cfg.page_tokens:
            lead, n = (cfg.num_pages,), cfg.page_tokens
            per_unit = cap // cfg.page_tokens
            if page_table is None:
                page_table = np.arange(B * H * per_unit, dtype=np.int32).reshape(B, H, per_unit)
            self.page_table = np.ascontiguousarray(page_table, np.int32)
            assert self.page_table.shape == (B, H, per_unit)
        else:
            lead, n = (B, H), cap
            self.page_table = None
        if cfg.layout == 2:
            self.k_codes = np.zeros(lead + (n, 4 * cfg.key_bits), np.uint32)
            self.v_codes = np.zeros(lead + ((n + 127) // 128, 128, 4 * cfg.value_bits), np.uint32)
        else:
            self.k_codes = np.zeros(lead + (n // 16, 64 * cfg.key_bits), np.uint32)
            self.v_codes = np.zeros(lead + (n // 16, 64 * cfg.value_bits), np.uint32)
        self.k_scale = np.zeros(lead + (n // G, 128), np.uint16)
        self.k_zero = np.zeros(lead + (n // G, 128), np.uint16)
        self.v_scale = np.zeros(lead + (n, 128 // G), np.uint16)
        self.v_zero = np.zeros(lead + (n, 128 // G), np.uint16)
        self.k_res = np.zeros((B, H, ring, 128), np.uint16)
        self.v_res = np.zeros((B, H, ring, 128), np.uint16)
        self.seq_len = np.zeros((B,), np.int64)
        # sparse outliers (one per quantized token and tensor): channel (0xffff: none) and fp16 value
        self.k_out_ch = np.full(lead + (n,), 0xFFFF, np.uint16)
        self.k_out_val = np.zeros(lead + (n,), np.uint16)
        self.v_out_ch = np.full(lead + (n,), 0xFFFF, np.uint16)
        self.v_out_val = np.zeros(lead + (n,), np.uint16)

    def c(self) -> _CCache:
        return _CCache(*(a.ctypes.data for a in (self.k_codes, self.v_codes, self.k_scale, self.k_zero,
                                                 self.v_scale, self.v_zero, self.k_res, self.v_res,
                                                 self.seq_len, self.k_out_ch, self.k_out_val, self.v_out_ch,
                                                 self.v_out_val)),
                       self.page_table.ctypes.data if self.page_table is not None else None)


def _u16(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.float16:
        a = a.view(np.uint16)
    assert a.dtype == np.uint16
    return a


def quantize_prefill(cfg: Config, cache: Cache, k: np.ndarray, v: np.ndarray, seq_lens, threads: int = 1) -> None:
    """k, v: fp16 [B][T][Hkv][128] (any element strides, last dim contiguous, same strides for both)."""
    k, v = _u16(k), _u16(v)
    assert k.strides == v.strides and k.strides[3] == 2
    sb, st, sh = (s // 2 for s in k.strides[:3])
    sl = np.ascontiguousarray(np.asarray(seq_lens, np.int64))
    cc, kc = cfg.c(), cache.c()
    rc = lib().kvq_ref_quantize_prefill(ctypes.byref(cc), ctypes.byref(kc), k.ctypes.data, v.ctypes.data,
                                        sb, st, sh, sl.ctypes.data, threads)
    if rc:
        raise ValueError(f"oracle prefill rejected the arguments (status {rc})")


def append_token(cfg: Config, cache: Cache, k_new: np.ndarray, v_new: np.ndarray) -> None:
    """k_new, v_new: fp16 [B][Hkv][128]."""
    k_new = np.ascontiguousarray(_u16(k_new))
    v_new = np.ascontiguousarray(_u16(v_new))
    cc, kc = cfg.c(), cache.c()
    rc = lib().kvq_ref_append_token(ctypes.byref(cc), ctypes.byref(kc), k_new.ctypes.data, v_new.ctypes.data)
    if rc:
        raise ValueError(f"oracle append rejected the arguments (status {rc})")


def decode(cfg: Config, cache: Cache, q: np.ndarray, sm_scale: float, threads: int = 1) -> np.ndarray:
    """q: fp16 [B][Hq][128] -> fp64 [B][Hq][128]."""
    q = np.ascontiguousarray(_u16(q))
    out = np.zeros((cfg.batch, cfg.num_q_heads, 128), np.float64)
    cc, kc = cfg.c(), cache.c()
    rc = lib().kvq_ref_decode(ctypes.byref(cc), ctypes.byref(kc), q.ctypes.data, float(sm_scale),
                              out.ctypes.data, threads)
    if rc:
        raise ValueError(f"oracle decode rejected the arguments (status {rc})")
    return out


# ---- single-step helpers (used by the oracle's pins) ----------------------------------------------

def f16_to_f32(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(_u16(h))
    out = np.empty(h.shape, np.float32)
    lib().kvq_ref_f16_to_f32(h.ctypes.data, out.ctypes.data, h.size)
    return out


def f32_to_f16(f: np.ndarray) -> np.ndarray:
    f = np.ascontiguousarray(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().kvq_ref_f32_to_f16(f.ctypes.data, out.ctypes.data, f.size)
    return out


def wht128_f32(x: np.ndarray) -> np.ndarray:
    y = np.array(x, np.float32, copy=True, order="C")
    assert y.shape == (128,)
    lib().kvq_ref_wht128_f32(y.ctypes.data)
    return y


def wht128_f64(x: np.ndarray) -> np.ndarray:
    y = np.array(x, np.float64, copy=True, order="C")
    assert y.shape == (128,)
    lib().kvq_ref_wht128_f64(y.ctypes.data)
    return y


def quantize_group(x: np.ndarray, bits: int):
    """One min/max group: returns (codes uint8[n], scale fp16 bits, zero fp16 bits)."""
    x = np.ascontiguousarray(_u16(x))
    codes = np.zeros(x.size, np.uint8)
    s = np.zeros(1, np.uint16)
    z = np.zeros(1, np.uint16)
    lib().kvq_ref_quantize_group(x.ctypes.data, x.size, bits, codes.ctypes.data, s.ctypes.data, z.ctypes.data)
    return codes, int(s[0]), int(z[0])


def key_word_bit(i: int, c: int, bits: int):
    w, b = ctypes.c_int(), ctypes.c_int()
    lib().kvq_ref_key_word_bit(i, c, bits, ctypes.byref(w), ctypes.byref(b))
    return w.value, b.value


def value_word_bit(i: int, c: int, bits: int):
    w, b = ctypes.c_int(), ctypes.c_int()
    lib().kvq_ref_value_word_bit(i, c, bits, ctypes.byref(w), ctypes.byref(b))
    return w.value, b.value


def key_word_bit_v2(t: int, c: int, bits: int):
    w, b = ctypes.c_int64(), ctypes.c_int()
    lib().kvq_ref_key_word_bit_v2(t, c, bits, ctypes.byref(w), ctypes.byref(b))
    return w.value, b.value


def value_word_bit_v2(t: int, c: int, bits: int):
    w, b = ctypes.c_int64(), ctypes.c_int()
    lib().kvq_ref_value_word_bit_v2(t, c, bits, ctypes.byref(w), ctypes.byref(b))
    return w.value, b.value


def key_param_pos(c: int) -> int:
    return lib().kvq_ref_key_param_pos(c)


def quantized_len(T: int, R: int, G: int) -> int:
    return lib().kvq_ref_quantized_len(T, R, G)


def check_f32_to_f16_range(lo: int, hi: int) -> int:
    return lib().kvq_ref_check_f32_to_f16_range(lo, hi)
