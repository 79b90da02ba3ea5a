"""CPU checks of the C ABI: the library loads without a GPU, exports every entry point that
include/kvq.h declares, reports buffer sizes from the layout's closed form, and rejects bad arguments
on the host before anything is launched (no device memory is touched by these calls)."""
import ctypes
import os
import re

import numpy as np
import pytest

import bit_kv_cache_prefill_b200 as kvq
from bit_kv_cache_prefill_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols():
    text = open(os.path.join(ROOT, "include", "kvq.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvq_[a-z_]+)\s*\(", text)))


def test_library_exports_every_declared_entry_point():
    names = _declared_symbols()
    assert names == ["kvq_append_token", "kvq_cache_buffer_bytes", "kvq_decode_attention",
                     "kvq_decode_attention_noalloc", "kvq_decode_status", "kvq_decode_workspace_bytes",
                     "kvq_outlier_buffer_bytes", "kvq_quantize_prefill", "kvq_status_string"]
    lib = ctypes.CDLL(kvq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
        assert hasattr(kvq, n), n  # the Python binding uses the same names


def test_status_strings():
    for s in (0, -1, -2, -3, -4, -5, -6):
        assert kvq.kvq_status_string(s) and kvq.kvq_status_string(s) != "unknown status"
    assert kvq.kvq_status_string(7) == "unknown status"


@pytest.mark.parametrize("B,Hq,Hkv,kb,vb,G,R,cap", [(8, 32, 32, 2, 2, 32, 128, 32768), (16, 32, 8, 2, 2, 64, 128, 131328),
                                                      (64, 32, 8, 4, 2, 32, 32, 16384), (1, 32, 8, 2, 2, 128, 128, 1 << 20)])
def test_buffer_bytes_closed_form(B, Hq, Hkv, kb, vb, G, R, cap):
    cfg = kvq.make_config(B, Hq, Hkv, kb, vb, G, R, 0, cap)
    got = kvq.kvq_cache_buffer_bytes(cfg)
    u = B * Hkv
    # codes: bits per element; key scale/zero: fp16 per (group, channel); value: fp16 per (token, group)
    want = [u * cap * 128 * kb // 8, u * cap * 128 * vb // 8, u * (cap // G) * 128 * 2, u * (cap // G) * 128 * 2,
            u * cap * (128 // G) * 2, u * cap * (128 // G) * 2, u * (R + G) * 128 * 2, u * (R + G) * 128 * 2]
    assert got == want
    assert kvq.kvq_decode_workspace_bytes(cfg) > 0


@pytest.mark.parametrize("cap", [4096, 4224, 1 << 20])
def test_buffer_bytes_rows_v2(cap):
    cfg = kvq.make_config(3, 8, 2, 4, 2, 32, 64, 0, cap, layout=kvq.KVQ_LAYOUT_ROWS_V2)
    got = kvq.kvq_cache_buffer_bytes(cfg)
    u = 3 * 2
    vcap = -(-cap // 128) * 128  # value rows come in whole 128-token blocks
    assert got[0] == u * cap * 4 * 4 * 4 and got[1] == u * vcap * 4 * 2 * 4
    assert got[2:] == kvq.kvq_cache_buffer_bytes(kvq.make_config(3, 8, 2, 4, 2, 32, 64, 0, cap))[2:]


def test_rows_v2_needs_whole_128_token_blocks():
    sizes = (ctypes.c_size_t * 8)()
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1056, layout=kvq.KVQ_LAYOUT_ROWS_V2)
    assert _status("kvq_cache_buffer_bytes", ctypes.byref(cfg), sizes) == kvq.KVQ_ERR_INVALID_ARG
    cfg.layout = kvq.KVQ_LAYOUT_TILE_V1
    assert _status("kvq_cache_buffer_bytes", ctypes.byref(cfg), sizes) == kvq.KVQ_OK


def _status(fn, *args):
    return getattr(_lib.lib, fn)(*args)


@pytest.mark.parametrize("field,value,status", [
    ("head_dim", 64, kvq.KVQ_ERR_UNSUPPORTED), ("key_bits", 3, kvq.KVQ_ERR_INVALID_ARG),
    ("value_bits", 8, kvq.KVQ_ERR_INVALID_ARG), ("group_size", 48, kvq.KVQ_ERR_INVALID_ARG),
    ("group_size", 256, kvq.KVQ_ERR_INVALID_ARG), ("num_q_heads", 33, kvq.KVQ_ERR_INVALID_ARG),
    ("num_q_heads", 64, kvq.KVQ_ERR_UNSUPPORTED), ("residual", -1, kvq.KVQ_ERR_INVALID_ARG),
    ("hadamard", 2, kvq.KVQ_ERR_INVALID_ARG), ("capacity", 100, kvq.KVQ_ERR_INVALID_ARG),
    ("layout", 3, kvq.KVQ_ERR_UNSUPPORTED), ("layout", 0, kvq.KVQ_ERR_UNSUPPORTED),
    ("batch", 0, kvq.KVQ_ERR_INVALID_ARG),
])
def test_config_validation(field, value, status):
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024)
    setattr(cfg, field, value)
    sizes = (ctypes.c_size_t * 8)()
    assert _status("kvq_cache_buffer_bytes", ctypes.byref(cfg), sizes) == status
    n = ctypes.c_size_t()
    assert _status("kvq_decode_workspace_bytes", ctypes.byref(cfg), ctypes.byref(n)) == status
    assert _status("kvq_cache_buffer_bytes", None, sizes) == kvq.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("layout,had,theta,status", [
    (2, 0, 10000.0, kvq.KVQ_OK), (2, 0, 0.0, kvq.KVQ_OK),
    (1, 0, 10000.0, kvq.KVQ_ERR_UNSUPPORTED),      # pre-RoPE keys need token-row keys (rows v2)
    (2, 1, 10000.0, kvq.KVQ_ERR_INVALID_ARG),      # RoPE and the Hadamard rotation exclude each other
    (2, 0, -1.0, kvq.KVQ_ERR_INVALID_ARG), (2, 0, float("nan"), kvq.KVQ_ERR_INVALID_ARG),
    (2, 0, float("inf"), kvq.KVQ_ERR_INVALID_ARG),
])
def test_rope_config_validation(layout, had, theta, status):
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, had, 1024, layout=layout, rope_theta=theta)
    sizes = (ctypes.c_size_t * 8)()
    assert _status("kvq_cache_buffer_bytes", ctypes.byref(cfg), sizes) == status
    n = ctypes.c_size_t()
    assert _status("kvq_decode_workspace_bytes", ctypes.byref(cfg), ctypes.byref(n)) == status


@pytest.mark.parametrize("cap", [1024, 1 << 20])
def test_rope_workspace_holds_the_angle_tables(cap):
    # the cache buffers do not change; the decode workspace gains the two angle tables,
    # (cos, sin) of every 32-token step start and of the 32 in-step offsets, after the partials
    base = kvq.make_config(1, 32, 8, 2, 2, 128, 128, 0, cap, layout=kvq.KVQ_LAYOUT_ROWS_V2)
    rope = kvq.make_config(1, 32, 8, 2, 2, 128, 128, 0, cap, layout=kvq.KVQ_LAYOUT_ROWS_V2, rope_theta=10000.0)
    assert kvq.kvq_cache_buffer_bytes(rope) == kvq.kvq_cache_buffer_bytes(base)
    records = 1 * 32 * 4  # one u32 status record per (sequence, query head) closes the workspace
    part = kvq.kvq_decode_workspace_bytes(base) - records  # partials, 256-byte aligned end
    tables = (-(-cap // 32) * 64 + 32 * 64) * 8
    assert kvq.kvq_decode_workspace_bytes(rope) == -(-(part + tables) // 256) * 256 + records


@pytest.mark.parametrize("layout,theta,value,status", [
    (1, 0.0, 1, kvq.KVQ_OK), (1, 0.0, 0, kvq.KVQ_OK),
    (2, 0.0, 1, kvq.KVQ_ERR_UNSUPPORTED),        # the outlier path exists for tile v1 only
    (2, 10000.0, 1, kvq.KVQ_ERR_UNSUPPORTED),    # and not with pre-RoPE keys
    (1, 0.0, 2, kvq.KVQ_ERR_INVALID_ARG), (1, 0.0, -1, kvq.KVQ_ERR_INVALID_ARG),
])
def test_outlier_config_validation(layout, theta, value, status):
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024, layout=layout, rope_theta=theta, outliers=value)
    sizes = (ctypes.c_size_t * 8)()
    assert _status("kvq_cache_buffer_bytes", ctypes.byref(cfg), sizes) == status
    out = (ctypes.c_size_t * 2)()
    assert _status("kvq_outlier_buffer_bytes", ctypes.byref(cfg), out) == status


@pytest.mark.parametrize("B,Hkv,cap", [(2, 2, 1024), (8, 32, 32768 + 1024), (1, 8, 1 << 20)])
def test_outlier_buffer_bytes(B, Hkv, cap):
    # one u32 (channel | fp16 value << 16) per (unit, token) for keys and for values; none when off
    on = kvq.make_config(B, 4 * Hkv if Hkv <= 8 else Hkv, Hkv, 2, 2, 32, 128, 0, cap, outliers=1)
    off = kvq.make_config(B, 4 * Hkv if Hkv <= 8 else Hkv, Hkv, 2, 2, 32, 128, 0, cap)
    assert kvq.kvq_outlier_buffer_bytes(on) == [B * Hkv * cap * 4] * 2
    assert kvq.kvq_outlier_buffer_bytes(off) == [0, 0]
    assert kvq.kvq_cache_buffer_bytes(on) == kvq.kvq_cache_buffer_bytes(off)
    assert _status("kvq_outlier_buffer_bytes", ctypes.byref(on), None) == kvq.KVQ_ERR_INVALID_ARG


def test_outlier_cache_needs_its_buffers():
    # outliers = 1 with null outlier pointers is rejected on the host before any launch
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024, outliers=1)
    c, host = _fake_cache(cfg, [0, 0])
    k = ctypes.c_void_p(0x100000)
    lens = np.array([64, 64], np.int64)
    st = _lib.lib.kvq_quantize_prefill(ctypes.byref(cfg), ctypes.byref(c), k, k, 64 * 2 * 128, 2 * 128, 128,
                                       lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
    c.k_out, c.v_out = 0x200000, 0x200008  # v_out not 16-byte aligned
    st = _lib.lib.kvq_quantize_prefill(ctypes.byref(cfg), ctypes.byref(c), k, k, 64 * 2 * 128, 2 * 128, 128,
                                       lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), None)
    assert st == kvq.KVQ_ERR_INVALID_ARG


def _fake_cache(cfg, lens):
    # Non-null, 16-byte aligned placeholder addresses: every call below is rejected on the host before
    # any of them could be used.
    host = np.asarray(lens, np.int64).copy()
    c = _lib.kvq_cache(*([0x10000 * (i + 1) for i in range(8)]),
                       host.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), 0x90000)
    return c, host


def test_prefill_rejects_lengths_beyond_capacity_and_bad_strides():
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024)
    c, host = _fake_cache(cfg, [0, 0])
    lens = np.array([1025, 5], np.int64)
    P = ctypes.POINTER(ctypes.c_int64)
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000, 0, 0, 0,
                   lens.ctypes.data_as(P), None) == kvq.KVQ_ERR_CAPACITY
    lens = np.array([10, -1], np.int64)
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000, 0, 0, 0,
                   lens.ctypes.data_as(P), None) == kvq.KVQ_ERR_CAPACITY
    lens = np.array([10, 5], np.int64)
    # misaligned input pointer, odd stride, null input, null lengths
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), 0x100002, 0x200000, 2048, 256, 128,
                   lens.ctypes.data_as(P), None) == kvq.KVQ_ERR_INVALID_ARG
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000, 2048, 256, 129,
                   lens.ctypes.data_as(P), None) == kvq.KVQ_ERR_INVALID_ARG
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), None, 0x200000, 2048, 256, 128,
                   lens.ctypes.data_as(P), None) == kvq.KVQ_ERR_INVALID_ARG
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000, 2048, 256, 128,
                   None, None) == kvq.KVQ_ERR_INVALID_ARG
    # a misaligned cache buffer
    c.k_scale = 0x30008
    assert _status("kvq_quantize_prefill", ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000, 2048, 256, 128,
                   lens.ctypes.data_as(P), None) == kvq.KVQ_ERR_INVALID_ARG
    assert list(host) == [0, 0]  # nothing changed on rejection


def test_append_rejects_capacity_overflow_without_side_effects():
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024)
    c, host = _fake_cache(cfg, [1024, 3])
    assert _status("kvq_append_token", ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000, None) == kvq.KVQ_ERR_CAPACITY
    assert list(host) == [1024, 3]
    assert _status("kvq_append_token", ctypes.byref(cfg), ctypes.byref(c), 0x100008, 0x200000, None) == kvq.KVQ_ERR_INVALID_ARG


def test_decode_rejects_small_workspace_and_bad_scale():
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024)
    c, _ = _fake_cache(cfg, [100, 3])
    need = kvq.kvq_decode_workspace_bytes(cfg)
    args = (ctypes.byref(cfg), ctypes.byref(c), 0x100000, 0x200000)
    assert _status("kvq_decode_attention", *args, ctypes.c_float(0.1), 0x300000, need - 1, None) == kvq.KVQ_ERR_WORKSPACE
    assert _status("kvq_decode_attention", *args, ctypes.c_float(0.1), None, need, None) == kvq.KVQ_ERR_WORKSPACE
    assert _status("kvq_decode_attention", *args, ctypes.c_float(0.1), 0x300010, need, None) == kvq.KVQ_ERR_WORKSPACE
    assert _status("kvq_decode_attention", *args, ctypes.c_float(0.0), 0x300000, need, None) == kvq.KVQ_ERR_INVALID_ARG
    assert _status("kvq_decode_attention", *args, ctypes.c_float(float("nan")), 0x300000, need, None) == kvq.KVQ_ERR_INVALID_ARG
    assert _status("kvq_decode_attention", ctypes.byref(cfg), ctypes.byref(c), None, 0x200000, ctypes.c_float(0.1),
                   0x300000, need, None) == kvq.KVQ_ERR_INVALID_ARG


@pytest.mark.parametrize("P,pages,layout,theta,status", [
    (128, 8, 1, 0.0, kvq.KVQ_OK), (512, 2, 1, 0.0, kvq.KVQ_OK), (1024, 1, 1, 0.0, kvq.KVQ_OK),
    (64, 8, 1, 0.0, kvq.KVQ_ERR_INVALID_ARG),     # not a multiple of 128
    (384, 8, 1, 0.0, kvq.KVQ_ERR_INVALID_ARG),    # does not divide the capacity
    (128, 0, 1, 0.0, kvq.KVQ_ERR_INVALID_ARG),    # an empty pool
    (-128, 8, 1, 0.0, kvq.KVQ_ERR_INVALID_ARG),
    (128, 8, 2, 0.0, kvq.KVQ_ERR_UNSUPPORTED),    # paging exists for tile v1 only
    (128, 8, 2, 10000.0, kvq.KVQ_ERR_UNSUPPORTED),
])
def test_paged_config_validation(P, pages, layout, theta, status):
    cfg = kvq.make_config(2, 8, 2, 2, 2, 32, 32, 0, 1024, layout=layout, rope_theta=theta, page_tokens=P,
                          num_pages=pages)
    sizes = (ctypes.c_size_t * 8)()
    assert _status("kvq_cache_buffer_bytes", ctypes.byref(cfg), sizes) == status


@pytest.mark.parametrize("P,pages,outliers", [(128, 37, 0), (512, 5, 1), (256, 1000, 1)])
def test_paged_buffer_bytes_are_pool_sized(P, pages, outliers):
    # the six per-token buffers (and the outlier words) hold num_pages pages of P tokens; the fp16
    # ring stays per unit
    B, Hkv, G, R, cap = 3, 2, 32, 64, 2048
    paged = kvq.make_config(B, 8, Hkv, 4, 2, G, R, 0, cap, outliers=outliers, page_tokens=P, num_pages=pages)
    got = kvq.kvq_cache_buffer_bytes(paged)
    want = [pages * P * 128 * 4 // 8, pages * P * 128 * 2 // 8, pages * (P // G) * 128 * 2,
            pages * (P // G) * 128 * 2, pages * P * (128 // G) * 2, pages * P * (128 // G) * 2]
    assert got[:6] == want
    contiguous = kvq.make_config(B, 8, Hkv, 4, 2, G, R, 0, cap, outliers=outliers)
    assert got[6:] == kvq.kvq_cache_buffer_bytes(contiguous)[6:]
    assert kvq.kvq_outlier_buffer_bytes(paged) == ([pages * P * 4] * 2 if outliers else [0, 0])


def _paged_fake_cache(cfg, lens, table):
    c, host = _fake_cache(cfg, lens)
    c.page_table_host = table.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))
    c.page_table_dev = 0xA0000
    return c, host


@pytest.mark.parametrize("bad", [-1, 4, 1 << 20])
def test_paged_prefill_rejects_table_entries_outside_the_pool(bad):
    # a page that would hold quantized tokens (T = 300, R = 32, G = 32: Q = 256, pages 0 and 1 of 128)
    # must map into the pool; the call is refused on the host before anything is copied or launched
    cfg = kvq.make_config(1, 2, 1, 2, 2, 32, 32, 0, 512, page_tokens=128, num_pages=4)
    table = np.array([[[0, bad, -1, -1]]], np.int32)
    c, _ = _paged_fake_cache(cfg, [0], table)
    k = ctypes.c_void_p(0x100000)
    lens = np.array([300], np.int64)
    st = _lib.lib.kvq_quantize_prefill(ctypes.byref(cfg), ctypes.byref(c), k, k, 300 * 128, 128, 128,
                                       lens.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), None)
    assert st == kvq.KVQ_ERR_INVALID_ARG


def test_paged_append_and_decode_check_the_table():
    # append: the flush that takes the quantized part into page 1 needs that page; decode: every page
    # of the quantized part
    cfg = kvq.make_config(1, 2, 1, 2, 2, 32, 32, 0, 512, page_tokens=128, num_pages=4)
    table = np.array([[[2, -1, -1, -1]]], np.int32)
    c, host = _paged_fake_cache(cfg, [159], table)  # Q = 96 -> 128 after this append: still page 0
    kn = ctypes.c_void_p(0x100000)
    host[0] = 191  # Q = 128 now; the append brings Q to 160, into page 1
    assert _lib.lib.kvq_append_token(ctypes.byref(cfg), ctypes.byref(c), kn, kn, None) == kvq.KVQ_ERR_INVALID_ARG
    host[0] = 200  # Q = 160: decode reads pages 0 and 1
    ws = ctypes.c_void_p(0x200000)
    st = _lib.lib.kvq_decode_attention(ctypes.byref(cfg), ctypes.byref(c), kn, kn, ctypes.c_float(0.1), ws,
                                       1 << 30, None)
    assert st == kvq.KVQ_ERR_INVALID_ARG
    c.page_table_host = None  # a paged cache without its table
    host[0] = 0
    assert _lib.lib.kvq_append_token(ctypes.byref(cfg), ctypes.byref(c), kn, kn, None) == kvq.KVQ_ERR_INVALID_ARG


def _header_struct(name, path=os.path.join("include", "kvq.h")):
    """Field (type, name) pairs of `typedef struct { ... } name;` in a C source, comments removed."""
    text = open(os.path.join(ROOT, path)).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = re.sub(r"//[^\n]*", "", text)
    body = re.search(r"typedef struct \{([^{}]*)\}\s*" + name + r";", text).group(1)
    fields = []
    for decl in body.split(";"):  # "type name", "type* name" or "type a, b, c"
        decl = decl.strip()
        if decl:
            base, rest = re.match(r"(\w+)\s*(.*)$", decl, flags=re.S).groups()
            for d in rest.split(","):
                d = d.strip()
                name = d.lstrip("*").strip()
                fields.append((base + "*" * (len(d) - len(d.lstrip("*"))), name))
    return fields


_CTYPE_OF = {"int32_t": ctypes.c_int32, "int64_t": ctypes.c_int64, "float": ctypes.c_float}
_SIZES = {"int32_t": 4, "float": 4, "int64_t": 8}


def _oracle_structs():
    import oracle
    return [("kvq_ref_config", oracle._CConfig), ("kvq_ref_cache", oracle._CCache)]


@pytest.mark.parametrize("name,binding,path", [
    ("kvq_config", _lib.kvq_config, os.path.join("include", "kvq.h")),
    ("kvq_cache", _lib.kvq_cache, os.path.join("include", "kvq.h")),
    ("kvq_ref_config", "oracle", os.path.join("oracle", "kvq_oracle.cpp")),
    ("kvq_ref_cache", "oracle", os.path.join("oracle", "kvq_oracle.cpp")),
])
def test_binding_structs_match_the_header(name, binding, path):
    # the ctypes structs (library binding and oracle wrapper) must list the C struct's fields in the
    # same order with the same types, and so have the same size: a drifted binding would pass every
    # argument one field off
    if binding == "oracle":
        binding = dict(_oracle_structs())[name]
    header = _header_struct(name, path)
    assert [n for _, n in header] == [n for n, _ in binding._fields_]
    for (ctype, fname), (_, btype) in zip(header, binding._fields_):
        if ctype.endswith("*"):
            assert btype is ctypes.c_void_p or issubclass(btype, ctypes._Pointer), fname
        else:
            assert btype is _CTYPE_OF[ctype], fname
    off = 0
    for ctype, _ in header:  # natural alignment, as the C compiler lays the struct out
        sz = 8 if ctype.endswith("*") else _SIZES[ctype]
        off = -(-off // sz) * sz + sz
    assert ctypes.sizeof(binding) == -(-off // 8) * 8


def test_decode_workspace_ends_with_one_status_record_per_query_head():
    """The workspace bound covers the split partials, the RoPE tables (pre-RoPE keys) and, 256-byte
    aligned at the end, one u32 status record per (sequence, query head)."""
    for B, Hq, Hkv, rope, layout in [(8, 32, 32, 0.0, 1), (16, 32, 8, 0.0, 1), (3, 8, 2, 10000.0, 2)]:
        cfg = kvq.make_config(B, Hq, Hkv, 2, 2, 32, 32, 0, 4096, layout=layout, rope_theta=rope)
        n = kvq.kvq_decode_workspace_bytes(cfg)
        assert (n - B * Hq * 4) % 256 == 0 and n > B * Hq * 4


def test_decode_status_rejects_bad_arguments():
    cfg = kvq.make_config(2, 4, 2, 2, 2, 32, 32, 0, 1024)
    assert _lib.lib.kvq_decode_status(ctypes.byref(cfg), None, None) == kvq.KVQ_ERR_INVALID_ARG
    assert _lib.lib.kvq_decode_status(ctypes.byref(cfg), ctypes.c_void_p(0x1001), None) == kvq.KVQ_ERR_INVALID_ARG
    bad = kvq.make_config(2, 4, 2, 3, 2, 32, 32, 0, 1024)
    assert _lib.lib.kvq_decode_status(ctypes.byref(bad), ctypes.c_void_p(0x1000), None) == kvq.KVQ_ERR_INVALID_ARG
