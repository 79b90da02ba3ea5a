"""GPU parity with paged storage (tile v1).

KVQuant review (Limitations, Future work, Sparks): blocked allocation instead of copying earlier
tokens' data on every update. With page_tokens = P the quantized part of a unit lives in pool pages
named by a page table; paging changes addresses only. The pool the GPU writes must equal the
oracle's pool for the same table bit for bit (codes, scales, zeros, outlier words), spare pages must
stay untouched, and decode attention must be within max-abs 2e-3 / relative L2 1e-3 of the oracle.
"""
import math

import numpy as np
import pytest
import torch

from bit_kv_cache_prefill_b200 import inputs

import _harness as H
from test_gpu_parity import _inputs_for

pytestmark = pytest.mark.gpu

W = inputs.Workload
POOL_ARRAYS = ("k_codes", "v_codes", "k_scale", "k_zero", "v_scale", "v_zero")


def _gpu_pool(w, cache, num_pages, P, outliers):
    G = w.group_size
    views = {
        "k_codes": cache.view("k_codes", torch.int32).cpu().numpy().view(np.uint32).reshape(num_pages, P // 16, 64 * w.key_bits),
        "v_codes": cache.view("v_codes", torch.int32).cpu().numpy().view(np.uint32).reshape(num_pages, P // 16, 64 * w.value_bits),
        "k_scale": cache.view("k_scale", torch.int16).cpu().numpy().view(np.uint16).reshape(num_pages, P // G, 128),
        "k_zero": cache.view("k_zero", torch.int16).cpu().numpy().view(np.uint16).reshape(num_pages, P // G, 128),
        "v_scale": cache.view("v_scale", torch.int16).cpu().numpy().view(np.uint16).reshape(num_pages, P, 128 // G),
        "v_zero": cache.view("v_zero", torch.int16).cpu().numpy().view(np.uint16).reshape(num_pages, P, 128 // G),
    }
    if outliers:
        for n in ("k_out", "v_out"):
            words = cache.view(n, torch.int32).cpu().numpy().view(np.uint32).reshape(num_pages, P)
            views[n + "_ch"] = (words & 0xFFFF).astype(np.uint16)
            views[n + "_val"] = (words >> 16).astype(np.uint16)
    return views


def _run(w, lens, cap, P, num_pages, table, appends=0, outliers=0, sink=0, alloc=None):
    """GPU and oracle on the same inputs and page table; `alloc(table, T)` (if given) hands out the
    pages a quantized part of T tokens reaches before each call."""
    import bit_kv_cache_prefill_b200 as kvq
    import oracle

    lens = np.asarray(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    cfg = kvq.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.key_bits, w.value_bits, w.group_size, w.residual,
                          w.hadamard, cap, sink=sink, outliers=outliers, page_tokens=P, num_pages=num_pages)
    cache = kvq.Cache(cfg, page_table=table.copy())
    ocfg = oracle.Config(w.batch, w.num_q_heads, w.num_kv_heads, w.key_bits, w.value_bits, w.group_size, w.residual,
                         w.hadamard, cap, sink=sink, outliers=outliers, page_tokens=P, num_pages=num_pages)
    oc = oracle.Cache(ocfg, page_table=cache.page_table_host)  # the oracle reads the same table array
    if alloc:
        for b in range(w.batch):
            alloc(cache.page_table_host, b, int(lens[b]))
    kvq.kvq_quantize_prefill(cfg, cache, k.cuda(), v.cuda(), lens)
    oracle.quantize_prefill(ocfg, oc, k.numpy(), v.numpy(), lens)
    for s in range(appends):
        if alloc:
            for b in range(w.batch):
                alloc(cache.page_table_host, b, int(lens[b]) + s + 1)
        kn, vn = inputs.append_tokens(w, s)
        kvq.kvq_append_token(cfg, cache, kn.cuda(), vn.cuda())
        oracle.append_token(ocfg, oc, kn.numpy(), vn.numpy())
    ws = torch.empty(kvq.kvq_decode_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
    kvq.kvq_decode_attention(cfg, cache, q.cuda(), out, 1 / math.sqrt(128), ws)
    torch.cuda.synchronize()
    ref = oracle.decode(ocfg, oc, q.numpy(), 1 / math.sqrt(128), threads=8)
    return cache, oc, out.cpu().numpy(), ref


def _check_pool(w, cache, oc, num_pages, P, outliers, lens_final):
    gv = _gpu_pool(w, cache, num_pages, P, outliers)
    table = cache.page_table_host
    G, R = w.group_size, w.residual
    touched = set()
    for b in range(w.batch):
        Q = max(int(lens_final[b]) - R, 0) // G * G
        for h in range(w.num_kv_heads):
            for j in range(-(-Q // P)):
                p = int(table[b, h, j])
                touched.add(p)
                n = min(P, Q - j * P)  # quantized tokens of this page
                for name, rows in (("k_codes", n // 16), ("v_codes", n // 16), ("k_scale", n // G), ("k_zero", n // G),
                                   ("v_scale", n), ("v_zero", n)):
                    np.testing.assert_array_equal(gv[name][p, :rows], getattr(oc, name)[p, :rows],
                                                  err_msg=f"{name} unit {b},{h} page {j} (pool page {p})")
                if outliers:
                    for name in ("k_out_ch", "k_out_val", "v_out_ch", "v_out_val"):
                        np.testing.assert_array_equal(gv[name][p, :n], getattr(oc, name)[p, :n],
                                                      err_msg=f"{name} unit {b},{h} page {j}")
    for p in set(range(num_pages)) - touched:  # the cache buffers start zeroed; nothing may write a spare page
        for name in POOL_ARRAYS:
            assert not gv[name][p].any(), f"{name}: spare pool page {p} was written"


def _shuffled(B, H, M, n, seed=5):
    return np.random.default_rng(seed).permutation(n)[: B * H * M].astype(np.int32).reshape(B, H, M)


CASES = [
    # name, workload, lengths, P
    ("k2v2_g32_r32_mha_p128", W("p1", 2, 2, 2, 2, 2, 32, 32, 0, 1000, seed=71), [1000, 517], 128),
    ("k4v2_g32_r32_wht_gqa4_p256", W("p2", 2, 8, 2, 4, 2, 32, 32, 1, 1500, seed=72), [1500, 33], 256),
    ("k2v2_g128_r128_gqa4_p512", W("p3", 1, 4, 1, 2, 2, 128, 128, 0, 3000, seed=73), [3000], 512),
    ("k4v4_g16_r0_gqa2_p128", W("p4", 2, 4, 2, 4, 4, 16, 0, 0, 777, seed=74), [777, 16], 128),
]


@pytest.mark.parametrize("outliers,sink", [(0, 0), (1, 1)], ids=["plain", "outliers_sink"])
@pytest.mark.parametrize("name,w,lens,P", CASES, ids=[c[0] for c in CASES])
def test_paged_prefill_bit_exact_and_decode(oracle_mod, name, w, lens, P, outliers, sink):
    cap = -(-max(lens) // P) * P  # a whole number of pages
    M = cap // P
    num_pages = w.batch * w.num_kv_heads * M + 5
    table = _shuffled(w.batch, w.num_kv_heads, M, num_pages)
    cache, oc, out, ref = _run(w, lens, cap, P, num_pages, table, outliers=outliers, sink=sink)
    _check_pool(w, cache, oc, num_pages, P, outliers, lens)
    H.check_attention(out, ref, name + " paged")


@pytest.mark.parametrize("outliers", [0, 1])
def test_paged_streaming_with_pages_handed_out_on_demand(oracle_mod, outliers):
    """Pages are handed out only when a quantized part first reaches them; the appends cross several
    page boundaries, and the library refreshes the table's device mirror itself."""
    P, T0, n = 128, 100, 420
    w = W("p5", 2, 4, 2, 2, 2, 32, 32, 0, T0, seed=75)
    cap = -(-(T0 + n) // P) * P
    M = cap // P
    num_pages = w.batch * w.num_kv_heads * M + 3
    free = list(np.random.default_rng(9).permutation(num_pages))

    def alloc(table, b, T):
        Q = max(T - w.residual, 0) // w.group_size * w.group_size
        for h in range(w.num_kv_heads):
            for j in range(-(-Q // P)):
                if table[b, h, j] < 0:
                    table[b, h, j] = free.pop()

    table = np.full((w.batch, w.num_kv_heads, M), -1, np.int32)
    cache, oc, out, ref = _run(w, [T0, T0], cap, P, num_pages, table, appends=n, outliers=outliers, alloc=alloc)
    _check_pool(w, cache, oc, num_pages, P, outliers, [T0 + n, T0 + n])
    H.check_attention(out, ref, "paged streaming")
