"""GPU: the sequence lengths reach the device as kernel arguments, so a caller's host length array in
pinned memory, rewritten by the library at every append, is never read late by a queued copy.

The library updates ``seq_len_host`` on the calling thread; a queued host-to-device copy of it could
run after the next append's increment and see a length one ahead. These tests put the array in
pinned memory and issue prefill and appends back to back with no synchronisation in between.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

from bit_kv_cache_prefill_b200 import inputs

import _harness as H

pytestmark = pytest.mark.gpu


def _pin_lengths(cache):
    """Point the cache's host length mirror at pinned memory (kept alive on the cache object)."""
    pinned = torch.zeros(cache.cfg.batch, dtype=torch.int64).pin_memory()
    cache.pinned_lengths = pinned
    cache.seq_len_host = pinned.numpy()
    cache.c.seq_len_host = ctypes.cast(pinned.data_ptr(), ctypes.POINTER(ctypes.c_int64))


@pytest.mark.parametrize("appends", [1, 40], ids=["one_append", "flushes"])
def test_pinned_host_lengths_prefill_then_appends(oracle_mod, appends):
    import bit_kv_cache_prefill_b200 as kvq

    w = inputs.Workload("pin", 3, 4, 2, 2, 2, 32, 32, 0, 700, seed=71)
    lens = np.array([700, 301, 33], np.int64)
    k, v = _inputs(w, lens)
    cfg = H.gpu_config(w.scaled(appends=appends))
    cache = kvq.Cache(cfg)
    _pin_lengths(cache)
    toks = [tuple(t.cuda() for t in inputs.append_tokens(w, s)) for s in range(appends)]
    kd, vd = k.cuda(), v.cuda()
    torch.cuda.synchronize()
    kvq.kvq_quantize_prefill(cfg, cache, kd, vd, lens)  # no synchronisation until the decode is queued
    for kn, vn in toks:
        kvq.kvq_append_token(cfg, cache, kn, vn)
    q = inputs.query(w)
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
    ws = torch.empty(kvq.kvq_decode_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    kvq.kvq_decode_attention(cfg, cache, q.cuda(), out, 1 / math.sqrt(128), ws)
    torch.cuda.synchronize()
    assert (cache.seq_len_host == lens + appends).all()
    assert (cache.seq_len_dev.cpu().numpy() == lens + appends).all()
    oc, ref = H.oracle_full(oracle_mod, w.scaled(appends=appends), k, v, lens, q, appends=appends)
    run = H.DeviceRun(cfg, cache, out, lens + appends)
    gv = H.gpu_views(w.scaled(appends=appends), run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]) + appends)
    H.check_attention(out.cpu().numpy(), ref, "pinned lengths")


def test_more_sequences_than_one_length_chunk(oracle_mod):
    """Batch 300 > 256 sequences per by-value length chunk: prefill and append launch once per chunk,
    and every sequence's length and flush come out right."""
    import bit_kv_cache_prefill_b200 as kvq

    w = inputs.Workload("chunks", 300, 1, 1, 2, 2, 16, 16, 0, 64, seed=72)
    lens = (np.arange(300, dtype=np.int64) * 7) % 61 + 3
    k, v = _inputs(w, lens)
    appends = 20
    cfg = H.gpu_config(w.scaled(appends=appends))
    cache = kvq.Cache(cfg)
    kvq.kvq_quantize_prefill(cfg, cache, k.cuda(), v.cuda(), lens)
    for s in range(appends):
        kn, vn = inputs.append_tokens(w, s)
        kvq.kvq_append_token(cfg, cache, kn.cuda(), vn.cuda())
    torch.cuda.synchronize()
    assert (cache.seq_len_dev.cpu().numpy() == lens + appends).all()
    oc, _ = H.oracle_full(oracle_mod, w.scaled(appends=appends), k, v, lens, inputs.query(w), appends=appends)
    run = H.DeviceRun(cfg, cache, torch.empty(0), lens + appends)
    gv = H.gpu_views(w.scaled(appends=appends), run)
    for b in range(w.batch):
        H.compare_unit_cache(w, gv, b, 0, oc, b, 0, int(lens[b]) + appends)


@pytest.mark.parametrize("layout", [1, 2])
def test_compact_prefill_grid_over_chunks(oracle_mod, layout):
    """A ragged batch of 300 sequences (0 to 768 tokens, half of the plain grid past the sequences' ends):
    on the tile layout the prefill launches only the blocks that exist, 256 sequences per launch (the
    rows layout keeps the plain grid), and every unit's codes, parameters and ring match the oracle bit
    for bit; the decode over them matches too."""

    w = inputs.Workload("compact", 300, 4, 2, 2, 2, 32, 32, 0, 768, seed=73)
    lens = (np.arange(300, dtype=np.int64) * 97) % 701
    lens[::37] = 0
    lens[5] = 768  # the longest sequence sets the plain grid's width
    assert 4 * (300 * 6 - int(np.sum((lens + 127) // 128))) > 300 * 6  # the compact grid is chosen
    k, v = _inputs(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=layout)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=layout)
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]), layout=layout)
    H.check_attention(run.out.cpu().numpy(), ref, f"compact grid, layout {layout}")


def _inputs(w, lens):
    k = torch.zeros(w.batch, int(lens.max()), w.num_kv_heads, 128, dtype=torch.float16)
    v = torch.zeros_like(k)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            ku, vu = inputs.unit_kv(w, b, h, int(lens[b]))
            k[b, : lens[b], h] = ku
            v[b, : lens[b], h] = vu
    return k, v
