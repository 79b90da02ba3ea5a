"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on the same seeded inputs.

Codes, scales, zero-points and the FP16 ring must match bit for bit; decode attention must be within
max-abs 2e-3 and relative L2 1e-3 of the oracle's fp64 result. Small cases span several 16-token
tiles, several key groups, ragged tails and the edge cases (empty sequence, one token, everything in
the FP16 window, R = 0, flush boundaries); the model-shaped workloads run at full size with the
oracle checking sampled (sequence, KV head) units.
"""
import math
import os

import numpy as np
import pytest
import torch

from bit_kv_cache_prefill_b200 import inputs

import _harness as H

pytestmark = pytest.mark.gpu

W = inputs.Workload

SMALL = [
    # name, workload, lengths
    ("k2v2_g32_r32_mha", W("t1", 2, 2, 2, 2, 2, 32, 32, 0, 1000, seed=11, outlier_channels=4,
                           outlier_per_head=True, outlier_scale=20.0), [1000, 517]),
    ("k2v2_g64_r128_gqa4", W("t2", 2, 8, 2, 2, 2, 64, 128, 0, 2125, seed=12), [2125, 300]),
    ("k4v2_g32_r32_wht_gqa4", W("t3", 3, 8, 2, 4, 2, 32, 32, 1, 1500, seed=13, outlier_channels=8,
                                outlier_per_head=False, outlier_scale=15.0), [1500, 33, 0]),
    ("k2v2_g128_r128_gqa4", W("t4", 1, 4, 1, 2, 2, 128, 128, 0, 3000, seed=14), [3000]),
    ("k4v4_g16_r0_gqa2", W("t5", 2, 4, 2, 4, 4, 16, 0, 0, 777, seed=15), [777, 16]),
    ("k2v4_g16_r5_wht_gqa3", W("t6", 2, 6, 2, 2, 4, 16, 5, 1, 401, seed=16), [401, 1]),
    ("all_in_window", W("t7", 2, 4, 1, 2, 2, 32, 256, 0, 200, seed=17), [200, 256]),
    # R = 0 with a partial group in the window: splits whose range is all window can get no token
    ("r0_window_tail_mha", W("t8", 2, 2, 2, 2, 2, 32, 0, 0, 777, seed=18), [777, 40]),
    ("r0_window_tail_gqa4_g16", W("t9", 1, 8, 2, 4, 2, 16, 0, 1, 1000, seed=19), [1000]),
]


def _lens_workload(w, lens):
    # capacity from the given lengths (round up to G)
    return w.scaled(seq_len=max(lens) if max(lens) > 0 else w.group_size)


def _inputs_for(w, lens):
    B = w.batch
    Tmax = max(max(lens), 1)
    k = torch.zeros(B, Tmax, w.num_kv_heads, 128, dtype=torch.float16)
    v = torch.zeros_like(k)
    mask = inputs.outlier_mask(w)
    for b in range(B):
        for h in range(w.num_kv_heads):
            if lens[b] > 0:
                ku, vu = inputs.unit_kv(w, b, h, lens[b], mask)
                k[b, : lens[b], h] = ku
                v[b, : lens[b], h] = vu
    return k, v


LAYOUTS = [1, 2]  # tile v1 (mma.sync kernel), rows v2 (tcgen05 kernel)


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
@pytest.mark.parametrize("name,w,lens", SMALL, ids=[s[0] for s in SMALL])
def test_small_prefill_bit_exact_and_decode(oracle_mod, name, w, lens, layout):
    w = _lens_workload(w, lens)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=layout)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=layout)
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]), layout=layout)
    H.check_attention(run.out.cpu().numpy(), ref, name)
    # empty sequences decode to exact zeros
    for b in range(w.batch):
        if lens[b] == 0:
            assert np.all(run.out[b].cpu().numpy() == 0)


@pytest.mark.parametrize("case", [
    dict(w=W("s1", 2, 8, 2, 2, 2, 32, 32, 0, 300, seed=21), T0=300, n=3 * 32 + 7),
    dict(w=W("s2", 2, 2, 2, 4, 2, 16, 0, 1, 100, seed=22), T0=100, n=40),
    dict(w=W("s3", 1, 4, 1, 2, 2, 64, 128, 0, 10, seed=23), T0=10, n=200),
], ids=["g32_r32_gqa4", "g16_r0_wht", "g64_r128_from_window"])
@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
def test_streaming_append_matches_oracle_and_bulk_prefill(oracle_mod, case, layout):
    w, T0, n = case["w"], case["T0"], case["n"]
    w = w.scaled(seq_len=T0, appends=n)
    lens = np.full(w.batch, T0, np.int64)
    k, v = _inputs_for(w, list(lens))
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, appends=n, layout=layout)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, appends=n, layout=layout)
    gv = H.gpu_views(w, run)
    assert np.array_equal(run.cache.seq_len_host, lens + n)
    assert np.array_equal(run.cache.seq_len_dev.cpu().numpy(), lens + n)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, T0 + n, layout=layout)
    H.check_attention(run.out.cpu().numpy(), ref, "streaming")
    # the GPU's own bulk prefill of all T0 + n tokens gives the same defined bits
    kk = torch.zeros(w.batch, T0 + n, w.num_kv_heads, 128, dtype=torch.float16)
    vv = torch.zeros_like(kk)
    kk[:, :T0], vv[:, :T0] = k, v
    for s in range(n):
        kn, vn = inputs.append_tokens(w, s)
        kk[:, T0 + s], vv[:, T0 + s] = kn, vn
    bulk = H.run_gpu(w, kk.cuda(), vv.cuda(), np.full(w.batch, T0 + n, np.int64), q, layout=layout)
    gb = H.gpu_views(w, bulk)
    G, R = w.group_size, w.residual
    T = T0 + n
    Q = max(T - R, 0) // G * G
    live = [t % (R + G) for t in range(Q, T)]
    if layout == 2:
        np.testing.assert_array_equal(gv["k_codes"][:, :, :Q], gb["k_codes"][:, :, :Q])
        nb, rem = divmod(Q, 128)
        np.testing.assert_array_equal(gv["v_codes"][:, :, :nb], gb["v_codes"][:, :, :nb])
        words = rem * w.value_bits // 32
        np.testing.assert_array_equal(gv["v_codes"][:, :, nb:nb + 1, :, :words], gb["v_codes"][:, :, nb:nb + 1, :, :words])
    else:
        for key in ("k_codes", "v_codes"):
            np.testing.assert_array_equal(gv[key][:, :, : Q // 16], gb[key][:, :, : Q // 16])
    for key in ("k_scale", "k_zero"):
        np.testing.assert_array_equal(gv[key][:, :, : Q // G], gb[key][:, :, : Q // G])
    for key in ("v_scale", "v_zero"):
        np.testing.assert_array_equal(gv[key][:, :, :Q], gb[key][:, :, :Q])
    for key in ("k_res", "v_res"):
        np.testing.assert_array_equal(gv[key][:, :, live], gb[key][:, :, live])
    np.testing.assert_array_equal(run.out.cpu().numpy(), bulk.out.cpu().numpy())


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
def test_sm_scale_and_single_token(oracle_mod, layout):
    w = W("one", 1, 4, 1, 2, 2, 32, 4, 0, 1, seed=31)
    lens = np.array([1], np.int64)
    k, v = _inputs_for(w, [1])
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, sm_scale=0.37, layout=layout)
    # one token: every head returns that token's value exactly (as fp16)
    for h in range(4):
        np.testing.assert_array_equal(run.out[0, h].cpu().numpy(), v[0, 0, 0].numpy())
    w2 = W("scl", 1, 4, 1, 2, 2, 32, 32, 0, 700, seed=32)
    k2, v2 = _inputs_for(w2, [700])
    q2 = inputs.query(w2)
    run2 = H.run_gpu(w2, k2.cuda(), v2.cuda(), np.array([700]), q2, sm_scale=0.02, layout=layout)
    _, ref2 = H.oracle_full(oracle_mod, w2, k2, v2, np.array([700]), q2, sm_scale=0.02)
    H.check_attention(run2.out.cpu().numpy(), ref2, "sm_scale 0.02")


# ---- model-shaped workloads at full size, in the launch configuration the bench uses: the oracle
#      runs the whole workload (multi-threaded) and every unit's cache and every output is compared
FULL = ["tiny", "llama2_7b_mha", "llama3_8b_gqa", "mistral_7b_ragged", "million_token"]


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
@pytest.mark.parametrize("name", FULL)
def test_full_size_workload_every_unit(oracle_mod, name, layout):
    w = inputs.WORKLOADS[name]
    k, v, lens = inputs.full_kv(w)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, appends=w.appends, layout=layout)
    gv = H.gpu_views(w, run)
    out = run.out.cpu().numpy()
    threads = len(os.sched_getaffinity(0))
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, appends=w.appends, layout=layout, threads=threads)
    del k, v
    units = 0
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]) + w.appends, layout=layout)
            units += 1
    assert units == w.batch * w.num_kv_heads
    H.check_attention(out, ref, f"{name}, all {w.batch * w.num_q_heads} query heads")
    assert np.array_equal(run.cache.seq_len_host, lens + w.appends)


def _signed_zero_kv(w, T, seed):
    """K/V of one sequence where many groups have a signed zero as min or max (random zero signs)."""
    rng = np.random.default_rng(seed)
    H = w.num_kv_heads

    def zeros(shape):
        return rng.choice(np.array([0x0000, 0x8000], np.uint16), size=shape)

    base = rng.standard_normal((T, H, 128)).astype(np.float16)
    k = base.view(np.uint16).copy()
    pos = np.abs(base).view(np.uint16)              # non-negative values
    neg = (-np.abs(base)).view(np.uint16)           # non-positive values
    zmask = rng.random((T, H, 128)) < 0.3
    # keys (per channel over tokens): a zero mix; zeros + positives (min a zero); zeros + negatives
    # (max a zero); only -0; only +0
    k[:, :, 0:16] = zeros((T, H, 16))
    k[:, :, 16:32] = np.where(zmask[:, :, 16:32], zeros((T, H, 16)), pos[:, :, 16:32])
    k[:, :, 32:48] = np.where(zmask[:, :, 32:48], zeros((T, H, 16)), neg[:, :, 32:48])
    k[:, :, 48:56] = 0x8000
    k[:, :, 56:64] = 0x0000
    # values (per token over channels): whole rows of zeros, zeros + positives, zeros + negatives
    v = rng.standard_normal((T, H, 128)).astype(np.float16).view(np.uint16).copy()
    vpos = np.abs(v.view(np.float16)).view(np.uint16)
    vneg = (-np.abs(v.view(np.float16))).view(np.uint16)
    sel = np.arange(T) % 4
    v[sel == 0] = zeros(((sel == 0).sum(), H, 128))
    v[sel == 1] = np.where(rng.random(((sel == 1).sum(), H, 128)) < 0.3, zeros(((sel == 1).sum(), H, 128)), vpos[sel == 1])
    v[sel == 2] = np.where(rng.random(((sel == 2).sum(), H, 128)) < 0.3, zeros(((sel == 2).sum(), H, 128)), vneg[sel == 2])
    kt = torch.from_numpy(k.view(np.float16)).unsqueeze(0).contiguous()
    vt = torch.from_numpy(v.view(np.float16)).unsqueeze(0).contiguous()
    return kt, vt


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
@pytest.mark.parametrize("G", [16, 32, 128])
def test_signed_zero_groups_bit_exact(oracle_mod, layout, G):
    """Groups whose min or max is -0 or +0 (the total order puts -0 below +0) match the oracle bit for
    bit, on every layout and with G = 16, 32 and 128."""
    T = 300
    w = W("z", 1, 4, 2, 2, 2, G, 8, 0, T, seed=51).scaled(seq_len=T)
    lens = np.array([T], np.int64)
    k, v = _signed_zero_kv(w, T, seed=G)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=layout)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=layout)
    gv = H.gpu_views(w, run)
    for h in range(w.num_kv_heads):
        H.compare_unit_cache(w, gv, 0, h, oc, 0, h, T, layout=layout)
    # rows v2 keeps key parameters in channel order: the all -0 channels have zero-point -0, the
    # all +0 ones +0
    if layout == 2:
        kz = gv["k_zero"][0, :, : (T - w.residual) // G]
        assert np.all(kz[:, :, 48:56] == 0x8000) and np.all(kz[:, :, 56:64] == 0x0000)
    H.check_attention(run.out.cpu().numpy(), ref, f"signed zeros G={G}")


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
def test_decode_status_is_ok_after_a_decode_that_finishes(layout):
    """kvq_decode_status reads the per-(sequence, query head) records the split combine writes at the
    end of the workspace: all clear after a decode whose kernels never gave up a wait (including a
    sequence of length 0)."""
    import bit_kv_cache_prefill_b200 as kvq

    name, w, lens = SMALL[2]
    w = _lens_workload(w, lens)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    cfg = H.gpu_config(w, layout)
    cache = kvq.Cache(cfg)
    kvq.kvq_quantize_prefill(cfg, cache, k.cuda(), v.cuda(), lens)
    ws = torch.full((kvq.kvq_decode_workspace_bytes(cfg),), 0xFF, dtype=torch.uint8, device="cuda")  # stale bits
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
    kvq.kvq_decode_attention(cfg, cache, inputs.query(w).cuda(), out, 1 / math.sqrt(128), ws)
    assert kvq.kvq_decode_status(cfg, ws) == kvq.KVQ_OK
    assert torch.isfinite(out.float()).all()


def test_tcgen05_bounded_wait_gives_up_and_reports(oracle_mod, monkeypatch):
    """KVQ_TEST_STALL_TC=1 makes one thread of every tcgen05 decode CTA wait on a barrier phase that
    nothing completes, with no copy and no MMA in flight (the CTA issues no quantized step): the bounded
    wait gives up after about 2 s, the outputs are NaN and kvq_decode_status reports KVQ_ERR_TIMEOUT.
    The next decode on the same context and workspace is correct and reports KVQ_OK."""
    import bit_kv_cache_prefill_b200 as kvq

    w = inputs.Workload("stall", 1, 4, 1, 2, 2, 32, 32, 0, 640, seed=91)
    lens = np.array([640], np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    cfg = H.gpu_config(w, 2)
    cache = kvq.Cache(cfg)
    kvq.kvq_quantize_prefill(cfg, cache, k.cuda(), v.cuda(), lens)
    ws = torch.zeros(kvq.kvq_decode_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
    monkeypatch.setenv("KVQ_TEST_STALL_TC", "1")
    kvq.kvq_decode_attention(cfg, cache, q.cuda(), out, 1 / math.sqrt(128), ws)
    assert kvq.kvq_decode_status(cfg, ws) == kvq.KVQ_ERR_TIMEOUT
    assert torch.isnan(out.float()).all()
    monkeypatch.delenv("KVQ_TEST_STALL_TC")
    kvq.kvq_decode_attention(cfg, cache, q.cuda(), out, 1 / math.sqrt(128), ws)
    assert kvq.kvq_decode_status(cfg, ws) == kvq.KVQ_OK
    _, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=2)
    H.check_attention(out.cpu().numpy(), ref, "decode after a give-up")


@pytest.mark.parametrize("sink", [0, 1], ids=["nosink", "sink"])
@pytest.mark.parametrize("name,w,lens", [c for c in SMALL if not c[1].hadamard][:6], ids=lambda x: x if isinstance(x, str) else "")
def test_cuda_core_control_matches_the_oracle(oracle_mod, monkeypatch, name, w, lens, sink):
    """KVQ_DECODE_CUDA_CORES=1 runs the CUDA-core control decode (the pre-RoPE kernel without its
    rotations) on a rows-v2 cache in place of the tcgen05 kernel: same outputs within tolerance."""
    monkeypatch.setenv("KVQ_DECODE_CUDA_CORES", "1")
    w = _lens_workload(w, lens).scaled(appends=3)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, appends=3, layout=2, sink=sink)
    _, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, appends=3, layout=2, sink=sink)
    H.check_attention(run.out.cpu().numpy(), ref, f"CUDA-core control {name}")
