"""GPU parity with the dense-and-sparse outliers on (tile v1).

KVQuant review, Method: a small share of the entries is kept in fp16 beside the low-bit codes, chosen
per vector. With outliers = 1 every quantized token keeps the largest-magnitude entry of its key and of
its value (ties: the lowest channel) as (channel, fp16 value); that entry stays out of its group's
min / max and codes to 0, and a key channel whose entries in a group are all outliers gets scale and
zero 0. Everything the oracle defines (codes, scales, zeros, the outlier channel and value, the fp16
window) must match bit for bit, and decode attention within max-abs 2e-3 / relative L2 1e-3.
"""
import numpy as np
import pytest
import torch

from bit_kv_cache_prefill_b200 import inputs

import _harness as H
from test_gpu_parity import SMALL, _inputs_for, _lens_workload

pytestmark = pytest.mark.gpu

W = inputs.Workload

OUT_SMALL = [s for s in SMALL if s[0] in (
    "k2v2_g32_r32_mha", "k2v2_g64_r128_gqa4", "k4v2_g32_r32_wht_gqa4", "k2v2_g128_r128_gqa4", "k4v4_g16_r0_gqa2",
    "k2v4_g16_r5_wht_gqa3", "all_in_window", "r0_window_tail_mha")]


def _check_all(w, run, oc, lens, ref, what, sink=0):
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]), sink=sink, outliers=1)
    H.check_attention(run.out.cpu().numpy(), ref, what)
    return gv


@pytest.mark.parametrize("sink", [0, 1], ids=["nosink", "sink"])
@pytest.mark.parametrize("name,w,lens", OUT_SMALL, ids=[s[0] for s in OUT_SMALL])
def test_outliers_prefill_bit_exact_and_decode(oracle_mod, name, w, lens, sink):
    w = _lens_workload(w, lens)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, sink=sink, outliers=1)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, sink=sink, outliers=1)
    _check_all(w, run, oc, lens, ref, name + " outliers", sink)


@pytest.mark.parametrize("case", [
    dict(w=W("o1", 2, 8, 2, 2, 2, 32, 32, 0, 0, seed=61), T0=0, n=4 * 32 + 9, sink=0),
    dict(w=W("o2", 2, 4, 2, 4, 2, 16, 0, 1, 0, seed=62), T0=0, n=50, sink=1),
    dict(w=W("o3", 1, 2, 1, 2, 4, 32, 5, 1, 70, seed=63), T0=70, n=100, sink=0),
    dict(w=W("o4", 2, 4, 1, 4, 4, 64, 16, 0, 300, seed=64), T0=300, n=90, sink=1),
], ids=["from_empty_g32_r32", "from_empty_g16_r0_wht_sink", "prefill_then_append_wht", "g64_gqa4_sink"])
def test_outliers_streaming_matches_oracle(oracle_mod, case):
    w, T0, n, sink = case["w"], case["T0"], case["n"], case["sink"]
    w = w.scaled(seq_len=T0, appends=n)
    lens = np.full(w.batch, T0, np.int64)
    k, v = _inputs_for(w, list(lens))
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, appends=n, sink=sink, outliers=1)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, appends=n, sink=sink, outliers=1)
    _check_all(w, run, oc, lens + n, ref, "outliers streaming", sink)


def test_outliers_all_in_one_key_channel_get_zero_parameters(oracle_mod):
    """A massive key channel holds every token's outlier: each of its key groups has no other entry,
    so its scale and zero are 0; every other channel's parameters and all codes still match."""
    w = W("o5", 2, 4, 2, 2, 2, 32, 32, 0, 700, seed=65)
    lens = np.array([700, 333], np.int64)
    k, v = _inputs_for(w, lens)
    t = torch.arange(k.shape[1], dtype=torch.float32)
    k[:, :, :, 37] = (300.0 + (t % 17))[None, :, None].to(torch.float16)  # far above the other channels
    v[:, :, :, 100] = (-250.0 - (t % 5))[None, :, None].to(torch.float16)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, outliers=1)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, outliers=1)
    gv = _check_all(w, run, oc, lens, ref, "massive channel")
    Q = (700 - 32) // 32 * 32
    assert (gv["k_out_ch"][0, :, :Q] == 37).all() and (gv["v_out_ch"][0, :, :Q] == 100).all()
    pos37 = 32 * ((37 & 7) >> 1) + 4 * (37 >> 4) + 2 * ((37 & 15) >> 3) + (37 & 1)  # tile-v1 parameter slot
    assert (gv["k_scale"][0, :, : Q // 32, pos37] == 0).all() and (gv["k_zero"][0, :, : Q // 32, pos37] == 0).all()


def test_outlier_ties_go_to_the_lowest_channel(oracle_mod):
    """Rows whose largest magnitude appears several times (with either sign) pick the lowest channel."""
    w = W("o6", 1, 2, 1, 2, 2, 32, 0, 0, 256, seed=66)
    lens = np.array([256], np.int64)
    k, v = _inputs_for(w, lens)
    g = torch.Generator().manual_seed(5)
    for tt in range(256):
        chans = torch.randperm(128, generator=g)[:3]
        k[0, tt, 0, chans] = torch.tensor([8.0, -8.0, 8.0], dtype=torch.float16)
        v[0, tt, 0, chans] = torch.tensor([-6.0, 6.0, -6.0], dtype=torch.float16)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, outliers=1)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, outliers=1)
    gv = _check_all(w, run, oc, lens, ref, "ties")
    kk = k[0, :, 0].numpy().view(np.uint16) & 0x7FFF
    assert (gv["k_out_ch"][0, 0, :256] == kk.argmax(axis=1)).all()  # argmax returns the first maximum


def test_outliers_off_leaves_the_cache_unchanged(oracle_mod):
    """outliers = 0 must give the same bytes as before the option existed (the oracle without it)."""
    name, w, lens = OUT_SMALL[0]
    w = _lens_workload(w, lens)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, outliers=0)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, outliers=0)
    gv = H.gpu_views(w, run)
    assert "k_out_ch" not in gv
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]))
    H.check_attention(run.out.cpu().numpy(), ref, name)
