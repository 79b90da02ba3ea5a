"""GPU parity with the attention sink on: the first token of every sequence stays in fp16.

KVQuant review, Method: the first token is kept in full precision. With the sink on, key group 0's
min/max leave token 0 out, token 0's codes and value scale / zero are 0, its fp16 key and value sit in
ring row R + G, and decode reads token 0 from that row only. Everything the oracle defines must match
bit for bit, and decode attention within max-abs 2e-3 / relative L2 1e-3 of the oracle.
"""
import numpy as np
import pytest
import torch

from bit_kv_cache_prefill_b200 import inputs

import _harness as H
from test_gpu_parity import LAYOUTS, SMALL, _inputs_for, _lens_workload

pytestmark = pytest.mark.gpu

W = inputs.Workload

# prefill cases: several groups and tiles, ragged tails, a one-token sequence, an empty one, R = 0 with
# Q = G (the sink group alone), everything in the window
SINK_SMALL = [s for s in SMALL if s[0] in (
    "k2v2_g32_r32_mha", "k4v2_g32_r32_wht_gqa4", "k4v4_g16_r0_gqa2", "k2v4_g16_r5_wht_gqa3", "all_in_window",
    "r0_window_tail_mha", "k2v2_g128_r128_gqa4")]


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
@pytest.mark.parametrize("name,w,lens", SINK_SMALL, ids=[s[0] for s in SINK_SMALL])
def test_sink_prefill_bit_exact_and_decode(oracle_mod, name, w, lens, layout):
    w = _lens_workload(w, lens)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=layout, sink=1)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=layout, sink=1)
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]), layout=layout, sink=1)
    H.check_attention(run.out.cpu().numpy(), ref, name + " sink")


@pytest.mark.parametrize("case", [
    dict(w=W("e1", 2, 8, 2, 2, 2, 32, 32, 0, 0, seed=41), T0=0, n=4 * 32 + 9),
    dict(w=W("e2", 2, 4, 2, 4, 2, 16, 0, 1, 0, seed=42), T0=0, n=50),
    dict(w=W("e3", 1, 2, 1, 2, 4, 32, 5, 1, 70, seed=43), T0=70, n=100),
], ids=["from_empty_g32_r32", "from_empty_g16_r0_wht", "prefill_then_append_wht"])
@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
def test_sink_streaming_matches_oracle(oracle_mod, case, layout):
    w, T0, n = case["w"], case["T0"], case["n"]
    w = w.scaled(seq_len=T0, appends=n)
    lens = np.full(w.batch, T0, np.int64)
    k, v = _inputs_for(w, list(lens))
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, appends=n, layout=layout, sink=1)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, appends=n, layout=layout, sink=1)
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, T0 + n, layout=layout, sink=1)
    H.check_attention(run.out.cpu().numpy(), ref, "sink streaming")


@pytest.mark.parametrize("layout", LAYOUTS, ids=["tile_v1", "rows_v2"])
def test_sink_off_and_on_differ_only_by_token_zero(oracle_mod, layout):
    """A huge first key shifts group 0's range with the sink off; with it on, the other tokens' codes
    equal those of a prefill where token 0 is replaced by a copy of token 1 (an in-range value)."""
    w = W("d1", 1, 2, 1, 2, 2, 32, 32, 0, 300, seed=44)
    lens = np.array([300], np.int64)
    k, v = _inputs_for(w, [300])
    k[0, 0] = 500.0  # far outside the other keys' range
    v[0, 0] = 1.5
    q = inputs.query(w)
    on = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=layout, sink=1)
    k2, v2 = k.clone(), v.clone()
    k2[0, 0], v2[0, 0] = k[0, 1], v[0, 1]
    ref = H.run_gpu(w, k2.cuda(), v2.cuda(), lens, q, layout=layout, sink=0, decode=False)
    g_on, g_ref = H.gpu_views(w, on), H.gpu_views(w, ref)
    # group 0 statistics: token 0 is left out, token 1 duplicated changes nothing
    np.testing.assert_array_equal(g_on["k_scale"][0, 0, 0], g_ref["k_scale"][0, 0, 0])
    np.testing.assert_array_equal(g_on["k_zero"][0, 0, 0], g_ref["k_zero"][0, 0, 0])
    np.testing.assert_array_equal(g_on["v_scale"][0, 0, 1:256], g_ref["v_scale"][0, 0, 1:256])
    assert np.all(g_on["v_scale"][0, 0, 0] == 0) and np.all(g_on["v_zero"][0, 0, 0] == 0)
    if layout == 2:  # token rows: tokens 1 .. 255 code alike, token 0 codes to 0
        np.testing.assert_array_equal(g_on["k_codes"][0, 0, 1:256], g_ref["k_codes"][0, 0, 1:256])
        assert np.all(g_on["k_codes"][0, 0, 0] == 0)
    # the sink row holds the fp16 first token
    ring = w.residual + w.group_size
    np.testing.assert_array_equal(g_on["k_res"][0, 0, ring], k[0, 0, 0].numpy().view(np.uint16))
    np.testing.assert_array_equal(g_on["v_res"][0, 0, ring], v[0, 0, 0].numpy().view(np.uint16))
    oc, ref_out = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=layout, sink=1)
    H.check_attention(on.out.cpu().numpy(), ref_out, "dominant sink")
