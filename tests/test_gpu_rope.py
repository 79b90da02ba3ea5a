"""GPU parity with pre-RoPE keys: keys are cached (and quantized) before RoPE and decode rotates each
dequantized key at its position (KVQuant review, Method and Key idea).

The cache bits must match the oracle exactly (quantization does not see the rotation), and decode
attention must be within max-abs 2e-3 / relative L2 1e-3 of the oracle's fp64 result, which applies
RoPE in fp64. Covers MHA and GQA, 2- and 4-bit codes, G = 16 .. 128, the sink token, the FP16 window
and streaming appends, on the rows-v2 layout (the one RoPE decode supports).
"""
import numpy as np
import pytest

from bit_kv_cache_prefill_b200 import inputs

import _harness as H
from test_gpu_parity import _inputs_for, _lens_workload

pytestmark = pytest.mark.gpu

W = inputs.Workload

CASES = [
    # name, workload, lengths, theta, sink
    ("k2v2_g32_r32_mha", W("r1", 2, 2, 2, 2, 2, 32, 32, 0, 1000, seed=71, outlier_channels=4,
                           outlier_per_head=True, outlier_scale=20.0), [1000, 517], 10000.0, 0),
    ("k2v2_g64_r128_gqa4", W("r2", 2, 8, 2, 2, 2, 64, 128, 0, 2125, seed=72), [2125, 300], 500000.0, 0),
    ("k4v2_g32_r32_gqa4_sink", W("r3", 3, 8, 2, 4, 2, 32, 32, 0, 1500, seed=73), [1500, 33, 0], 10000.0, 1),
    ("k2v4_g16_r5_gqa3", W("r4", 2, 6, 2, 2, 4, 16, 5, 0, 401, seed=74), [401, 1], 1000000.0, 0),
    ("k4v4_g128_r0_gqa2", W("r5", 1, 4, 2, 4, 4, 128, 0, 0, 3000, seed=75), [3000], 10000.0, 1),
    ("all_in_window", W("r6", 2, 4, 1, 2, 2, 32, 256, 0, 200, seed=76), [200, 256], 10000.0, 0),
    # 2-bit values (P.V on the tensor cores) at every group size and head ratio: n-blocks of 4, 2 and 1
    # value groups, channel tiles of one group (G = 16) up to one group per 8 tiles (G = 128)
    ("k2v2_g16_r16_gqa2", W("r7", 2, 4, 2, 2, 2, 16, 16, 0, 700, seed=77), [700, 129], 10000.0, 0),
    ("k2v2_g128_r64_mha", W("r8", 1, 2, 2, 2, 2, 128, 64, 0, 1500, seed=78), [1500], 10000.0, 1),
    ("k4v2_g64_r32_gqa2", W("r9", 2, 4, 2, 4, 2, 64, 32, 0, 1100, seed=79), [1100, 97], 500000.0, 0),
    ("k2v2_g16_r0_mha_ragged", W("r10", 3, 2, 2, 2, 2, 16, 0, 0, 333, seed=80), [333, 31, 65], 10000.0, 1),
]


@pytest.mark.parametrize("name,w,lens,theta,sink", CASES, ids=[c[0] for c in CASES])
def test_rope_prefill_bit_exact_and_decode(oracle_mod, name, w, lens, theta, sink):
    w = _lens_workload(w, lens)
    lens = np.array(lens, np.int64)
    k, v = _inputs_for(w, lens)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=2, sink=sink, rope=theta)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, layout=2, sink=sink, rope=theta)
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, int(lens[b]), layout=2, sink=sink)
    H.check_attention(run.out.cpu().numpy(), ref, name + " rope")


@pytest.mark.parametrize("sink", [0, 1])
def test_rope_streaming_matches_oracle(oracle_mod, sink):
    w = W("rs", 2, 8, 2, 2, 2, 32, 32, 0, 300, seed=77).scaled(seq_len=300, appends=3 * 32 + 7)
    n = w.appends
    lens = np.full(w.batch, 300, np.int64)
    k, v = _inputs_for(w, list(lens))
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, appends=n, layout=2, sink=sink, rope=10000.0)
    oc, ref = H.oracle_full(oracle_mod, w, k, v, lens, q, appends=n, layout=2, sink=sink, rope=10000.0)
    gv = H.gpu_views(w, run)
    for b in range(w.batch):
        for h in range(w.num_kv_heads):
            H.compare_unit_cache(w, gv, b, h, oc, b, h, 300 + n, layout=2, sink=sink)
    H.check_attention(run.out.cpu().numpy(), ref, "rope streaming")


def test_rope_long_context_sampled_units(oracle_mod):
    """A 64K-token sequence (positions far into the angle range, many splits): sampled units against
    the oracle's per-unit decode."""
    w = W("rl", 1, 8, 2, 2, 2, 64, 128, 0, 65536, seed=78)
    k, v, lens = inputs.full_kv(w)
    q = inputs.query(w)
    run = H.run_gpu(w, k.cuda(), v.cuda(), lens, q, layout=2, rope=500000.0)
    out = run.out.cpu().numpy()
    for h in range(w.num_kv_heads):
        ocfg = H.oracle_config(oracle_mod, w, batch=1, hq=w.gqa, hkv=1, layout=2, rope=500000.0)
        oc = oracle_mod.Cache(ocfg)
        ku, vu = inputs.unit_kv(w, 0, h, int(lens[0]))
        oracle_mod.quantize_prefill(ocfg, oc, ku.numpy()[None, :, None, :], vu.numpy()[None, :, None, :], [int(lens[0])])
        qq = q[0:1, h * w.gqa:(h + 1) * w.gqa].contiguous().numpy()
        ref = oracle_mod.decode(ocfg, oc, qq, 1 / np.sqrt(128), threads=8)[0]
        H.check_attention(out[0, h * w.gqa:(h + 1) * w.gqa], ref, f"rope 64K unit {h}")
