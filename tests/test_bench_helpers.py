"""CPU checks of bench.py's accounting: the algorithmic byte counts behind every GB/s figure, the
rank reduction's inputs, and the committed-counter lookup that fills roofline.traffic."""
import json
import os

import numpy as np

import bench
from bit_kv_cache_prefill_b200 import inputs


def test_decode_bytes_closed_form():
    # llama2_7b_mha: 8 sequences x 32 heads x 32768 tokens, 2/2-bit, G = 32, R = 128
    w = inputs.WORKLOADS["llama2_7b_mha"]
    T, G, R = 32768, 32, 128
    Q = (T - R) // G * G
    per_unit = Q * 128 * 4 // 8 + (Q // G) * 128 * 4 + Q * (128 // G) * 4 + (T - Q) * 128 * 4
    want = 8 * 32 * per_unit + 2 * 8 * 32 * 128 * 2
    assert bench.decode_bytes(w, np.full(8, T)) == want
    assert abs(want / 1e6 - 819) < 1  # 819 MB per call
    # the sink adds the first token's fp16 key and value row once a group is quantized
    assert bench.decode_bytes(w, np.full(8, T), sink=1) == want + 8 * 32 * 512
    assert bench.decode_bytes(w, np.full(8, 100), sink=1) == bench.decode_bytes(w, np.full(8, 100))
    # outliers: a 4-byte key and a 4-byte value word per quantized token
    Q = (T - w.residual) // w.group_size * w.group_size
    assert bench.decode_bytes(w, np.full(8, T), outliers=1) == want + 8 * w.num_kv_heads * Q * 8


def test_prefill_bytes_closed_form():
    w = inputs.WORKLOADS["million_token"]
    T, G, R = 1 << 20, 128, 128
    Q = (T - R) // G * G
    per_unit = T * 128 * 4 + Q * 128 * 4 // 8 + (Q // G) * 128 * 4 + Q * (128 // G) * 4 + (T - Q) * 128 * 4
    assert bench.prefill_bytes(w, np.array([T])) == 8 * per_unit
    assert bench.prefill_bytes(w, np.array([T]), sink=1) == 8 * (per_unit + 512)


def _sources_hash(root, files):
    import hashlib
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(root, f), "rb").read())
    return h.hexdigest()


def test_traffic_counters_are_used_only_while_their_sources_match():
    # every committed counter names its workload, kernel sources and their hash; a record is used only
    # while the hash matches (else the traffic is null), and it scales by the units processed (or, for a
    # capture at a reduced length, by the (token, KV head) pairs)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    entries = json.load(open(os.path.join(root, "profiles", "decode_traffic_counters.txt")))
    assert {"decode", "prefill"} <= {e.get("kind", "decode") for e in entries.values()}
    for e in entries.values():
        kind = e.get("kind", "decode")
        w = inputs.WORKLOADS[e["workload"]]
        got = bench.measured_traffic(w, e["layout"], kind)
        if _sources_hash(root, e["kernel_sources"]) != e["sources_sha256"]:
            assert got is None  # the kernel changed since the capture
            continue
        if "capture_tokens" in e:
            scale = float(np.sum(w.seq_lens())) * w.num_kv_heads / e["capture_tokens"]
        else:
            scale = w.batch * w.num_kv_heads / e["capture_units"]
        assert got == round((e["dram_read_bytes"] + e["dram_write_bytes"]) * scale)
        # the captured DRAM bytes stay within a few percent of the algorithmic bytes of the workload
        lens = w.seq_lens()
        algorithmic = bench.decode_bytes(w, lens + w.appends) if kind == "decode" else bench.prefill_bytes(w, lens)
        assert 0.95 < got / algorithmic < 1.06, (e["workload"], kind, got / algorithmic)


def test_traffic_lookup_is_none_for_other_layouts_and_kernels():
    w = inputs.WORKLOADS["llama2_7b_mha"]
    assert bench.measured_traffic(w, 2, "decode") is None
    assert bench.measured_traffic(inputs.WORKLOADS["tiny"], 1, "decode") is None
    # the records were taken with the sink and RoPE off: other options get no traffic figure
    assert bench.measured_traffic(w, 1, "decode", sink=1) is None
    assert bench.measured_traffic(inputs.WORKLOADS["llama3_8b_gqa"], 1, "prefill", sink=1) is None
    assert bench.measured_traffic(w, 2, "decode", rope=10000.0) is None


def test_flush_steps_and_scanned_tokens():
    # G = 32, R = 128: from T = 160 (Q = 32) the append that makes T = 192 flushes (Q 32 -> 64), then
    # every 32nd append; with ragged lengths any sequence's flush counts
    w = inputs.WORKLOADS["llama2_7b_mha"].scaled(batch=2)
    flags = bench.flush_steps(w, np.array([160, 160]), 70)
    assert [i for i, f in enumerate(flags) if f] == [31, 63]
    flags = bench.flush_steps(w, np.array([160, 170]), 40)
    assert [i for i, f in enumerate(flags) if f] == [21, 31]
    assert not any(bench.flush_steps(w, np.array([10, 20]), 100))  # still inside the window (T < R + G)
    assert bench.kv_tokens(w, np.array([100, 200])) == 300 * w.num_kv_heads


def test_oracle_sample_reports_one_thread_time():
    res = bench.oracle_decode_sample(inputs.WORKLOADS["tiny"], budget_s=0.05, single_thread_s=0.01)
    assert res.gbs > 0 and res.threads >= 1 and res.single_thread_gbs > 0 and "one thread" in res.sample
    assert res.prefill_gbs > 0
    assert bench.oracle_decode_sample(inputs.WORKLOADS["tiny"], budget_s=0.01).single_thread_gbs is None


def test_reference_arm_prints_one_line(capsys, monkeypatch):
    # --impl reference on the tiny workload: the oracle timed on the host, one JSON line with the
    # fields the line needs (the same metric and config keys as the GPU arm); each sample is cut short
    import sys
    real = bench.oracle_decode_sample
    monkeypatch.setattr(bench, "oracle_decode_sample", lambda *a, **k: real(*a, **{**k, "budget_s": 0.05}))
    argv = sys.argv
    sys.argv = ["bench.py", "--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "0"]
    try:
        assert bench.main() == 0
    finally:
        sys.argv = argv
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["prefill_value"] > 0
    assert line["config"]["workload"] == "tiny" and line["e2e"]["h2d_bytes_per_step"] == 0


def test_input_digest_names_the_inputs():
    w = inputs.WORKLOADS["tiny"]
    k, v, _ = inputs.full_kv(w)
    d1 = bench.input_digest(k.numpy(), v.numpy(), inputs.query(w).numpy())
    k2, v2, _ = inputs.full_kv(w)  # the same seeds give the same bytes
    assert bench.input_digest(k2.numpy(), v2.numpy(), inputs.query(w).numpy()) == d1
    v2[0, 0, 0, 0] += 1
    assert bench.input_digest(k2.numpy(), v2.numpy(), inputs.query(w).numpy()) != d1


def test_append_summary():
    assert bench.append_summary([], []) is None
    got = bench.append_summary([0.004, 0.010, 0.006], [False, True, False])
    assert got == {"n": 3, "mean_us": 6.67, "flush_us": 10.0, "n_flush": 1, "noflush_us": 5.0}
    assert bench.append_summary([0.004], [False])["flush_us"] is None
