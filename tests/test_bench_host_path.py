"""CPU run of bench.py's GPU arm with every CUDA call replaced by a host stand-in.

The stand-ins compute nothing (the library calls only move the length counters, the events return a
fixed tick), so no number printed here means anything. What the test checks is the arm's host logic:
that it runs from argument parsing to the printed JSON line, and that the line carries every key the
result contract needs, with the byte and token bookkeeping consistent with the workload. The real
arm runs only on a GPU.
"""
import json
import sys
import types

import numpy as np
import pytest
import torch

import bench
import bit_kv_cache_prefill_b200 as pkg
from bit_kv_cache_prefill_b200 import inputs


class _Event:
    clock = [0.0]

    def __init__(self, enable_timing=False):
        self.t = 0.0

    def record(self, stream=None):
        _Event.clock[0] += 0.01  # 10 µs per recorded event
        self.t = _Event.clock[0]

    def elapsed_time(self, other):
        return other.t - self.t


class _Stream:
    cuda_stream = 0

    def synchronize(self):
        pass


class _Cache:
    def __init__(self, cfg, device="cuda", page_table=None):
        self.cfg = cfg
        self.seq_len_host = np.zeros(cfg.batch, np.int64)


@pytest.fixture
def host_cuda(monkeypatch):
    monkeypatch.setattr(torch.cuda, "set_device", lambda d: None)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a: None)
    monkeypatch.setattr(torch.cuda, "current_stream", lambda *a: _Stream())
    monkeypatch.setattr(torch.cuda, "Event", _Event)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    monkeypatch.setattr(torch.Tensor, "cuda", lambda self, *a, **k: self)
    monkeypatch.setattr(torch.Tensor, "pin_memory", lambda self, *a, **k: self)
    real_empty = torch.empty
    monkeypatch.setattr(torch, "empty", lambda *a, device=None, **k: real_empty(*a, **k))
    calls = {"prefill": 0, "append": 0, "decode": 0}

    def make_config(batch, *a, **k):
        return types.SimpleNamespace(batch=batch)

    def prefill(cfg, cache, k, v, lens, stream=None):
        calls["prefill"] += 1
        cache.seq_len_host[:] = lens

    def append(cfg, cache, kn, vn, stream=None):
        calls["append"] += 1
        cache.seq_len_host += 1

    def decode(cfg, cache, q, out, sm_scale, ws, stream=None):
        calls["decode"] += 1

    for name, fn in (("make_config", make_config), ("Cache", _Cache), ("kvq_quantize_prefill", prefill),
                     ("kvq_append_token", append), ("kvq_decode_attention", decode),
                     ("kvq_decode_workspace_bytes", lambda cfg: 256)):
        monkeypatch.setattr(pkg, name, fn, raising=False)
    real_sample = bench.oracle_decode_sample
    monkeypatch.setattr(bench, "oracle_decode_sample",
                        lambda *a, **k: real_sample(*a, **{**k, "budget_s": 0.02, "single_thread_s": 0.01}))
    w = inputs.Workload("hostpath", 2, 4, 2, 2, 2, 32, 32, 0, 300, seed=5, appends=40)
    monkeypatch.setitem(inputs.WORKLOADS, "hostpath", w)
    return calls, w


@pytest.mark.parametrize("opts,launches", [([], 3), (["--layout", "2", "--sink", "1"], 3),
                                           (["--layout", "2", "--rope", "10000"], 4),
                                           (["--outliers", "1"], 3), (["--page-tokens", "128", "--outliers", "1"], 3)],
                         ids=["tile_v1", "rows_v2_sink", "rows_v2_rope", "outliers", "paged_outliers"])
def test_gpu_arm_host_logic_prints_a_complete_line(host_cuda, capsys, monkeypatch, opts, launches):
    calls, w = host_cuda
    steps, warmup = 4, 3
    monkeypatch.setattr(sys, "argv", ["bench.py", "--workload", "hostpath", "--steps", str(steps),
                                      "--warmup", str(warmup), "--prefill-iters", "2"] + opts)
    assert bench.main() == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks", "prefill", "input_sha256", "workload_appends"):
        assert key in line, key
    assert line["metric"] == bench.METRIC and line["steps"] == steps and line["gpu_launches"] == launches * steps
    assert set(line["roofline"]) >= {"bound", "achieved", "peak", "unit", "frac", "traffic"}
    assert set(line["cpu_baseline"]) >= {"value", "unit", "cores", "kind", "sample"}
    assert set(line["e2e"]) >= {"value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"}
    # the workload's 40 appends, the warm-up steps, the padding that puts a group flush inside the
    # timed steps, the timed steps, then the end-to-end steps
    pad = bench.align_pad(w, np.full(w.batch, 300 + 40 + warmup, np.int64), steps)
    assert calls["prefill"] == 3 and calls["append"] == 40 + warmup + pad + 2 * steps
    assert calls["decode"] == warmup + 2 * steps
    assert line["workload_appends"]["n"] == 40
    assert line["append_flush_us"] is not None  # a flush fell inside the timed steps
    # bytes per timed step from the lengths each decode saw: prefill 300 + 40 appends + warm-up + padding
    lens = np.full(w.batch, 300 + 40 + warmup + pad, np.int64)
    want = sum(bench.decode_bytes(w, lens + i + 1, sink=1 if "--sink" in opts else 0,
                                  outliers=1 if "--outliers" in opts else 0) for i in range(steps))
    assert line["value"] == pytest.approx(want / (line["ms_per_step"] * steps * 1e-3) / 1e9, rel=1e-3)
    k, v, _ = inputs.full_kv(w)
    assert line["input_sha256"] == bench.input_digest(k.numpy(), v.numpy(), inputs.query(w).numpy())
