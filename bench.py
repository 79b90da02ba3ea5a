#!/usr/bin/env python3
"""Benchmark: decode steps on the packed low-bit KV cache, B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl kvq|reference]

One step is one serving decode step of the whole batch on the resident cache: append the new token of
every sequence (Hadamard rotation of the key when enabled, group flush every G steps) and decode
attention of one query per sequence over the packed cache plus the FP16 window (query prep, split-K
attention, split combine). Prefill quantization of the full prompt (fp16 K/V -> codes, scales, window)
is timed separately in the same run. The headline value is effective decode bandwidth: the bytes the
method must read per step (packed codes, scales, zero-points, FP16 window, query and output) divided
by the device time per step; inputs (> L2) are resident in HBM when timing starts.

With --gpus N > 1 (torchrun) every rank runs its own replica of the workload (the path has no
exchange step): weak scaling, value = bytes of all ranks / max-over-ranks time.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time
from typing import List, NamedTuple, Optional

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_kv_cache_prefill_b200 import inputs  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 2**20
METRIC = "decode-attn effective KV HBM GB/s (fraction of B200 peak); tokens/s"


# ---------------------------------------------------------------------------------------------------
# algorithmic bytes (what the method must move), per unit of work
# ---------------------------------------------------------------------------------------------------
def decode_bytes(w: inputs.Workload, lens: np.ndarray, sink: int = 0, outliers: int = 0) -> int:
    """Bytes one decode call must read/write: packed codes + key group scale/zero + value token
    scale/zero for the quantized tokens (and with the outliers on, one 4-byte key and one value
    outlier word per quantized token), fp16 K/V for the window (and for the first token when the
    sink is on), q in and out."""
    G, R = w.group_size, w.residual
    total = 0
    for T in lens:
        T = int(T)
        Q = max(T - R, 0) // G * G
        per_unit = Q * 128 * (w.key_bits + w.value_bits) // 8 + (Q // G) * 128 * 4 + Q * (128 // G) * 4 + (T - Q) * 128 * 4
        if sink and Q > 0:
            per_unit += 128 * 4
        if outliers:
            per_unit += Q * 8
        total += w.num_kv_heads * per_unit
    return total + 2 * w.batch * w.num_q_heads * 128 * 2


def prefill_bytes(w: inputs.Workload, lens: np.ndarray, sink: int = 0, outliers: int = 0) -> int:
    """fp16 K and V read + codes, scales, zero-points and window (and the sink row, and the outlier
    words) written."""
    G, R = w.group_size, w.residual
    total = 0
    for T in lens:
        T = int(T)
        Q = max(T - R, 0) // G * G
        total += w.num_kv_heads * (T * 128 * 4 + Q * 128 * (w.key_bits + w.value_bits) // 8
                                   + (Q // G) * 128 * 4 + Q * (128 // G) * 4 + (T - Q) * 128 * 4
                                   + (128 * 4 if sink and T > 0 else 0) + (Q * 8 if outliers else 0))
    return total


def append_bytes(w: inputs.Workload) -> int:
    return 2 * w.batch * w.num_kv_heads * 128 * 2


def flush_steps(w: inputs.Workload, lens_before: np.ndarray, steps: int) -> List[bool]:
    """For each of `steps` appends starting from lengths lens_before: whether it flushes a group out
    of the fp16 window in some sequence (its quantized length grows)."""
    G, R = w.group_size, w.residual
    q = lambda T: np.maximum(T - R, 0) // G * G  # noqa: E731
    return [bool((q(lens_before + i + 1) > q(lens_before + i)).any()) for i in range(steps)]


def align_pad(w: inputs.Workload, lens: np.ndarray, steps: int) -> int:
    """Appends to make before `steps` timed appends from lengths `lens` so that the first append that
    flushes a group (in the longest sequence) is timed step steps // 2 (0 if it would already fall
    inside the timed steps without padding before that point)."""
    G, R = w.group_size, w.residual
    T = int(np.max(lens))
    # append i (0-based) makes the length T + i + 1; it flushes when (T + i + 1 - R) is a positive multiple of G
    first = next(i for i in range(G) if T + i + 1 - R > 0 and (T + i + 1 - R) % G == 0)
    want = min(steps // 2, G - 1)
    return (first - want) % G


def align_appends(w: inputs.Workload, lens: np.ndarray, steps: int):
    """The padding appends of align_pad (seeded tokens after the workload's own)."""
    n = align_pad(w, lens, steps)
    return [inputs.append_tokens(w, 10_000 + s) for s in range(n)]


def kv_tokens(w: inputs.Workload, lens: np.ndarray) -> int:
    """Cached (token, KV head) pairs one decode call scans."""
    return int(np.asarray(lens, np.int64).sum()) * w.num_kv_heads


def input_digest(*arrays) -> str:
    """SHA-256 of the arrays' bytes in order (C-contiguous numpy arrays): names the exact synthetic
    inputs a run used."""
    import hashlib
    h = hashlib.sha256()
    for a in arrays:
        h.update(memoryview(np.ascontiguousarray(a)))
    return h.hexdigest()


def append_summary(ms: List[float], flush: List[bool]) -> Optional[dict]:
    """Mean µs of a run of appends, overall and split by whether the append flushed a group."""
    if not ms:
        return None
    fl = [m for m, f in zip(ms, flush) if f]
    pl = [m for m, f in zip(ms, flush) if not f]
    us = lambda xs: round(statistics.mean(xs) * 1e3, 2) if xs else None  # noqa: E731
    return {"n": len(ms), "mean_us": us(ms), "flush_us": us(fl), "n_flush": len(fl), "noflush_us": us(pl)}


def cpu_model() -> Optional[str]:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


# ---------------------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except FileNotFoundError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def reduce_over_ranks(dist, device, ms: float, *sums: float):
    """Whole-job aggregates of a replicated run: the max of the per-rank times `ms` (the job ends with its
    slowest rank) and the sums of `sums` (bytes, tokens) over the ranks. Without a process group the
    values are returned unchanged."""
    if dist is None:
        return (float(ms),) + tuple(float(x) for x in sums)
    t = torch.tensor([ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    out = (float(t.item()),)
    if sums:
        s = torch.tensor(list(sums), device=device, dtype=torch.float64)
        dist.all_reduce(s)
        out += tuple(float(x) for x in s.tolist())
    return out


def measured_traffic(w: inputs.Workload, layout: int, kind: str = "decode", sink: int = 0, rope: float = 0.0,
                     outliers: int = 0, page_tokens: int = 0):
    """DRAM bytes per launch of the decode-split (kind "decode") or bulk-prefill (kind "prefill")
    kernel from the committed ncu counters (profiles/decode_traffic_counters.txt, JSON), scaled from
    the captured batch to this one by the units processed; None if there is no capture for this
    workload, layout, kernel and options (sink, RoPE, outliers, pages; a record without them was taken
    with them off) or the kernel sources changed since it was taken."""
    import hashlib
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles", "decode_traffic_counters.txt")
    try:
        entries = json.load(open(path))
    except (OSError, ValueError):
        return None
    root = os.path.dirname(os.path.abspath(__file__))
    for e in entries.values():
        if e.get("workload") != w.name or e.get("layout") != layout or e.get("kind", "decode") != kind:
            continue
        if (e.get("sink", 0) != sink or e.get("rope_theta", 0.0) != rope or e.get("outliers", 0) != outliers
                or e.get("page_tokens", 0) != page_tokens):
            continue
        h = hashlib.sha256()
        for f in e["kernel_sources"]:
            h.update(open(os.path.join(root, f), "rb").read())
        if h.hexdigest() != e["sources_sha256"]:
            return None
        # traffic grows with the units processed; a capture at a reduced prefill length records its
        # (token, KV head) pairs, and then scales by those instead
        if "capture_tokens" in e:
            scale = float(np.sum(w.seq_lens())) * w.num_kv_heads / e["capture_tokens"]
        else:
            scale = w.batch * w.num_kv_heads / e["capture_units"]
        return int(round((e["dram_read_bytes"] + e["dram_write_bytes"]) * scale))
    return None


def measured_hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------------------------------
# CPU oracle baseline (bounded sample)
# ---------------------------------------------------------------------------------------------------
class OracleSample(NamedTuple):
    gbs: float                          # algorithmic decode bytes / s, on `threads` threads
    threads: int
    sample: str                         # what was timed
    single_thread_gbs: Optional[float]  # the same on one thread (when asked for)
    prefill_gbs: float                  # the sample's quantize_prefill: algorithmic prefill bytes / s


def oracle_decode_sample(w: inputs.Workload, budget_s: float = 15.0, layout: int = 1, sink: int = 0,
                         rope: float = 0.0, outliers: int = 0, single_thread_s: float = 0.0) -> OracleSample:
    """Time the oracle's decode on a bounded sample of the workload: whole (sequence, KV head) units
    batched into one oracle problem (enough units to give every host core a query head), decoded
    repeatedly until about budget_s seconds have passed; with single_thread_s > 0, then on one thread
    for about that long (at least one call)."""
    import oracle as ref

    cores = len(os.sched_getaffinity(0))
    g = w.gqa
    lens_all = w.seq_lens() + w.appends
    units = [(b, h) for b in range(w.batch) for h in range(w.num_kv_heads)]
    n = max(1, min(len(units), -(-cores // g)))
    while n > 1 and n * int(lens_all.max()) > (4 << 20):  # keep the sample's host memory bounded
        n -= 1
    stride = max(1, len(units) // n)
    picked = units[::stride][:n]
    lens = np.array([int(lens_all[b]) for b, _ in picked], np.int64)
    Tmax = int(lens.max())
    cap = int(math.ceil(Tmax / w.group_size) * w.group_size)
    if layout == 2:
        cap = -(-cap // 128) * 128
    ocfg = ref.Config(n, g, 1, w.key_bits, w.value_bits, w.group_size, w.residual, w.hadamard, cap,
                      layout=layout, sink=sink, rope_theta=rope, outliers=outliers)
    k = np.zeros((n, Tmax, 1, 128), np.float16)
    v = np.zeros_like(k)
    qs = np.zeros((n, g, 128), np.float16)
    q = inputs.query(w).numpy()
    for i, (b, h) in enumerate(picked):
        ku, vu = inputs.unit_kv(w, b, h, int(lens[i]))
        k[i, : lens[i], 0] = ku.numpy()
        v[i, : lens[i], 0] = vu.numpy()
        qs[i] = q[b, h * g:(h + 1) * g]
    oc = ref.Cache(ocfg)
    t_pre = time.perf_counter()
    ref.quantize_prefill(ocfg, oc, k, v, lens, threads=cores)
    t_pre = time.perf_counter() - t_pre
    threads = min(cores, n * g)
    calls, spent = 0, 0.0
    while spent < budget_s or calls == 0:
        t0 = time.perf_counter()
        ref.decode(ocfg, oc, qs, 1 / math.sqrt(128), threads=threads)
        spent += time.perf_counter() - t0
        calls += 1
    per_call = decode_bytes(w.scaled(batch=n, num_q_heads=g, num_kv_heads=1), lens, sink, outliers)
    desc = f"{n} (sequence, KV head) units of {w.name} ({int(lens.sum())} tokens), decode x{calls}"
    single = None
    if single_thread_s > 0:
        st_calls, st_spent = 0, 0.0
        while st_spent < single_thread_s or st_calls == 0:
            t0 = time.perf_counter()
            ref.decode(ocfg, oc, qs, 1 / math.sqrt(128), threads=1)
            st_spent += time.perf_counter() - t0
            st_calls += 1
        single = per_call * st_calls / st_spent / 1e9
        desc += f"; one thread: decode x{st_calls}"
    pre = prefill_bytes(w.scaled(batch=n, num_q_heads=g, num_kv_heads=1), lens, sink)
    return OracleSample(per_call * calls / spent / 1e9, threads, desc, single, pre / t_pre / 1e9)


def workload_config(w: inputs.Workload, args) -> dict:
    """The JSON line's config, the same for both arms (a function of the workload and the options only:
    the read size quoted is that of a decode at the workload's lengths after its own appends)."""
    step_bytes = decode_bytes(w, w.seq_lens() + w.appends, args.sink, args.outliers)
    return {"workload": w.name, "batch": w.batch, "seq_len": w.seq_len, "num_q_heads": w.num_q_heads,
            "num_kv_heads": w.num_kv_heads, "key_bits": w.key_bits, "value_bits": w.value_bits,
            "group_size": w.group_size, "residual": w.residual, "hadamard": w.hadamard,
            "ragged": bool(w.ragged_min), "parallelism": f"replicas{args.gpus}", "layout": args.layout,
            "sink": args.sink, "rope_theta": args.rope, "outliers": args.outliers,
            "page_tokens": getattr(args, "page_tokens", 0), "cuda_cores": getattr(args, "cuda_cores", 0), "l2": f"inputs larger than L2 ({step_bytes / 2**20:.0f} MiB read per decode > 126 MiB)"}


def run_reference(args, w):
    """--impl reference: the CPU oracle as it stands, timed on the host cores."""
    import oracle as ref

    ref.build()
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    lens = w.seq_lens() + w.appends
    per_step = []
    budget = max(2.0, 60.0 / max(1, args.steps + args.warmup))
    for i in range(args.warmup + args.steps):
        res = oracle_decode_sample(w, budget_s=budget, layout=args.layout, sink=args.sink, rope=args.rope,
                                   outliers=args.outliers)
        cores, sample, pre_gbs = res.threads, res.sample, res.prefill_gbs
        if i >= args.warmup:
            per_step.append(res.gbs)
    value = statistics.mean(per_step)
    step_bytes = decode_bytes(w, lens, args.sink, args.outliers)
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(step_bytes / (value * 1e9) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": sample,
                         "prefill_value": round(pre_gbs, 4), "cpu_model": cpu_model()},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="llama3_8b_gqa", choices=sorted(inputs.WORKLOADS))
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--prefill-iters", type=int, default=3)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (profiling captures)")
    ap.add_argument("--seq-len", type=int, default=0,
                    help="override the workload's prefill length (profiling captures of single-sequence workloads)")
    ap.add_argument("--layout", type=int, default=1, choices=[1, 2],
                    help="packed layout: 1 = tile v1 (mma.sync decode), 2 = rows v2 (tcgen05 decode)")
    ap.add_argument("--sink", type=int, default=0, choices=[0, 1],
                    help="1: keep every sequence's first token in fp16 (attention sink)")
    ap.add_argument("--rope", type=float, default=0.0,
                    help="> 0: cache keys before RoPE with this theta and rotate them in decode (needs --layout 2)")
    ap.add_argument("--page-tokens", type=int, default=0,
                    help="> 0: paged storage with pages of this many tokens (a multiple of 128; needs --layout 1); "
                         "each unit's pages are consecutive pool pages")
    ap.add_argument("--cuda-cores", type=int, default=0, choices=[0, 1],
                    help="1: decode with the CUDA-core control kernel instead of the tensor-core one (needs --layout 2, "
                         "no RoPE, no Hadamard rotation); for measuring the tensor-core gain")
    ap.add_argument("--outliers", type=int, default=0, choices=[0, 1],
                    help="1: keep each quantized token's largest key / value entry in fp16 (needs --layout 1)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    w0 = inputs.WORKLOADS[args.workload]
    if args.batch > 0:
        w0 = w0.scaled(batch=args.batch)
    if args.seq_len > 0:
        w0 = w0.scaled(seq_len=args.seq_len, ragged_min=min(w0.ragged_min, args.seq_len))

    if args.impl == "reference":
        return run_reference(args, w0)

    import bit_kv_cache_prefill_b200 as kvq

    if args.cuda_cores:
        if args.layout != 2 or args.rope > 0 or w0.hadamard:
            raise SystemExit("--cuda-cores 1 needs --layout 2, no RoPE and a workload without the Hadamard rotation")
        os.environ["KVQ_DECODE_CUDA_CORES"] = "1"  # read by the library at each decode call
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()

    # capacity for the prefill plus every appended token of this run
    n_app = w0.appends + args.warmup + args.steps + w0.group_size + (1 if not args.no_e2e else 0) * (args.steps + args.warmup)
    w = w0.scaled(appends=n_app)
    lens0 = w0.seq_lens()
    k, v, _ = inputs.full_kv(w0)  # CPU, seeded
    digest = input_digest(k.numpy(), v.numpy(), inputs.query(w0).numpy())
    kd, vd = k.cuda(), v.cuda()
    del k, v
    cap = w.capacity()
    if args.page_tokens > 0:
        cap = -(-cap // args.page_tokens) * args.page_tokens  # a whole number of pages
    if args.layout == 2:
        cap = -(-cap // 128) * 128  # rows v2 stores values in whole 128-token blocks
    cfg = kvq.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.key_bits, w.value_bits, w.group_size, w.residual,
                          w.hadamard, cap, layout=args.layout, sink=args.sink, rope_theta=args.rope,
                          outliers=args.outliers, page_tokens=args.page_tokens,
                          num_pages=w.batch * w.num_kv_heads * cap // max(args.page_tokens, 1) if args.page_tokens else 0)
    cache = kvq.Cache(cfg)
    stream = torch.cuda.current_stream()

    # ---- prefill quantization, timed separately (same input each iteration)
    pre_ms = []
    for i in range(args.prefill_iters + 1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        kvq.kvq_quantize_prefill(cfg, cache, kd, vd, lens0)
        e1.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            pre_ms.append(e0.elapsed_time(e1))
    pre_bytes = prefill_bytes(w0, lens0, args.sink, args.outliers)
    del kd, vd
    torch.cuda.empty_cache()

    # the workload's own streaming appends (e.g. 256 new tokens per sequence) before decode, each
    # timed with CUDA events on the stream (its inputs already on the device)
    wl_app = [tuple(t.cuda() for t in inputs.append_tokens(w0, s)) for s in range(w0.appends)]
    wl_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in wl_app]
    for (kn, vn), (ea, eb) in zip(wl_app, wl_ev):
        ea.record(stream)
        kvq.kvq_append_token(cfg, cache, kn, vn)
        eb.record(stream)
    torch.cuda.synchronize()
    wl_app_ms = [ea.elapsed_time(eb) for ea, eb in wl_ev]
    del wl_app

    q = inputs.query(w0).cuda()
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
    ws = torch.empty(kvq.kvq_decode_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
    sm_scale = 1 / math.sqrt(128)
    steps_tok = [inputs.append_tokens(w0, w0.appends + s) for s in range(args.warmup + args.steps)]
    app_k = [t[0].cuda() for t in steps_tok]
    app_v = [t[1].cuda() for t in steps_tok]

    def step(i, ev=None):
        if ev is not None:
            ev[0].record(stream)
        kvq.kvq_append_token(cfg, cache, app_k[i], app_v[i])
        if ev is not None:
            ev[1].record(stream)
        kvq.kvq_decode_attention(cfg, cache, q, out, sm_scale, ws)
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    # untimed appends (at most G - 1) so that the first group flush after warm-up falls in the middle of
    # the timed steps: the timed region then holds the flush cost of one step in G
    for kn, vn in align_appends(w0, cache.seq_len_host, args.steps):
        kvq.kvq_append_token(cfg, cache, kn.cuda(), vn.cuda())
    barrier()
    lens_before = cache.seq_len_host.copy()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    visible = os.environ.get("CUDA_VISIBLE_DEVICES")
    gpu_id = visible.split(",")[local] if visible else str(local)
    with ClockSampler(gpu_id) as clocks:
        time.sleep(0.25)
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(args.steps):
            step(args.warmup + i, evs[i])
        t_end.record(stream)
        barrier()
    total_ms = t_start.elapsed_time(t_end)
    decode_ms = [e[1].elapsed_time(e[2]) for e in evs]
    append_ms = [e[0].elapsed_time(e[1]) for e in evs]
    # bytes per step from the lengths each decode actually saw (append happens first)
    step_bytes = [decode_bytes(w0, lens_before + i + 1, args.sink, args.outliers) for i in range(args.steps)]
    total_bytes = float(sum(step_bytes))
    tokens = w.batch * args.steps

    # max over ranks of the time, sums of the work
    total_ms, total_bytes, tokens = reduce_over_ranks(dist, "cuda", total_ms, total_bytes, float(tokens))
    tokens = int(tokens)

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    e2e = None
    if not args.no_e2e:
        q_cpu = inputs.query(w0)
        out_host = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16).pin_memory()
        # each step's inputs (new K, new V, q) in one pinned buffer, so one host->device copy per step
        nk, nq = steps_tok[0][0].numel(), q_cpu.numel()
        in_host = [torch.cat([t[0].reshape(-1), t[1].reshape(-1), q_cpu.reshape(-1)]).pin_memory() for t in steps_tok]
        in_dev = torch.empty(2 * nk + nq, dtype=torch.float16, device="cuda")
        kn_dev = in_dev[:nk].view(app_k[0].shape)
        vn_dev = in_dev[nk:2 * nk].view(app_v[0].shape)
        q_dev = in_dev[2 * nk:].view(q.shape)
        lens_e = cache.seq_len_host.copy()
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(args.steps):
            j = (args.warmup + i) % len(in_host)
            in_dev.copy_(in_host[j], non_blocking=True)
            kvq.kvq_append_token(cfg, cache, kn_dev, vn_dev)
            kvq.kvq_decode_attention(cfg, cache, q_dev, out, sm_scale, ws)
            out_host.copy_(out, non_blocking=True)
            stream.synchronize()  # the step's result is on the host
        e1.record(stream)
        barrier()
        e2e_ms = e0.elapsed_time(e1)
        e2e_bytes = float(sum(decode_bytes(w0, lens_e + i + 1, args.sink, args.outliers) for i in range(args.steps)))
        e2e_ms, e2e_bytes = reduce_over_ranks(dist, "cuda", e2e_ms, e2e_bytes)
        h2d = in_host[0].numel() * 2
        d2h = out_host.numel() * 2
        e2e = {"value": round(e2e_bytes / (e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h),
               "tokens_per_s": round(w.batch * world * args.steps / (e2e_ms * 1e-3), 1)}

    if rank != 0:
        if dist is not None:
            dist.destroy_process_group()
        return 0

    peak, peak_kind = measured_hbm_peak()
    flush = flush_steps(w0, lens_before, args.steps)
    app_flush = [a for a, f in zip(append_ms, flush) if f]
    app_plain = [a for a, f in zip(append_ms, flush) if not f]
    scanned = float(sum(kv_tokens(w0, lens_before + i + 1) for i in range(args.steps)))
    value = total_bytes / (total_ms * 1e-3) / 1e9
    mean_decode_ms = statistics.mean(decode_ms)
    achieved = statistics.mean(step_bytes) / (mean_decode_ms * 1e-3) / 1e9
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "u2/u4 codes, fp16 in/out, fp32 accumulate",
        "data": "synthetic",
        "config": workload_config(w0, args),
        "tokens_per_s": round(tokens / (total_ms * 1e-3), 1),
        "frac_of_nominal_8tbs": round(value / NOMINAL_HBM_GBS, 4),
        "decode_ms": round(mean_decode_ms, 4),
        "append_us": round(statistics.mean(append_ms) * 1e3, 2),
        # appends that flush a group out of the window in some sequence, and the others
        "append_flush_us": round(statistics.mean(app_flush) * 1e3, 2) if app_flush else None,
        "append_noflush_us": round(statistics.mean(app_plain) * 1e3, 2) if app_plain else None,
        "kv_tokens_scanned_per_s": round(scanned / (sum(decode_ms) * 1e-3), 1),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": measured_traffic(w0, args.layout, "decode", args.sink, args.rope, args.outliers, args.page_tokens), "peak_kind": peak_kind,
                     "kernel": ("decode_rope_kernel" if args.rope > 0 else
                                "decode_rope_kernel without rotations (CUDA-core control)" if args.cuda_cores else
                                "decode_split_kernel" if args.layout == 1 else "decode_tc_kernel")
                     + " + decode_combine_kernel (one kvq_decode_attention call)"},
        "prefill": {"gbs": round(pre_bytes / (statistics.mean(pre_ms) * 1e-3) / 1e9, 1),
                    "elements_per_s": round(2 * 128 * kv_tokens(w0, lens0) / (statistics.mean(pre_ms) * 1e-3), 1),
                    "ms": round(statistics.mean(pre_ms), 3), "bytes": pre_bytes, "bound": "hbm", "peak": peak,
                    "frac": round(pre_bytes / (statistics.mean(pre_ms) * 1e-3) / 1e9 / peak, 4),
                    "traffic": measured_traffic(w0, args.layout, "prefill", args.sink, args.rope, args.outliers, args.page_tokens),
                    "kernel": "prefill_block_kernel (one kvq_quantize_prefill call)"},
        # per step: append (one launch per 256 sequences), then the decode split kernel + combine (+ the
        # RoPE angle tables)
        "gpu_launches": (-(-w.batch // 256) + (3 if args.rope > 0 else 2)) * args.steps,
        "clocks": clocks.summary(),
        "input_sha256": digest,  # prefill K, V (fp16 [B][T][Hkv][128], zero past each length) and q
        # the workload's own appends before the timed steps (e.g. 256 per sequence), one event pair each
        "workload_appends": append_summary(wl_app_ms, flush_steps(w0, lens0, len(wl_app_ms))),
    }
    if e2e is not None:
        line["e2e"] = e2e
    if args.gpus == 1 and not args.no_cpu_baseline:
        import oracle as ref

        ref.build()
        res = oracle_decode_sample(w0, layout=args.layout, sink=args.sink, rope=args.rope, outliers=args.outliers,
                                   single_thread_s=3.0)
        line["cpu_baseline"] = {"value": round(res.gbs, 4), "unit": "GB/s", "cores": res.threads, "kind": "oracle",
                                "sample": res.sample, "single_thread_value": round(res.single_thread_gbs, 4),
                                "prefill_value": round(res.prefill_gbs, 4), "cpu_model": cpu_model()}
    print(json.dumps(line), flush=True)
    if dist is not None:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
