"""Shared helpers for the tests: run one workload through the CUDA library (C ABI) and through the
CPU oracle on the same seeded inputs, and compare."""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np
import torch

from bit_kv_cache_prefill_b200 import inputs

MAX_ABS_TOL = 2e-3  # decode attention output, absolute
REL_L2_TOL = 1e-3   # decode attention output, relative L2 over all compared outputs


def capacity(w: inputs.Workload, layout: int) -> int:
    """Workload capacity, rounded up to whole 128-token blocks for the rows-v2 layout."""
    cap = w.capacity()
    return -(-cap // 128) * 128 if layout == 2 else cap


def oracle_config(oracle, w: inputs.Workload, batch=None, hq=None, hkv=None, layout: int = 1, sink: int = 0,
                  rope: float = 0.0, outliers: int = 0):
    return oracle.Config(batch or w.batch, hq or w.num_q_heads, hkv or w.num_kv_heads, w.key_bits, w.value_bits,
                         w.group_size, w.residual, w.hadamard, capacity(w, layout), layout=layout, sink=sink,
                         rope_theta=rope, outliers=outliers)


def gpu_config(w: inputs.Workload, layout: int = 1, sink: int = 0, rope: float = 0.0, outliers: int = 0):
    import bit_kv_cache_prefill_b200 as kvq

    return kvq.make_config(w.batch, w.num_q_heads, w.num_kv_heads, w.key_bits, w.value_bits, w.group_size,
                           w.residual, w.hadamard, capacity(w, layout), layout=layout, sink=sink, rope_theta=rope,
                           outliers=outliers)


@dataclass
class DeviceRun:
    cfg: object
    cache: object
    out: torch.Tensor  # fp16 [B][Hq][128] on the device
    lens: np.ndarray
    layout: int = 1
    sink: int = 0
    outliers: int = 0


def run_gpu(w: inputs.Workload, k: torch.Tensor, v: torch.Tensor, lens: np.ndarray, q: torch.Tensor,
            appends: int = 0, sm_scale: Optional[float] = None, layout: int = 1, decode: bool = True,
            sink: int = 0, rope: float = 0.0, outliers: int = 0) -> DeviceRun:
    """Prefill (k, v on the device), `appends` streaming appends, one decode (unless decode=False)."""
    import bit_kv_cache_prefill_b200 as kvq

    cfg = gpu_config(w, layout, sink, rope, outliers)
    cache = kvq.Cache(cfg)
    kvq.kvq_quantize_prefill(cfg, cache, k, v, lens)
    for step in range(appends):
        kn, vn = inputs.append_tokens(w, step)
        kvq.kvq_append_token(cfg, cache, kn.cuda(), vn.cuda())
    out = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
    if decode:
        ws = torch.empty(kvq.kvq_decode_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
        kvq.kvq_decode_attention(cfg, cache, q.cuda(), out, sm_scale or 1 / math.sqrt(128), ws)
    torch.cuda.synchronize()
    return DeviceRun(cfg, cache, out, lens + appends, layout, sink, outliers)


def code_shapes(w: inputs.Workload, layout: int):
    B, H, cap = w.batch, w.num_kv_heads, capacity(w, layout)
    if layout == 2:
        return (B, H, cap, 4 * w.key_bits), (B, H, cap // 128, 128, 4 * w.value_bits)
    return (B, H, cap // 16, 64 * w.key_bits), (B, H, cap // 16, 64 * w.value_bits)


def gpu_views(w: inputs.Workload, run: DeviceRun) -> Dict[str, np.ndarray]:
    """GPU cache buffers as numpy arrays with the oracle's shapes."""
    B, H, cap, G = w.batch, w.num_kv_heads, capacity(w, run.layout), w.group_size
    ring = w.residual + G + run.sink  # ring slots, then the sink row
    c = run.cache
    ks, vs = code_shapes(w, run.layout)
    extra = {}
    if run.outliers:  # u32 per (unit, token): channel | fp16 value << 16
        for n in ("k_out", "v_out"):
            words = c.view(n, torch.int32).cpu().numpy().view(np.uint32).reshape(B, H, cap)
            extra[n + "_ch"] = (words & 0xFFFF).astype(np.uint16)
            extra[n + "_val"] = (words >> 16).astype(np.uint16)
    return extra | {
        "k_codes": c.view("k_codes", torch.int32).cpu().numpy().view(np.uint32).reshape(ks),
        "v_codes": c.view("v_codes", torch.int32).cpu().numpy().view(np.uint32).reshape(vs),
        "k_scale": c.view("k_scale", torch.int16).cpu().numpy().view(np.uint16).reshape(B, H, cap // G, 128),
        "k_zero": c.view("k_zero", torch.int16).cpu().numpy().view(np.uint16).reshape(B, H, cap // G, 128),
        "v_scale": c.view("v_scale", torch.int16).cpu().numpy().view(np.uint16).reshape(B, H, cap, 128 // G),
        "v_zero": c.view("v_zero", torch.int16).cpu().numpy().view(np.uint16).reshape(B, H, cap, 128 // G),
        "k_res": c.view("k_res", torch.int16).cpu().numpy().view(np.uint16).reshape(B, H, ring, 128),
        "v_res": c.view("v_res", torch.int16).cpu().numpy().view(np.uint16).reshape(B, H, ring, 128),
    }


def compare_unit_cache(w: inputs.Workload, gv: Dict[str, np.ndarray], b: int, h: int, oc, ob: int, oh: int, T: int,
                       layout: int = 1, sink: int = 0, outliers: int = 0) -> None:
    """Bit-exact comparison of everything that is defined for one unit of length T."""
    G, R = w.group_size, w.residual
    Q = max(T - R, 0) // G * G
    if outliers:  # the (channel, fp16 value) of every quantized token's key and value outlier
        for key in ("k_out_ch", "k_out_val", "v_out_ch", "v_out_val"):
            np.testing.assert_array_equal(gv[key][b, h, :Q], getattr(oc, key)[ob, oh, :Q], err_msg=f"{key} unit {b},{h}")
    ring = R + G
    if layout == 2:
        np.testing.assert_array_equal(gv["k_codes"][b, h, :Q], oc.k_codes[ob, oh, :Q], err_msg=f"k_codes unit {b},{h}")
        nb, rem = divmod(Q, 128)
        np.testing.assert_array_equal(gv["v_codes"][b, h, :nb], oc.v_codes[ob, oh, :nb], err_msg=f"v_codes unit {b},{h}")
        if rem:  # a partial block: only the words of the quantized token pairs are defined
            words = rem * w.value_bits // 32
            np.testing.assert_array_equal(gv["v_codes"][b, h, nb, :, :words], oc.v_codes[ob, oh, nb, :, :words],
                                          err_msg=f"v_codes unit {b},{h} partial block")
    else:
        np.testing.assert_array_equal(gv["k_codes"][b, h, : Q // 16], oc.k_codes[ob, oh, : Q // 16], err_msg=f"k_codes unit {b},{h}")
        np.testing.assert_array_equal(gv["v_codes"][b, h, : Q // 16], oc.v_codes[ob, oh, : Q // 16], err_msg=f"v_codes unit {b},{h}")
    np.testing.assert_array_equal(gv["k_scale"][b, h, : Q // G], oc.k_scale[ob, oh, : Q // G], err_msg=f"k_scale unit {b},{h}")
    np.testing.assert_array_equal(gv["k_zero"][b, h, : Q // G], oc.k_zero[ob, oh, : Q // G], err_msg=f"k_zero unit {b},{h}")
    np.testing.assert_array_equal(gv["v_scale"][b, h, :Q], oc.v_scale[ob, oh, :Q], err_msg=f"v_scale unit {b},{h}")
    np.testing.assert_array_equal(gv["v_zero"][b, h, :Q], oc.v_zero[ob, oh, :Q], err_msg=f"v_zero unit {b},{h}")
    live = [t % ring for t in range(Q, T)]
    np.testing.assert_array_equal(gv["k_res"][b, h, live], oc.k_res[ob, oh, live], err_msg=f"k_res unit {b},{h}")
    np.testing.assert_array_equal(gv["v_res"][b, h, live], oc.v_res[ob, oh, live], err_msg=f"v_res unit {b},{h}")
    if sink and T > 0:  # the sink token's fp16 row
        for key in ("k_res", "v_res"):
            np.testing.assert_array_equal(gv[key][b, h, ring], getattr(oc, key)[ob, oh, ring], err_msg=f"{key} sink row {b},{h}")


def fp16_ulp(x: np.ndarray) -> np.ndarray:
    """Spacing of binary16 values at |x| (2^-24 in the subnormal range)."""
    e = np.floor(np.log2(np.maximum(np.abs(x), 2.0 ** -14)))
    return 2.0 ** (e - 10)


def check_attention(gpu_out: np.ndarray, ref: np.ndarray, what: str) -> Tuple[float, float]:
    """Max-abs and relative-L2 error of the fp16 output against the fp64 oracle. The absolute bound is
    MAX_ABS_TOL where fp16 can hold it, i.e. for |out| < 4; a larger output element (a planted value
    outlier of hundreds) is held to one fp16 spacing at its magnitude, since rounding the output to
    fp16 alone moves it by up to half of one."""
    gpu = gpu_out.astype(np.float64)
    err = np.abs(gpu - ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(ref))
    rel = float(np.linalg.norm(gpu - ref) / denom) if denom > 0 else float(np.linalg.norm(gpu))
    tol = np.maximum(MAX_ABS_TOL, fp16_ulp(ref))
    if err.size and not (err <= tol).all():
        i = int(np.argmax(err - tol))
        raise AssertionError(f"{what}: max abs error {err.flat[i]:.3e} > {tol.flat[i]:.3e} at |out| = {abs(ref.flat[i]):.3g}")
    assert rel <= REL_L2_TOL, f"{what}: relative L2 error {rel:.3e} > {REL_L2_TOL}"
    return max_abs, rel


def oracle_full(oracle, w: inputs.Workload, k: torch.Tensor, v: torch.Tensor, lens: np.ndarray, q: torch.Tensor,
                appends: int = 0, sm_scale: Optional[float] = None, threads: int = 8, layout: int = 1, sink: int = 0,
                rope: float = 0.0, outliers: int = 0):
    ocfg = oracle_config(oracle, w, layout=layout, sink=sink, rope=rope, outliers=outliers)
    oc = oracle.Cache(ocfg)
    oracle.quantize_prefill(ocfg, oc, k.numpy(), v.numpy(), lens, threads=threads)
    for step in range(appends):
        kn, vn = inputs.append_tokens(w, step)
        oracle.append_token(ocfg, oc, kn.numpy(), vn.numpy())
    out = oracle.decode(ocfg, oc, q.numpy(), sm_scale or 1 / math.sqrt(128), threads=threads)
    return oc, out


def oracle_unit(oracle, w: inputs.Workload, b: int, h: int, T0: int, q: torch.Tensor, appends: int = 0,
                sm_scale: Optional[float] = None, threads: int = 4, layout: int = 1):
    """Oracle on the (sequence b, KV head h) sub-problem only (batch 1, one KV head, its g query heads)."""
    g = w.gqa
    ocfg = oracle_config(oracle, w, batch=1, hq=g, hkv=1, layout=layout)
    oc = oracle.Cache(ocfg)
    ku, vu = inputs.unit_kv(w, b, h, T0)
    oracle.quantize_prefill(ocfg, oc, ku.numpy()[None, :, None, :], vu.numpy()[None, :, None, :], [T0])
    for step in range(appends):
        kn, vn = inputs.append_tokens(w, step)
        oracle.append_token(ocfg, oc, kn[b:b + 1, h:h + 1].numpy(), vn[b:b + 1, h:h + 1].numpy())
    qq = q[b:b + 1, h * g:(h + 1) * g].contiguous().numpy()
    out = oracle.decode(ocfg, oc, qq, sm_scale or 1 / math.sqrt(128), threads=threads)
    return oc, out[0]
