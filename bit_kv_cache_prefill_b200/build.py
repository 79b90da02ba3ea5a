"""Build libkvq.so in-tree for sm_100a with nvcc (no GPU needed; nvcc cross-compiles).

    python -m bit_kv_cache_prefill_b200.build [--ptxas-verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkvq.so")
SOURCES = ["kvq_api.cu", "kvq_prefill.cu", "kvq_quantize.cu", "kvq_decode.cu", "kvq_decode_tc.cu", "kvq_decode_rope.cu",
           "kvq_static.cu"]
HEADERS = ["kvq_common.cuh", "kvq_decode_common.cuh", "kvq_internal.h"]

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-lineinfo", "-std=c++17",
    "-Xcompiler", "-fPIC", "-shared",
    "--expt-relaxed-constexpr",
]


def _nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, s) for s in SOURCES + HEADERS] + [os.path.join(INCLUDE, "kvq.h")]
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every source to an object in parallel (one nvcc per file), then link libkvq.so."""
    if not (force or ptxas_verbose or _stale()):
        return LIB
    import concurrent.futures
    import tempfile

    common = [_nvcc(), *[f for f in NVCC_FLAGS if f != "-shared"], "-I", INCLUDE, "-I", CSRC]
    if ptxas_verbose:
        common += ["-Xptxas", "-v"]
    with tempfile.TemporaryDirectory(prefix="kvq_build_") as objdir:
        objs = [os.path.join(objdir, os.path.splitext(s)[0] + ".o") for s in SOURCES]

        def compile_one(i: int) -> None:
            subprocess.check_call([*common, "-c", os.path.join(CSRC, SOURCES[i]), "-o", objs[i]])

        workers = max(1, min(len(SOURCES), os.cpu_count() or 1))
        with concurrent.futures.ThreadPoolExecutor(workers) as pool:
            list(pool.map(compile_one, range(len(SOURCES))))  # re-raises the first failure
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.check_call([_nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-shared", "-o", tmp, *objs])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, ptxas_verbose="--ptxas-verbose" in sys.argv)
    print(LIB)
