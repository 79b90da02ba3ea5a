"""Decode attention for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc: for example a plugin inside a host framework
that owns all device memory through its own pool, or a serving loop that forbids allocation after
start-up. ``kvq_decode_attention_noalloc`` keeps the split partials in a fixed scratch array inside the
library instead of a caller-provided workspace. This file checks it through the C ABI against
``kvq_decode_attention`` (the entry point that takes a workspace) on two calls in a row, with different
caches and queries, so that content left in the shared scratch by the first call cannot leak into the
second. It is named to be collected last.
"""
import math

import numpy as np
import pytest
import torch

import bit_kv_cache_prefill_b200 as kvq
from bit_kv_cache_prefill_b200 import inputs

import _harness as H

pytestmark = pytest.mark.gpu


def _prepared(w: inputs.Workload, layout: int = 1, sink: int = 0, rope: float = 0.0):
    k, v, lens = inputs.full_kv(w)
    cfg = H.gpu_config(w, layout=layout, sink=sink, rope=rope)
    cache = kvq.Cache(cfg)
    kvq.kvq_quantize_prefill(cfg, cache, k.cuda(), v.cuda(), lens)
    return cfg, cache


# (workload, layout, sink, rope_theta): tile v1 (mma.sync decode); rows v2 (tcgen05 decode, its own
# split length); rows v2 with pre-RoPE keys (the RoPE angle tables share the scratch, behind the
# split partials)
CASES = {
    "tile_v1": [(inputs.Workload("na1", 4, 16, 4, 2, 2, 32, 64, 0, 3000, seed=41, ragged_min=700), 1, 0, 0.0),
                (inputs.Workload("na2", 2, 8, 8, 4, 2, 64, 32, 1, 5000, seed=42), 1, 0, 0.0)],
    "rows_v2": [(inputs.Workload("na3", 3, 8, 2, 2, 2, 32, 32, 0, 2500, seed=43), 2, 1, 0.0),
                (inputs.Workload("na4", 2, 4, 4, 2, 2, 128, 128, 0, 4000, seed=44), 2, 0, 0.0)],
    "rope": [(inputs.Workload("na5", 2, 8, 2, 2, 2, 64, 64, 0, 3000, seed=45), 2, 1, 10000.0),
             (inputs.Workload("na6", 3, 4, 4, 2, 2, 32, 32, 0, 2000, seed=46, ragged_min=500), 2, 0, 500000.0)],
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_noalloc_decode_matches_workspace_decode_on_two_calls(case):
    runs = []
    for w, layout, sink, rope in CASES[case]:
        cfg, cache = _prepared(w, layout, sink, rope)
        q = inputs.query(w).cuda()
        ws = torch.empty(kvq.kvq_decode_workspace_bytes(cfg), dtype=torch.uint8, device="cuda")
        ref = torch.empty(w.batch, w.num_q_heads, 128, dtype=torch.float16, device="cuda")
        kvq.kvq_decode_attention(cfg, cache, q, ref, 1 / math.sqrt(128), ws)
        runs.append((cfg, cache, q, ref))
    outs = []
    for cfg, cache, q, ref in runs:  # two no-alloc calls in a row on the shared scratch
        out = torch.full_like(ref, float("nan"))
        kvq.kvq_decode_attention_noalloc(cfg, cache, q, out, 1 / math.sqrt(128))
        outs.append(out)
    torch.cuda.synchronize()
    for (cfg, cache, q, ref), out in zip(runs, outs):
        H.check_attention(out.cpu().numpy(), ref.cpu().numpy().astype(np.float64), "no-alloc vs workspace decode")


def test_noalloc_rejects_configs_beyond_the_fixed_scratch():
    # 4096 sequences x 8 KV heads x 4 query heads need more split space than the fixed 16 MiB.
    cfg = kvq.make_config(4096, 32, 8, 2, 2, 32, 32, 0, 1024)
    assert kvq.kvq_decode_workspace_bytes(cfg) > kvq.STATIC_SCRATCH_BYTES
    cache = kvq.Cache(kvq.make_config(1, 4, 1, 2, 2, 32, 32, 0, 64))  # any valid buffers; rejected first
    q = torch.zeros(1, 4, 128, dtype=torch.float16, device="cuda")
    with pytest.raises(kvq.KvqError) as e:
        kvq.kvq_decode_attention_noalloc(cfg, cache, q, q.clone(), 0.1)
    assert e.value.status == kvq.KVQ_ERR_WORKSPACE
