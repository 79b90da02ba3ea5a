"""Seeded synthetic inputs for the KV-cache workloads.

This module only draws random numbers and lays them out; it contains none of the quantization or
attention arithmetic, so both the CUDA path and the CPU oracle can consume the same bytes.

Workloads mirror the model shapes the pages evaluate on (LLaMA / Llama-2 / Llama-3 / Mistral decode
layers, KVQuant review, Validation; million-token single sequence, KVQuant review, Goal). Datasets and
trained weights are not used: keys, values and queries are N(0, 1) draws cast to fp16, with a few key
channels scaled up to model the fixed large-magnitude key channels the pages describe (KV cache
quantization wiki page, KIVI notes; KVQuant review, figure caption on pre-RoPE key outliers).

Every (sequence, KV head) unit is drawn from its own ``torch.Generator`` seeded from
(workload seed, b, kvh), so any unit can be regenerated on its own (used for sampled full-size checks).
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace
from typing import List, Optional, Tuple

import numpy as np
import torch

HEAD_DIM = 128


@dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    key_bits: int
    value_bits: int
    group_size: int
    residual: int
    hadamard: int
    seq_len: int  # prefill length (max length for ragged workloads)
    seed: int
    ragged_min: int = 0  # >0: lengths uniform in [ragged_min, seq_len]
    appends: int = 0  # tokens appended per sequence after prefill (before decode)
    outlier_channels: int = 0  # number of (kv head, channel) pairs scaled by outlier_scale
    outlier_per_head: bool = False  # True: the same channels in every head; False: pairs drawn over (head, channel)
    outlier_scale: float = 1.0

    @property
    def gqa(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    def seq_lens(self) -> np.ndarray:
        if self.ragged_min > 0:
            g = torch.Generator().manual_seed(self.seed * 7919 + 17)
            return torch.randint(self.ragged_min, self.seq_len + 1, (self.batch,), generator=g).numpy().astype(np.int64)
        return np.full((self.batch,), self.seq_len, np.int64)

    def capacity(self) -> int:
        need = int(self.seq_lens().max()) + self.appends
        return int(math.ceil(need / self.group_size) * self.group_size)

    def final_lens(self) -> np.ndarray:
        return self.seq_lens() + self.appends

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads (model-shaped decode layers). Sizes are the full ones; tests shrink them with
# ``Workload.scaled`` when the oracle has to see every output.
WORKLOADS = {
    "tiny": Workload("tiny", 1, 1, 1, 2, 2, 32, 32, 0, 4096, seed=1001,
                     outlier_channels=4, outlier_per_head=True, outlier_scale=20.0),
    "llama2_7b_mha": Workload("llama2_7b_mha", 8, 32, 32, 2, 2, 32, 128, 0, 32768, seed=1002,
                              outlier_channels=41, outlier_per_head=False, outlier_scale=15.0),
    "llama3_8b_gqa": Workload("llama3_8b_gqa", 16, 32, 8, 2, 2, 64, 128, 0, 131072, seed=1003, appends=256),
    "mistral_7b_ragged": Workload("mistral_7b_ragged", 64, 32, 8, 4, 2, 32, 32, 1, 16384, seed=1004,
                                  ragged_min=1024),
    "million_token": Workload("million_token", 1, 32, 8, 2, 2, 128, 128, 0, 1048576, seed=1005),
}


def outlier_mask(w: Workload) -> np.ndarray:
    """[Hkv][128] float32 multipliers for the key channels (1 everywhere except the outlier pairs)."""
    m = np.ones((w.num_kv_heads, HEAD_DIM), np.float32)
    if w.outlier_channels <= 0:
        return m
    g = torch.Generator().manual_seed(w.seed * 31 + 5)
    if w.outlier_per_head:
        ch = torch.randperm(HEAD_DIM, generator=g)[: w.outlier_channels].numpy()
        m[:, ch] = w.outlier_scale
    else:
        flat = torch.randperm(w.num_kv_heads * HEAD_DIM, generator=g)[: w.outlier_channels].numpy()
        m.reshape(-1)[flat] = w.outlier_scale
    return m


def _unit_gen(w: Workload, b: int, kvh: int, salt: int) -> torch.Generator:
    return torch.Generator().manual_seed(((w.seed * 1_000_003 + b) * 4099 + kvh) * 8 + salt)


def unit_kv(w: Workload, b: int, kvh: int, T: int, mask: Optional[np.ndarray] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Keys and values of one (sequence, KV head): fp16 [T][128] each (CPU tensors)."""
    if mask is None:
        mask = outlier_mask(w)
    g = _unit_gen(w, b, kvh, 0)
    k = torch.randn(T, HEAD_DIM, generator=g)
    k.mul_(torch.from_numpy(mask[kvh]))
    g = _unit_gen(w, b, kvh, 1)
    v = torch.randn(T, HEAD_DIM, generator=g)
    return k.to(torch.float16), v.to(torch.float16)


def full_kv(w: Workload, T: Optional[int] = None, device: str = "cpu") -> Tuple[torch.Tensor, torch.Tensor, np.ndarray]:
    """Prefill keys/values as fp16 [B][Tmax][Hkv][128] on ``device`` plus the per-sequence lengths.

    Tokens past a sequence's length are zero.
    """
    lens = w.seq_lens() if T is None else np.full((w.batch,), T, np.int64)
    Tmax = int(lens.max())
    mask = outlier_mask(w)
    k = torch.zeros(w.batch, Tmax, w.num_kv_heads, HEAD_DIM, dtype=torch.float16, device=device)
    v = torch.zeros_like(k)
    for b in range(w.batch):
        Tb = int(lens[b])
        for h in range(w.num_kv_heads):
            ku, vu = unit_kv(w, b, h, Tb, mask)
            k[b, :Tb, h].copy_(ku, non_blocking=False)
            v[b, :Tb, h].copy_(vu, non_blocking=False)
    return k, v, lens


def append_tokens(w: Workload, step: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """The token appended to every sequence at decode step ``step``: fp16 [B][Hkv][128] keys and values."""
    mask = torch.from_numpy(outlier_mask(w))
    g = torch.Generator().manual_seed(w.seed * 104729 + 2 * step + 1)
    k = torch.randn(w.batch, w.num_kv_heads, HEAD_DIM, generator=g) * mask
    v = torch.randn(w.batch, w.num_kv_heads, HEAD_DIM, generator=g)
    return k.to(torch.float16), v.to(torch.float16)


def query(w: Workload, step: int = 0) -> torch.Tensor:
    """Decode queries: fp16 [B][Hq][128]."""
    g = torch.Generator().manual_seed(w.seed * 15485863 + step)
    return torch.randn(w.batch, w.num_q_heads, HEAD_DIM, generator=g).to(torch.float16)
