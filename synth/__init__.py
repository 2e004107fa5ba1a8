"""Seeded synthetic inputs shaped like the pages' workloads.

Shared by the tests (which feed the same tensors to the CUDA library and to the
oracle) and by the benchmark.  This module draws random numbers only; it holds
none of the method's arithmetic.

Shapes come from the pages' models: the Llama-3-8B GQA skeleton of the record
"kv-efficiency/kivi-2bit-llama3-8b-gqa-8k" ("Model": 32 layers, 8 kv heads,
32 query heads, head_dim 128, 8K context) and the Llama-2 7B/13B MHA models
that record's "notes" and "Methodology" fields mention.  The key distribution
carries the structure "KIVI: A Tuning-Free Asymmetric 2bit Quantization for
KV Cache" reports (keys have outlier channels, values do not): either a few
channels scaled x10, or a log-normal scale per channel.  The pages' real
workloads (LongBench prompts through trained Llama weights) are not available;
these tensors stand in for them.
"""
from __future__ import annotations

import dataclasses

import torch

BASE_SEED = 0x4B495649


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_layers: int
    num_kv_heads: int
    num_q_heads: int
    head_dim: int
    context: int          # prefill length
    bits: int
    decode_steps: int     # append + attend steps after the prefill
    key_dist: str         # "outlier4x10" or "lognormal"
    index: int            # position in WORKLOADS, mixed into the seed

    @property
    def seed(self) -> int:
        return BASE_SEED + self.index

    def with_batch(self, batch: int) -> "Workload":
        return dataclasses.replace(self, batch=batch)


WORKLOADS = {
    w.name: w
    for w in [
        Workload("tiny", 1, 1, 2, 4, 64, 512, 2, 1, "outlier4x10", 0),
        Workload("llama2_7b_mha_layer", 8, 1, 32, 32, 128, 4096, 2, 64, "lognormal", 1),
        Workload("llama3_8b_gqa_8k", 16, 32, 8, 32, 128, 8192, 2, 64, "lognormal", 2),
        Workload("llama3_8b_gqa_8k_4bit", 32, 32, 8, 32, 128, 8192, 4, 1, "lognormal", 3),
        Workload("llama2_13b_mha_sweep", 16, 40, 40, 40, 128, 4096, 2, 1, "lognormal", 4),
    ]
}

# Tensor tags mixed into the per-tensor seed.
_TAG_KEY_SCALE, _TAG_K, _TAG_V, _TAG_Q, _TAG_KNEW, _TAG_VNEW, _TAG_QPROMPT = 1, 2, 3, 4, 5, 6, 7


def _gen(w: Workload, tag: int, layer: int, step: int, device) -> torch.Generator:
    seed = (w.seed * 1_000_003 + tag * 10_007 + layer * 101 + step) % (2**63 - 1)
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def key_channel_scale(w: Workload, layer: int, device="cpu") -> torch.Tensor:
    """Per (kv head, channel) key scale of a layer, fp32 [Hkv][D].

    outlier4x10: 1 everywhere except 4 channels per kv head (a seeded random
    choice) scaled x10.  lognormal: exp(N(0, 1)) per channel.
    """
    H, D = w.num_kv_heads, w.head_dim
    g = _gen(w, _TAG_KEY_SCALE, layer, 0, "cpu")
    if w.key_dist == "outlier4x10":
        s = torch.ones(H, D)
        for h in range(H):
            idx = torch.randperm(D, generator=g)[:4]
            s[h, idx] = 10.0
    elif w.key_dist == "lognormal":
        s = torch.exp(torch.randn(H, D, generator=g))
    else:
        raise ValueError(w.key_dist)
    return s.to(device)


def prefill_kv(w: Workload, layer: int, S: int | None = None, device="cpu"):
    """Prompt keys and values, bf16 [B][Hkv][S][D] each."""
    S = w.context if S is None else S
    shape = (w.batch, w.num_kv_heads, S, w.head_dim)
    sk = key_channel_scale(w, layer, device)[None, :, None, :]
    k = torch.randn(shape, generator=_gen(w, _TAG_K, layer, 0, device), device=device)
    k = (k * sk).to(torch.bfloat16)
    v = torch.randn(shape, generator=_gen(w, _TAG_V, layer, 0, device), device=device)
    return k, v.to(torch.bfloat16)


def step_kv(w: Workload, layer: int, step: int, device="cpu"):
    """Keys and values appended at decode step `step`, bf16 [B][Hkv][D] each."""
    shape = (w.batch, w.num_kv_heads, w.head_dim)
    sk = key_channel_scale(w, layer, device)[None]
    k = torch.randn(shape, generator=_gen(w, _TAG_KNEW, layer, step, device), device=device)
    v = torch.randn(shape, generator=_gen(w, _TAG_VNEW, layer, step, device), device=device)
    return (k * sk).to(torch.bfloat16), v.to(torch.bfloat16)


def query(w: Workload, layer: int, step: int, device="cpu"):
    """Decode query of step `step`, bf16 [B][Hq][D]."""
    shape = (w.batch, w.num_q_heads, w.head_dim)
    q = torch.randn(shape, generator=_gen(w, _TAG_Q, layer, step, device), device=device)
    return q.to(torch.bfloat16)


def prompt_query(w: Workload, layer: int, S: int | None = None, device="cpu"):
    """Queries of the prompt's positions (prefill attention), bf16 [B][Hq][S][D]."""
    S = w.context if S is None else S
    shape = (w.batch, w.num_q_heads, S, w.head_dim)
    q = torch.randn(shape, generator=_gen(w, _TAG_QPROMPT, layer, 0, device), device=device)
    return q.to(torch.bfloat16)


def bf16_bits(t: torch.Tensor):
    """numpy uint16 view of a bf16 tensor's bit patterns (host copy)."""
    import numpy as np

    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
