"""Seeded synthetic inputs for mixed-head (DuoAttention) attention.

This module is shared by the CUDA path's tests/benchmarks and by the oracle's
tests. It holds only input recipes (shapes, seeds, value distributions, the
retrieval/streaming head assignment); none of the attention arithmetic.

Workloads follow the MHA and GQA models the DuoAttention pages evaluate
(Llama-2-7B-32K-shaped MHA with 25 % retrieval heads, Llama-3-8B-shaped GQA
with 50 % retrieval KV heads; DuoAttention abstract and project card, "Limitations
& Caveats"). Values are N(0, 1) rounded to bf16.

Token stream: every (layer, position) owns q/k/v rows drawn from a torch
generator seeded per 4096-position block, so any range of positions can be
produced on its own and a decode step at position p sees the same rows a
longer prefill would (decode inputs continue the prefill stream).
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Sequence

import torch

BLOCK = 4096  # positions per independently seeded block


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    sink: int
    recent: int
    retrieval_ratio: float
    num_layers: int = 1
    prefill_len: int = 0      # tokens pre-filled through chunked prefill
    chunk: int = 4096         # prefill chunk length
    decode_steps: int = 0     # decode steps after the prefill
    context: int = 0          # for decode-only workloads: cache pre-filled by append
    sink_key_scale: int = 0   # if >0: K rows at positions < 4 multiplied by this
    seed: int = 0
    explicit_retrieval: Optional[Sequence[int]] = None  # per-KV-head 0/1 override

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def retrieval_mask(w: Workload, layer: int = 0) -> List[int]:
    """Per-KV-head retrieval flags (1 = retrieval, 0 = streaming).

    round(ratio * Hkv) heads are retrieval; which ones is a seeded random
    permutation (torch.randperm, seed = w.seed + layer).
    """
    if w.explicit_retrieval is not None:
        return [int(x) for x in w.explicit_retrieval]
    h = w.num_kv_heads
    n_r = int(round(w.retrieval_ratio * h))
    g = torch.Generator().manual_seed(1_000_003 * (w.seed + layer) + 17)
    perm = torch.randperm(h, generator=g).tolist()
    chosen = set(perm[:n_r])
    return [1 if i in chosen else 0 for i in range(h)]


def _block_seed(seed: int, layer: int, block: int, what: int) -> int:
    return ((seed * 1_000_003 + layer) * 100_003 + block) * 7 + what


def _normal_bf16(shape, seed: int, device) -> torch.Tensor:
    dev = torch.device(device)
    g = torch.Generator(device=dev).manual_seed(seed)
    return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)


def tokens(w: Workload, layer: int, p0: int, n: int, device="cpu", which="qkv"):
    """q [B,n,Hq,D], k [B,n,Hkv,D], v [B,n,Hkv,D] (bf16) for positions [p0, p0+n).

    `which` selects the tensors returned (subset of "qkv", in that order).
    """
    B, Hq, Hkv, D = w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim
    out = {}
    specs = {"q": (Hq, 0), "k": (Hkv, 1), "v": (Hkv, 2)}
    for name in which:
        heads, tag = specs[name]
        parts = []
        blocks = range(p0 // BLOCK, (p0 + n - 1) // BLOCK + 1) if n > 0 else range(0)
        for blk in blocks:
            full = _normal_bf16((B, BLOCK, heads, D), _block_seed(w.seed, layer, blk, tag), device)
            lo = max(p0, blk * BLOCK) - blk * BLOCK
            hi = min(p0 + n, (blk + 1) * BLOCK) - blk * BLOCK
            parts.append(full[:, lo:hi])
        t = torch.cat(parts, dim=1) if parts else torch.empty((B, 0, heads, D), dtype=torch.bfloat16, device=device)
        if name == "k" and w.sink_key_scale and p0 < 4:
            m = min(4, p0 + n) - p0
            t[:, :m] = t[:, :m] * w.sink_key_scale  # power of two: exact in bf16
        out[name] = t.contiguous()
    return tuple(out[c] for c in which)


# The five workloads (sizes use binary K: 32K = 32768, 1M = 2**20).
TINY_MHA = Workload("tiny_mha_d64", batch=1, num_q_heads=4, num_kv_heads=4, head_dim=64,
                    sink=4, recent=64, retrieval_ratio=0.5, prefill_len=512, chunk=512,
                    decode_steps=16, explicit_retrieval=(1, 0, 1, 0))
LLAMA2_MHA = Workload("llama2_7b_mha_32k", batch=1, num_q_heads=32, num_kv_heads=32, head_dim=128,
                      sink=64, recent=256, retrieval_ratio=0.25, prefill_len=32768, chunk=4096,
                      decode_steps=128, sink_key_scale=8)
LLAMA3_GQA = Workload("llama3_8b_gqa_128k_decode_b4", batch=4, num_q_heads=32, num_kv_heads=8,
                      head_dim=128, sink=64, recent=256, retrieval_ratio=0.5, context=131072,
                      decode_steps=1)
GQA_STACK_1M = Workload("gqa_32layer_1m_decode", batch=1, num_q_heads=32, num_kv_heads=8, head_dim=128,
                        sink=64, recent=256, retrieval_ratio=0.5, num_layers=32, context=1 << 20,
                        decode_steps=1)


def mha_sweep(ratio: float, recent: int = 256, batch: int = 8, prefill: bool = False) -> Workload:
    if prefill:
        return Workload(f"mha_sweep_prefill_r{int(ratio*100)}_R{recent}", batch=1, num_q_heads=32,
                        num_kv_heads=32, head_dim=128, sink=64, recent=recent, retrieval_ratio=ratio,
                        prefill_len=65536, chunk=4096)
    return Workload(f"mha_sweep_decode_r{int(ratio*100)}_R{recent}", batch=batch, num_q_heads=32,
                    num_kv_heads=32, head_dim=128, sink=64, recent=recent, retrieval_ratio=ratio,
                    context=65536, decode_steps=1)
