"""Head-sharded mixed-head attention: one process per GPU, KV heads split across ranks.

DuoAttention's heads are independent during attention: a retrieval head reads
only its own full cache and a streaming head only its own sink + recent cache
(DuoAttention abstract, pith.science review page, "read the original
abstract"). A layer therefore shards by KV head with no exchange inside
attention; the only collective is the gather of the head outputs that the
model's output projection needs, and it sits outside the kernels.

Retrieval heads are the heavy units (their caches grow with the context,
streaming caches stay at sink + recent tokens), so the partition balances them:
every rank owns the same number of KV heads of every layer, and both per layer
and over the whole stack no rank holds more than one retrieval head above
another (partition_kv_heads).

Each rank keeps an ordinary duo_cache (libduo) over its own heads and runs the
same kernels on them. Its inputs are the tensors of its own heads, in the order
`local_q_heads(layer)` / `local_kv_heads(layer)` give (a tensor-parallel model
computes exactly these heads in its QKV projection; `shard` slices them out of
full-head tensors for callers that have those). `gather` all-gathers the
ranks' outputs over the process group (NCCL on GPUs) and puts every head back
at its global index.

This module is host plumbing: partition, per-rank cache set-up, and one
all-gather per call. Every attention step runs in libduo's kernels.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch

from . import DuoCache


def partition_kv_heads(is_retrieval: Sequence[int], num_layers: int, num_kv_heads: int, world: int) -> List[List[List[int]]]:
    """KV heads owned by each rank, per layer: plan[layer][rank] = sorted global KV head indices.

    is_retrieval: flat [num_layers * num_kv_heads] 0/1 flags. Needs num_kv_heads
    divisible by world: every rank owns num_kv_heads / world heads of each layer,
    so the per-rank caches share one layout and the gathered outputs have equal
    sizes. Layer by layer, every rank gets floor(n_retrieval / world) retrieval
    heads and the remaining n_retrieval mod world go, one each, to the ranks that
    hold the fewest retrieval heads over the layers so far (lowest rank first on
    a tie); streaming heads fill the other places. So per layer and over the
    stack, no rank holds more than one retrieval head above any other."""
    if world < 1 or num_kv_heads % world != 0:
        raise ValueError(f"num_kv_heads={num_kv_heads} must be a positive multiple of world={world}")
    mask = [int(x) for x in is_retrieval]
    if len(mask) != num_layers * num_kv_heads or any(x not in (0, 1) for x in mask):
        raise ValueError("is_retrieval must hold num_layers * num_kv_heads flags of 0 or 1")
    per_rank = num_kv_heads // world
    totals = [0] * world
    plan = []
    for layer in range(num_layers):
        m = mask[layer * num_kv_heads:(layer + 1) * num_kv_heads]
        retr = [g for g in range(num_kv_heads) if m[g]]
        strm = [g for g in range(num_kv_heads) if not m[g]]
        base, extra = divmod(len(retr), world)
        favoured = set(sorted(range(world), key=lambda r: (totals[r], r))[:extra])
        quota = [base + (1 if r in favoured else 0) for r in range(world)]
        owned = [[] for _ in range(world)]
        it = iter(retr)
        for r in range(world):
            owned[r].extend(next(it) for _ in range(quota[r]))
            totals[r] += quota[r]
        it = iter(strm)
        for r in range(world):
            owned[r].extend(next(it) for _ in range(per_rank - quota[r]))
        plan.append([sorted(o) for o in owned])
    return plan


def _world_and_rank(group):
    dist = torch.distributed
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


class HeadShardPlan:
    """Which heads this rank owns, and the gather that puts all ranks' head
    outputs back in global head order (no cache; see ShardedDuoLayers).

    is_retrieval: flat [num_layers * num_kv_heads] 0/1 flags; `group` is the
    process group (None: the default group when torch.distributed is
    initialised, else a single rank). `world` and `rank`, when given, replace
    the group's (to lay out one rank's share without a process group; such a
    plan assembles outputs with `assemble`, not `gather`)."""

    def __init__(self, num_layers: int, num_q_heads: int, num_kv_heads: int, is_retrieval: Sequence[int],
                 group=None, world: Optional[int] = None, rank: Optional[int] = None):
        if num_kv_heads < 1 or num_q_heads % num_kv_heads != 0:
            raise ValueError("num_q_heads must be a multiple of num_kv_heads")
        self.group = group
        self.world, self.rank = _world_and_rank(group) if world is None else (world, rank)
        self._explicit = world is not None
        if not 0 <= self.rank < self.world:
            raise ValueError(f"rank {self.rank} outside world {self.world}")
        self.G = num_q_heads // num_kv_heads
        self.num_layers, self.num_q_heads, self.num_kv_heads = num_layers, num_q_heads, num_kv_heads
        self.plan = partition_kv_heads(is_retrieval, num_layers, num_kv_heads, self.world)
        mask = [int(x) for x in is_retrieval]
        self.kv_heads = [self.plan[l][self.rank] for l in range(num_layers)]
        # the rank's own retrieval flags, [num_layers][num_kv_heads / world] flattened
        self.local_mask = [mask[l * num_kv_heads + g] for l in range(num_layers) for g in self.kv_heads[l]]
        # Gathered order: rank-major, each rank's query heads in its local order.
        self._gathered = [torch.tensor([g * self.G + i for r in range(self.world) for g in self.plan[l][r]
                                        for i in range(self.G)], dtype=torch.long) for l in range(num_layers)]
        self._dev_index = {}

    # ------------------------------------------------------------------ heads
    def local_kv_heads(self, layer: int) -> List[int]:
        return list(self.kv_heads[layer])

    def local_q_heads(self, layer: int) -> List[int]:
        return [g * self.G + i for g in self.kv_heads[layer] for i in range(self.G)]

    def shard(self, layer: int, q, k, v):
        """This rank's heads of full-head tensors (head axis = -2): q [..., Hq, D],
        k, v [..., Hkv, D]. Returns contiguous (q_local, k_local, v_local)."""
        qi = self._index(layer, "q", q.device)
        ki = self._index(layer, "kv", k.device)
        return (q.index_select(-2, qi).contiguous(), k.index_select(-2, ki).contiguous(),
                v.index_select(-2, ki).contiguous())

    def _index(self, layer, kind, device):
        key = (layer, kind, str(device))
        if key not in self._dev_index:
            heads = self.local_q_heads(layer) if kind == "q" else self.local_kv_heads(layer)
            self._dev_index[key] = torch.tensor(heads, dtype=torch.long, device=device)
        return self._dev_index[key]

    # ------------------------------------------------------------------ gather
    def assemble(self, layer: int, outs, out=None):
        """Place the ranks' outputs (a list, rank order, each [..., Hq / world, D]) at
        their global query heads: returns (or fills `out`) [..., Hq, D]."""
        if len(outs) != self.world:
            raise ValueError(f"expected {self.world} rank outputs, got {len(outs)}")
        first = outs[0]
        lead = tuple(first.shape[:-2])
        hl, D = first.shape[-2], first.shape[-1]
        nd = len(lead)
        gathered = torch.cat(list(outs), dim=nd) if self.world > 1 else first  # [*lead, world * hl, D]
        if out is None:
            out = torch.empty(lead + (self.num_q_heads, D), dtype=first.dtype, device=first.device)
        out.index_copy_(nd, self._gathered[layer].to(out.device), gathered)
        return out

    def gather(self, layer: int, out_local, out=None):
        """All-gather every rank's [..., Hq / world, D] output over the process group
        and return (or fill `out`) the [..., Hq, D] tensor with every query head at
        its global index."""
        if self.world == 1:
            return self.assemble(layer, [out_local], out)
        if self._explicit:
            raise RuntimeError("a plan laid out with explicit world/rank has no process group: use assemble()")
        flat = out_local.contiguous().view(-1)
        buf = torch.empty(self.world * flat.numel(), dtype=out_local.dtype, device=out_local.device)
        torch.distributed.all_gather_into_tensor(buf, flat, group=self.group)  # rank-major concatenation
        parts = buf.view((self.world,) + tuple(out_local.shape)).unbind(0)
        return self.assemble(layer, parts, out)


class ShardedDuoLayers(HeadShardPlan):
    """This rank's share of a head-sharded mixed-head attention stack: the
    HeadShardPlan of its heads and a DuoCache over them.

    Arguments as DuoCache, with the full model's head counts and the flat
    [num_layers * num_kv_heads] retrieval mask."""

    def __init__(self, num_layers: int, batch: int, num_q_heads: int, num_kv_heads: int, head_dim: int, sink: int,
                 recent: int, max_len: int, is_retrieval: Sequence[int], softmax_scale: float = 0.0,
                 device="cuda", group=None, world: Optional[int] = None, rank: Optional[int] = None):
        super().__init__(num_layers, num_q_heads, num_kv_heads, is_retrieval, group, world, rank)
        self.cache = DuoCache(num_layers, batch, num_q_heads // self.world, num_kv_heads // self.world, head_dim,
                              sink, recent, max_len, self.local_mask, softmax_scale=softmax_scale, device=device)

    def prefill_local(self, layer: int, q_local, k_local, v_local, stream=None):
        """duo_prefill over this rank's heads: returns its [B, C, Hq / world, D] output."""
        o = torch.empty_like(q_local)
        self.cache.prefill(layer, q_local, k_local, v_local, o, stream)
        return o

    def decode_local(self, layer: int, q_local, k_new_local, v_new_local, stream=None):
        """duo_decode over this rank's heads: returns its [B, Hq / world, D] output."""
        o = torch.empty_like(q_local)
        self.cache.decode(layer, q_local, k_new_local, v_new_local, o, stream)
        return o

    def prefill(self, layer: int, q_local, k_local, v_local, out=None, stream=None):
        """Prefill of this rank's heads, then the gather of all heads' outputs."""
        return self.gather(layer, self.prefill_local(layer, q_local, k_local, v_local, stream), out)

    def append(self, layer: int, k_local, v_local, stream=None):
        self.cache.append(layer, k_local, v_local, stream)

    def decode(self, layer: int, q_local, k_new_local, v_new_local, out=None, stream=None):
        """Decode step of this rank's heads, then the gather of all heads' outputs."""
        return self.gather(layer, self.decode_local(layer, q_local, k_new_local, v_new_local, stream), out)

    def close(self):
        self.cache.close()
