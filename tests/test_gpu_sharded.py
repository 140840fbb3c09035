"""Head-sharded layers on the GPU, against the fp64 oracle.

  - world size 1 (no process group): ShardedDuoLayers runs the library's
    kernels over every head and gathers trivially;
  - the shares of 2 and 4 ranks laid out in one process on one GPU (explicit
    world/rank, no collective, the ranks run one after the other): each rank's
    cache holds only its own heads with its own retrieval flags, and the
    assembled outputs of all ranks equal the oracle's over the full layer.
Chunked prefill, cache append and decode steps, GQA groups of 4, a 3-layer
stack whose retrieval heads differ per layer.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from duo_harness import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sharded():
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    from mixed_head_kv_b200 import sharded as mod
    return mod


W = workloads.Workload("sharded", batch=2, num_q_heads=16, num_kv_heads=4, head_dim=128, sink=8, recent=96,
                       retrieval_ratio=0.5, num_layers=3, seed=21)
CHUNKS = [300, 129]
STEPS = 3


def _run(sharded, world):
    masks = [workloads.retrieval_mask(W, l) for l in range(W.num_layers)]
    flat = [m for ms in masks for m in ms]
    T = sum(CHUNKS) + STEPS
    kw = {} if world == 1 else {"world": world}
    ranks = [sharded.ShardedDuoLayers(W.num_layers, W.batch, W.num_q_heads, W.num_kv_heads, W.head_dim, W.sink,
                                      W.recent, T + 8, flat, **(dict(kw, rank=r) if kw else {}))
             for r in range(world)]
    outs = {}
    for layer in range(W.num_layers):
        q, k, v = (x.cuda() for x in workloads.tokens(W, layer, 0, T))
        rows = []
        p = 0
        for c in CHUNKS:
            parts = []
            for rk in ranks:
                ql, kl, vl = rk.shard(layer, q[:, p:p + c], k[:, p:p + c], v[:, p:p + c])
                parts.append(rk.prefill_local(layer, ql, kl, vl))
                rk.append(layer, kl, vl)
            rows.append(ranks[0].assemble(layer, parts))
            p += c
        for _ in range(STEPS):
            parts = []
            for rk in ranks:
                ql, kl, vl = rk.shard(layer, q[:, p], k[:, p], v[:, p])
                parts.append(rk.decode_local(layer, ql, kl, vl))
            rows.append(ranks[0].assemble(layer, parts)[:, None])
            p += 1
        outs[layer] = torch.cat(rows, dim=1)
    torch.cuda.synchronize()
    for rk in ranks:
        assert rk.cache.error_flags() == 0
        rk.close()
    return outs, masks


@pytest.mark.parametrize("world", [1, 2, 4])
def test_sharded_layers_match_oracle(sharded, world):
    outs, masks = _run(sharded, world)
    T = sum(CHUNKS) + STEPS
    for layer in range(W.num_layers):
        q, k, v = workloads.tokens(W, layer, 0, T)
        ref = oracle.attention(q.permute(0, 2, 1, 3), np.arange(T), k.permute(0, 2, 1, 3), v.permute(0, 2, 1, 3),
                               masks[layer], W.sink, W.recent).transpose(0, 2, 1, 3)
        assert_close(outs[layer].cpu(), ref, f"world {world} layer {layer}")


def test_sharded_world_size_1_gather_through_the_group_path(sharded):
    """Without explicit world/rank and no process group the plan is one rank and
    gather() returns the outputs in head order unchanged."""
    lay = sharded.ShardedDuoLayers(1, 1, 8, 2, 64, 4, 16, 64, [1, 0])
    assert (lay.world, lay.rank) == (1, 0)
    q, k, v = (x.cuda() for x in workloads.tokens(
        workloads.Workload("s1", batch=1, num_q_heads=8, num_kv_heads=2, head_dim=64, sink=4, recent=16,
                           retrieval_ratio=0.5, explicit_retrieval=(1, 0)), 0, 0, 40))
    out = lay.prefill(0, *lay.shard(0, q, k, v))
    ref = oracle.attention(q.cpu().permute(0, 2, 1, 3), np.arange(40), k.cpu().permute(0, 2, 1, 3),
                           v.cpu().permute(0, 2, 1, 3), [1, 0], 4, 16).transpose(0, 2, 1, 3)
    torch.cuda.synchronize()
    assert_close(out.cpu(), ref, "world 1 prefill")
    lay.close()
