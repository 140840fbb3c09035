"""Head-sharded layers, host side (no GPU): the partition of KV heads across
ranks and the gather of the ranks' head outputs, with world size 2 on the
gloo backend (two CPU processes). Stand-in attention outputs carry each query
head's global index, so a head that lands in the wrong place, or twice, shows.
"""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import workloads
from mixed_head_kv_b200.sharded import HeadShardPlan, partition_kv_heads


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _check_plan(plan, mask, layers, hkv, world):
    totals = [0] * world
    for l in range(layers):
        owned = [h for r in range(world) for h in plan[l][r]]
        assert sorted(owned) == list(range(hkv)), f"layer {l}: every KV head owned exactly once"
        assert all(len(plan[l][r]) == hkv // world for r in range(world))
        cnt = [sum(mask[l * hkv + g] for g in plan[l][r]) for r in range(world)]
        assert max(cnt) - min(cnt) <= 1, f"layer {l}: retrieval heads per rank {cnt}"
        totals = [t + c for t, c in zip(totals, cnt)]
    assert max(totals) - min(totals) <= 1, f"retrieval heads over the stack per rank {totals}"


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_partition_balances_retrieval_heads(world):
    w = workloads.GQA_STACK_1M  # 32 layers x 8 KV heads, half of them retrieval, chosen per layer by seed
    mask = [m for l in range(w.num_layers) for m in workloads.retrieval_mask(w, l)]
    _check_plan(partition_kv_heads(mask, w.num_layers, w.num_kv_heads, world), mask, w.num_layers,
                w.num_kv_heads, world)


def test_partition_random_masks_and_rejections():
    g = torch.Generator().manual_seed(3)
    for _ in range(300):
        world = [1, 2, 4, 8][int(torch.randint(0, 4, (1,), generator=g))]
        hkv = world * int(torch.randint(1, 5, (1,), generator=g))
        layers = int(torch.randint(1, 7, (1,), generator=g))
        mask = torch.randint(0, 2, (layers * hkv,), generator=g).tolist()
        _check_plan(partition_kv_heads(mask, layers, hkv, world), mask, layers, hkv, world)
    with pytest.raises(ValueError):
        partition_kv_heads([1, 0, 1], 1, 3, 2)  # 3 KV heads over 2 ranks
    with pytest.raises(ValueError):
        partition_kv_heads([1, 0], 2, 2, 1)  # wrong mask length
    with pytest.raises(ValueError):
        partition_kv_heads([2, 0], 1, 2, 1)  # not a 0/1 flag


def _rank_main(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = workloads.Workload("shard", batch=3, num_q_heads=16, num_kv_heads=4, head_dim=8, sink=4, recent=16,
                               retrieval_ratio=0.5, num_layers=3)
        mask = [m for l in range(3) for m in workloads.retrieval_mask(w, l)]
        plan = HeadShardPlan(3, 16, 4, mask)
        assert (plan.world, plan.rank) == (world, rank)
        # every rank computes the same partition
        plans = [None] * world
        torch.distributed.all_gather_object(plans, plan.plan)
        assert all(p == plan.plan for p in plans)
        for layer in range(3):
            qh = plan.local_q_heads(layer)
            assert qh == [g * 4 + i for g in plan.local_kv_heads(layer) for i in range(4)]
            assert plan.local_mask[layer * 2:(layer + 1) * 2] == [mask[layer * 4 + g] for g in plan.local_kv_heads(layer)]
            # shard(): full-head tensors whose head h holds the value h
            T = 5
            q = torch.arange(16, dtype=torch.float32).view(1, 1, 16, 1).expand(3, T, 16, 8).contiguous()
            k = torch.arange(4, dtype=torch.float32).view(1, 1, 4, 1).expand(3, T, 4, 8).contiguous()
            ql, kl, vl = plan.shard(layer, q, k, k)
            assert ql.shape == (3, T, 8, 8) and kl.shape == (3, T, 2, 8)
            assert ql[0, 0, :, 0].tolist() == [float(h) for h in qh]
            assert kl[0, 0, :, 0].tolist() == [float(g) for g in plan.local_kv_heads(layer)]
            # gather(): stand-in outputs carrying (global head, position, rank) come back in head order
            pos = torch.arange(T, dtype=torch.float32).view(1, T, 1, 1)
            out_local = ql * 1000 + pos + 0.25 * rank
            full = plan.gather(layer, out_local)
            assert full.shape == (3, T, 16, 8)
            owner = {h: r for r in range(world) for g in plan.plan[layer][r] for h in range(g * 4, g * 4 + 4)}
            for h in range(16):
                expect = h * 1000 + pos[0, :, 0, 0] + 0.25 * owner[h]
                assert torch.equal(full[1, :, h, 3], expect), (layer, h)
            # decode-shaped outputs [batch, heads, D] and a caller-provided output tensor
            dec = torch.empty(3, 16, 8)
            plan.gather(layer, ql[:, 0] + 0.5, out=dec)
            assert torch.equal(dec[:, :, 0], torch.arange(16, dtype=torch.float32).expand(3, 16) + 0.5)
        open(os.path.join(result_dir, f"rank{rank}.ok"), "w").write("ok")
    finally:
        torch.distributed.destroy_process_group()


def test_gather_world_size_2_gloo(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    assert sorted(os.listdir(tmp_path)) == ["rank0.ok", "rank1.ok"]
