"""The benchmark's multi-rank plumbing on CPU (gloo, world size 2): replicas
agree on the max step time, and the algorithmic-work formulas match brute force."""
import os
import socket

import numpy as np
import torch
import torch.multiprocessing as mp

import bench
import oracle
import workloads


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    bench.init_dist(world, "gloo")
    w, r, _ = bench.dist_env()
    got = bench.max_over_ranks(10.0 + 5.0 * r)
    bench.barrier()
    out[r] = got
    torch.distributed.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 15.0, 1: 15.0}


def test_single_rank_is_identity():
    assert bench.max_over_ranks(3.5) == 3.5


def test_prefill_flops_counts_unmasked_pairs():
    w = workloads.Workload("t", batch=2, num_q_heads=4, num_kv_heads=2, head_dim=8, sink=2, recent=3,
                           retrieval_ratio=0.5, explicit_retrieval=(1, 0))
    mask = workloads.retrieval_mask(w)
    p0, n = 5, 9
    pairs = 0
    for h in range(4):
        g = h // 2
        for p in range(p0, p0 + n):
            pairs += sum(oracle.key_allowed(mask[g], p, j, w.sink, w.recent) for j in range(p + 1))
    assert bench.prefill_flops(w, mask, p0, n) == 4 * 8 * 2 * pairs


def test_append_bytes_counts_written_slots():
    w = workloads.Workload("t", batch=1, num_q_heads=2, num_kv_heads=2, head_dim=8, sink=3, recent=4,
                           retrieval_ratio=0.5, explicit_retrieval=(1, 0))
    mask = workloads.retrieval_mask(w)
    for L, n in [(0, 2), (0, 10), (2, 5), (7, 20), (1, 1)]:
        pos = np.arange(L, L + n)
        kept = [p for p in pos if p < w.sink or p >= L + n - w.recent]
        rows = n + len(kept)
        assert bench.append_bytes(w, mask, L, n) == rows * 2 * 8 * 2 * 2, (L, n)


def test_reference_arm_line():
    """`bench.py --impl reference` (the oracle timed on the host cores) prints one
    line with the headline's metric, unit, direction and config, its own
    cpu_baseline and an e2e block without host-device copies."""
    import json
    import subprocess
    import sys

    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "1",
                          "--cpu-budget", "1"], cwd=root, env=env, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    w = workloads.LLAMA2_MHA
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "tokens/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 1 and d["warmup"] == 1
    assert d["config"] == bench.main_config(w, workloads.retrieval_mask(w), 1)
    assert d["value"] > 0 and d["value"] == d["cpu_baseline"]["value"] == d["e2e"]["value"]
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
