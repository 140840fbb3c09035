"""Benchmark of mixed-head (DuoAttention) attention on B200.

One step = the whole hot path over one sequence batch of the Llama-2-7B-shaped
MHA layer (32 heads, head_dim 128, 25 % retrieval heads chosen by seed, sink 64
+ recent 256, first 4 keys x8): chunked prefill of 32768 tokens in chunks of
4096 (duo_prefill + duo_cache_append per chunk), then 128 decode steps
(duo_decode). The cache length is reset to 0 at the start of each step.

Prints one JSON line. `value` = tokens processed per second (prefill + decode
tokens, all ranks), inputs resident in HBM. Sub-metrics: prefill TFLOP/s over
unmasked positions, decode KV-read GB/s and tokens/s. `e2e` repeats the step
through the same C ABI from pinned host buffers with the copies timed.

At N = 1 the line also carries `secondary`: every other configuration of the
benchmark definition (Llama-3-8B-shaped GQA decode at 128K, the MHA
retrieval-ratio sweep of decode and chunked prefill at 64K, the 32-layer GQA
stack at 1M), each with its own device time, roofline fraction and clock record.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--no-secondary]

Under torchrun (N > 1) every rank runs an independent replica (the method has
no cross-GPU exchange); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "decode KV-read GB/s & tokens/s; prefill unmasked TFLOP/s (mixed-head attn)"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0


# ----------------------------------------------------------------------------- rank plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import datetime
    if world > 1 and not torch.distributed.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank scalar (identity when not distributed)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device is not None and device.type == "cuda":
            torch.distributed.barrier(device_ids=[device.index])
        else:
            torch.distributed.barrier()


# ----------------------------------------------------------------------------- algorithmic work
def keys_seen(is_retr: int, p: np.ndarray, S: int, R: int) -> np.ndarray:
    """|K(p)|: keys a query at position p attends to (retrieval: p+1; streaming: min(p+1, S+R))."""
    return p + 1 if is_retr else np.minimum(p + 1, S + R)


def prefill_flops(w, mask, p0: int, n: int) -> float:
    """QK^T + PV flops over unmasked (query, key) pairs of positions [p0, p0+n)."""
    p = np.arange(p0, p0 + n, dtype=np.float64)
    tot = 0.0
    for g in range(w.num_kv_heads):
        tot += w.group * float(keys_seen(mask[g], p, w.sink, w.recent).sum())
    return tot * 4.0 * w.head_dim * w.batch


def decode_bytes(w, mask, L: int, retr_elem: int = 2) -> float:
    """Bytes one decode step at cache length L must move: every visible K/V row once
    (the new token's from the input), the new token's write, q and out. Retrieval
    rows take retr_elem bytes per element (2: bf16, 1: E4M3 codes)."""
    D, B = w.head_dim, w.batch
    retr = sum(L + 1 for g in range(w.num_kv_heads) if mask[g])
    strm = sum(min(L + 1, w.sink + w.recent) for g in range(w.num_kv_heads) if not mask[g])
    return B * ((retr * retr_elem + strm * 2) * 2 * D + w.num_kv_heads * 2 * D * 2 + 2 * w.num_q_heads * D * 2)


def append_bytes(w, mask, L: int, n: int) -> float:
    """Rows written by one append of n tokens at length L, K and V, read + written."""
    rows = 0
    for g in range(w.num_kv_heads):
        if mask[g]:
            rows += n
        else:
            sinks = max(0, min(L + n, w.sink) - L)
            rows += sinks + max(0, min(n - sinks, w.recent))
    return w.batch * rows * 2 * w.head_dim * 2 * 2


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(path))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def samples(self) -> int:
        try:
            return sum(1 for line in open(self.path) if line.strip())
        except OSError:
            return 0

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, smax, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            r = [x.strip() for x in r]
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except (ValueError, IndexError):
                continue
            for nm, val in zip(names, r[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- GPU arm
class Step:
    """Device-resident inputs and the launch sequence of one step."""

    def __init__(self, duo, w, device):
        self.duo, self.w, self.dev = duo, w, device
        self.mask = workloads.retrieval_mask(w)
        self.T = w.prefill_len + w.decode_steps
        self.C = w.chunk
        self.n_chunks = (w.prefill_len + self.C - 1) // self.C
        q, k, v = workloads.tokens(w, 0, 0, self.T, device=device)
        self.q, self.k, self.v = q, k, v
        P = w.prefill_len
        self.chunks = []
        for i in range(self.n_chunks):
            a, b = i * self.C, min(P, (i + 1) * self.C)
            qc, kc, vc = (x[:, a:b].contiguous() for x in (q, k, v))
            self.chunks.append((a, b - a, qc, kc, vc, torch.empty_like(qc)))
        self.dec = []
        for t in range(w.decode_steps):
            p = P + t
            qd, kd, vd = (x[:, p].contiguous() for x in (q, k, v))
            self.dec.append((p, qd, kd, vd, torch.empty_like(qd)))
        self.cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent,
                                  self.T, self.mask, device=device)
        self.h = self.cache.handle
        # Per chunk: the retrieval-item prefill kernel and the streaming-item one (each
        # only when the layer has heads of that kind), and the append; one decode per token.
        r = int(sum(self.mask))
        self.prefill_launches_per_chunk = int(r > 0) + int(r < len(self.mask))
        self.launches_per_step = (self.prefill_launches_per_chunk + 1) * self.n_chunks + w.decode_steps

    def run(self, stream_ptr, events=None):
        """Enqueue one step. events: dict kind -> list of (start, end) to record around launches."""
        lib = self.duo._lib
        self.duo.duo_cache_set_len(self.h, 0, 0)
        for (p0, n, qc, kc, vc, oc) in self.chunks:
            if events is not None:
                e0, e1 = events["prefill"].pop()
                e0.record()
            st = lib.duo_prefill(self.h, 0, qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), oc.data_ptr(), n,
                                 stream_ptr)
            if events is not None:
                e1.record()
                e2, e3 = events["append"].pop()
                e2.record()
            st |= lib.duo_cache_append(self.h, 0, kc.data_ptr(), vc.data_ptr(), n, stream_ptr)
            if events is not None:
                e3.record()
            if st:
                raise RuntimeError(f"prefill/append failed: {self.duo.duo_status_str(st)}")
        if events is not None:
            e0, e1 = events["decode"].pop()
            e0.record()  # one pair around the decode loop: consecutive decodes overlap (PDL)
        for (p, qd, kd, vd, od) in self.dec:
            st = lib.duo_decode(self.h, 0, qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), stream_ptr)
            if st:
                raise RuntimeError(f"decode failed: {self.duo.duo_status_str(st)}")
        if events is not None:
            e1.record()

    def work(self):
        w, m = self.w, self.mask
        pf = [prefill_flops(w, m, p0, n) for (p0, n, *_r) in self.chunks]
        ab = [append_bytes(w, m, p0, n) for (p0, n, *_r) in self.chunks]
        db = [decode_bytes(w, m, p) for (p, *_r) in self.dec]
        return pf, ab, db


def make_events(step, k):
    mk = lambda: (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    return {"prefill": [mk() for _ in range(step.n_chunks * k)],
            "append": [mk() for _ in range(step.n_chunks * k)],
            "decode": [mk() for _ in range(k)]}


def run_gpu(args):
    world, rank, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    init_dist(world, "nccl")
    import __graft_entry__
    __graft_entry__.build()
    import mixed_head_kv_b200 as duo

    w = workloads.LLAMA2_MHA
    step = Step(duo, w, device)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    # Clocks are sampled from the start of warm-up to the end of the timed region
    # (the timed region alone is shorter than nvidia-smi's start-up).
    clocks = ClockSampler(local)
    clocks.start()
    t_warm = time.perf_counter()
    while True:
        for _ in range(args.warmup):
            step.run(sp)
        torch.cuda.synchronize()
        if clocks.samples() >= 3 or time.perf_counter() - t_warm > 10.0:
            break
    if step.cache.error_flags() != 0:
        raise RuntimeError("device error flag set during warm-up")

    events = make_events(step, args.steps)
    all_events = {kname: list(v) for kname, v in events.items()}
    for v in events.values():
        v.reverse()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    torch.cuda.synchronize()
    t0.record()
    for _ in range(args.steps):
        step.run(sp, events)
    t1.record()
    torch.cuda.synchronize()
    barrier(device)
    clk = clocks.stop()
    ms_local = t0.elapsed_time(t1)
    ms = max_over_ranks(ms_local, device) / args.steps

    dur = {kname: [a.elapsed_time(b) for a, b in v] for kname, v in all_events.items()}
    pf, ab, db = step.work()
    tok_per_step = w.batch * (w.prefill_len + w.decode_steps)
    peaks = load_peaks()
    t_pf = sum(dur["prefill"]) / args.steps
    t_ap = sum(dur["append"]) / args.steps
    t_dc = sum(dur["decode"]) / args.steps
    prefill_tflops = sum(pf) / (t_pf * 1e-3) / 1e12
    decode_gbs = sum(db) / (t_dc * 1e-3) / 1e9
    append_gbs = sum(ab) / (t_ap * 1e-3) / 1e9
    decode_tok_s = w.batch * w.decode_steps / (t_dc * 1e-3)
    kernels = {
        # Every prefill launch is timed on its own (CUDA events around it): the burst peak applies.
        "prefill": {"bound": "tensor", "achieved": prefill_tflops, "peak": peaks["bf16_tflops"],
                    "unit": "TFLOP/s", "ms_per_step": t_pf,
                    "launches_per_step": step.prefill_launches_per_chunk * step.n_chunks},
        "decode": {"bound": "hbm", "achieved": decode_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "ms_per_step": t_dc, "launches_per_step": w.decode_steps},
        "append": {"bound": "hbm", "achieved": append_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                   "ms_per_step": t_ap, "launches_per_step": step.n_chunks},
    }
    for kv in kernels.values():
        kv["frac"] = kv["achieved"] / kv["peak"]
    dom = max(kernels, key=lambda kname: kernels[kname]["ms_per_step"])
    traffic = load_traffic(dom)
    roof = {k2: kernels[dom][k2] for k2 in ("bound", "achieved", "peak", "unit", "frac")}
    roof.update({"kernel": dom, "traffic": traffic, "peak_source": peaks["source"]})

    e2e = run_e2e(duo, step, args, sp, device)
    cpu = None
    if rank == 0:
        cpu = cpu_baseline(step, budget_s=args.cpu_budget)
    secondary = None
    if world == 1 and not args.no_secondary:
        step.cache.close()
        del step.chunks, step.dec
        torch.cuda.empty_cache()
        secondary = run_secondary(duo, peaks)
    res = {
        "metric": METRIC, "value": world * tok_per_step / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": main_config(w, step.mask, world),
        "prefill": {"unmasked_tflops": prefill_tflops, "ms": t_pf, "unmasked_flop": sum(pf),
                    "frac_of_measured_burst": prefill_tflops / peaks["bf16_tflops"],
                    "frac_of_nominal_2250": prefill_tflops / 2250.0},
        "decode": {"kv_read_gbs": decode_gbs, "tokens_per_s": decode_tok_s, "us_per_step": 1e3 * t_dc / w.decode_steps,
                   "frac_of_measured_hbm": decode_gbs / peaks["hbm_gbs"], "frac_of_nominal_8000": decode_gbs / 8000.0},
        "append": {"gbs": append_gbs, "ms": t_ap},
        "roofline": roof, "kernels": kernels, "e2e": e2e,
        "gpu_launches": step.launches_per_step * args.steps,
        "clocks": dict(clk, window="warm-up through timed region"),
    }
    if cpu is not None:
        res["cpu_baseline"] = cpu
    if secondary is not None:
        res["secondary"] = secondary
    if rank == 0:
        print(json.dumps(res))
    step.cache.close()
    if world > 1:
        torch.distributed.destroy_process_group()


def load_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if it is current."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(path))
        return d.get(kernel, {}).get("bytes_per_launch")
    except Exception:
        return None


def gpu_local_cpus(device):
    """CPUs of the GPU's own NUMA node (sysfs, read only), within this process's
    allowed set; None when unknown."""
    try:
        pr = torch.cuda.get_device_properties(device)
        path = (f"/sys/bus/pci/devices/{pr.pci_domain_id:04x}:{pr.pci_bus_id:02x}:{pr.pci_device_id:02x}.0/"
                "local_cpulist")
        cpus = set()
        for part in open(path).read().strip().split(","):
            a, _, b = part.partition("-")
            cpus.update(range(int(a), int(b or a) + 1))
        cpus &= os.sched_getaffinity(0)
        return cpus or None
    except Exception:
        return None


def run_e2e(duo, step, args, sp, device):
    """See run_e2e_on: the host thread runs on the GPU's NUMA node while the pinned
    buffers are allocated and filled, so the copies read node-local memory."""
    old = os.sched_getaffinity(0)
    local = gpu_local_cpus(device)
    if local:
        os.sched_setaffinity(0, local)
    try:
        out = run_e2e_on(duo, step, args, sp, device)
    finally:
        if local:
            os.sched_setaffinity(0, old)
    out["host_cpus"] = len(local) if local else "unchanged"
    return out


def run_e2e_on(duo, step, args, sp, device):
    """The same step from pinned host buffers through the same C ABI: every input is
    copied host -> device and every output device -> host inside the timed region.
    Copies run on their own streams and overlap the kernels: the upload of chunk i+1
    runs while chunk i computes, each output is read back as soon as it is ready, and
    consecutive steps use alternate device buffers, so the next step's uploads start
    while this step decodes (the kernels themselves stay in order on one stream)."""
    lib = duo._lib
    hc = [(qc.cpu().pin_memory(), kc.cpu().pin_memory(), vc.cpu().pin_memory(),
           torch.empty_like(oc, device="cpu").pin_memory()) for (_p, _n, qc, kc, vc, oc) in step.chunks]
    # The decode steps' inputs travel as one [steps, 3, ...] block and their outputs as
    # one [steps, ...] block (one copy each way instead of hundreds of small ones).
    n_dec = len(step.dec)
    q0, k0 = step.dec[0][1], step.dec[0][2]
    nq, nk = q0.numel(), k0.numel()
    dec_in_h = torch.stack([torch.cat([qd.flatten(), kd.flatten(), vd.flatten()])
                            for (_p, qd, kd, vd, _od) in step.dec]).cpu().pin_memory()
    dec_out_h = torch.empty((n_dec,) + tuple(q0.shape), dtype=torch.bfloat16).pin_memory()
    h2d = sum(a.numel() * 2 + b.numel() * 2 + c.numel() * 2 for a, b, c, _ in hc) + dec_in_h.numel() * 2
    d2h = sum(o.numel() * 2 for *_x, o in hc) + dec_out_h.numel() * 2

    def dec_set():
        din = torch.empty_like(dec_in_h, device=device)
        dout = torch.empty_like(dec_out_h, device=device)
        views = [(p, din[t, :nq].view(q0.shape), din[t, nq:nq + nk].view(k0.shape),
                  din[t, nq + nk:].view(k0.shape), dout[t]) for t, (p, *_r) in enumerate(step.dec)]
        return din, dout, views

    # two sets of device buffers: the step's own chunk tensors and a copy of their shapes
    sets = [(step.chunks, dec_set()),
            ([(p0, n, torch.empty_like(qc), torch.empty_like(kc), torch.empty_like(vc), torch.empty_like(oc))
              for (p0, n, qc, kc, vc, oc) in step.chunks], dec_set())]
    main = torch.cuda.current_stream()
    up = torch.cuda.Stream(device=device)
    down = torch.cuda.Stream(device=device)
    n_c = len(step.chunks)
    ev_in = [[torch.cuda.Event() for _ in range(n_c + 1)] for _ in range(2)]
    ev_out = [[torch.cuda.Event() for _ in range(n_c + 1)] for _ in range(2)]
    done = [None, None]  # per buffer set: the last read-back of the step that used it

    def one(s):
        chunks, (din, dout, dec) = sets[s]
        with torch.cuda.stream(up):
            if done[s] is not None:
                up.wait_event(done[s])  # that step's kernels and read-backs are finished with the set
            for i, ((hq, hk, hv, _ho), (_p, _n, qc, kc, vc, _oc)) in enumerate(zip(hc, chunks)):
                qc.copy_(hq, non_blocking=True)
                kc.copy_(hk, non_blocking=True)
                vc.copy_(hv, non_blocking=True)
                ev_in[s][i].record(up)
            din.copy_(dec_in_h, non_blocking=True)
            ev_in[s][n_c].record(up)
        duo.duo_cache_set_len(step.h, 0, 0)
        for i, (p0, n, qc, kc, vc, oc) in enumerate(chunks):
            main.wait_event(ev_in[s][i])
            st = lib.duo_prefill(step.h, 0, qc.data_ptr(), kc.data_ptr(), vc.data_ptr(), oc.data_ptr(), n, sp)
            ev_out[s][i].record(main)
            st |= lib.duo_cache_append(step.h, 0, kc.data_ptr(), vc.data_ptr(), n, sp)
            if st:
                raise RuntimeError(f"prefill/append failed: {duo.duo_status_str(st)}")
        main.wait_event(ev_in[s][n_c])
        for (p, qd, kd, vd, od) in dec:
            st = lib.duo_decode(step.h, 0, qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), od.data_ptr(), sp)
            if st:
                raise RuntimeError(f"decode failed: {duo.duo_status_str(st)}")
        ev_out[s][n_c].record(main)
        with torch.cuda.stream(down):
            for i, ((_hq, _hk, _hv, ho), (_p, _n, _qc, _kc, _vc, oc)) in enumerate(zip(hc, chunks)):
                down.wait_event(ev_out[s][i])
                ho.copy_(oc, non_blocking=True)
            down.wait_event(ev_out[s][n_c])
            dec_out_h.copy_(dout, non_blocking=True)
            done[s] = torch.cuda.Event()
            done[s].record(down)

    for i in range(max(2, args.warmup)):
        one(i % 2)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(device)
    t0.record()
    up.wait_stream(main)  # the first uploads start after t0
    for i in range(args.steps):
        one(i % 2)
    main.wait_stream(down)  # the last read-back is inside the timed region
    t1.record()
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), device) / args.steps
    world = dist_env()[0]
    tok = step.w.batch * step.T
    return {"value": world * tok / (ms * 1e-3), "unit": "tokens/s", "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "overlap": "uploads, kernels and read-backs on separate streams; alternate device buffers per step"}


# ----------------------------------------------------------------------------- oracle (CPU) timing
def oracle_sample(w, q, k, v, mask, positions):
    """Run the fp64 oracle for all heads at the given query positions; returns seconds."""
    import oracle
    pos = np.asarray(positions, dtype=np.int64)
    T = int(pos.max()) + 1
    qs = q[:, pos].permute(0, 2, 1, 3).contiguous()
    ks = k[:, :T].permute(0, 2, 1, 3).contiguous()
    vs = v[:, :T].permute(0, 2, 1, 3).contiguous()
    t = time.perf_counter()
    oracle.attention(qs, pos, ks, vs, mask, w.sink, w.recent)
    return time.perf_counter() - t


def sample_positions(w, stride):
    """Every `stride`-th prefill position plus the first and last decode positions."""
    pre = list(range(stride // 2, w.prefill_len, stride))
    dec = [w.prefill_len, w.prefill_len + w.decode_steps - 1]
    return pre + dec


def cpu_baseline(step_or_inputs, budget_s=15.0, stride=None):
    """Time the oracle as it stands on a bounded sample of the step's query positions."""
    import oracle
    oracle.build()
    if isinstance(step_or_inputs, Step):
        w, mask = step_or_inputs.w, step_or_inputs.mask
        q, k, v = (x.cpu() for x in (step_or_inputs.q, step_or_inputs.k, step_or_inputs.v))
    else:
        w, mask, (q, k, v) = step_or_inputs
    if stride is None:
        # Calibrate on a tiny sample, then pick the stride that fills about budget_s.
        probe = sample_positions(w, 8192)
        t = oracle_sample(w, q, k, v, mask, probe)
        per_pos = t / len(probe)
        n = max(4, int(budget_s / max(per_pos, 1e-6)))
        stride = max(16, w.prefill_len // n)
    pos = sample_positions(w, stride)
    t = oracle_sample(w, q, k, v, mask, pos)
    return {"value": w.batch * len(pos) / t, "unit": "tokens/s", "cores": oracle.num_threads(), "kind": "oracle",
            "seconds": t,
            "sample": f"{len(pos)} query positions (every {stride}th of the 32768 prefill positions + 2 decode "
                      f"positions), all {w.num_q_heads} heads, batch {w.batch}; fp64 C oracle, OpenMP"}


def main_config(w, mask, world):
    """The `config` of the headline line, shared by both arms."""
    return {"workload": w.name, "batch": w.batch, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "retrieval_kv_heads": int(sum(mask)), "sink": w.sink, "recent": w.recent,
            "prefill_len": w.prefill_len, "chunk": w.chunk, "decode_steps": w.decode_steps,
            "seq_len": w.prefill_len + w.decode_steps, "global_batch": w.batch * world,
            "parallelism": "replicas" if world > 1 else "single", "l2": "inputs larger than L2"}


def run_reference(args):
    world, rank, local = dist_env()
    if world > 1 and rank != 0:
        return
    w = workloads.LLAMA2_MHA
    mask = workloads.retrieval_mask(w)
    T = w.prefill_len + w.decode_steps
    q, k, v = workloads.tokens(w, 0, 0, T)
    inputs = (w, mask, (q, k, v))
    probe = cpu_baseline(inputs, stride=4096)  # calibration
    per_tok = 1.0 / probe["value"]
    total_budget = args.cpu_budget
    n_tok = max(4, int(total_budget / max(1, args.steps + args.warmup) / per_tok))
    stride = max(16, w.prefill_len // n_tok)
    for _ in range(args.warmup):
        cpu_baseline(inputs, stride=stride)
    secs, toks = 0.0, 0
    for _ in range(args.steps):
        r = cpu_baseline(inputs, stride=stride)
        secs += r["seconds"]
        toks += int(round(r["value"] * r["seconds"]))
    val = toks / secs
    res = {"impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": main_config(w, mask, world),
           "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                            "sample": r["sample"] + " per step"},
           "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(res))


# ----------------------------------------------------------------------------- secondary workloads
L2_BYTES = 126 * 2**20


def _fill_cache(duo, cache, w, layer, L, block=1 << 16):
    for c0 in range(0, L, block):
        n = min(block, L - c0)
        kk, vv = workloads.tokens(w, layer, c0, n, device="cuda", which="kv")
        cache.append(layer, kk, vv)


def _with_clocks(fn, min_reps=3, max_s=10.0):
    """Run fn() as warm-up until nvidia-smi has sampled at least 3 clock readings
    (at least min_reps times, at most max_s seconds), then once more as the timed
    run. Returns (the timed run's result, clocks over warm-up and timed run)."""
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    t0 = time.perf_counter()
    reps = 0
    while reps < min_reps or (clocks.samples() < 3 and time.perf_counter() - t0 < max_s):
        fn()
        reps += 1
    res = fn()
    clk = clocks.stop()
    return res, dict(clk, window="warm-up through timed run", warmup_reps=reps)


class DecodeCase:
    """Decode steps of one workload (one launch per layer per step) on an
    append-filled cache; device time per step with CUDA events."""

    def __init__(self, duo, w, layers, steps, kv_format=0):
        self.duo, self.w, self.layers, self.steps = duo, w, layers, steps
        self.kv_format = kv_format
        self.L = L = w.context
        self.masks = [workloads.retrieval_mask(w, l) for l in range(w.num_layers)]
        self.cache = duo.DuoCache(w.num_layers, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink,
                                  w.recent, L + steps + 1, [m for ms in self.masks for m in ms], kv_format=kv_format)
        for l in layers:
            _fill_cache(duo, self.cache, w, l, L)
        qkv = [workloads.tokens(w, l, L, steps, device="cuda") for l in layers]
        self.ins = [[tuple(x[:, t].contiguous() for x in qkv[i]) for t in range(steps)] for i in range(len(layers))]
        self.out = torch.empty_like(self.ins[0][0][0])
        elem = 1 if kv_format == duo.DUO_KV_E4M3 else 2
        self.bytes_per_step = sum(statistics.fmean(decode_bytes(w, self.masks[l], L + s, elem) for s in range(steps))
                                  for l in layers)
        # A step whose reads fit in L2 would be served from L2 on the next step:
        # flush L2 between timed steps then (a real model runs its other layers in between).
        self.flush = (torch.empty(4 * L2_BYTES, dtype=torch.uint8, device="cuda")
                      if self.bytes_per_step < 2 * L2_BYTES else None)

    def run(self):
        lib, sp = self.duo._lib, torch.cuda.current_stream().cuda_stream
        for l in self.layers:
            self.cache.set_length(l, self.L)
        ev = []
        if self.flush is None:
            ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
            ev[0][0].record()
        for t in range(self.steps):
            if self.flush is not None:
                self.flush.fill_(t & 0xFF)
                ev.append((torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)))
                ev[-1][0].record()
            for i, l in enumerate(self.layers):
                q, k, v = self.ins[i][t]
                if lib.duo_decode(self.cache.handle, l, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                  self.out.data_ptr(), sp):
                    raise RuntimeError("decode failed")
            if self.flush is not None:
                ev[-1][1].record()
        if self.flush is None:
            ev[0][1].record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) * 1e-3 / self.steps

    def result(self, peaks):
        t, clk = _with_clocks(self.run)
        if self.cache.error_flags():
            raise RuntimeError("device error flag set")
        w, gbs = self.w, self.bytes_per_step / t / 1e9
        return {"workload": w.name + ("_e4m3" if self.kv_format else ""), "phase": "decode",
                "retrieval_kv_format": "e4m3" if self.kv_format else "bf16",
                "batch": w.batch, "context": self.L, "layers": len(self.layers),
                "retrieval_kv_heads_per_layer": int(sum(self.masks[self.layers[0]])),
                "steps": self.steps, "us_per_step": t * 1e6, "tokens_per_s": w.batch / t, "kv_read_gbs": gbs,
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                             "frac": gbs / peaks["hbm_gbs"], "peak_source": peaks["source"]},
                "frac_of_nominal_8000": gbs / 8000.0,
                "l2": "flushed between steps" if self.flush is not None else "per-step reads larger than L2",
                "clocks": clk}

    def close(self):
        self.cache.close()
        del self.cache, self.ins, self.flush


class PrefillCase:
    """Chunked prefill of one workload (duo_prefill + duo_cache_append per chunk);
    device time of the prefill launches with CUDA events around each."""

    def __init__(self, duo, w):
        self.duo, self.w = duo, w
        self.mask = workloads.retrieval_mask(w)
        self.cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent,
                                  w.prefill_len, self.mask)
        q, k, v = workloads.tokens(w, 0, 0, w.prefill_len, device="cuda")
        self.chunks = [(p0, tuple(x[:, p0:p0 + w.chunk].contiguous() for x in (q, k, v)))
                       for p0 in range(0, w.prefill_len, w.chunk)]
        self.out = torch.empty_like(self.chunks[0][1][0])
        self.flop = sum(prefill_flops(w, self.mask, p0, w.chunk) for p0, _ in self.chunks)

    def run(self):
        self.cache.set_length(0, 0)
        ev = []
        for p0, (qc, kc, vc) in self.chunks:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            self.cache.prefill(0, qc, kc, vc, self.out)
            e1.record()
            ev.append((e0, e1))
            self.cache.append(0, kc, vc)
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) * 1e-3

    def result(self, peaks):
        t, clk = _with_clocks(self.run)
        if self.cache.error_flags():
            raise RuntimeError("device error flag set")
        w, tf = self.w, self.flop / t / 1e12
        return {"workload": w.name, "phase": "prefill", "batch": w.batch, "context": w.prefill_len, "chunk": w.chunk,
                "retrieval_kv_heads": int(sum(self.mask)), "ms_prefill_kernels": t * 1e3, "unmasked_tflops": tf,
                "unmasked_flop": self.flop,
                "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                             "frac": tf / peaks["bf16_tflops"], "peak_source": peaks["source"]},
                "frac_of_nominal_2250": tf / 2250.0, "l2": "inputs larger than L2", "clocks": clk}

    def close(self):
        self.cache.close()
        del self.cache, self.chunks


def secondary_cases():
    """(kind, workload, layers, steps) of every other configuration of the benchmark
    definition: GQA decode at 128K, the MHA retrieval-ratio sweep (decode and
    chunked prefill, recent 256 and 1024) and the 32-layer GQA stack at 1M; the
    two GQA decodes also with E4M3 retrieval caches (the quantized cache the
    pages' longest contexts rely on)."""
    cases = [("decode", workloads.LLAMA3_GQA, [0], 20), ("decode_e4m3", workloads.LLAMA3_GQA, [0], 20)]
    for ratio in (0.0, 0.25, 0.5, 0.75, 1.0):
        cases.append(("decode", workloads.mha_sweep(ratio, recent=256), [0], 10))
    for ratio in (0.0, 0.25):
        cases.append(("decode", workloads.mha_sweep(ratio, recent=1024), [0], 10))
    cases.append(("decode", workloads.GQA_STACK_1M, list(range(workloads.GQA_STACK_1M.num_layers)), 4))
    cases.append(("decode_e4m3", workloads.GQA_STACK_1M, list(range(workloads.GQA_STACK_1M.num_layers)), 4))
    for ratio in (0.0, 0.25, 0.5, 0.75, 1.0):
        cases.append(("prefill", workloads.mha_sweep(ratio, recent=256, prefill=True), None, None))
    cases.append(("prefill", workloads.mha_sweep(0.0, recent=1024, prefill=True), None, None))
    return cases


def case_name(kind, w):
    return w.name + ("_e4m3" if kind == "decode_e4m3" else "")


def run_secondary(duo, peaks, emit=None, only=None):
    out = []
    for kind, w, layers, steps in secondary_cases():
        if only is not None and case_name(kind, w) not in only:
            continue
        if kind == "prefill":
            case = PrefillCase(duo, w)
        else:
            case = DecodeCase(duo, w, layers, steps, duo.DUO_KV_E4M3 if kind == "decode_e4m3" else duo.DUO_KV_BF16)
        try:
            r = case.result(peaks)
        finally:
            case.close()
            torch.cuda.empty_cache()
        out.append(r)
        if emit is not None:
            emit(r)
    return out


def run_sweep(args):
    """The other workloads of the benchmark definition, one JSON line each
    (device time, clocks sampled per line)."""
    torch.cuda.set_device(0)
    import __graft_entry__
    __graft_entry__.build()
    import mixed_head_kv_b200 as duo
    return run_secondary(duo, load_peaks(), emit=lambda d: print(json.dumps(d), flush=True), only=args.case)


# ----------------------------------------------------------------------------- memory footprint
# Model shapes for the footprint table: (name, layers, q heads, KV heads, head_dim, retrieval ratio,
# parameters). The parameter counts are the public sizes of the models these shapes follow; they
# only add the bf16 weights to both sides of the whole-model ratio.
FOOTPRINT_MODELS = (
    ("llama2_7b_mha", 32, 32, 32, 128, 0.25, 6.74e9),
    ("llama3_8b_gqa", 32, 32, 8, 128, 0.5, 8.03e9),
)


def memory_footprint(duo, name, layers, hq, hkv, d, ratio, params, context, sink=64, recent=256, batch=1):
    """KV-cache bytes of full attention against the mixed-head cache the library sizes
    (duo_cache_alloc without a buffer), for one batch at `context` tokens."""
    w = workloads.Workload(name, batch=batch, num_q_heads=hq, num_kv_heads=hkv, head_dim=d, sink=sink,
                           recent=recent, retrieval_ratio=ratio, num_layers=layers)
    mask = [m for l in range(layers) for m in workloads.retrieval_mask(w, l)]
    lay = duo.make_layout(layers, batch, hq, hkv, d, sink, recent, context)
    st, required, _ = duo.duo_cache_alloc(lay, mask)
    if st != duo.DUO_OK:
        raise RuntimeError(duo.duo_status_str(st))
    n_retr = sum(mask)
    kv_full = layers * batch * hkv * context * d * 2 * 2
    kv_duo = (n_retr * context + (len(mask) - n_retr) * (sink + recent)) * batch * d * 2 * 2
    weights = params * 2
    return {"model": name, "context": context, "batch": batch, "retrieval_kv_heads": n_retr,
            "kv_full_bytes": kv_full, "kv_duo_bytes": kv_duo, "duo_required_bytes": required,
            "kv_ratio": kv_full / kv_duo, "with_weights_ratio": (weights + kv_full) / (weights + required)}


def run_memory(args):
    import mixed_head_kv_b200 as duo
    for m in FOOTPRINT_MODELS:
        for context in (32768, 131072, 1 << 20):
            print(json.dumps(memory_footprint(duo, *m, context)), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="duo", choices=["duo", "reference"])
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="seconds of oracle work for the CPU baseline")
    ap.add_argument("--sweep", action="store_true",
                    help="time only the other workloads (GQA decode at 128K and 1M, MHA ratio sweep), a line each")
    ap.add_argument("--case", action="append", default=None,
                    help="with --sweep: only this workload (repeatable), e.g. llama3_8b_gqa_128k_decode_b4_e4m3")
    ap.add_argument("--no-secondary", action="store_true",
                    help="leave the other workloads out of the main line (they run by default at N=1)")
    ap.add_argument("--memory", action="store_true",
                    help="print the KV-cache footprint of full attention against the mixed-head cache (no GPU)")
    args = ap.parse_args(argv)
    if args.memory:
        run_memory(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.warmup < 3 and args.impl != "reference":
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
