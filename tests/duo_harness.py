"""Shared helpers for the GPU parity tests: run a sequence of prefill chunks and
decode steps through the C ABI and compute the oracle for the same inputs."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads

ATOL = 2e-2
RTOL = 2e-2


def make_workload(B=1, Hq=4, Hkv=4, D=128, S=4, R=64, mask=None, seed=0, sink_key_scale=0):
    return workloads.Workload("case", batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D, sink=S, recent=R,
                              retrieval_ratio=0.5, seed=seed, sink_key_scale=sink_key_scale,
                              explicit_retrieval=tuple(mask) if mask is not None else None)


def run_gpu(w, chunks, decode_steps, max_len=None, device="cuda", qkv=None, layer=0):
    """Prefill `chunks` (lengths) then `decode_steps` decodes. Returns (cache,
    outputs [B, T, Hq, D] bf16 on CPU, (q, k, v) CPU inputs [B, T, H, D])."""
    import mixed_head_kv_b200 as duo
    T = sum(chunks) + decode_steps
    if qkv is None:
        qkv = workloads.tokens(w, layer, 0, T)
    q, k, v = qkv
    mask = workloads.retrieval_mask(w, layer)
    cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent,
                         max_len or T + 8, mask, device=device)
    outs = []
    p = 0
    for c in chunks:
        qc, kc, vc = (x[:, p:p + c].to(device) for x in (q, k, v))
        o = torch.full_like(qc, float("nan"))
        cache.prefill(0, qc, kc, vc, o)
        cache.append(0, kc, vc)
        outs.append(o)
        p += c
    for _ in range(decode_steps):
        o = torch.full((w.batch, w.num_q_heads, w.head_dim), float("nan"), dtype=torch.bfloat16, device=device)
        cache.decode(0, q[:, p].to(device), k[:, p].to(device), v[:, p].to(device), o)
        outs.append(o[:, None])
        p += 1
    torch.cuda.synchronize()
    out = torch.cat(outs, dim=1).cpu() if outs else torch.empty(0)
    return cache, out, (q, k, v)


def oracle_out(w, q, k, v, positions, layer=0):
    """Oracle rows for query positions `positions` (q: [B, T, Hq, D] full stream)."""
    pos = np.asarray(positions, dtype=np.int64)
    T = int(pos.max()) + 1
    qs = q[:, pos].permute(0, 2, 1, 3)
    ks = k[:, :T].permute(0, 2, 1, 3)
    vs = v[:, :T].permute(0, 2, 1, 3)
    ref = oracle.attention(qs, pos, ks, vs, workloads.retrieval_mask(w, layer), w.sink, w.recent)
    return ref.transpose(0, 2, 1, 3)  # [B, n, Hq, D]


def assert_close(gpu, ref, what=""):
    g = gpu.float().numpy() if isinstance(gpu, torch.Tensor) else gpu
    err = np.abs(g - ref)
    tol = ATOL + RTOL * np.abs(ref)
    bad = ~(err <= tol)  # NaN counts as bad
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())}/{bad.size} outside |err| <= {ATOL} + {RTOL}|ref|; "
                             f"max err {np.nanmax(err):.3e}; first bad {idx.tolist()}")
    return float(err.max()) if err.size else 0.0


def check_cache_bits(cache, w, k, v, length, max_len, layer=0):
    """Cache contents must equal, bit for bit, the input rows at the positions the
    oracle's slot model assigns to each slot (empty slots stay zero)."""
    mask = workloads.retrieval_mask(w, layer)
    W = w.sink + w.recent
    for g in range(w.num_kv_heads):
        ck, cv, r = cache.head_view(0, g)
        assert r == mask[g]
        nslots = max_len if r else W
        pos = oracle.slot_positions(r, w.sink, w.recent, length, nslots)
        ek = torch.zeros((w.batch, nslots, w.head_dim), dtype=torch.bfloat16)
        ev = torch.zeros_like(ek)
        held = np.nonzero(pos >= 0)[0]
        ek[:, held] = k[:, pos[held], g]
        ev[:, held] = v[:, pos[held], g]
        gk = ck.cpu().view(torch.int16)
        gv = cv.cpu().view(torch.int16)
        assert torch.equal(gk, ek.view(torch.int16)), f"K cache of head {g} differs"
        assert torch.equal(gv, ev.view(torch.int16)), f"V cache of head {g} differs"
