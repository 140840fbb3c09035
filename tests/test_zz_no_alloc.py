"""duo_decode_static_scratch: the decode step for callers that cannot allocate.

Callers such as an inference-engine plugin that only receives a memory arena
planned before the run, or a serving loop that must not let cudaMalloc/cudaFree
synchronize the device, cannot allocate scratch when they call in. This entry
point keeps duo_decode's split-KV partial results in a file-scope device array
of the library instead. These tests run it through the C ABI next to
duo_decode on identical caches, for two calls in a row, and require
  - the fp64 oracle's outputs within the tolerance of the other parity tests,
  - duo_decode's outputs within the same tolerance,
on uniform, GQA (G = 8) and ragged batches, and on batches whose full split
plan does not fit the array (fewer, longer splits are used then), on both the
tensor-core and the CUDA-core decode kernels.

This file is collected last on purpose and also passes when run on its own.
"""
import numpy as np
import pytest
import torch

import __graft_entry__
import oracle
import workloads
from duo_harness import ATOL, RTOL, assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def duo():
    __graft_entry__.build()
    torch.cuda.set_device(0)
    import mixed_head_kv_b200
    return mixed_head_kv_b200


def _workload(shape, seed=5):
    return workloads.Workload("no_alloc", batch=shape["batch"], num_q_heads=shape["num_q_heads"],
                              num_kv_heads=shape["num_kv_heads"], head_dim=shape["head_dim"], sink=shape["sink"],
                              recent=shape["recent"], retrieval_ratio=0.5, explicit_retrieval=shape["mask"],
                              seed=seed)


def _caches(duo, w, max_len):
    mask = workloads.retrieval_mask(w)
    return [duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, max_len, mask)
            for _ in range(2)]


def _oracle_rows(w, q, k, v, b, p):
    """Oracle output [Hq, D] of sequence b's query at position p (q, k, v: CPU [B, T, H, D])."""
    ref = oracle.attention(q[b:b + 1, p:p + 1].permute(0, 2, 1, 3), np.array([p]),
                           k[b:b + 1, :p + 1].permute(0, 2, 1, 3), v[b:b + 1, :p + 1].permute(0, 2, 1, 3),
                           workloads.retrieval_mask(w), w.sink, w.recent)
    return ref[0, :, 0]


def _decode_pair(duo, ref_cache, static_cache, qd, kd, vd):
    a = torch.full_like(qd, float("nan"))
    b = torch.full_like(qd, float("nan"))
    assert duo.duo_decode(ref_cache.handle, 0, qd, kd, vd, a) == duo.DUO_OK
    assert duo.duo_decode_static_scratch(static_cache.handle, 0, qd, kd, vd, b) == duo.DUO_OK
    torch.cuda.synchronize()
    return a.float().cpu().numpy(), b.cpu()


def _close_to_decode(ra, rb, what):
    rb = rb.float().numpy()
    assert np.all(np.isfinite(rb)), what
    assert np.all(np.abs(rb - ra) <= ATOL + RTOL * np.abs(ra)), f"{what}: max diff {np.abs(rb - ra).max()}"


@pytest.mark.parametrize("shape", [
    dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, sink=64, recent=256, mask=(1, 0), T=9000),
    dict(batch=1, num_q_heads=4, num_kv_heads=4, head_dim=64, sink=4, recent=64, mask=(1, 0, 1, 0), T=700),
    dict(batch=2, num_q_heads=16, num_kv_heads=2, head_dim=128, sink=8, recent=100, mask=(0, 1), T=5000),
], ids=["gqa4_d128", "mha_d64", "gqa8_d128"])
def test_static_scratch_decode_matches_oracle_and_duo_decode(duo, shape):
    w = _workload(shape)
    T = shape["T"]
    ref_cache, static_cache = _caches(duo, w, T + 8)
    q, k, v = workloads.tokens(w, 0, 0, T + 2)
    qg, kg, vg = (x.cuda() for x in (q, k, v))
    for c in (ref_cache, static_cache):  # chunked prefill then append, as a serving loop would
        out = torch.empty_like(qg[:, :T])
        c.prefill(0, qg[:, :T].contiguous(), kg[:, :T].contiguous(), vg[:, :T].contiguous(), out)
        c.append(0, kg[:, :T].contiguous(), vg[:, :T].contiguous())
    for step in range(2):  # two calls in a row: the array keeps the first call's contents
        p = T + step
        ra, rb = _decode_pair(duo, ref_cache, static_cache, *(x[:, p].contiguous() for x in (qg, kg, vg)))
        for b in range(w.batch):
            assert_close(rb[b], _oracle_rows(w, q, k, v, b, p), f"step {step} seq {b} vs oracle")
        _close_to_decode(ra, rb, f"step {step} vs duo_decode")
        assert static_cache.length(0) == ref_cache.length(0) == p + 1
    assert static_cache.error_flags() == 0


def test_static_scratch_ragged_batch(duo):
    """Sequences at different cache lengths (one still inside its sinks): each
    appends and attends at its own length."""
    w = _workload(dict(batch=3, num_q_heads=8, num_kv_heads=2, head_dim=128, sink=16, recent=64, mask=(1, 0)))
    lens = [4100, 9, 1500]
    T = max(lens) + 3
    q, k, v = workloads.tokens(w, 0, 0, T)
    ref_cache, static_cache = _caches(duo, w, T + 8)
    mx = max(lens)
    kp = torch.zeros((w.batch, mx, w.num_kv_heads, w.head_dim), dtype=torch.bfloat16)
    vp = torch.zeros_like(kp)
    for b in range(w.batch):
        kp[b, :lens[b]] = k[b, :lens[b]]
        vp[b, :lens[b]] = v[b, :lens[b]]
    for c in (ref_cache, static_cache):
        c.append_ragged(0, kp.cuda(), vp.cuda(), lens)
    for step in range(2):
        rows = [lens[b] + step for b in range(w.batch)]
        qd, kd, vd = (torch.stack([x[b, rows[b]] for b in range(w.batch)]).cuda() for x in (q, k, v))
        ra, rb = _decode_pair(duo, ref_cache, static_cache, qd, kd, vd)
        for b in range(w.batch):
            assert_close(rb[b], _oracle_rows(w, q, k, v, b, rows[b]), f"step {step} seq {b} vs oracle")
        _close_to_decode(ra, rb, f"step {step} vs duo_decode")
    assert static_cache.seq_lens(0) == [x + 2 for x in lens]
    assert static_cache.error_flags() == 0


def _planned_splits(batch, n_retr, n_strm, rows, strm_rows, num_sms, G, D):
    """The split count duo_decode would pick (restated here only to check that the
    shapes below really exceed the static array; the library's own plan decides).
    Query groups of 4 and 8 with head_dim 128 run one tensor-core CTA per SM; the
    CUDA-core kernel runs 3 CTAs per SM for groups of 2 and 4, 2 otherwise."""
    per_sm = 1 if (G in (4, 8) and D == 128) else (3 if G in (2, 4) else 2)
    slots = num_sms * per_sm
    best, best_cost = 1, None
    for ns in range(1, min(256, max(1, (rows + 255) // 256)) + 1):
        waves = (batch * n_retr * ns + batch * n_strm + slots - 1) // slots
        longest = max((rows + ns - 1) // ns, strm_rows if n_strm else 0)
        cost = waves * (longest + 64)
        if best_cost is None or cost < best_cost:
            best, best_cost = ns, cost
    return best


@pytest.mark.parametrize("shape", [
    # tensor-core decode: 64 sequences x 4 retrieval KV heads x G = 8, head_dim 128, 8K context
    dict(batch=64, num_q_heads=128, num_kv_heads=16, head_dim=128, L=8192, retr=(0, 3, 5, 12)),
    # CUDA-core decode: 64 sequences x 3 retrieval KV heads x G = 8, head_dim 64, 16K context
    dict(batch=64, num_q_heads=256, num_kv_heads=32, head_dim=64, L=16384, retr=(1, 9, 30)),
], ids=["tensor_core_path", "cuda_core_path"])
def test_static_scratch_clamps_splits_to_the_array(duo, shape):
    """The full split plan needs more partials than the array holds, so the call
    serves the step with fewer, longer splits; outputs still match the oracle and
    duo_decode."""
    mask = tuple(1 if g in shape["retr"] else 0 for g in range(shape["num_kv_heads"]))
    shape = dict(shape, sink=64, recent=256, mask=mask)
    w = _workload(shape, seed=11)
    L = shape["L"]
    G, D = w.group, w.head_dim
    n_retr = sum(mask)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    counters = (w.batch * w.num_kv_heads * 4 + 255) // 256 * 256
    fit = (duo.DUO_STATIC_SCRATCH_BYTES - counters - 256) // (w.batch * n_retr * G * (D + 1) * 4)
    planned = _planned_splits(w.batch, n_retr, w.num_kv_heads - n_retr, L + 1, w.sink + w.recent, sms, G, D)
    assert 1 <= fit < planned, (fit, planned)  # the premise: the plan does not fit the array
    ref_cache, static_cache = _caches(duo, w, L + 8)
    for c0 in range(0, L, 4096):
        kk, vv = workloads.tokens(w, 0, c0, 4096, device="cuda", which="kv")
        for c in (ref_cache, static_cache):
            c.append(0, kk, vv)
    q, k, v = workloads.tokens(w, 0, L, 2, device="cuda")
    sampled = (0, 17, w.batch - 1)
    kh, vh = workloads.tokens(w, 0, 0, L, device="cuda", which="kv")
    hist = [torch.cat([h, x], dim=1)[list(sampled)].cpu() for h, x in ((kh, k), (vh, v))]
    del kh, vh
    for step in range(2):
        ra, rb = _decode_pair(duo, ref_cache, static_cache, *(x[:, step].contiguous() for x in (q, k, v)))
        _close_to_decode(ra, rb, f"step {step} vs duo_decode")
        p = L + step
        for i, b in enumerate(sampled):
            ref = oracle.attention(q[b:b + 1, step:step + 1].cpu().permute(0, 2, 1, 3), np.array([p]),
                                   hist[0][i:i + 1, :p + 1].permute(0, 2, 1, 3),
                                   hist[1][i:i + 1, :p + 1].permute(0, 2, 1, 3), mask, w.sink, w.recent)
            assert_close(rb[b], ref[0, :, 0], f"step {step} seq {b} vs oracle")
    assert static_cache.error_flags() == 0


def test_static_scratch_rejects_oversized_requests(duo):
    """128 sequences x 32 retrieval KV heads x 8 query heads each need
    128*32*8*129*4 bytes (16.9 MB) of partials for a single split: more than the
    array holds, so the call is refused before any launch."""
    cache = duo.DuoCache(1, 128, 256, 32, 128, 0, 1, 2, [1] * 32)
    q = torch.zeros((128, 256, 128), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((128, 32, 128), dtype=torch.bfloat16, device="cuda")
    st = duo.duo_decode_static_scratch(cache.handle, 0, q, kv, kv, torch.empty_like(q))
    assert st == duo.DUO_ERR_SCRATCH_LIMIT
    assert "static decode scratch" in duo.duo_status_str(st)
    assert cache.length(0) == 0
