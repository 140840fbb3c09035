"""Ragged batches: sequences of one batch at different cache lengths.

Each sequence b reads its own seeded token stream (row p = position p); the
cache is filled with duo_cache_append_ragged (per-sequence token counts in a
padded [batch, max_tok, H, D] tensor) and decoded with duo_decode, every
sequence appending at its own length. Oracle parity per sequence (B = 1 oracle
calls over that sequence's history); caches compared bit-exactly per sequence
against the oracle's slot model.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from duo_harness import assert_close, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def duo():
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    import mixed_head_kv_b200
    return mixed_head_kv_b200


def _check_seq_cache(cache, w, b, k, v, length):
    mask = workloads.retrieval_mask(w)
    for g in range(w.num_kv_heads):
        ck, cv, r = cache.head_view(0, g)
        nslots = ck.shape[1]
        pos = torch.from_numpy(oracle.slot_positions(r, w.sink, w.recent, length, nslots))
        held = pos >= 0
        for c, src in ((ck, k), (cv, v)):
            got = c[b].cpu()
            exp = torch.zeros_like(got)
            exp[held] = src[b, pos[held], g]
            assert torch.equal(got.view(torch.int16), exp.view(torch.int16)), f"seq {b} head {g} cache differs"


def _run_ragged(duo, w, lens, steps, fill_chunks=1):
    """Fill sequence b with its first lens[b] tokens (in `fill_chunks` ragged appends),
    then `steps` decodes. Returns decode outputs [steps, B, Hq, D] (CPU) and inputs."""
    B = w.batch
    T = max(lens) + steps + 1
    q, k, v = workloads.tokens(w, 0, 0, T)  # [B, T, H, D] CPU
    mask = workloads.retrieval_mask(w)
    cache = duo.DuoCache(1, B, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, T + 8, mask)
    # ragged fill: chunk c carries rows [c*step_b, ...) of each sequence, padded
    done = [0] * B
    for c in range(fill_chunks):
        n_tok = [(lens[b] * (c + 1)) // fill_chunks - done[b] for b in range(B)]
        mx = max(max(n_tok), 1)
        kp = torch.zeros((B, mx, w.num_kv_heads, w.head_dim), dtype=torch.bfloat16)
        vp = torch.zeros_like(kp)
        for b in range(B):
            kp[b, :n_tok[b]] = k[b, done[b]:done[b] + n_tok[b]]
            vp[b, :n_tok[b]] = v[b, done[b]:done[b] + n_tok[b]]
        cache.append_ragged(0, kp.cuda(), vp.cuda(), n_tok)
        done = [done[b] + n_tok[b] for b in range(B)]
    assert cache.seq_lens(0) == list(lens)
    outs = []
    for t in range(steps):
        rows = [lens[b] + t for b in range(B)]
        qd = torch.stack([q[b, rows[b]] for b in range(B)]).cuda()
        kd = torch.stack([k[b, rows[b]] for b in range(B)]).cuda()
        vd = torch.stack([v[b, rows[b]] for b in range(B)]).cuda()
        o = torch.full_like(qd, float("nan"))
        cache.decode(0, qd, kd, vd, o)
        outs.append(o)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    assert cache.seq_lens(0) == [lens[b] + steps for b in range(B)]
    return cache, torch.stack(outs).cpu(), (q, k, v)


def _oracle_decode(w, q, k, v, b, pos):
    mask = workloads.retrieval_mask(w)
    qs = q[b:b + 1, pos:pos + 1].permute(0, 2, 1, 3)
    ks = k[b:b + 1, :pos + 1].permute(0, 2, 1, 3)
    vs = v[b:b + 1, :pos + 1].permute(0, 2, 1, 3)
    return oracle.attention(qs, np.array([pos]), ks, vs, mask, w.sink, w.recent)[0, :, 0]  # [Hq, D]


@pytest.mark.parametrize("G,lens,fill_chunks", [
    (1, [100, 37, 260], 1),     # MHA, ring and sink edges at different lengths
    (2, [3, 64, 70, 500], 2),   # GQA, one sequence still inside the sinks, two ragged fills
    (4, [5000, 301], 1),        # long vs short: the short sequence's later splits hold no rows
])
def test_ragged_append_and_decode(duo, G, lens, fill_chunks):
    Hkv = 4 if G < 4 else 2
    mask = [1, 0, 1, 0][:Hkv]
    w = make_workload(B=len(lens), Hq=Hkv * G, Hkv=Hkv, D=64, S=4, R=64, mask=mask)
    steps = 6
    cache, out, (q, k, v) = _run_ragged(duo, w, lens, steps, fill_chunks)
    for b in range(w.batch):
        for t in range(steps):
            ref = _oracle_decode(w, q, k, v, b, lens[b] + t)
            assert_close(out[t, b], ref, f"seq {b} step {t}")
        _check_seq_cache(cache, w, b, k, v, lens[b] + steps)


def test_ragged_state_rules(duo):
    w = make_workload(B=2, Hq=4, Hkv=4, D=64, S=4, R=16, mask=[1, 0, 1, 0])
    cache = duo.DuoCache(1, 2, 4, 4, 64, 4, 16, 64, workloads.retrieval_mask(w))
    cache.set_seq_lens(0, [10, 20])
    assert cache.seq_lens(0) == [10, 20]
    st, _ = duo.duo_cache_len(cache.handle, 0)
    assert st == duo.DUO_ERR_STATE  # no single length
    q = torch.zeros((2, 8, 4, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(q)
    assert duo.duo_prefill_ragged(cache.handle, 0, q, q, q, o, [9, 1], 8) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_prefill_ragged(cache.handle, 0, q, q, q, o, [8, 8], 8) == duo.DUO_OK  # 18, 28 <= 64
    kv = torch.zeros((2, 50, 4, 64), dtype=torch.bfloat16, device="cuda")
    # capacity is checked per sequence, before anything is written
    assert duo.duo_cache_append_ragged(cache.handle, 0, kv, kv, [40, 50], 50) == duo.DUO_ERR_CAPACITY
    assert duo.duo_cache_append_ragged(cache.handle, 0, kv, kv, [51, 0], 50) == duo.DUO_ERR_INVALID_ARG
    assert cache.seq_lens(0) == [10, 20]
    assert duo.duo_cache_set_seq_lens(cache.handle, 0, [65, 0]) == duo.DUO_ERR_INVALID_ARG
    cache.set_length(0, 7)
    assert cache.seq_lens(0) == [7, 7] and cache.length(0) == 7


def test_ragged_batch_limit(duo):
    B = duo.DUO_MAX_RAGGED_BATCH + 1
    w = make_workload(B=B, Hq=2, Hkv=2, D=64, S=4, R=16, mask=[1, 0])
    cache = duo.DuoCache(1, B, 2, 2, 64, 4, 16, 64, workloads.retrieval_mask(w))
    lens = [5] * B
    lens[-1] = 6
    cache.set_seq_lens(0, lens)
    x = torch.zeros((B, 2, 64), dtype=torch.bfloat16, device="cuda")
    assert duo.duo_decode(cache.handle, 0, x, x, x, torch.empty_like(x)) == duo.DUO_ERR_STATE
    cache.set_length(0, 5)  # uniform lengths work at any batch size
    assert duo.duo_decode(cache.handle, 0, x, x, x, torch.empty_like(x)) == duo.DUO_OK
    torch.cuda.synchronize()


@pytest.mark.parametrize("G,lens,n_tok", [
    (1, [100, 37, 260], [50, 129, 7]),   # the third sequence's second query tile is empty
    (2, [0, 300, 3], [200, 1, 130]),     # a fresh sequence, a one-token chunk, a chunk over the sinks
    (1, [40, 0, 200], [0, 150, 129]),    # a sequence without a chunk; full and partial query tiles
])
def test_ragged_prefill_then_decode(duo, G, lens, n_tok):
    Hkv = 4
    w = make_workload(B=len(lens), Hq=Hkv * G, Hkv=Hkv, D=64, S=4, R=64, mask=[1, 0, 1, 0])
    B, steps = w.batch, 3
    T = max(l + n for l, n in zip(lens, n_tok)) + steps + 1
    q, k, v = workloads.tokens(w, 0, 0, T)
    mask = workloads.retrieval_mask(w)
    cache = duo.DuoCache(1, B, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, T + 8, mask)

    def padded(x, starts, counts, rows):
        out = torch.zeros((B, rows) + tuple(x.shape[2:]), dtype=torch.bfloat16)
        for b in range(B):
            out[b, :counts[b]] = x[b, starts[b]:starts[b] + counts[b]]
        return out.cuda()

    mx = max(max(lens), 1)
    cache.append_ragged(0, padded(k, [0] * B, lens, mx), padded(v, [0] * B, lens, mx), lens)
    C = max(n_tok)
    qc, kc, vc = (padded(x, lens, n_tok, C) for x in (q, k, v))
    out = torch.full_like(qc, float("nan"))
    cache.prefill_ragged(0, qc, kc, vc, out, n_tok)
    cache.append_ragged(0, kc, vc, n_tok)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    out = out.cpu()
    for b in range(B):
        pos = np.arange(lens[b], lens[b] + n_tok[b])
        if len(pos):
            ref = oracle.attention(q[b:b + 1, pos].permute(0, 2, 1, 3), pos,
                                   k[b:b + 1, :pos[-1] + 1].permute(0, 2, 1, 3),
                                   v[b:b + 1, :pos[-1] + 1].permute(0, 2, 1, 3), mask, w.sink, w.recent)
            assert_close(out[b, :n_tok[b]], ref[0].transpose(1, 0, 2), f"seq {b} prefill")
        assert torch.isnan(out[b, n_tok[b]:].float()).all(), f"seq {b}: rows past its chunk were written"
    base = [l + n for l, n in zip(lens, n_tok)]
    assert cache.seq_lens(0) == base
    for t in range(steps):
        rows = [base[b] + t for b in range(B)]
        qd, kd, vd = (torch.stack([x[b, rows[b]] for b in range(B)]).cuda() for x in (q, k, v))
        o = torch.full_like(qd, float("nan"))
        cache.decode(0, qd, kd, vd, o)
        o = o.cpu()
        for b in range(B):
            assert_close(o[b], _oracle_decode(w, q, k, v, b, rows[b]), f"seq {b} decode {t}")
    for b in range(B):
        _check_seq_cache(cache, w, b, k, v, base[b] + steps)
