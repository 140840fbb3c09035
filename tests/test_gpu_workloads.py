"""Parity at the benchmark workloads' full sizes, in the launch configuration
bench.py times (same chunking, same decode loop), on sampled outputs the oracle
can compute one by one; caches compared bit-exactly.

Inputs are generated on the GPU (seeded torch generator, workloads.tokens) and
read back for the oracle; nothing the oracle sees comes from the CUDA path.
"""
import numpy as np
import pytest
import torch

import __graft_entry__
import oracle
import workloads
from duo_harness import assert_close

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


@pytest.fixture(scope="module")
def duo():
    __graft_entry__.build()
    torch.cuda.set_device(0)
    import mixed_head_kv_b200
    return mixed_head_kv_b200


def _oracle_rows(w, q_rows, positions, k_hist, v_hist, mask):
    """q_rows [B, n, Hq, D] at absolute `positions`; k/v_hist [B, T, Hkv, D] (CPU bf16)."""
    ref = oracle.attention(q_rows.permute(0, 2, 1, 3), np.asarray(positions), k_hist.permute(0, 2, 1, 3),
                           v_hist.permute(0, 2, 1, 3), mask, w.sink, w.recent)
    return ref.transpose(0, 2, 1, 3)


def _check_cache_gpu(cache, w, k_dev, v_dev, length, layer=0):
    """Bit-exact cache check on the device: expected rows gathered from the inputs
    at the oracle's slot positions (empty slots must be zero)."""
    mask = workloads.retrieval_mask(w, layer)
    for g in range(w.num_kv_heads):
        ck, cv, r = cache.head_view(layer, g)
        nslots = ck.shape[1]
        pos = torch.from_numpy(oracle.slot_positions(r, w.sink, w.recent, length, nslots)).to(ck.device)
        held = pos >= 0
        for c, src in ((ck, k_dev), (cv, v_dev)):
            exp = torch.zeros_like(c)
            exp[:, held] = src[:, pos[held], g]
            assert torch.equal(c.view(torch.int16), exp.view(torch.int16)), f"layer {layer} head {g} cache differs"


def test_llama2_mha_32k_chunked_prefill_and_decode(duo):
    """Llama-2-7B-shaped MHA layer: 32K prefill in 4096-token chunks + 128 decodes."""
    w = workloads.LLAMA2_MHA
    mask = workloads.retrieval_mask(w)
    T = w.prefill_len + w.decode_steps
    q, k, v = workloads.tokens(w, 0, 0, T, device="cuda")
    cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, T, mask)
    out = torch.full_like(q, float("nan"))
    for c0 in range(0, w.prefill_len, w.chunk):
        sl = slice(c0, c0 + w.chunk)
        o = torch.empty_like(q[:, sl])
        cache.prefill(0, q[:, sl].contiguous(), k[:, sl].contiguous(), v[:, sl].contiguous(), o)
        cache.append(0, k[:, sl].contiguous(), v[:, sl].contiguous())
        out[:, sl] = o
    _check_cache_gpu(cache, w, k, v, w.prefill_len)
    for t in range(w.decode_steps):
        p = w.prefill_len + t
        o = torch.empty_like(q[:, p])
        cache.decode(0, q[:, p].contiguous(), k[:, p].contiguous(), v[:, p].contiguous(), o)
        out[:, p] = o
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    _check_cache_gpu(cache, w, k, v, T)
    # Sampled rows: every 61st prefill row, the edges of every chunk, all decode rows.
    rows = set(range(0, w.prefill_len, 61))
    for c0 in range(0, w.prefill_len, w.chunk):
        rows |= {c0, c0 + 1, c0 + 127, c0 + 128, c0 + w.chunk - 2, c0 + w.chunk - 1}
    rows |= set(range(w.prefill_len, T))
    rows = np.array(sorted(rows))
    qc, kc, vc = q.cpu(), k.cpu(), v.cpu()
    ref = _oracle_rows(w, qc[:, rows], rows, kc, vc, mask)
    assert_close(out[:, rows].cpu(), ref, "llama2 32K sampled rows")


def _decode_workload(duo, w, steps=2, fill_chunk=16384):
    mask = workloads.retrieval_mask(w)
    L = w.context
    cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, L + steps, mask)
    for c0 in range(0, L, fill_chunk):
        kk, vv = workloads.tokens(w, 0, c0, min(fill_chunk, L - c0), device="cuda", which="kv")
        cache.append(0, kk, vv)
    q, k, v = workloads.tokens(w, 0, L, steps, device="cuda")
    outs = []
    for t in range(steps):
        o = torch.full_like(q[:, t], float("nan"))
        cache.decode(0, q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), o)
        outs.append(o)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    out = torch.stack(outs, dim=1).cpu()
    # Oracle over the whole history, regenerated from the same seeds.
    kh, vh = workloads.tokens(w, 0, 0, L + steps, device="cuda", which="kv")
    ref = _oracle_rows(w, q.cpu(), np.arange(L, L + steps), kh.cpu(), vh.cpu(), mask)
    assert_close(out, ref, w.name)
    _check_cache_gpu(cache, w, kh, vh, L + steps)
    return cache


def test_llama3_gqa_decode_b4_128k(duo):
    """Llama-3-8B-shaped GQA layer: batch 4, 128K cached tokens, 50 % retrieval KV heads."""
    _decode_workload(duo, workloads.LLAMA3_GQA)


SWEEP = [(r, 256) for r in (0.0, 0.25, 0.5, 0.75, 1.0)] + [(0.0, 1024), (0.25, 1024), (0.5, 1024)]


def test_llama3_gqa_decode_b4_128k_e4m3(duo):
    """The Llama-3-8B-shaped GQA decode (batch 4, 128K) over E4M3 retrieval caches
    with per-head scales, in the benchmark's launch configuration (tensor-core
    decode, codes converted to f16): every output against the oracle's attention
    over the codes (streaming heads over bf16 rows), and the codes of a
    retrieval head bit-exact against the oracle's quantizer."""
    w = workloads.LLAMA3_GQA
    mask = workloads.retrieval_mask(w)
    L, steps, G = w.context, 2, w.group
    ks = [0.5 + 0.25 * g for g in range(w.num_kv_heads)]
    vs = [1.5 - 0.125 * g for g in range(w.num_kv_heads)]
    cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, L + steps, mask,
                         kv_format=duo.DUO_KV_E4M3)
    cache.set_kv_scales(0, ks, vs)
    for c0 in range(0, L, 16384):
        kk, vv = workloads.tokens(w, 0, c0, 16384, device="cuda", which="kv")
        cache.append(0, kk, vv)
    q, k, v = workloads.tokens(w, 0, L, steps, device="cuda")
    outs = []
    for t in range(steps):
        o = torch.full_like(q[:, t], float("nan"))
        cache.decode(0, q[:, t].contiguous(), k[:, t].contiguous(), v[:, t].contiguous(), o)
        outs.append(o)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    kh, vh = (x.cpu() for x in workloads.tokens(w, 0, 0, L + steps, device="cuda", which="kv"))
    qc = q.cpu()
    inv = lambda x: float(np.float32(1.0) / np.float32(x))
    g0 = mask.index(1)
    ck, cv, _ = cache.head_view(0, g0)
    for b in range(w.batch):
        assert np.array_equal(ck[b, :L + steps].cpu().numpy(), oracle.e4m3_quantize(kh[b, :, g0], inv(ks[g0])))
        assert np.array_equal(cv[b, :L + steps].cpu().numpy(), oracle.e4m3_quantize(vh[b, :, g0], inv(vs[g0])))
    scale = 1.0 / np.sqrt(w.head_dim)
    for t in range(steps):
        p = L + t
        ref = _oracle_rows(w, qc[:, t:t + 1], np.array([p]), kh[:, :p + 1], vh[:, :p + 1], mask)[:, 0]
        for g in range(w.num_kv_heads):
            if not mask[g]:
                continue
            for b in range(w.batch):
                kc = oracle.e4m3_quantize(kh[b, :p + 1, g], inv(ks[g]))
                vc = oracle.e4m3_quantize(vh[b, :p + 1, g], inv(vs[g]))
                for h in range(g * G, (g + 1) * G):
                    ref[b, h], _ = oracle.attend_rows_e4m3(qc[b, t, h], kc, vc, ks[g], vs[g], scale)
        assert_close(outs[t].cpu(), ref, f"e4m3 step {t}")


@pytest.mark.parametrize("ratio,recent", SWEEP)
def test_mha_sweep_decode_b8_64k(duo, ratio, recent):
    """MHA retrieval-ratio sweep: 32 heads, batch 8, 64K cached tokens."""
    _decode_workload(duo, workloads.mha_sweep(ratio, recent=recent), steps=1)


@pytest.mark.parametrize("ratio,recent", SWEEP)
def test_mha_sweep_prefill_chunk_64k(duo, ratio, recent):
    """Prefill chunks of the MHA sweep one chunk deep into a 64K context (cache
    filled by append, chunk at [61440, 65536)), in the launch configuration the
    benchmark times; sampled rows (every 97th, the first three, the last)."""
    w = workloads.mha_sweep(ratio, recent=recent, prefill=True)
    mask = workloads.retrieval_mask(w)
    L0 = w.prefill_len - w.chunk
    cache = duo.DuoCache(1, 1, 32, 32, 128, w.sink, w.recent, w.prefill_len, mask)
    for c0 in range(0, L0, 16384):
        kk, vv = workloads.tokens(w, 0, c0, min(16384, L0 - c0), device="cuda", which="kv")
        cache.append(0, kk, vv)
    q, k, v = workloads.tokens(w, 0, L0, w.chunk, device="cuda")
    o = torch.full_like(q, float("nan"))
    cache.prefill(0, q, k, v, o)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    rows = np.array(sorted(set(range(0, w.chunk, 97)) | {0, 1, 2, w.chunk - 1}))
    kh, vh = workloads.tokens(w, 0, 0, w.prefill_len, device="cuda", which="kv")
    ref = _oracle_rows(w, q.cpu()[:, rows], L0 + rows, kh.cpu(), vh.cpu(), mask)
    assert_close(o.cpu()[:, rows], ref, w.name)


def test_gqa_32_layer_stack_1m_decode(duo):
    """32-layer GQA stack at 1M (2**20) cached tokens, batch 1, one decode step per
    layer, in the launch configuration the benchmark times. Every layer is checked
    against the oracle on two of its KV heads, its first retrieval head and its
    first streaming head, with all 4 query heads of each (the oracle reads those
    heads' full 1M-token history); each layer's retrieval head cache and streaming
    head cache are compared bit-exactly; every output is finite."""
    w = workloads.GQA_STACK_1M
    L = w.context
    G = w.group
    masks = [workloads.retrieval_mask(w, l) for l in range(w.num_layers)]
    flat = [m for ms in masks for m in ms]
    cache = duo.DuoCache(w.num_layers, 1, 32, 8, 128, w.sink, w.recent, L + 1, flat)
    fill = 1 << 17
    for l in range(w.num_layers):
        for c0 in range(0, L, fill):
            kk, vv = workloads.tokens(w, l, c0, fill, device="cuda", which="kv")
            duo.duo_cache_append(cache.handle, l, kk, vv, fill)
    outs = []
    for l in range(w.num_layers):
        q, k, v = workloads.tokens(w, l, L, 1, device="cuda")
        o = torch.full_like(q[:, 0], float("nan"))
        assert duo.duo_decode(cache.handle, l, q[:, 0].contiguous(), k[:, 0].contiguous(), v[:, 0].contiguous(),
                              o) == duo.DUO_OK
        outs.append(o)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    for l in range(w.num_layers):
        assert torch.isfinite(outs[l].float()).all(), l
        q = workloads.tokens(w, l, L, 1, device="cuda", which="q")[0]
        kh, vh = workloads.tokens(w, l, 0, L + 1, device="cuda", which="kv")
        for g in (masks[l].index(1), masks[l].index(0)):
            # bit-exact cache of this head, then the oracle over its history alone
            ck, cv, r = cache.head_view(l, g)
            pos = torch.from_numpy(oracle.slot_positions(r, w.sink, w.recent, L + 1, ck.shape[1])).to(ck.device)
            held = pos >= 0
            for c, src in ((ck, kh), (cv, vh)):
                exp = torch.zeros_like(c)
                exp[:, held] = src[:, pos[held], g]
                assert torch.equal(c.view(torch.int16), exp.view(torch.int16)), f"layer {l} head {g} cache differs"
            ref = oracle.attention(q[:, :, g * G:(g + 1) * G].cpu().permute(0, 2, 1, 3), np.array([L]),
                                   kh[:, :, g:g + 1].cpu().permute(0, 2, 1, 3),
                                   vh[:, :, g:g + 1].cpu().permute(0, 2, 1, 3), [masks[l][g]], w.sink, w.recent)
            assert_close(outs[l].cpu()[:, g * G:(g + 1) * G], ref[:, :, 0], f"layer {l} KV head {g}")
        del kh, vh
