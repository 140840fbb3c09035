"""E4M3 retrieval caches: append stores the oracle's codes bit for bit, decode
matches the oracle's attention over those codes with the per-head scales, and
streaming heads stay bf16."""
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


def _setup(duo, w, L, steps, k_scale, v_scale):
    T = L + steps
    q, k, v = workloads.tokens(w, 0, 0, T)
    mask = workloads.retrieval_mask(w)
    cache = duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, T + 8, mask,
                         kv_format=duo.DUO_KV_E4M3)
    cache.set_kv_scales(0, k_scale, v_scale)
    cache.append(0, k[:, :L].cuda(), v[:, :L].cuda())
    return cache, (q, k, v), mask


def _inv(s):
    return float(np.float32(1.0) / np.float32(s))


@pytest.mark.parametrize("G,D", [(1, 128), (4, 64), (4, 128), (8, 128)])
def test_fp8_append_codes_and_decode(duo, G, D):
    """Groups of 4 and 8 with head_dim 128 run the tensor-core decode (codes
    converted to f16 in shared memory); the others the CUDA-core kernel."""
    Hkv = 4
    w = make_workload(B=2, Hq=Hkv * G, Hkv=Hkv, D=D, S=4, R=64, mask=[1, 0, 1, 0])
    L, steps = 700, 4
    k_scale = [0.37, 1.0, 2.5, 1.0]
    v_scale = [1.7, 1.0, 0.05, 1.0]
    cache, (q, k, v), mask = _setup(duo, w, L, steps, k_scale, v_scale)
    outs = []
    for t in range(steps):
        p = L + t
        o = torch.full((w.batch, w.num_q_heads, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        cache.decode(0, q[:, p].cuda(), k[:, p].cuda(), v[:, p].cuda(), o)
        outs.append(o.cpu())
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    T = L + steps
    # caches: retrieval heads hold the oracle's codes of every token, streaming heads bf16 rows
    for g in range(Hkv):
        ck, cv, r = cache.head_view(0, g)
        if r:
            for b in range(w.batch):
                kc = oracle.e4m3_quantize(k[b, :T, g], _inv(k_scale[g]))
                vc = oracle.e4m3_quantize(v[b, :T, g], _inv(v_scale[g]))
                assert np.array_equal(ck[b, :T].cpu().numpy(), kc), f"K codes, head {g} seq {b}"
                assert np.array_equal(cv[b, :T].cpu().numpy(), vc), f"V codes, head {g} seq {b}"
        else:
            pos = torch.from_numpy(oracle.slot_positions(0, w.sink, w.recent, T, ck.shape[1]))
            held = pos >= 0
            exp = torch.zeros_like(ck.cpu())
            exp[:, held] = k[:, pos[held], g]
            assert torch.equal(ck.cpu().view(torch.int16), exp.view(torch.int16))
    # outputs: retrieval heads over the codes with the scales, streaming heads as before
    scale = 1.0 / np.sqrt(D)
    for t in range(steps):
        p = L + t
        ref_all = oracle.attention(q[:, p:p + 1].permute(0, 2, 1, 3), np.array([p]),
                                   k[:, :p + 1].permute(0, 2, 1, 3), v[:, :p + 1].permute(0, 2, 1, 3), mask,
                                   w.sink, w.recent)[:, :, 0]  # [B, Hq, D], bf16 definition
        ref = ref_all.copy()
        for b in range(w.batch):
            for h in range(w.num_q_heads):
                g = h // G
                if mask[g]:
                    kc = oracle.e4m3_quantize(k[b, :p + 1, g], _inv(k_scale[g]))
                    vc = oracle.e4m3_quantize(v[b, :p + 1, g], _inv(v_scale[g]))
                    ref[b, h], _ = oracle.attend_rows_e4m3(q[b, p, h], kc, vc, k_scale[g], v_scale[g], scale)
        assert_close(outs[t], ref, f"decode step {t}")


def test_fp8_state_rules(duo):
    w = make_workload(B=1, Hq=2, Hkv=2, D=64, S=4, R=16, mask=[1, 0])
    cache = duo.DuoCache(1, 1, 2, 2, 64, 4, 16, 64, workloads.retrieval_mask(w), kv_format=duo.DUO_KV_E4M3)
    assert duo.duo_cache_set_kv_scales(cache.handle, 0, [0.0, 1.0], [1.0, 1.0]) == duo.DUO_ERR_INVALID_ARG
    x = torch.zeros((1, 8, 2, 64), dtype=torch.bfloat16, device="cuda")
    o = torch.empty_like(x)
    assert duo.duo_prefill(cache.handle, 0, x, x, x, o, 8) == duo.DUO_OK  # first chunk: no cache tiles
    cache.append(0, x, x)
    assert duo.duo_prefill(cache.handle, 0, x, x, x, o, 8) == duo.DUO_ERR_STATE
    plain = duo.DuoCache(1, 1, 2, 2, 64, 4, 16, 64, workloads.retrieval_mask(w))
    assert duo.duo_cache_set_kv_scales(plain.handle, 0, [1.0, 1.0], [1.0, 1.0]) == duo.DUO_ERR_STATE
    torch.cuda.synchronize()


def _fp8_ref(q_row, k_hist, v_hist, mask, G, w, k_scale, v_scale, p):
    """Oracle for one decode position p: streaming heads over bf16 rows (the
    definition), retrieval heads over the E4M3 codes of their whole history."""
    scale = 1.0 / np.sqrt(w.head_dim)
    ref = oracle.attention(q_row.permute(0, 2, 1, 3), np.array([p]), k_hist.permute(0, 2, 1, 3),
                           v_hist.permute(0, 2, 1, 3), mask, w.sink, w.recent)[:, :, 0]
    for b in range(w.batch):
        for h in range(w.num_q_heads):
            g = h // G
            if mask[g]:
                kc = oracle.e4m3_quantize(k_hist[b, :p + 1, g], _inv(k_scale[g]))
                vc = oracle.e4m3_quantize(v_hist[b, :p + 1, g], _inv(v_scale[g]))
                ref[b, h], _ = oracle.attend_rows_e4m3(q_row[b, 0, h], kc, vc, k_scale[g], v_scale[g], scale)
    return ref


@pytest.mark.parametrize("G", [2, 4])
@pytest.mark.parametrize("entry", ["duo_decode", "duo_decode_static_scratch"])
def test_fp8_long_context_split_decode(duo, entry, G):
    """20K cached tokens (many splits and the log-sum-exp merge), GQA G = 2 (CUDA
    cores) and 4 (tensor cores), both decode entry points; sink-like keys (x8) in
    the first positions."""
    w = workloads.Workload("fp8_long", batch=1, num_q_heads=4 * G, num_kv_heads=4, head_dim=128, sink=64, recent=256,
                           retrieval_ratio=0.5, explicit_retrieval=(0, 1, 1, 0), seed=9, sink_key_scale=8)
    L, steps = 20000, 2
    k_scale, v_scale = [1.0, 0.125, 0.75, 1.0], [1.0, 0.5, 3.0, 1.0]
    cache, (q, k, v), mask = _setup(duo, w, L, steps, k_scale, v_scale)
    call = getattr(duo, entry)
    for t in range(steps):
        p = L + t
        o = torch.full((1, 4 * G, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert call(cache.handle, 0, q[:, p].cuda(), k[:, p].cuda(), v[:, p].cuda(), o) == duo.DUO_OK
        torch.cuda.synchronize()
        ref = _fp8_ref(q[:, p:p + 1], k[:, :p + 1], v[:, :p + 1], mask, G, w, k_scale, v_scale, p)
        assert_close(o.cpu(), ref, f"{entry} step {t}")
    assert cache.error_flags() == 0


def test_fp8_one_chunk_prefill_then_decode(duo):
    """The supported prefill flow of an E4M3 cache: the prompt in one chunk (no
    cached retrieval tokens yet; the chunk's own bf16 keys are used), the append
    that quantizes it, then decode steps over the codes."""
    w = make_workload(B=1, Hq=4, Hkv=2, D=128, S=16, R=64, mask=[1, 0], seed=4)
    C, steps = 600, 3
    q, k, v = workloads.tokens(w, 0, 0, C + steps)
    mask = workloads.retrieval_mask(w)
    cache = duo.DuoCache(1, 1, 4, 2, 128, w.sink, w.recent, C + steps + 8, mask, kv_format=duo.DUO_KV_E4M3)
    ks, vs = [0.5, 1.0], [0.25, 1.0]
    cache.set_kv_scales(0, ks, vs)
    o = torch.empty_like(q[:, :C]).cuda()
    cache.prefill(0, q[:, :C].cuda(), k[:, :C].cuda(), v[:, :C].cuda(), o)
    cache.append(0, k[:, :C].cuda(), v[:, :C].cuda())
    torch.cuda.synchronize()
    ref = oracle.attention(q[:, :C].permute(0, 2, 1, 3), np.arange(C), k[:, :C].permute(0, 2, 1, 3),
                           v[:, :C].permute(0, 2, 1, 3), mask, w.sink, w.recent).transpose(0, 2, 1, 3)
    assert_close(o.cpu(), ref, "one-chunk prefill")
    for t in range(steps):
        p = C + t
        od = torch.full((1, 4, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
        cache.decode(0, q[:, p].cuda(), k[:, p].cuda(), v[:, p].cuda(), od)
        torch.cuda.synchronize()
        assert_close(od.cpu(), _fp8_ref(q[:, p:p + 1], k[:, :p + 1], v[:, :p + 1], mask, 2, w, ks, vs, p),
                     f"decode {t}")
    assert cache.error_flags() == 0

