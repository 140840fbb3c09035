"""Device-side failure detection, exercised without any fault.

Every kernel wait on an asynchronous copy is bounded; when it runs out the
kernel sets a bit in the cache's error word and returns. The test hook
duo_cache_test_wait_timeout makes one copy of the next decode launch never be
issued (nothing else changes, nothing is left in flight), so the wait for it
gives up after a short limit. The tests check that the launch returns, the
error word reports the decode-copy bit, the cache update of that step still
happened, and the next normal step is correct again.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import workloads
from duo_harness import assert_close, check_cache_bits, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def duo():
    import __graft_entry__
    __graft_entry__.build()
    torch.cuda.set_device(0)
    import mixed_head_kv_b200
    return mixed_head_kv_b200


@pytest.mark.parametrize("kv_format", [0, 1], ids=["bf16", "e4m3"])
def test_decode_wait_timeout_is_reported_and_recovered(duo, kv_format):
    w = make_workload(B=1, Hq=4, Hkv=2, D=128, S=8, R=64, mask=[1, 0], seed=13)
    L = 3000
    q, k, v = workloads.tokens(w, 0, 0, L + 2)
    mask = workloads.retrieval_mask(w)
    cache = duo.DuoCache(1, 1, 4, 2, 128, w.sink, w.recent, L + 8, mask, kv_format=kv_format)
    cache.append(0, k[:, :L].cuda(), v[:, :L].cuda())
    torch.cuda.synchronize()
    assert cache.error_flags() == 0

    assert duo.duo_cache_test_wait_timeout(cache.handle, duo.DUO_TEST_WAIT_DECODE, 2_000_000) == duo.DUO_OK
    o = torch.zeros((1, 4, 128), dtype=torch.bfloat16, device="cuda")
    t0 = time.perf_counter()
    cache.decode(0, q[:, L].cuda(), k[:, L].cuda(), v[:, L].cuda(), o)
    flags = cache.error_flags()  # synchronizes
    assert time.perf_counter() - t0 < 5.0  # the 2 ms limit, not the default second, and no hang
    assert flags == duo.DUO_ERR_BIT_DECODE_COPY
    assert cache.error_flags() == 0  # read-and-clear
    assert cache.length(0) == L + 1
    if kv_format == 0:
        check_cache_bits(cache, w, k, v, L + 1, L + 8)  # the step's own token was appended

    # The next step is armed by nothing and is correct.
    o2 = torch.full((1, 4, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    cache.decode(0, q[:, L + 1].cuda(), k[:, L + 1].cuda(), v[:, L + 1].cuda(), o2)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    p = L + 1
    ref = oracle.attention(q[:, p:p + 1].permute(0, 2, 1, 3), np.array([p]), k[:, :p + 1].permute(0, 2, 1, 3),
                           v[:, :p + 1].permute(0, 2, 1, 3), mask, w.sink, w.recent)[:, :, 0]
    if kv_format == 1:  # the retrieval head reads E4M3 codes (scale 1)
        kc = oracle.e4m3_quantize(k[0, :p + 1, 0], 1.0)
        vc = oracle.e4m3_quantize(v[0, :p + 1, 0], 1.0)
        for h in range(2):
            ref[0, h], _ = oracle.attend_rows_e4m3(q[0, p, h], kc, vc, 1.0, 1.0, 1.0 / np.sqrt(128))
    assert_close(o2.cpu(), ref, "step after the reported timeout")


def test_test_hook_rejects_bad_arguments(duo):
    cache = duo.DuoCache(1, 1, 2, 2, 64, 4, 16, 64, [1, 0])
    assert duo.duo_cache_test_wait_timeout(cache.handle, 4, 2_000_000) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_test_wait_timeout(cache.handle, 1, 10) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_test_wait_timeout(cache.handle, 1, 2_000_000_000) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_test_wait_timeout(None, 1, 2_000_000) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_test_wait_timeout(cache.handle, 0, 2_000_000) == duo.DUO_OK  # disarm


def test_prefill_wait_timeout_is_reported_and_recovered(duo):
    """The first CTA of one prefill launch never gets its first K tile: its MMA
    issuer gives up after 2 ms, the CTA unwinds, the error word reports it; the
    next prefill of the same chunk is correct."""
    w = make_workload(B=1, Hq=4, Hkv=4, D=128, S=4, R=64, mask=[1, 0, 1, 0], seed=17)
    C = 700
    q, k, v = (x.cuda() for x in workloads.tokens(w, 0, 0, C))
    mask = workloads.retrieval_mask(w)
    cache = duo.DuoCache(1, 1, 4, 4, 128, w.sink, w.recent, C + 8, mask)
    assert duo.duo_cache_test_wait_timeout(cache.handle, duo.DUO_TEST_WAIT_PREFILL, 2_000_000) == duo.DUO_OK
    o = torch.zeros_like(q)
    t0 = time.perf_counter()
    cache.prefill(0, q, k, v, o)
    flags = cache.error_flags()
    assert time.perf_counter() - t0 < 5.0
    assert flags == duo.DUO_ERR_BIT_PREFILL_WAIT
    o2 = torch.full_like(q, float("nan"))
    cache.prefill(0, q, k, v, o2)
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
    ref = oracle.attention(q.cpu().permute(0, 2, 1, 3), np.arange(C), k.cpu().permute(0, 2, 1, 3),
                           v.cpu().permute(0, 2, 1, 3), mask, w.sink, w.recent).transpose(0, 2, 1, 3)
    assert_close(o2.cpu(), ref, "prefill after the reported timeout")
