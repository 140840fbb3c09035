"""duo_decode_static_scratch: the decode step for callers that cannot allocate.

Callers such as an inference-engine plugin that only receives a memory arena
planned before the run, or a serving loop that must not let cudaMalloc/cudaFree
synchronize the device, cannot allocate scratch when they call in. This entry
point keeps duo_decode's split-KV partial results in a file-scope device array
of the library instead. These tests run it through the C ABI next to
duo_decode on identical caches and require the same outputs, within the
tolerance of the other parity tests, for two calls in a row.

This file is collected last on purpose and also passes when run on its own.
"""
import numpy as np
import pytest
import torch

import __graft_entry__

pytestmark = pytest.mark.gpu

ATOL = 2e-2
RTOL = 2e-2


@pytest.fixture(scope="module")
def duo():
    __graft_entry__.build()
    torch.cuda.set_device(0)
    import mixed_head_kv_b200
    return mixed_head_kv_b200


def _pair_of_caches(duo, w, T_prefill, max_len):
    import workloads
    mask = workloads.retrieval_mask(w)
    caches = [duo.DuoCache(1, w.batch, w.num_q_heads, w.num_kv_heads, w.head_dim, w.sink, w.recent, max_len, mask)
              for _ in range(2)]
    q, k, v = workloads.tokens(w, 0, 0, T_prefill + 2, device="cuda")
    for c in caches:
        out = torch.empty_like(q[:, :T_prefill])
        c.prefill(0, q[:, :T_prefill].contiguous(), k[:, :T_prefill].contiguous(), v[:, :T_prefill].contiguous(), out)
        c.append(0, k[:, :T_prefill].contiguous(), v[:, :T_prefill].contiguous())
    return caches, (q, k, v)


@pytest.mark.parametrize("shape", [
    dict(batch=2, num_q_heads=8, num_kv_heads=2, head_dim=128, sink=64, recent=256, mask=(1, 0), T=9000),
    dict(batch=1, num_q_heads=4, num_kv_heads=4, head_dim=64, sink=4, recent=64, mask=(1, 0, 1, 0), T=700),
])
def test_static_scratch_decode_matches_duo_decode(duo, shape):
    import workloads
    w = workloads.Workload("no_alloc", batch=shape["batch"], num_q_heads=shape["num_q_heads"],
                           num_kv_heads=shape["num_kv_heads"], head_dim=shape["head_dim"], sink=shape["sink"],
                           recent=shape["recent"], retrieval_ratio=0.5, explicit_retrieval=shape["mask"], seed=5)
    T = shape["T"]
    (ref_cache, static_cache), (q, k, v) = _pair_of_caches(duo, w, T, T + 8)
    for step in range(2):  # two calls in a row: the array keeps the first call's contents
        p = T + step
        qd, kd, vd = (x[:, p].contiguous() for x in (q, k, v))
        a = torch.full_like(qd, float("nan"))
        b = torch.full_like(qd, float("nan"))
        assert duo.duo_decode(ref_cache.handle, 0, qd, kd, vd, a) == duo.DUO_OK
        assert duo.duo_decode_static_scratch(static_cache.handle, 0, qd, kd, vd, b) == duo.DUO_OK
        torch.cuda.synchronize()
        ra, rb = a.float().cpu().numpy(), b.float().cpu().numpy()
        assert np.all(np.isfinite(rb))
        assert np.all(np.abs(rb - ra) <= ATOL + RTOL * np.abs(ra)), f"step {step}: max diff {np.abs(rb - ra).max()}"
        assert static_cache.length(0) == ref_cache.length(0) == p + 1
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
