"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Outputs: |gpu - oracle| <= 2e-2 + 2e-2 |oracle| element-wise (bf16 inputs,
fp32 accumulation, bf16 outputs). Caches: bit-exact against the oracle's slot
model applied to the input rows.
"""
import numpy as np
import pytest
import torch

import __graft_entry__
from duo_harness import assert_close, check_cache_bits, make_workload, oracle_out, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    __graft_entry__.build()
    torch.cuda.set_device(0)


def _full_check(w, chunks, steps, max_len=None):
    T = sum(chunks) + steps
    max_len = max_len or T + 8
    cache, out, (q, k, v) = run_gpu(w, chunks, steps, max_len=max_len)
    ref = oracle_out(w, q, k, v, np.arange(T))
    err = assert_close(out, ref, f"chunks={chunks} steps={steps}")
    check_cache_bits(cache, w, k, v, T, max_len)
    assert cache.error_flags() == 0
    return err, out, ref, (q, k, v)


def test_tiny_mha_config():
    """1 batch, 4 heads (0, 2 retrieval; 1, 3 streaming), D=64, sink 4 + recent 64,
    prefill 512 in one chunk then 16 decode steps."""
    w = make_workload(B=1, Hq=4, Hkv=4, D=64, S=4, R=64, mask=(1, 0, 1, 0))
    _full_check(w, [512], 16)


@pytest.mark.parametrize("chunks,steps", [([100, 300, 37], 5), ([1, 1, 129], 3), ([256, 256], 0), ([0], 4)])
def test_mha_d128_chunks(chunks, steps):
    w = make_workload(B=1, Hq=4, Hkv=4, D=128, S=4, R=40, mask=(1, 0, 0, 1))
    _full_check(w, [c for c in chunks if c], steps)


@pytest.mark.parametrize("C", [1, 7, 64, 65, 200])
def test_chunk_size_sweep(C):
    w = make_workload(B=1, Hq=2, Hkv=2, D=128, S=3, R=50, mask=(1, 0), seed=C)
    T = 260
    chunks = [C] * (T // C) + ([T % C] if T % C else [])
    _full_check(w, chunks, 2)


@pytest.mark.parametrize("G", [2, 4, 8])
def test_gqa_groups(G):
    w = make_workload(B=2, Hq=2 * G, Hkv=2, D=128, S=8, R=130, mask=(0, 1), seed=G)
    _full_check(w, [129, 256, 1, 64], 3)


@pytest.mark.parametrize("S,R", [(0, 1), (0, 128), (200, 30), (4, 1000), (130, 129), (1, 257)])
def test_sink_window_edges(S, R):
    """Degenerate windows (only the query itself), a window wider than the
    context (streaming = full), chunks straddling the sink boundary, windows
    that are not tile multiples."""
    w = make_workload(B=1, Hq=4, Hkv=2, D=128, S=S, R=R, mask=(0, 1), seed=S + R)
    _full_check(w, [150, 100, 300], 4)


@pytest.mark.parametrize("mask", [(1, 1), (0, 0)])
def test_all_retrieval_and_all_streaming_layers(mask):
    w = make_workload(B=1, Hq=4, Hkv=2, D=64, S=16, R=100, mask=mask)
    _full_check(w, [333, 200], 3)


def test_sink_like_keys():
    """First 4 keys scaled x8 (attention-sink-like scores) exercise the stale-max rescale."""
    w = make_workload(B=1, Hq=4, Hkv=4, D=128, S=64, R=256, mask=(1, 0, 1, 0), sink_key_scale=8)
    _full_check(w, [700, 512], 3)


def test_first_query_returns_v0_exactly():
    w = make_workload(B=2, Hq=4, Hkv=2, D=128, S=2, R=8, mask=(1, 0))
    cache, out, (q, k, v) = run_gpu(w, [64], 0)
    G = 2
    for h in range(4):
        assert torch.equal(out[:, 0, h].view(torch.int16), v[:, 0, h // G].view(torch.int16))


def test_decode_after_prefill_equals_longer_prefill():
    """Prefill 300 + 20 decodes gives the rows a 320-token prefill gives."""
    w = make_workload(B=1, Hq=4, Hkv=4, D=128, S=4, R=64, mask=(1, 0, 1, 0), seed=3)
    _, a, qkv = run_gpu(w, [300], 20)
    _, b, _ = run_gpu(w, [320], 0, qkv=qkv)
    d = (a.float() - b.float()).abs()
    assert float(d.max()) <= 2e-2 + 2e-2 * float(b.float().abs().max())


def test_long_context_decode_splits():
    """Decode with many split-KV partials (cache of 20000 tokens, B=2, GQA)."""
    w = make_workload(B=2, Hq=8, Hkv=2, D=128, S=64, R=256, mask=(1, 0), seed=11)
    _full_check(w, [4096, 4096, 4096, 4096, 3616], 4)


def test_abi_errors_on_device():
    import mixed_head_kv_b200 as duo
    w = make_workload(B=1, Hq=2, Hkv=2, D=128, S=2, R=4, mask=(1, 0))
    cache = duo.DuoCache(1, 1, 2, 2, 128, 2, 4, 16, [1, 0])
    x = torch.zeros((1, 20, 2, 128), dtype=torch.bfloat16, device="cuda")
    o = torch.zeros_like(x)
    h = cache.handle
    assert duo.duo_prefill(h, 0, x, x, x, o, 17) == duo.DUO_ERR_CAPACITY
    assert duo.duo_cache_append(h, 0, x, x, 17) == duo.DUO_ERR_CAPACITY
    assert duo.duo_prefill(h, 1, x, x, x, o, 4) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_prefill(h, 0, x, x, x, o, -1) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_prefill(h, 0, None, x, x, o, 4) == duo.DUO_ERR_INVALID_ARG
    mis = x.view(-1)[1:].data_ptr()
    assert duo.duo_prefill(h, 0, mis, x, x, o, 4) == duo.DUO_ERR_ALIGNMENT
    assert duo.duo_cache_append(h, 0, x, mis, 4) == duo.DUO_ERR_ALIGNMENT
    assert duo.duo_decode(h, 0, x, x, mis, o) == duo.DUO_ERR_ALIGNMENT
    assert cache.length(0) == 0  # nothing changed
    assert duo.duo_cache_append(h, 0, x, x, 16) == duo.DUO_OK
    assert duo.duo_decode(h, 0, x, x, x, o) == duo.DUO_ERR_CAPACITY
    assert cache.length(0) == 16
    cache.set_length(0, 3)
    assert cache.length(0) == 3
    assert duo.duo_cache_set_len(h, 0, 17) == duo.DUO_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert cache.error_flags() == 0
