"""Footprint report (bench.py --memory): full-attention KV bytes against the mixed-head
cache the library sizes. Host-only: duo_cache_alloc without a buffer only sizes."""
import pytest

import bench
import mixed_head_kv_b200 as duo


def _fp(ratio, context, layers=2, hq=8, hkv=4, d=64, sink=4, recent=60, params=0.0):
    return bench.memory_footprint(duo, "t", layers, hq, hkv, d, ratio, params, context, sink=sink, recent=recent)


def test_all_retrieval_keeps_the_full_cache():
    r = _fp(1.0, 4096)
    assert r["kv_duo_bytes"] == r["kv_full_bytes"]
    assert r["kv_ratio"] == 1.0


@pytest.mark.parametrize("mult", [1, 4, 16])
def test_all_streaming_cache_is_constant_length(mult):
    # sink + recent = 64 slots per head, whatever the context
    r = _fp(0.0, 64 * mult)
    assert r["kv_duo_bytes"] == 2 * 1 * 4 * 64 * 64 * 2 * 2
    assert r["kv_ratio"] == pytest.approx(mult)


def test_mixed_ratio_and_library_sizing():
    r = _fp(0.5, 8192)
    # half the KV heads keep 8192 slots, half keep 64
    assert r["retrieval_kv_heads"] == 4
    assert r["kv_duo_bytes"] == (4 * 8192 + 4 * 64) * 64 * 2 * 2
    # the library's buffer holds the two pools plus a decode scratch that does not grow with context
    scratch = r["duo_required_bytes"] - r["kv_duo_bytes"]
    assert 0 < scratch < (1 << 20)
    assert _fp(0.5, 4 * 8192)["duo_required_bytes"] - _fp(0.5, 4 * 8192)["kv_duo_bytes"] == scratch
    assert r["kv_ratio"] == pytest.approx(8 * 8192 / (4 * 8192 + 4 * 64))


def test_weights_dilute_the_ratio():
    r = _fp(0.25, 1 << 16, params=1e9)
    assert 1.0 < r["with_weights_ratio"] < r["kv_ratio"]
