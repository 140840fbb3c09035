"""Pins for the fp64 oracle: it is checked against things other than itself.

- hand-derived key sets and a hand-derived worked example (tests/golden/);
- special cases that reduce to a library routine (PyTorch's causal and masked
  scaled_dot_product_attention in float64);
- an evict-oldest cache simulation (a second derivation of the streaming key
  set from the abstract's fixed-size cache of sink and latest tokens);
- closed forms, invariants and exact special cases.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import brute, cache_model

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16)


def _to_oracle_layout(x):
    """[B, T, H, D] -> [B, H, T, D] contiguous."""
    return x.permute(0, 2, 1, 3).contiguous()


def _sdpa(q, k, v, mask=None, causal=False, scale=None):
    """PyTorch's attention in float64 on [B, H, T, D] (GQA: repeat KV heads)."""
    G = q.shape[1] // k.shape[1]
    k = k.double().repeat_interleave(G, dim=1)
    v = v.double().repeat_interleave(G, dim=1)
    return torch.nn.functional.scaled_dot_product_attention(
        q.double(), k, v, attn_mask=mask, is_causal=causal, scale=scale).numpy()


def test_golden_keysets():
    data = json.load(open(os.path.join(GOLDEN, "keysets.json")))
    for c in data["cases"]:
        retr = 1 if c["kind"] == "retrieval" else 0
        got = [j for j in range(c["p"] + 1) if oracle.key_allowed(retr, c["p"], j, c["sink"], c["recent"])]
        assert got == c["keys"], c


def test_streaming_keyset_size_is_constant_length():
    # A streaming head's cache has constant length sink + recent once full.
    for S in range(0, 5):
        for R in range(1, 6):
            for p in range(0, 30):
                n = sum(oracle.key_allowed(0, p, j, S, R) for j in range(p + 1))
                assert n == min(p + 1, S + R), (S, R, p)


def test_golden_worked_example():
    data = json.load(open(os.path.join(GOLDEN, "worked_example.json")))
    D = data["D"]
    q = torch.tensor([data["q"]], dtype=torch.bfloat16).reshape(1, 1, 1, D)
    k = torch.tensor(data["k"], dtype=torch.bfloat16).reshape(1, 1, 3, D)
    v = torch.tensor(data["v"], dtype=torch.bfloat16).reshape(1, 1, 3, D)
    for c in data["cases"]:
        retr = [1 if c["kind"] == "retrieval" else 0]
        out = oracle.attention(q, [2], k, v, retr, c["sink"], c["recent"])
        np.testing.assert_allclose(out[0, 0, 0], c["out"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2)])
def test_all_retrieval_equals_causal_attention(Hq, Hkv):
    B, T, D = 2, 37, 16
    q, k, v = _rand_bf16((B, Hq, T, D), 1), _rand_bf16((B, Hkv, T, D), 2), _rand_bf16((B, Hkv, T, D), 3)
    out = oracle.attention(q, np.arange(T), k, v, [1] * Hkv, sink=2, recent=3)
    ref = _sdpa(q, k, v, causal=True)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_streaming_head_with_wide_window_equals_full_head():
    B, H, T, D = 1, 3, 40, 8
    q, k, v = _rand_bf16((B, H, T, D), 4), _rand_bf16((B, H, T, D), 5), _rand_bf16((B, H, T, D), 6)
    for S, R in [(0, 40), (4, 36), (4, 600), (40, 1)]:
        out = oracle.attention(q, np.arange(T), k, v, [0] * H, sink=S, recent=R)
        ref = _sdpa(q, k, v, causal=True)
        np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("S,R", [(0, 1), (1, 1), (2, 3), (4, 5), (3, 11)])
def test_all_streaming_equals_evict_oldest_cache(S, R):
    """The key set of a streaming query is what an evict-oldest cache of
    S sinks + R recent tokens holds right after the query's token arrives."""
    B, Hq, Hkv, T, D = 1, 4, 2, 33, 8
    q, k, v = _rand_bf16((B, Hq, T, D), 7), _rand_bf16((B, Hkv, T, D), 8), _rand_bf16((B, Hkv, T, D), 9)
    mask = torch.zeros(T, T, dtype=torch.bool)
    for p in range(T):
        for j in cache_model.retained_positions(False, S, R, p + 1):
            mask[p, j] = True
    ref = _sdpa(q, k, v, mask=mask)
    out = oracle.attention(q, np.arange(T), k, v, [0] * Hkv, sink=S, recent=R)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_dense_brute_force_matches_mixed_heads():
    B, Hq, Hkv, T, D = 2, 6, 3, 29, 8
    q, k, v = _rand_bf16((B, Hq, T, D), 10), _rand_bf16((B, Hkv, T, D), 11), _rand_bf16((B, Hkv, T, D), 12)
    kinds = [1, 0, 0]
    bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    ref = brute.attention(bits(q), bits(k), bits(v), kinds, sink=2, recent=5)
    out = oracle.attention(q, np.arange(T), k, v, kinds, sink=2, recent=5)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_softmax_weights_sum_to_one():
    B, H, T, D = 1, 4, 50, 16
    q, k, v = _rand_bf16((B, H, T, D), 13), _rand_bf16((B, H, T, D), 14), _rand_bf16((B, H, T, D), 15)
    _, ws = oracle.attention(q, np.arange(T), k, v, [1, 0, 1, 0], sink=3, recent=7, with_wsum=True)
    assert np.max(np.abs(ws - 1.0)) < 1e-12


def test_query_at_position_zero_returns_v0_exactly():
    B, H, T, D = 1, 2, 5, 8
    q, k, v = _rand_bf16((B, H, T, D), 16), _rand_bf16((B, H, T, D), 17), _rand_bf16((B, H, T, D), 18)
    out = oracle.attention(q[:, :, :1], [0], k, v, [1, 0], sink=0, recent=1)
    np.testing.assert_array_equal(out[:, :, 0], v[:, :, 0].double().numpy())


def test_constant_values_give_that_value():
    B, H, T, D = 1, 2, 20, 8
    q, k = _rand_bf16((B, H, T, D), 19), _rand_bf16((B, H, T, D), 20)
    u = _rand_bf16((D,), 21)
    v = u.expand(B, H, T, D).contiguous()
    out = oracle.attention(q, np.arange(T), k, v, [1, 0], sink=1, recent=4)
    np.testing.assert_allclose(out, np.broadcast_to(u.double().numpy(), out.shape), rtol=0, atol=1e-14)


def test_scale_argument():
    B, H, T, D = 1, 2, 12, 8
    q, k, v = _rand_bf16((B, H, T, D), 22), _rand_bf16((B, H, T, D), 23), _rand_bf16((B, H, T, D), 24)
    out = oracle.attention(q, np.arange(T), k, v, [1, 1], sink=1, recent=4, scale=0.3)
    ref = _sdpa(q, k, v, causal=True, scale=0.3)
    np.testing.assert_allclose(out, ref, rtol=1e-12, atol=1e-12)


def test_slot_map_closed_form_matches_simulation():
    for S in range(0, 6):
        for R in range(1, 7):
            W = S + R
            for L in range(0, 41):
                pos = oracle.slot_positions(0, S, R, L, W)
                sim = cache_model.ring_slots(S, R, L)
                for s in range(W):
                    assert pos[s] == sim.get(s, -1), (S, R, L, s)
                held = sorted(int(p) for p in pos if p >= 0)
                assert held == cache_model.retained_positions(False, S, R, L), (S, R, L)
            rpos = oracle.slot_positions(1, S, R, 9, 12)
            assert list(rpos) == list(range(9)) + [-1, -1, -1]


@pytest.mark.parametrize("S,R", [(4, 8), (0, 5), (3, 1), (6, 40)])
def test_decode_over_cache_slots_equals_masked_prefill(S, R):
    """A decode step attends over the slots of the cache after appending its own
    token; that equals the masked attention of the same query in a prefill."""
    T, D = 30, 8
    q, k, v = _rand_bf16((1, 1, T, D), 25), _rand_bf16((1, 1, T, D), 26), _rand_bf16((1, 1, T, D), 27)
    scale = 1.0 / math.sqrt(D)
    full = oracle.attention(q, np.arange(T), k, v, [0], sink=S, recent=R)
    for p in range(T):
        pos = oracle.slot_positions(0, S, R, p + 1, S + R)
        held = [int(x) for x in pos if x >= 0]
        out, _ = oracle.attend_rows(q[0, 0, p], k[0, 0, held], v[0, 0, held], scale)
        np.testing.assert_allclose(out, full[0, 0, p], rtol=1e-12, atol=1e-13)


def test_ring_order_does_not_matter():
    T, D, S, R = 25, 8, 2, 6
    q, k, v = _rand_bf16((1, 1, T, D), 28), _rand_bf16((1, 1, T, D), 29), _rand_bf16((1, 1, T, D), 30)
    scale = 1.0 / math.sqrt(D)
    pos = [int(x) for x in oracle.slot_positions(0, S, R, T, S + R) if x >= 0]
    a, _ = oracle.attend_rows(q[0, 0, T - 1], k[0, 0, pos], v[0, 0, pos], scale)
    perm = list(reversed(pos))
    b, _ = oracle.attend_rows(q[0, 0, T - 1], k[0, 0, perm], v[0, 0, perm], scale)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-14)


def test_queries_are_independent_of_batching():
    """Chunked prefill equals one prefill: each query row only sees keys <= p,
    so computing rows in chunks of any size gives the same rows."""
    B, H, T, D = 1, 2, 40, 8
    q, k, v = _rand_bf16((B, H, T, D), 31), _rand_bf16((B, H, T, D), 32), _rand_bf16((B, H, T, D), 33)
    full = oracle.attention(q, np.arange(T), k, v, [1, 0], sink=2, recent=5)
    for C in (1, 7, 13):
        for c0 in range(0, T, C):
            c1 = min(T, c0 + C)
            part = oracle.attention(q[:, :, c0:c1], np.arange(c0, c1), k[:, :, :c1], v[:, :, :c1], [1, 0],
                                    sink=2, recent=5)
            np.testing.assert_array_equal(part, full[:, :, c0:c1])
