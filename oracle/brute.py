"""Dense-mask NumPy restatement of mixed-head attention, for tiny inputs only.

TEST INFRASTRUCTURE ONLY (see oracle/__init__.py). It materialises the full
T x T boolean mask of every head and the full softmax matrix, so a reader can
check it against the DuoAttention abstract by eye: retrieval heads see every
previous token, streaming heads see the attention sinks and the recent window.
"""
from __future__ import annotations

import numpy as np


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def head_mask(T: int, is_retrieval: bool, sink: int, recent: int) -> np.ndarray:
    """mask[p, j] = True when a query at position p attends to key position j."""
    p = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    causal = j <= p
    if is_retrieval:
        return causal
    return causal & ((j < sink) | (p - j < recent))


def attention(q_bits, k_bits, v_bits, is_retrieval, sink, recent, scale=None):
    """q: [B, Hq, T, D], k/v: [B, Hkv, T, D] as bf16 bit patterns (uint16), all
    positions 0..T-1 (query row p sits at position p). Returns [B, Hq, T, D] f64."""
    q = bf16_bits_to_f64(np.asarray(q_bits))
    k = bf16_bits_to_f64(np.asarray(k_bits))
    v = bf16_bits_to_f64(np.asarray(v_bits))
    B, Hq, T, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.empty_like(q)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            m = head_mask(T, bool(is_retrieval[g]), sink, recent)
            s = scale * (q[b, h] @ k[b, g].T)
            s = np.where(m, s, -np.inf)
            s = s - s.max(axis=1, keepdims=True)
            e = np.where(m, np.exp(s), 0.0)
            a = e / e.sum(axis=1, keepdims=True)
            out[b, h] = a @ v[b, g]
    return out
