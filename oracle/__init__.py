"""Oracle for mixed-head (DuoAttention) attention: plain, slow, fp64, CPU.

TEST INFRASTRUCTURE ONLY: imported by tests/, by the smoke check and by the
benchmark's CPU-baseline leg, never by the product package. It shares no code
with the CUDA path.

Parts:
  duo_oracle.c   the masked attention and the cache slot model (fp64, OpenMP)
  brute.py       a dense-mask NumPy restatement for tiny inputs
  cache_model.py an evict-oldest cache simulation for tiny inputs
This module wraps duo_oracle.c through ctypes, taking numpy/torch arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "duo_oracle.c")
_LIB = os.path.join(_HERE, "libduo_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile duo_oracle.c with gcc (-O2 -fopenmp) into libduo_oracle.so."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.duo_oracle_attention.restype = i64
        lib.duo_oracle_attention.argtypes = [P, P, P, P, P, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                             i64, i64, ctypes.c_int, i64, i64, ctypes.c_double, P, P]
        lib.duo_oracle_attend_rows.restype = ctypes.c_int
        lib.duo_oracle_attend_rows.argtypes = [P, P, P, i64, ctypes.c_int, ctypes.c_double, P, P]
        lib.duo_oracle_slot_positions.restype = None
        lib.duo_oracle_slot_positions.argtypes = [ctypes.c_int, i64, i64, i64, i64, P]
        lib.duo_oracle_key_allowed.restype = ctypes.c_int
        lib.duo_oracle_key_allowed.argtypes = [ctypes.c_int, i64, i64, i64, i64]
        lib.duo_oracle_num_threads.restype = ctypes.c_int
        lib.duo_oracle_e4m3_value.restype = ctypes.c_double
        lib.duo_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.duo_oracle_e4m3_code.restype = ctypes.c_uint8
        lib.duo_oracle_e4m3_code.argtypes = [ctypes.c_double]
        lib.duo_oracle_attend_rows_e4m3.restype = ctypes.c_int
        lib.duo_oracle_attend_rows_e4m3.argtypes = [P, P, P, i64, ctypes.c_int, ctypes.c_double, ctypes.c_double,
                                                    ctypes.c_double, P, P]
        lib.duo_oracle_e4m3_quantize.restype = None
        lib.duo_oracle_e4m3_quantize.argtypes = [P, i64, ctypes.c_float, P]
        _lib = lib
    return _lib


def _bits(a) -> np.ndarray:
    """bf16 tensor/array -> contiguous uint16 bit patterns."""
    try:
        import torch
        if isinstance(a, torch.Tensor):
            assert a.dtype == torch.bfloat16
            return np.ascontiguousarray(a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))
    except ImportError:  # pragma: no cover
        pass
    a = np.asarray(a)
    assert a.dtype == np.uint16
    return np.ascontiguousarray(a)


def num_threads() -> int:
    return int(_load().duo_oracle_num_threads())


def key_allowed(is_retrieval: int, p: int, j: int, sink: int, recent: int) -> bool:
    return bool(_load().duo_oracle_key_allowed(int(is_retrieval), p, j, sink, recent))


def attention(q, qpos, k, v, is_retrieval, sink: int, recent: int, scale: float | None = None,
              with_wsum: bool = False):
    """Mixed-head attention in fp64.

    q: [B, Hq, NQ, D] bf16 (query i at absolute position qpos[i]);
    k, v: [B, Hkv, T, D] bf16 (row j = position j); is_retrieval: [Hkv] 0/1.
    Returns out [B, Hq, NQ, D] float64 (and the softmax weight sums).
    """
    lib = _load()
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    B, Hq, NQ, D = qb.shape
    _, Hkv, T, _ = kb.shape
    assert kb.shape == vb.shape and Hq % Hkv == 0
    qp = np.ascontiguousarray(np.asarray(qpos, dtype=np.int64).reshape(-1))
    assert qp.shape[0] == NQ
    kind = np.ascontiguousarray(np.asarray(is_retrieval, dtype=np.uint8).reshape(-1))
    assert kind.shape[0] == Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    out = np.zeros((B, Hq, NQ, D), dtype=np.float64)
    ws = np.zeros((B, Hq, NQ), dtype=np.float64)
    failed = lib.duo_oracle_attention(qb.ctypes.data, qp.ctypes.data, kb.ctypes.data, vb.ctypes.data,
                                      kind.ctypes.data, B, Hq, Hkv, NQ, T, D, sink, recent,
                                      float(scale), out.ctypes.data, ws.ctypes.data)
    if failed:
        raise ValueError(f"{failed} query rows have an empty key set")
    return (out, ws) if with_wsum else out


def attend_rows(q, keys, vals, scale: float):
    """Softmax attention of one query q[D] over explicit key/value rows [n, D] (bf16)."""
    lib = _load()
    qb, kb, vb = _bits(q), _bits(keys), _bits(vals)
    n, D = kb.shape
    out = np.zeros(D, dtype=np.float64)
    ws = np.zeros(1, dtype=np.float64)
    rc = lib.duo_oracle_attend_rows(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, n, D, float(scale),
                                    out.ctypes.data, ws.ctypes.data)
    if rc != 0:
        raise ValueError("empty key list")
    return out, float(ws[0])


def slot_positions(is_retrieval: int, sink: int, recent: int, length: int, nslots: int) -> np.ndarray:
    """Absolute position held by each cache slot after `length` appended tokens (-1 = empty)."""
    lib = _load()
    pos = np.zeros(nslots, dtype=np.int64)
    lib.duo_oracle_slot_positions(int(is_retrieval), sink, recent, length, nslots, pos.ctypes.data)
    return pos


def e4m3_value(code: int) -> float:
    """Value of an FP8 E4M3 code (NaN for 0x7F / 0xFF)."""
    return float(_load().duo_oracle_e4m3_value(int(code)))


def e4m3_code(x: float) -> int:
    """E4M3 code of x: nearest, ties to even, saturating to +-448."""
    return int(_load().duo_oracle_e4m3_code(float(x)))


def e4m3_quantize(x, inv_scale: float) -> np.ndarray:
    """Codes of bf16 values x times inv_scale (product rounded to fp32 first)."""
    xb = _bits(x)
    out = np.zeros(xb.shape, dtype=np.uint8)
    _load().duo_oracle_e4m3_quantize(xb.ctypes.data, xb.size, float(inv_scale), out.ctypes.data)
    return out


def attend_rows_e4m3(q, k_codes, v_codes, k_scale: float, v_scale: float, scale: float):
    """attend_rows over key/value rows [n, D] stored as E4M3 codes with per-head scales."""
    lib = _load()
    qb = _bits(q)
    kc = np.ascontiguousarray(k_codes, dtype=np.uint8)
    vc = np.ascontiguousarray(v_codes, dtype=np.uint8)
    n, D = kc.shape
    out = np.zeros(D, dtype=np.float64)
    ws = np.zeros(1, dtype=np.float64)
    rc = lib.duo_oracle_attend_rows_e4m3(qb.ctypes.data, kc.ctypes.data, vc.ctypes.data, n, D, float(k_scale),
                                         float(v_scale), float(scale), out.ctypes.data, ws.ctypes.data)
    if rc != 0:
        raise ValueError("empty key list")
    return out, float(ws[0])
