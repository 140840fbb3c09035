"""Python binding of libduo (include/duo.h): mixed-head (DuoAttention) attention on B200.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libduo.so. PyTorch supplies device memory and streams. The module
refuses to load when libduo.so has not been built (run
`python mixed_head_kv_b200/build.py` or `__graft_entry__.build()`); there is
no fallback path.

Functions keep the C names: duo_cache_alloc, duo_cache_free, duo_cache_append,
duo_prefill, duo_decode, duo_cache_len, duo_cache_set_len, duo_cache_views,
duo_cache_error, duo_status_str. `DuoCache` bundles a cache handle with the
torch buffer that backs it.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libduo.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libduo.so is not built at {LIB_PATH}; run `python mixed_head_kv_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

DUO_OK = 0
DUO_ERR_INVALID_ARG = 1
DUO_ERR_CAPACITY = 2
DUO_ERR_ALIGNMENT = 3
DUO_ERR_CUDA = 4
DUO_ERR_STATE = 5
DUO_ERR_DEVICE = 6
DUO_ERR_SCRATCH_LIMIT = 7
DUO_STATIC_SCRATCH_BYTES = 16 * 1024 * 1024
DUO_MAX_Q_HEADS = 256
DUO_MAX_KV_HEADS = 128

DUO_MAX_RAGGED_BATCH = 64  # sequences of different lengths per batch (include/duo.h)
DUO_KV_BF16 = 0  # cache formats of the retrieval heads (include/duo.h)
DUO_KV_E4M3 = 1

EXPORTED = ("duo_cache_alloc", "duo_cache_free", "duo_cache_append", "duo_prefill", "duo_decode",
            "duo_cache_len", "duo_cache_set_len", "duo_cache_views", "duo_cache_error", "duo_status_str",
            "duo_decode_static_scratch", "duo_cache_append_ragged", "duo_cache_seq_lens",
            "duo_cache_set_seq_lens", "duo_prefill_ragged", "duo_cache_set_kv_scales",
            "duo_cache_test_wait_timeout")
DUO_TEST_WAIT_DECODE = 1  # duo_cache_test_wait_timeout kinds and duo_cache_error bits (include/duo.h)
DUO_TEST_WAIT_PREFILL = 2
DUO_ERR_BIT_PREFILL_WAIT = 1
DUO_ERR_BIT_DECODE_COPY = 2


class duo_layout(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32), ("sink", ctypes.c_int32),
                ("recent", ctypes.c_int32), ("kv_format", ctypes.c_int32), ("max_len", ctypes.c_int64),
                ("softmax_scale", ctypes.c_float), ("reserved1", ctypes.c_int32)]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_ST = ctypes.c_int

_lib.duo_status_str.restype = ctypes.c_char_p
_lib.duo_status_str.argtypes = [_ST]
_lib.duo_cache_alloc.restype = _ST
_lib.duo_cache_alloc.argtypes = [ctypes.POINTER(duo_layout), _P, _P, ctypes.c_size_t,
                                 ctypes.POINTER(ctypes.c_size_t), _P, ctypes.POINTER(_P)]
_lib.duo_cache_free.restype = _ST
_lib.duo_cache_free.argtypes = [_P]
_lib.duo_cache_append.restype = _ST
_lib.duo_cache_append.argtypes = [_P, _I32, _P, _P, _I64, _P]
_lib.duo_prefill.restype = _ST
_lib.duo_prefill.argtypes = [_P, _I32, _P, _P, _P, _P, _I64, _P]
_lib.duo_decode.restype = _ST
_lib.duo_decode.argtypes = [_P, _I32, _P, _P, _P, _P, _P]
_lib.duo_decode_static_scratch.restype = _ST
_lib.duo_decode_static_scratch.argtypes = [_P, _I32, _P, _P, _P, _P, _P]
_lib.duo_cache_len.restype = _ST
_lib.duo_cache_len.argtypes = [_P, _I32, ctypes.POINTER(_I64)]
_lib.duo_cache_set_len.restype = _ST
_lib.duo_cache_set_len.argtypes = [_P, _I32, _I64]
_lib.duo_cache_views.restype = _ST
_lib.duo_cache_views.argtypes = [_P, _I32, _I32, ctypes.POINTER(_P), ctypes.POINTER(_P), ctypes.POINTER(_I64),
                                 ctypes.POINTER(_I32)]
_lib.duo_cache_append_ragged.restype = _ST
_lib.duo_cache_append_ragged.argtypes = [_P, _I32, _P, _P, ctypes.POINTER(_I64), _I64, _P]
_lib.duo_cache_set_kv_scales.restype = _ST
_lib.duo_cache_set_kv_scales.argtypes = [_P, _I32, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_float), _P]
_lib.duo_prefill_ragged.restype = _ST
_lib.duo_prefill_ragged.argtypes = [_P, _I32, _P, _P, _P, _P, ctypes.POINTER(_I64), _I64, _P]
_lib.duo_cache_seq_lens.restype = _ST
_lib.duo_cache_seq_lens.argtypes = [_P, _I32, ctypes.POINTER(_I64)]
_lib.duo_cache_set_seq_lens.restype = _ST
_lib.duo_cache_set_seq_lens.argtypes = [_P, _I32, ctypes.POINTER(_I64)]
_lib.duo_cache_test_wait_timeout.restype = _ST
_lib.duo_cache_test_wait_timeout.argtypes = [_P, _I32, ctypes.c_uint64]
_lib.duo_cache_error.restype = _ST
_lib.duo_cache_error.argtypes = [_P, _P, ctypes.POINTER(ctypes.c_uint32)]


class DuoError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {duo_status_str(status)} (status {status})")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != DUO_OK:
        raise DuoError(status, where)


def _ptr(x) -> Optional[int]:
    """Device pointer of a tensor, or an int/None passed through."""
    if x is None or isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        raw = getattr(torch._C, "_cuda_getCurrentRawStream", None)
        if raw is not None:  # the current stream's handle without building a Stream object
            return raw(torch.cuda.current_device())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def duo_status_str(status: int) -> str:
    return _lib.duo_status_str(status).decode()


def make_layout(num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, recent, max_len,
                softmax_scale=0.0, kv_format=0) -> duo_layout:
    return duo_layout(num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, recent, kv_format, max_len,
                      softmax_scale, 0)


def _mask_buf(is_retrieval: Sequence[int]):
    vals = [int(x) for x in is_retrieval]
    return (ctypes.c_uint8 * max(1, len(vals)))(*vals)


def duo_cache_alloc(layout: duo_layout, is_retrieval: Sequence[int], dev_buf=None, buf_bytes: int = 0,
                    stream=None):
    """Returns (status, required_bytes, handle). With dev_buf None only sizes the cache."""
    req = ctypes.c_size_t(0)
    handle = _P()
    mask = _mask_buf(is_retrieval)
    s = _stream(stream) if dev_buf is not None else None
    st = _lib.duo_cache_alloc(ctypes.byref(layout), ctypes.cast(mask, _P), _ptr(dev_buf), buf_bytes,
                              ctypes.byref(req), s, ctypes.byref(handle))
    return st, req.value, handle.value


def duo_cache_free(handle) -> int:
    return _lib.duo_cache_free(handle)


def duo_cache_append(handle, layer, k, v, n_tok, stream=None) -> int:
    return _lib.duo_cache_append(handle, layer, _ptr(k), _ptr(v), n_tok, _stream(stream))


def duo_prefill(handle, layer, q, k, v, out, n_tok, stream=None) -> int:
    return _lib.duo_prefill(handle, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), n_tok, _stream(stream))


def duo_decode(handle, layer, q, k_new, v_new, out, stream=None) -> int:
    return _lib.duo_decode(handle, layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out), _stream(stream))


def duo_decode_static_scratch(handle, layer, q, k_new, v_new, out, stream=None) -> int:
    """duo_decode with its split-KV scratch in the library's static device array
    (for callers that cannot allocate device memory at call time)."""
    return _lib.duo_decode_static_scratch(handle, layer, _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                          _stream(stream))


def duo_cache_len(handle, layer):
    n = _I64(0)
    st = _lib.duo_cache_len(handle, layer, ctypes.byref(n))
    return st, n.value


def duo_cache_set_len(handle, layer, length) -> int:
    return _lib.duo_cache_set_len(handle, layer, length)


def duo_cache_append_ragged(handle, layer, k, v, n_tok: Sequence[int], max_tok: int, stream=None) -> int:
    """Sequence b appends rows [0, n_tok[b]) of k/v [batch][max_tok][Hkv][D]."""
    n = (_I64 * max(1, len(n_tok)))(*[int(x) for x in n_tok])
    return _lib.duo_cache_append_ragged(handle, layer, _ptr(k), _ptr(v), n, max_tok,
                                        _stream(stream) if k is not None else None)


def duo_prefill_ragged(handle, layer, q, k, v, out, n_tok: Sequence[int], max_tok: int, stream=None) -> int:
    """Sequence b's chunk is rows [0, n_tok[b]) of q/k/v [batch][max_tok][H][D]."""
    n = (_I64 * max(1, len(n_tok)))(*[int(x) for x in n_tok])
    return _lib.duo_prefill_ragged(handle, layer, _ptr(q), _ptr(k), _ptr(v), _ptr(out), n, max_tok,
                                   _stream(stream) if q is not None else None)


def duo_cache_set_kv_scales(handle, layer, k_scale: Sequence[float], v_scale: Sequence[float], stream=None) -> int:
    """Per-KV-head scales of an E4M3 cache (host lists [num_kv_heads])."""
    k = (ctypes.c_float * max(1, len(k_scale)))(*[float(x) for x in k_scale])
    v = (ctypes.c_float * max(1, len(v_scale)))(*[float(x) for x in v_scale])
    return _lib.duo_cache_set_kv_scales(handle, layer, k, v, _stream(stream))


def duo_cache_seq_lens(handle, layer, batch: int):
    lens = (_I64 * batch)()
    st = _lib.duo_cache_seq_lens(handle, layer, lens)
    return st, list(lens)


def duo_cache_set_seq_lens(handle, layer, lens: Sequence[int]) -> int:
    arr = (_I64 * max(1, len(lens)))(*[int(x) for x in lens])
    return _lib.duo_cache_set_seq_lens(handle, layer, arr)


def duo_cache_views(handle, layer, kv_head):
    k, v, slots, r = _P(), _P(), _I64(0), _I32(0)
    st = _lib.duo_cache_views(handle, layer, kv_head, ctypes.byref(k), ctypes.byref(v), ctypes.byref(slots),
                              ctypes.byref(r))
    return st, k.value, v.value, slots.value, r.value


def duo_cache_test_wait_timeout(handle, launches: int, timeout_ns: int) -> int:
    """Arm the next launch of the given kinds to test the bounded waits (include/duo.h)."""
    return _lib.duo_cache_test_wait_timeout(handle, launches, timeout_ns)


def duo_cache_error(handle, stream=None):
    f = ctypes.c_uint32(0)
    st = _lib.duo_cache_error(handle, _stream(stream), ctypes.byref(f))
    return st, f.value


class DuoCache:
    """A cache handle plus the torch uint8 buffer that backs it (owned here)."""

    def __init__(self, num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, recent, max_len,
                 is_retrieval: Sequence[int], softmax_scale=0.0, device="cuda", stream=None, kv_format=0):
        import torch
        self.layout = make_layout(num_layers, batch, num_q_heads, num_kv_heads, head_dim, sink, recent, max_len,
                                  softmax_scale, kv_format)
        self.is_retrieval = [int(x) for x in is_retrieval]
        st, req, _ = duo_cache_alloc(self.layout, self.is_retrieval)
        _check(st, "duo_cache_alloc(size)")
        self.nbytes = req
        self.buffer = torch.empty(req + 256, dtype=torch.uint8, device=device)
        off = (-self.buffer.data_ptr()) % 256
        self._base = self.buffer.data_ptr() + off
        st, _, handle = duo_cache_alloc(self.layout, self.is_retrieval, self._base, req, stream)
        _check(st, "duo_cache_alloc")
        self.handle = handle

    def close(self):
        if getattr(self, "handle", None):
            duo_cache_free(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:  # interpreter shutdown: module globals may already be gone
            pass

    def append(self, layer, k, v, stream=None):
        _check(duo_cache_append(self.handle, layer, k, v, k.shape[1], stream), "duo_cache_append")

    def append_ragged(self, layer, k, v, n_tok, stream=None):
        """Per-sequence token counts n_tok[b] <= k.shape[1] (rows past them are not read)."""
        _check(duo_cache_append_ragged(self.handle, layer, k, v, n_tok, k.shape[1], stream),
               "duo_cache_append_ragged")

    def prefill_ragged(self, layer, q, k, v, out, n_tok, stream=None):
        _check(duo_prefill_ragged(self.handle, layer, q, k, v, out, n_tok, q.shape[1], stream), "duo_prefill_ragged")

    def seq_lens(self, layer):
        st, lens = duo_cache_seq_lens(self.handle, layer, self.layout.batch)
        _check(st, "duo_cache_seq_lens")
        return lens

    def set_seq_lens(self, layer, lens):
        _check(duo_cache_set_seq_lens(self.handle, layer, lens), "duo_cache_set_seq_lens")

    def prefill(self, layer, q, k, v, out, stream=None):
        _check(duo_prefill(self.handle, layer, q, k, v, out, q.shape[1], stream), "duo_prefill")

    def decode(self, layer, q, k_new, v_new, out, stream=None):
        _check(duo_decode(self.handle, layer, q, k_new, v_new, out, stream), "duo_decode")

    def length(self, layer) -> int:
        st, n = duo_cache_len(self.handle, layer)
        _check(st, "duo_cache_len")
        return n

    def set_length(self, layer, n):
        _check(duo_cache_set_len(self.handle, layer, n), "duo_cache_set_len")

    def error_flags(self, stream=None) -> int:
        st, f = duo_cache_error(self.handle, stream)
        _check(st, "duo_cache_error")
        return f

    def head_view(self, layer, kv_head):
        """(k, v, is_retrieval): torch views [batch, slots, head_dim] of one KV head's cache
        (bf16, or uint8 E4M3 codes for the retrieval heads of an E4M3 cache)."""
        import torch
        st, kp, vp, slots, r = duo_cache_views(self.handle, layer, kv_head)
        _check(st, "duo_cache_views")
        B, D = self.layout.batch, self.layout.head_dim
        codes = bool(r) and self.layout.kv_format == DUO_KV_E4M3
        n = B * slots * D * (1 if codes else 2)  # bytes

        def view(ptr):
            start = ptr - self.buffer.data_ptr()
            raw = self.buffer[start:start + n]
            return (raw if codes else raw.view(torch.bfloat16)).view(B, slots, D)
        return view(kp), view(vp), r

    def set_kv_scales(self, layer, k_scale, v_scale, stream=None):
        _check(duo_cache_set_kv_scales(self.handle, layer, k_scale, v_scale, stream), "duo_cache_set_kv_scales")
