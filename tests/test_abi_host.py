"""Host-only checks of the C ABI (no GPU): the library loads, exports every
symbol include/duo.h declares, sizes caches as documented, and rejects bad
arguments before touching the device."""
import ctypes
import os
import re
import subprocess

import pytest

import __graft_entry__

__graft_entry__.build()
import mixed_head_kv_b200 as duo  # noqa: E402

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "duo.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^DUO_API\s+[\w\s\*]+?\b(duo_\w+)\s*\(", text, flags=re.M)))


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("duo_cache_alloc", "duo_cache_append", "duo_prefill", "duo_decode"):
        assert n in names
    assert set(names) == set(duo.EXPORTED)


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", duo.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for name in _declared():
        assert name in exported, name
        getattr(duo._lib, name)  # resolvable through ctypes


def _layout(**kw):
    base = dict(num_layers=2, batch=3, num_q_heads=8, num_kv_heads=4, head_dim=128, sink=4, recent=60,
                max_len=1000)
    base.update(kw)
    return duo.make_layout(**base)


def _expected_bytes(L, mask):
    """The documented layout: K and V pools per kind, decode scratch, counters, error word."""
    a = lambda x: (x + 255) // 256 * 256
    nr = sum(mask)
    ns = len(mask) - nr
    D, B, W, G = L.head_dim, L.batch, L.sink + L.recent, L.num_q_heads // L.num_kv_heads
    H = L.num_kv_heads
    max_retr = max(sum(mask[l * H:(l + 1) * H]) for l in range(L.num_layers))
    items = B * max_retr * 256  # partials: retrieval heads only, per layer
    return (2 * a(nr * B * L.max_len * D * 2) + 2 * a(ns * B * W * D * 2) + a(items * G * D * 4)
            + a(items * G * 4) + a(B * L.num_kv_heads * 4) + a(4))


@pytest.mark.parametrize("mask", [[1, 0, 0, 1, 0, 0, 0, 1], [0] * 8, [1] * 8])
def test_required_bytes(mask):
    L = _layout()
    st, req, handle = duo.duo_cache_alloc(L, mask)
    assert st == duo.DUO_OK and handle is None
    assert req == _expected_bytes(L, mask)


def test_memory_reduction_shape():
    """Streaming heads hold sink + recent slots instead of max_len: the cache of a
    25 %-retrieval MHA layer at 32K context is about a quarter of the full one."""
    L = _layout(num_layers=1, batch=1, num_q_heads=32, num_kv_heads=32, sink=64, recent=256, max_len=32768)
    _, full, _ = duo.duo_cache_alloc(L, [1] * 32)
    _, mixed, _ = duo.duo_cache_alloc(L, [1] * 8 + [0] * 24)
    pools_full = 2 * 32 * 32768 * 128 * 2
    pools_mixed = 2 * (8 * 32768 + 24 * 320) * 128 * 2
    scratch = lambda n_retr: n_retr * 256 * 128 * 4 + n_retr * 256 * 4  # split-KV partials of retrieval heads
    assert full - mixed == pools_full - pools_mixed + scratch(32) - scratch(8)


@pytest.mark.parametrize("bad", [
    dict(num_layers=0), dict(batch=0), dict(num_kv_heads=0), dict(num_q_heads=6), dict(num_q_heads=12),
    dict(num_q_heads=12, num_kv_heads=4), dict(head_dim=96), dict(head_dim=256), dict(sink=-1),
    dict(recent=0), dict(max_len=0), dict(num_kv_heads=129, num_q_heads=129),
    dict(num_q_heads=512, num_kv_heads=128)])
def test_bad_layouts_rejected(bad):
    L = _layout(**bad)
    n = L.num_layers * max(L.num_kv_heads, 1)
    st, _, _ = duo.duo_cache_alloc(L, [0] * n)
    assert st == duo.DUO_ERR_INVALID_ARG, bad


def test_bad_mask_and_scale_rejected():
    L = _layout()
    assert duo.duo_cache_alloc(L, [2] + [0] * 7)[0] == duo.DUO_ERR_INVALID_ARG
    L2 = _layout()
    L2.softmax_scale = -1.0
    assert duo.duo_cache_alloc(L2, [0] * 8)[0] == duo.DUO_ERR_INVALID_ARG
    L3 = _layout()
    L3.softmax_scale = float("nan")
    assert duo.duo_cache_alloc(L3, [0] * 8)[0] == duo.DUO_ERR_INVALID_ARG
    st = duo._lib.duo_cache_alloc(ctypes.byref(L), None, None, 0, None, None, None)
    assert st == duo.DUO_ERR_INVALID_ARG


def test_buffer_checks_before_device_work():
    L = _layout()
    mask = [1, 0] * 4
    _, req, _ = duo.duo_cache_alloc(L, mask)
    assert duo.duo_cache_alloc(L, mask, dev_buf=0x1000, buf_bytes=req - 1, stream=0)[0] == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_alloc(L, mask, dev_buf=0x1010, buf_bytes=req, stream=0)[0] == duo.DUO_ERR_ALIGNMENT
    st = duo._lib.duo_cache_alloc(ctypes.byref(L), ctypes.cast(duo._mask_buf(mask), ctypes.c_void_p), 0x1000, req,
                                  None, None, None)
    assert st == duo.DUO_ERR_INVALID_ARG  # no out pointer


def test_null_cache_rejected():
    assert duo.duo_cache_len(None, 0)[0] == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_set_len(None, 0, 1) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_views(None, 0, 0)[0] == duo.DUO_ERR_INVALID_ARG
    assert duo._lib.duo_cache_append(None, 0, None, None, 1, None) == duo.DUO_ERR_INVALID_ARG
    assert duo._lib.duo_prefill(None, 0, None, None, None, None, 1, None) == duo.DUO_ERR_INVALID_ARG
    assert duo._lib.duo_decode(None, 0, None, None, None, None, None) == duo.DUO_ERR_INVALID_ARG
    assert duo.duo_cache_free(None) == duo.DUO_OK


def test_status_strings():
    for s in range(8):
        assert duo.duo_status_str(s) and duo.duo_status_str(s) != "unknown status"
    assert duo.duo_status_str(99) == "unknown status"


def test_e4m3_cache_sizes():
    """E4M3 retrieval pools take one byte per element instead of two; the cache
    gains a region of 4 fp32 scales per (layer, KV head)."""
    mask = [1, 0, 1, 0, 1, 1, 0, 0]
    _, b16, _ = duo.duo_cache_alloc(duo.make_layout(2, 1, 8, 4, 128, 64, 256, 4096), mask)
    _, b8, _ = duo.duo_cache_alloc(duo.make_layout(2, 1, 8, 4, 128, 64, 256, 4096, kv_format=duo.DUO_KV_E4M3), mask)
    assert b16 - b8 == 2 * 4 * 4096 * 128 - 256
    st, _, _ = duo.duo_cache_alloc(duo.make_layout(2, 1, 8, 4, 128, 64, 256, 4096, kv_format=2), mask)
    assert st == duo.DUO_ERR_INVALID_ARG
