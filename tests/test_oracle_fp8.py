"""Pins of the oracle's FP8 E4M3 encoding (the format of the quantized
retrieval caches, a next step of the library): every code's value against
torch's float8_e4m3fn, round trips, ties to even at every midpoint, agreement
with torch's rounding on random in-range values, saturation, and the error
bound of quantize-then-dequantize."""
import math

import numpy as np
import torch

import oracle

FINITE = [c for c in range(256) if c not in (0x7F, 0xFF)]


def test_every_code_value_matches_torch_float8():
    codes = torch.arange(256, dtype=torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).tolist()
    for c in range(256):
        v = oracle.e4m3_value(c)
        if c in (0x7F, 0xFF):
            assert math.isnan(v) and math.isnan(ref[c])
        else:
            assert v == ref[c], (hex(c), v, ref[c])
    assert oracle.e4m3_value(0x7E) == 448.0 and oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x08) == 2.0 ** -6 and oracle.e4m3_value(0x38) == 1.0


def test_round_trip_of_every_finite_code():
    for c in FINITE:
        assert oracle.e4m3_code(oracle.e4m3_value(c)) == c, hex(c)


def test_midpoints_round_to_the_even_code():
    pos = sorted((oracle.e4m3_value(c), c) for c in FINITE if c < 0x80)
    for (v0, c0), (v1, c1) in zip(pos, pos[1:]):
        mid = (v0 + v1) / 2
        even = c0 if c0 % 2 == 0 else c1
        assert oracle.e4m3_code(mid) == even, (v0, v1)
        assert oracle.e4m3_code(-mid) == even | 0x80
        eps = (v1 - v0) / 1024
        assert oracle.e4m3_code(mid - eps) == c0 and oracle.e4m3_code(mid + eps) == c1


def test_random_values_match_torch_rounding():
    g = torch.Generator().manual_seed(0)
    x = (torch.rand(20000, generator=g, dtype=torch.float64) * 2 - 1) * 448.0
    x = torch.cat([x, x * 2.0 ** -8, x * 2.0 ** -14])  # normal and subnormal ranges
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).tolist()
    got = [oracle.e4m3_code(v) for v in x.tolist()]
    assert got == ref


def test_saturation_and_nan():
    for v in (448.5, 463.0, 464.0, 500.0, 1e30, math.inf):
        assert oracle.e4m3_code(v) == 0x7E and oracle.e4m3_code(-v) == 0xFE
    assert oracle.e4m3_code(math.nan) == 0x7F
    assert oracle.e4m3_code(0.0) == 0x00 and oracle.e4m3_code(-0.0) == 0x80
    assert oracle.e4m3_code(2.0 ** -11) == 0x00  # below half the smallest subnormal


def test_quantize_is_fp32_product_then_nearest_code():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(4096, generator=g) * 3).to(torch.bfloat16)
    for inv in (1.0, 0.37, 25.0):
        codes = oracle.e4m3_quantize(x, inv)
        prod = x.float().numpy() * np.float32(inv)  # fp32 product, independent of the oracle
        assert codes.tolist() == [oracle.e4m3_code(float(p)) for p in prod]
        back = np.array([oracle.e4m3_value(c) for c in codes]) / np.float64(np.float32(inv))
        xs = x.double().numpy()
        a = np.abs(prod.astype(np.float64))
        normal = (a >= 2.0 ** -6) & (a <= 448.0)
        # half a unit in the last place: 2^-4 relative for normals, 2^-10 absolute (scaled) below
        assert np.all(np.abs(back - xs)[normal] <= 2.0 ** -4 * np.abs(xs)[normal] * (1 + 1e-6))
        assert np.all(np.abs(back - xs)[a < 2.0 ** -6] <= 2.0 ** -10 / np.float32(inv) * (1 + 1e-6))


def _grid_rows(g, n, D, lo=-2.0, hi=2.0):
    """Random rows whose values are E4M3 codes in [lo, hi] (exact in bf16 too)."""
    codes = [c for c in FINITE if lo <= oracle.e4m3_value(c) <= hi]
    idx = torch.randint(0, len(codes), (n, D), generator=g)
    c = np.array(codes, dtype=np.uint8)[idx.numpy()]
    vals = np.vectorize(oracle.e4m3_value)(c)
    return c, torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16)


def test_fp8_rows_equal_bf16_rows_when_values_are_exact():
    g = torch.Generator().manual_seed(2)
    D, n = 64, 37
    kc, kb = _grid_rows(g, n, D)
    vc, vb = _grid_rows(g, n, D)
    q = torch.randn(D, generator=g).to(torch.bfloat16)
    for ks, vs in ((1.0, 1.0), (0.25, 8.0)):  # powers of two scale exactly
        got, wsum = oracle.attend_rows_e4m3(q, kc, vc, ks, vs, 0.125)
        ref, _ = oracle.attend_rows(q, (kb.double() * ks).to(torch.bfloat16), (vb.double() * vs).to(torch.bfloat16),
                                    0.125)
        assert np.array_equal(got, ref)
        assert abs(wsum - 1.0) < 1e-12


def test_fp8_rows_constant_value_rows_return_that_value():
    g = torch.Generator().manual_seed(3)
    D, n = 32, 50
    kc, _ = _grid_rows(g, n, D)
    vc = np.full((n, D), oracle.e4m3_code(0.75), dtype=np.uint8)
    q = torch.randn(D, generator=g).to(torch.bfloat16)
    got, _ = oracle.attend_rows_e4m3(q, kc, vc, 1.7, 3.0, 0.2)
    assert np.allclose(got, 0.75 * 3.0, rtol=0, atol=1e-12)
