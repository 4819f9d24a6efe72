"""Pins for oracle/formats.py against library conversions, exact arithmetic
and the format definitions (no GPU)."""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle.formats as F


def test_fraction_to_f32_matches_numpy_rounding():
    # numpy's float64 -> float32 cast is IEEE round-to-nearest-even.
    rng = np.random.default_rng(0)
    x = np.concatenate([
        rng.standard_normal(2000) * 10.0 ** rng.integers(-30, 30, 2000),
        rng.standard_normal(200) * 1e-42,            # fp32 subnormal range
        np.ldexp(1.0 + np.arange(1, 200) * 2.0 ** -24, 3),   # exact fp32 midpoints (ties)
        -np.ldexp(1.0 + np.arange(1, 200) * 2.0 ** -24, -5),
    ])
    for xi in x:
        assert F.fraction_to_f32(Fraction(float(xi))) == float(np.float32(xi)), xi


def test_fraction_to_f32_tie_and_sticky():
    one = Fraction(1)
    ulp = Fraction(1, 2 ** 23)
    # exactly halfway between 1 and 1+ulp -> even (1); a hair above -> up
    assert F.fraction_to_f32(one + ulp / 2) == 1.0
    assert F.fraction_to_f32(one + ulp / 2 + Fraction(1, 2 ** 80)) == float(1 + ulp)
    # halfway between 1+ulp and 1+2ulp -> even (1+2ulp)
    assert F.fraction_to_f32(one + ulp + ulp / 2) == float(1 + 2 * ulp)
    assert F.fraction_to_f32(Fraction(1, 3)) == float(np.float32(1 / 3))


def test_exact_mean_matches_fraction_brute_force():
    g = torch.Generator().manual_seed(1)
    x = (torch.randn(300, 5, generator=g) * 3 + 7).to(torch.bfloat16).double().numpy()
    x[7, 2] = float(torch.tensor(1e-30).to(torch.bfloat16))   # widely spread exponents
    x[8, 2] = float(torch.tensor(-3e4).to(torch.bfloat16))
    got = F.exact_mean_f32(x[None])[0]
    for c in range(5):
        s = sum((Fraction(float(v)) for v in x[:, c]), Fraction(0))
        assert got[c] == np.float32(F.fraction_to_f32(s / 300))


def test_exact_mean_is_order_independent_and_not_naive():
    # Values whose fp32 running sum loses the small terms; the exact mean keeps them.
    x = np.array([2.0 ** 24, 1.0, 1.0, 1.0, -(2.0 ** 24)])[:, None]
    assert F.exact_mean_f32(x[None])[0, 0] == np.float32(3.0 / 5.0)
    perm = x[[4, 1, 0, 3, 2]]
    assert F.exact_mean_f32(perm[None])[0, 0] == np.float32(3.0 / 5.0)


def test_bf16_round_matches_torch():
    g = torch.Generator().manual_seed(2)
    x = torch.randn(10000, generator=g) * 100
    ref = x.to(torch.bfloat16).double().numpy()     # torch: fp32 -> bf16, RN-even
    np.testing.assert_array_equal(F.bf16_round(x.double().numpy()), ref)


def test_e4m3_all_codes_round_trip_and_match_torch_decode():
    codes = np.arange(256, dtype=np.uint8)
    dec = F.e4m3_decode(codes)
    tdec = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(tdec)
    assert nan.sum() == 2 and np.isnan(dec[nan]).all()
    np.testing.assert_array_equal(dec[~nan], tdec[~nan])
    np.testing.assert_array_equal(F.e4m3_encode(dec[~nan]), codes[~nan])
    assert dec[~nan].max() == 448.0 and dec[0x7E] == 448.0
    assert dec[1] == 2.0 ** -9 and dec[8] == 2.0 ** -6


def test_e4m3_rounding_matches_torch_cast_in_range():
    g = torch.Generator().manual_seed(3)
    x = torch.cat([torch.randn(20000, generator=g) * s for s in (1e-3, 0.1, 1, 30, 120)])
    x = x.clamp(-448, 448).float()
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()     # RN-even cast
    got = F.e4m3_encode(x.double().numpy())
    np.testing.assert_array_equal(got, ref)


def test_e4m3_ties_saturation_and_sign():
    # ties between neighbours go to the even mantissa
    assert F.e4m3_round(1.0 + 1 / 16) == 1.0          # 1.0 (m=0) vs 1.125 (m=1)
    assert F.e4m3_round(1.125 + 1 / 16) == 1.25       # 1.125 (m=1) vs 1.25 (m=2)
    assert F.e4m3_round(2.0 ** -10) == 0.0            # half of the subnormal step -> 0
    assert F.e4m3_round(3 * 2.0 ** -10) == 2 * 2.0 ** -9
    assert F.e4m3_round(464.0) == 448.0               # above max -> satfinite
    assert F.e4m3_round(1e9) == 448.0 and F.e4m3_round(-1e9) == -448.0
    assert F.e4m3_encode(np.array([-0.0]))[0] == 0x80
    assert F.e4m3_encode(np.array([-1e-6]))[0] == 0x80
    assert F.e4m3_encode(np.array([448.0]))[0] == 0x7E


def test_e2m1_table_ties_and_saturation():
    codes = np.arange(16, dtype=np.uint8)
    dec = F.e2m1_decode(codes)
    np.testing.assert_array_equal(dec[:8], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(dec[8:], -dec[:8])
    np.testing.assert_array_equal(F.e2m1_encode(dec[1:]), codes[1:])
    # ties to even mantissa
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, 100.0, -0.25, -5.0])
    np.testing.assert_array_equal(F.e2m1_round(x), [0, 1, 1, 2, 2, 4, 4, 6, 6, -0.0, -4])
    # non-ties go to the nearest value
    x = np.array([0.26, 0.74, 1.3, 2.6, 4.9, 5.1])
    np.testing.assert_array_equal(F.e2m1_round(x), [0.5, 0.5, 1.5, 3, 4, 6])


def test_e2m1_nearest_by_brute_force():
    rng = np.random.default_rng(4)
    x = rng.uniform(-7, 7, 5000)
    grid = np.concatenate([-F.E2M1_GRID[::-1], F.E2M1_GRID])
    d = np.abs(x[:, None] - grid[None, :])
    nearest = grid[np.argmin(d, axis=1)]
    np.testing.assert_array_equal(np.abs(F.e2m1_round(x)), np.abs(nearest))


def test_pack_order():
    codes = np.array([[1, 2, 3, 4]], dtype=np.uint8)
    p = F.pack_e2m1(codes)
    np.testing.assert_array_equal(p, [[0x21, 0x43]])
    np.testing.assert_array_equal(F.unpack_e2m1(p), codes)


@pytest.mark.parametrize("sign", [1, -1])
def test_e4m3_monotone_over_all_fp32_bins(sign):
    # every code's value rounds to itself; midpoints between neighbours round to the even one
    vals = np.sort(F.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)))
    mids = (vals[:-1] + vals[1:]) / 2
    r = F.e4m3_round(sign * mids)
    lo, hi = sign * vals[:-1], sign * vals[1:]
    codes_lo = F.e4m3_encode(lo) & 1
    expect = np.where(codes_lo == 0, lo, hi)
    np.testing.assert_array_equal(r, expect)
