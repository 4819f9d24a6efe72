"""Number formats used by the quantized-attention oracle.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` use it.

Everything here is written from the formats' definitions:

* fp32 / bf16 rounding: IEEE 754 round-to-nearest, ties to even.
* FP8 E4M3 ("e4m3fn", the OCP 8-bit float used for V and P in the
  INT8-QK / FP8-PV kernel, thu-ml/sageattention llms.txt,
  "sageattn_qk_int8_pv_fp8_cuda"): 1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits; no infinities; exponent 15 with mantissa 7 is NaN, so the
  largest finite magnitude is 1.75 * 2**8 = 448; subnormals step by 2**-9.
* FP4 E2M1 (the NVFP4 element format of "flashinfer.nvfp4_attention_sm120_fwd",
  16-element vectors with an FP8 scale each): 1 sign bit, 2 exponent bits
  with bias 1, 1 mantissa bit; magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}.

Encoders round to nearest with ties to the even code and saturate to the
largest finite magnitude (the "rn.satfinite" conversion).  The sign of a
value that rounds to zero is kept in the code (the code of -0.0 is 0x80 for
E4M3 and 0x8 for E2M1).
"""
from __future__ import annotations

import math
from fractions import Fraction

import numpy as np

E4M3_MAX = 448.0
E2M1_MAX = 6.0
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


# ---------------------------------------------------------------- fp32/bf16
def f32(x):
    """Round float64 values to the nearest fp32 value (ties to even)."""
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def bf16_round(x):
    """Round float64 values to the nearest bf16 value (8 significant bits),
    ties to even, returned as float64.  Values are assumed finite and within
    the bf16 normal range (true for attention outputs here)."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    _, ex = np.frexp(np.where(mag > 0, mag, 1.0))     # mag = m * 2**ex, m in [0.5, 1)
    quantum = np.ldexp(1.0, ex - 8)                    # 8 significant bits
    r = np.rint(x / quantum) * quantum                 # x/quantum is exact (power of 2)
    return np.where(mag > 0, r, x)


def fraction_to_f32(x: Fraction) -> float:
    """Correctly rounded fp32 value of an exact rational (ties to even).

    Returns a Python float holding an fp32-representable value.
    """
    if x == 0:
        return 0.0
    neg = x < 0
    x = -x if neg else x
    num, den = x.numerator, x.denominator
    # e = floor(log2(x)):  2**e <= x < 2**(e+1)
    e = num.bit_length() - den.bit_length()
    if (num << max(0, -e)) < (den << max(0, e)):
        e -= 1
    binade = max(e, -126)                  # below 2**-126 the quantum stays 2**-149
    qexp = binade - 23
    scaled = x / (Fraction(2) ** qexp)     # exact
    m = scaled.numerator // scaled.denominator
    rem = scaled - m
    half = Fraction(1, 2)
    if rem > half or (rem == half and m % 2 == 1):
        m += 1
    val = math.ldexp(m, qexp)              # m <= 2**24: exact in float64
    if val > float(np.finfo(np.float32).max):
        val = math.inf
    return -val if neg else val


def exact_column_sums(x2d):
    """Exact sums over axis 0 of a 2-D array of fp32-representable values.

    Returns a list of ``fractions.Fraction``, one per column.  Each value is
    split as M * 2**E with an integer M (|M| < 2**24); for every column the
    integers of equal E are added (exactly: the partial sums stay below
    2**53), and the per-exponent totals are combined in Python integers.
    """
    x2d = np.asarray(x2d, dtype=np.float64)
    R, C = x2d.shape
    m, e = np.frexp(x2d)                   # x = m * 2**e, |m| in [0.5, 1) or 0
    M = np.ldexp(m, 24)
    if not np.all(M == np.rint(M)):
        raise ValueError("exact_column_sums expects fp32-representable inputs")
    if R == 0:
        return [Fraction(0)] * C
    e = np.where(x2d == 0, e.max(initial=0), e)
    emin = int(e.min())
    span = int(e.max()) - emin + 1
    key = (np.arange(C)[None, :] * span + (e - emin)).ravel()
    sums = np.bincount(key, weights=M.ravel(), minlength=C * span).reshape(C, span)
    out = []
    for c in range(C):
        tot = 0
        for j in np.nonzero(sums[c])[0]:
            tot += int(sums[c, j]) << int(j)
        out.append(Fraction(tot) * (Fraction(2) ** (emin - 24)))
    return out


def exact_mean_f32(x, count=None):
    """Mean over axis -2 (tokens) of ``x[..., N, C]``, computed exactly and
    rounded once to fp32.  ``count`` (default N) is the divisor.

    This is the K channel mean of the ``smooth_k`` step: the plain meaning of
    "the mean of each K channel over tokens" with a single final rounding.
    """
    x = np.asarray(x, dtype=np.float64)
    lead = x.shape[:-2]
    N, C = x.shape[-2:]
    count = N if count is None else count
    flat = x.reshape((-1, N, C))
    res = np.zeros((flat.shape[0], C), dtype=np.float32)
    for i in range(flat.shape[0]):
        sums = exact_column_sums(flat[i])
        res[i] = [fraction_to_f32(s / count) for s in sums]
    return res.reshape(lead + (C,))


# ---------------------------------------------------------------- FP8 E4M3
def e4m3_round(x):
    """Nearest E4M3 value (ties to even), saturated to +-448, as float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    binade = np.maximum(ex - 1, -6)           # floor(log2 a); subnormals share 2**-6's quantum
    quantum = np.ldexp(1.0, binade - 3)       # 3 mantissa bits
    val = np.minimum(np.rint(a / quantum) * quantum, E4M3_MAX)
    return np.where(np.signbit(x), -val, val)


def e4m3_encode(x):
    """E4M3 codes (uint8) of float64 values: round to nearest even, satfinite."""
    r = e4m3_round(x)
    sign = np.signbit(r).astype(np.uint16)
    a = np.abs(r)
    sub = a < 2.0 ** -6
    m, ex = np.frexp(np.where(sub, 1.0, a))    # a = m * 2**ex, m in [0.5, 1)
    exp_bits = (ex - 1) + 7
    man_bits = np.rint(m * 16 - 8)            # (2m - 1) * 8
    normal = (exp_bits * 8 + man_bits).astype(np.uint16)
    subn = np.rint(a / 2.0 ** -9).astype(np.uint16)
    code = np.where(sub, subn, normal) | (sign << 7)
    return code.astype(np.uint8)


def e4m3_decode(code):
    """float64 values of E4M3 codes (NaN for the two NaN codes)."""
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    s = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = c & 0x7
    val = np.where(e == 0, np.ldexp(m.astype(np.float64), -9),
                   np.ldexp(1.0 + m / 8.0, e - 7))
    val = np.where((e == 15) & (m == 7), np.nan, val)
    return s * val


# ---------------------------------------------------------------- FP4 E2M1
def e2m1_round(x):
    """Nearest E2M1 value (ties to even), saturated to +-6, as float64."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))
    binade = np.maximum(ex - 1, 0)            # values below 1 share the quantum 0.5
    quantum = np.ldexp(1.0, binade - 1)       # 1 mantissa bit
    val = np.minimum(np.rint(a / quantum) * quantum, E2M1_MAX)
    return np.where(np.signbit(x), -val, val)


def e2m1_encode(x):
    """E2M1 codes (uint8 holding 0..15) of float64 values."""
    r = e2m1_round(x)
    a = np.abs(r)
    idx = np.searchsorted(E2M1_GRID, a)       # a is exactly a grid value
    return (idx | (np.signbit(r).astype(np.int64) << 3)).astype(np.uint8)


def e2m1_decode(code):
    c = np.asarray(code, dtype=np.uint8).astype(np.int64)
    val = E2M1_GRID[c & 7]
    return np.where(c & 8, -val, val)


def pack_e2m1(codes):
    """Pack E2M1 codes two per byte along the last axis: element 2i in the
    low nibble, element 2i+1 in the high nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def unpack_e2m1(packed):
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out
