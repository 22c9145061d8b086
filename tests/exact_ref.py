"""Independent exact arithmetic used to pin the oracle.

Nothing here is shared with the oracle or the CUDA path: rationals are Python
``Fraction``s, the rounding to binary32 is written out from the IEEE 754
definition (nearest, ties to even, subnormals, overflow to infinity), and the
rounding of a binary32 to E4M3 is delegated to torch's ``float8_e4m3fn`` cast
(a library routine) inside its non-saturating range; past 464 the
saturating-finite rule of the quantizer sends every magnitude to 448.
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np
import torch

F32_MIN_EXP = -126          # smallest normal exponent
F32_MANT = 23               # stored mantissa bits
E4M3_SAT = 0x7E


def fraction_of_f32(x) -> Fraction:
    return Fraction(float(np.float32(x)))


def round_to_f32(q: Fraction, negative_zero: bool = False) -> np.float32:
    """Round an exact rational to binary32, nearest-even."""
    if q == 0:
        return np.float32(-0.0) if negative_zero else np.float32(0.0)
    sign = -1 if q < 0 else 1
    a = abs(q)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    e_eff = max(e, F32_MIN_EXP)
    ulp = Fraction(2) ** (e_eff - F32_MANT)
    n = a / ulp
    whole = n.numerator // n.denominator
    rest = n - whole
    if rest > Fraction(1, 2) or (rest == Fraction(1, 2) and whole % 2 == 1):
        whole += 1
    v = whole * ulp
    if v >= Fraction(2) ** 128:
        return np.float32(sign * np.inf)
    return np.float32(sign * float(v))


def e4m3_of_f32(y: np.ndarray) -> np.ndarray:
    """E4M3 code of binary32 values: torch's nearest-even cast below the
    saturation region, +-0x7E at and beyond 464."""
    y = np.asarray(y, dtype=np.float32)
    mag = np.abs(y)
    t = torch.from_numpy(np.where(mag > 464.0, np.float32(0.0), y).astype(np.float32))
    codes = t.to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()
    sat = mag > 464.0
    codes[sat] = E4M3_SAT | np.where(np.signbit(y[sat]), 0x80, 0).astype(np.uint8)
    return codes


def e4m3_value(code: np.ndarray) -> np.ndarray:
    """Decode E4M3 codes with torch (fp32 result)."""
    c = torch.from_numpy(np.asarray(code, dtype=np.uint8).copy())
    return c.view(torch.float8_e4m3fn).to(torch.float32).numpy()


ONE_E_MINUS_12_F32 = round_to_f32(Fraction(1, 10 ** 12))


def group_ref(xs_f32: np.ndarray):
    """Exact reference of one 128-group: (scale, codes)."""
    vals = [Fraction(float(v)) for v in xs_f32]
    amax = max(abs(v) for v in vals)
    floor = max(amax, Fraction(float(ONE_E_MINUS_12_F32)))
    s = round_to_f32(floor / 448)
    quot = [round_to_f32(v / Fraction(float(s)), negative_zero=bool(np.signbit(x)))
            for v, x in zip(vals, xs_f32)]
    return s, e4m3_of_f32(np.array(quot, dtype=np.float32))


def tensor_codes_ref(xs_f32: np.ndarray, scale) -> np.ndarray:
    """Exact E4M3(fp32(x / scale)) of each element (per-tensor scale)."""
    s = Fraction(float(np.float32(scale)))
    quot = [round_to_f32(Fraction(float(v)) / s, negative_zero=bool(np.signbit(v)))
            for v in xs_f32]
    return e4m3_of_f32(np.array(quot, dtype=np.float32))


def quotient_f32(x_f32: np.ndarray, scale) -> np.ndarray:
    """fp32(x / scale), correctly rounded, vectorised.

    The quotient is first formed in binary64 (one rounding).  Rounding that
    binary64 value to binary32 gives the correctly rounded binary32 quotient
    unless it sits exactly on a binary32 rounding midpoint (any binary32
    midpoint is a binary64 number, so the exact quotient cannot lie across one
    from its binary64 rounding); those elements are redone with rationals."""
    x = np.asarray(x_f32, dtype=np.float32)
    s32 = np.float32(scale)
    q64 = x.astype(np.float64) / np.float64(s32)
    r32 = q64.astype(np.float32)
    up = np.nextafter(r32, np.float32(np.inf))
    dn = np.nextafter(r32, np.float32(-np.inf))
    mid_up = (r32.astype(np.float64) + up.astype(np.float64)) / 2
    mid_dn = (r32.astype(np.float64) + dn.astype(np.float64)) / 2
    amb = (q64 == mid_up) | (q64 == mid_dn)
    out = r32.copy()
    for i in np.flatnonzero(amb.reshape(-1)):
        xv = x.reshape(-1)[i]
        out.reshape(-1)[i] = round_to_f32(Fraction(float(xv)) / Fraction(float(s32)),
                                          negative_zero=bool(np.signbit(xv)))
    return out


def tensor_codes_fast(x_f32: np.ndarray, scale) -> np.ndarray:
    """Vectorised E4M3(fp32(x / scale)) for a per-tensor scale."""
    return e4m3_of_f32(quotient_f32(x_f32, scale))
