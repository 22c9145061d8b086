"""Pins of the oracle's E4M3 encoder (no GPU).

The encoder is checked against (a) closed-form values of the format in
tests/golden/e4m3_values.txt, (b) torch's float8_e4m3fn cast, a library
routine, over a dense sweep of binary32 values, (c) the saturating-finite rule
beyond 448, and (d) nearest-even at every midpoint of the grid.
"""
import os

import numpy as np

import oracle
from exact_ref import e4m3_of_f32, e4m3_value

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_values():
    rows = []
    with open(os.path.join(GOLDEN, "e4m3_values.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if line:
                code, val = line.split()
                rows.append((int(code, 16), float.fromhex(val)))
    return rows


def test_closed_form_values_encode_to_their_codes():
    rows = _golden_values()
    assert len(rows) >= 10
    for code, val in rows:
        assert int(oracle.e4m3_encode([val])[0]) == code, (hex(code), val)


def test_closed_form_values_agree_with_torch_decode():
    # the golden table itself is checked against the library decoder
    for code, val in _golden_values():
        dec = float(e4m3_value([code])[0])
        assert dec == val and np.signbit(dec) == np.signbit(val), (hex(code), val, dec)


def test_every_finite_code_round_trips():
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], dtype=np.uint8)
    vals = e4m3_value(codes)
    assert np.array_equal(oracle.e4m3_encode(vals), codes)


def _sweep_values():
    """Binary32 values over exponents 2^-30 .. 2^9: every pattern of the top 11
    mantissa bits, with low bits 0, 1, 0x7FF, 0x800, 0x801, 0xFFF (around the
    E4M3 midpoints, which all have a zero tail), both signs."""
    exps = np.arange(127 - 30, 127 + 10, dtype=np.uint32)
    top = np.arange(1 << 11, dtype=np.uint32) << 12
    low = np.array([0, 1, 0x7FF, 0x800, 0x801, 0xFFF], dtype=np.uint32)
    bits = (exps[:, None, None] << 23) | top[None, :, None] | low[None, None, :]
    bits = bits.reshape(-1)
    bits = np.concatenate([bits, bits | np.uint32(0x80000000)])
    # binary32 subnormals and zeros as well
    sub = np.arange(0, 1 << 23, 4099, dtype=np.uint32)
    bits = np.concatenate([bits, sub, sub | np.uint32(0x80000000)])
    return bits.view(np.float32)


def test_matches_torch_cast_on_dense_sweep():
    y = _sweep_values()
    inside = np.abs(y) <= 464.0
    y = y[inside]
    got = oracle.e4m3_encode(y)
    want = e4m3_of_f32(y)
    bad = np.flatnonzero(got != want)
    assert bad.size == 0, [(float(y[i]), hex(got[i]), hex(want[i])) for i in bad[:5]]


def test_matches_torch_cast_on_random_values():
    g = np.random.Generator(np.random.Philox(1234))
    e = g.integers(-40, 10, size=1_000_000)
    m = g.random(1_000_000)
    y = (np.ldexp(1.0 + m, e) * np.where(g.random(1_000_000) < 0.5, -1, 1)).astype(np.float32)
    assert np.array_equal(oracle.e4m3_encode(y), e4m3_of_f32(y))


def test_saturates_to_448_beyond_the_grid():
    big = np.array([448.0, 450.0, 463.99, 464.0, 464.01, 480.0, 896.0, 1e6, 3.4e38],
                   dtype=np.float32)
    assert np.all(oracle.e4m3_encode(big) == 0x7E)
    assert np.all(oracle.e4m3_encode(-big) == 0xFE)


def test_midpoints_round_to_even_mantissa():
    pos = np.array([c for c in range(0x7F)], dtype=np.uint8)  # 0x00 .. 0x7E
    vals = e4m3_value(pos).astype(np.float64)
    for c in range(len(pos) - 1):
        lo, hi = vals[c], vals[c + 1]
        mid = np.float32((lo + hi) / 2)  # exact: at most 5 significant bits
        assert float(mid) == (lo + hi) / 2
        even = c if c % 2 == 0 else c + 1
        assert int(oracle.e4m3_encode([mid])[0]) == even, (c, float(mid))
        above = np.nextafter(mid, np.float32(np.inf))
        below = np.nextafter(mid, np.float32(-np.inf))
        assert int(oracle.e4m3_encode([above])[0]) == c + 1
        assert int(oracle.e4m3_encode([below])[0]) == c
        assert int(oracle.e4m3_encode([-mid])[0]) == (0x80 | even)


def test_signed_zero_and_tiny_values():
    assert int(oracle.e4m3_encode([0.0])[0]) == 0x00
    assert int(oracle.e4m3_encode([-0.0])[0]) == 0x80
    # below half the smallest subnormal: zero of the same sign
    assert int(oracle.e4m3_encode([2.0 ** -11])[0]) == 0x00
    assert int(oracle.e4m3_encode([-(2.0 ** -11)])[0]) == 0x80
    # exactly half the smallest subnormal ties to zero (even)
    assert int(oracle.e4m3_encode([2.0 ** -10])[0]) == 0x00
    assert int(oracle.e4m3_encode([3 * 2.0 ** -10])[0]) == 0x02
