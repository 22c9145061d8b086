"""Pins of the oracle's per-token 1x128-group quantizer (no GPU).

Checked against: the hand-worked group in tests/golden, exact rational
arithmetic (tests/exact_ref.py) on random groups of several shapes of value,
closed forms (scale 1 when amax is 448, the floor scale of an all-zero group),
the saturation boundary, the dequantization error bound, and the invariant
that each group's largest element encodes to +-448.
"""
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads
from exact_ref import (ONE_E_MINUS_12_F32, e4m3_of_f32, e4m3_value, group_ref,
                       round_to_f32)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _group_row(values):
    x = np.zeros(128, dtype=np.float32)
    x[:len(values)] = values
    return workloads.to_bf16_bits(x)


def test_handworked_group():
    rows, scale_bits = [], None
    with open(os.path.join(GOLDEN, "group_quant_handworked.txt")) as fh:
        for line in fh:
            line = line.split("#")[0].strip()
            if not line:
                continue
            parts = line.split()
            if parts[0] == "SCALE":
                scale_bits = int(parts[1], 16)
            else:
                rows.append((int(parts[0]), float.fromhex(parts[1]), int(parts[3], 16)))
    x = np.zeros(128, dtype=np.float32)
    want = np.zeros(128, dtype=np.uint8)
    for idx, val, code in rows:
        x[idx] = val
        want[idx] = code
    bits = workloads.bf16_bits_of(x)            # every value is bf16-exact
    q, s = oracle.group_quant(bits.reshape(1, 128))
    assert s.view(np.uint32)[0, 0] == scale_bits
    assert np.array_equal(q[0], want), [(i, hex(q[0, i]), hex(want[i])) for i in range(9)]


def test_amax_448_gives_unit_scale_and_plain_codes():
    g = np.random.Generator(np.random.Philox(7))
    x = (g.standard_normal(128) * 50).astype(np.float32)
    x[3] = 448.0
    bits = workloads.to_bf16_bits(np.clip(x, -448, 448))
    q, s = oracle.group_quant(bits.reshape(1, 128))
    assert s[0, 0] == np.float32(1.0)
    assert np.array_equal(q[0], e4m3_of_f32(oracle.bf16_to_f32(bits)))


def test_all_zero_group_uses_the_floor_scale():
    bits = np.zeros((2, 256), dtype=np.uint16)
    bits[1, 5] = 0x8000                          # a -0 in the second row
    q, s = oracle.group_quant(bits)
    floor_scale = round_to_f32(Fraction(float(ONE_E_MINUS_12_F32)) / 448)
    assert np.all(s.view(np.uint32) == np.float32(floor_scale).view(np.uint32))
    expect = np.zeros((2, 256), dtype=np.uint8)
    expect[1, 5] = 0x80
    assert np.array_equal(q, expect)


def _random_groups(n, g):
    kinds = []
    for i in range(n):
        kind = i % 6
        if kind == 0:
            x = g.standard_normal(128)
        elif kind == 1:
            x = g.standard_normal(128) * (g.random(128) < 0.05) * 30 + g.standard_normal(128)
        elif kind == 2:
            x = g.standard_normal(128) * 1e-6
        elif kind == 3:
            x = g.standard_normal(128) * 1e4
        elif kind == 4:
            x = np.ldexp(1.0, g.integers(-30, 10, 128)) * np.sign(g.standard_normal(128))
        else:
            x = g.standard_normal(128) * 1e-30     # deep in the floor region
        kinds.append(x.astype(np.float32))
    return workloads.to_bf16_bits(np.stack(kinds))


def test_random_groups_match_exact_arithmetic():
    g = np.random.Generator(np.random.Philox(11))
    bits = _random_groups(48, g)
    q, s = oracle.group_quant(bits.reshape(1, -1))
    xf = oracle.bf16_to_f32(bits)
    for i in range(bits.shape[0]):
        s_ref, q_ref = group_ref(xf[i])
        assert s[0, i].view(np.uint32) == np.float32(s_ref).view(np.uint32), i
        assert np.array_equal(q[0, i * 128:(i + 1) * 128], q_ref), i


def test_saturation_boundary_never_produces_nan():
    # bf16 amax values for which the fp32 quotient amax / fp32(amax/448) lands
    # above 448: the code must saturate to 0x7E, never the NaN code 0x7F.
    amax_bits = np.arange(0x0080, 0x7F80, dtype=np.uint16)      # positive normals
    amax = oracle.bf16_to_f32(amax_bits)
    keep = amax > np.float32(1e-12)                              # above the floor
    amax_bits, amax = amax_bits[keep], amax[keep]
    s = (amax / np.float32(448.0)).astype(np.float32)          # fp32 division
    over = (amax / s).astype(np.float32) > np.float32(448.0)
    assert over.any(), "no boundary case found: the pin would not bite"
    picks = amax_bits[over][:64]
    rows = np.zeros((len(picks), 128), dtype=np.uint16)
    rows[:, 0] = picks
    rows[:, 1] = picks | 0x8000
    q, _ = oracle.group_quant(rows.reshape(1, -1))
    q = q.reshape(len(picks), 128)
    assert np.all(q[:, 0] == 0x7E) and np.all(q[:, 1] == 0xFE)


def test_largest_element_of_every_group_encodes_to_448():
    bits = workloads.prefill_quant(64, 5120)
    q, s = oracle.group_quant(bits)
    xf = oracle.bf16_to_f32(bits).reshape(64, 40, 128)
    qg = q.reshape(64, 40, 128)
    idx = np.argmax(np.abs(xf), axis=2)
    top = np.take_along_axis(qg, idx[..., None], axis=2)[..., 0]
    nonzero = np.abs(xf).max(axis=2) > 0
    assert np.all((top[nonzero] & 0x7F) == 0x7E)
    assert np.all(top[~nonzero] == 0x00)


def test_dequantization_error_bound():
    bits = workloads.prefill_quant(32, 5120)
    q, s = oracle.group_quant(bits)
    x = oracle.bf16_to_f32(bits).astype(np.float64).reshape(32, 40, 128)
    sc = s.astype(np.float64)[..., None]
    deq = e4m3_value(q).astype(np.float64).reshape(32, 40, 128)
    unsat = (q.reshape(32, 40, 128) & 0x7F) != 0x7E
    mag = np.abs(deq)
    ulp = np.where(mag >= 2.0 ** -6, np.ldexp(1.0, np.floor(np.log2(np.maximum(mag, 2.0 ** -6))).astype(int) - 3),
                   2.0 ** -9)
    bound = (0.5 * ulp + np.abs(x / sc) * 2.0 ** -24) * sc
    err = np.abs(deq * sc - x)
    assert np.all(err[unsat] <= bound[unsat] * (1 + 1e-12))


def test_strided_rows_equal_packed_rows():
    bits = workloads.normal_activation(5, 384, 99, 0, 0)
    padded = np.full((5, 384 + 72), 0x7F7F, dtype=np.uint16)   # huge bf16 pad
    padded[:, :384] = bits
    q1, s1 = oracle.group_quant(bits)
    q2, s2 = oracle.group_quant_strided(padded, 5, 384, 384 + 72)
    assert np.array_equal(q1, q2) and np.array_equal(s1.view(np.uint32), s2.view(np.uint32))


def test_rejects_k_not_multiple_of_128():
    with pytest.raises(ValueError):
        oracle.group_quant(np.zeros((2, 200), dtype=np.uint16))


def test_empty_input():
    q, s = oracle.group_quant(np.zeros((0, 256), dtype=np.uint16))
    assert q.shape == (0, 256) and s.shape == (0, 2)
