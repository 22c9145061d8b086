"""Pins of the oracle's K-major quantization for a padded FP8 GEMM
(decode_w8a8_quant_act, "spark_model/layers/ops/dispatch_proj_decode.rs"):
codes of the phantom rows zeroed up to m_pad, the 1x128 scales laid out
[K/128, m_pad] with the pad columns zero.

Each pin is independent of the oracle's own code: exact rational arithmetic
per group, and a block-scaled product that reads the scales token-contiguous
and must reproduce the bf16 activation within the E4M3 rounding bound (a
transposed or row-major scale array fails it, which the last test shows).
"""
import numpy as np
import pytest

import oracle
import workloads
from exact_ref import e4m3_value, group_ref


def _ulp_bound(deq, x, sc):
    mag = np.abs(deq)
    ulp = np.where(mag >= 2.0 ** -6,
                   np.ldexp(1.0, np.floor(np.log2(np.maximum(mag, 2.0 ** -6))).astype(int) - 3),
                   2.0 ** -9)
    return (0.5 * ulp + np.abs(x / sc) * 2.0 ** -24) * sc


def _dequant_with(scale_of, q, m, k):
    """Dequantize the live rows, taking row r, group g's scale from scale_of(g, r)."""
    kg = k // 128
    sc = np.array([[scale_of(g, r) for g in range(kg)] for r in range(m)], dtype=np.float64)
    deq = e4m3_value(q[:m]).astype(np.float64).reshape(m, kg, 128)
    return deq, sc[..., None]


def test_tiny_case_against_exact_groups():
    """3 live rows of 256 (strided source), m_pad 16: every live group equals
    the exact rational reference, every phantom byte and scale is zero."""
    m, k, stride, m_pad = 3, 256, 264, 16
    live = workloads.normal_activation(m, k, 7, 3, 256, std=3.0)
    buf = np.full((m, stride), 0x7FC0, dtype=np.uint16)      # NaN in the row padding
    buf[:, :k] = live
    q, skm = oracle.group_quant_kmajor(buf, m, k, stride, m_pad)
    assert q.shape == (m_pad, k) and skm.shape == (k // 128, m_pad)
    xf = oracle.bf16_to_f32(live)
    for r in range(m):
        for g in range(k // 128):
            s, codes = group_ref(xf[r, 128 * g:128 * (g + 1)])
            assert skm[g, r].view(np.uint32) == np.float32(s).view(np.uint32), (r, g)
            assert np.array_equal(q[r, 128 * g:128 * (g + 1)], codes), (r, g)
    assert not q[m:].any()
    assert not skm[:, m:].view(np.uint32).any()          # +0.0 exactly, no -0.0


@pytest.mark.parametrize("m", [5, 11, 16])
def test_block_scaled_product_reads_token_contiguous_scales(m):
    """Decode band (5..16 rows padded to 16), K = 5120: with the scale of
    (row r, group g) read at [g, r], dequantized codes reproduce x within half
    an E4M3 ulp; a 16-row product against a weight gives x @ w.T within the
    summed bound on live rows and exactly 0 on phantom rows."""
    k, m_pad = 5120, 16
    bits = workloads.normal_activation(m, k, 11, m)
    q, skm = oracle.group_quant_kmajor(bits, m, k, k, m_pad)
    x = oracle.bf16_to_f32(bits).astype(np.float64).reshape(m, k // 128, 128)
    deq, sc = _dequant_with(lambda g, r: skm[g, r], q, m, k)
    unsat = (q[:m].reshape(m, k // 128, 128) & 0x7F) != 0x7E
    bound = _ulp_bound(deq, x, sc)
    err = np.abs(deq * sc - x)
    assert np.all(err[unsat] <= bound[unsat] * (1 + 1e-12))

    w = workloads.generator(11, 99).standard_normal((8, k))
    full_scales = np.repeat(skm.T.astype(np.float64), 128, axis=1)     # [m_pad, k]
    full = e4m3_value(q).astype(np.float64) * full_scales
    out = full @ w.T
    ref = x.reshape(m, k) @ w.T
    tol = (np.maximum(bound, err).reshape(m, k)) @ np.abs(w).T
    assert np.all(np.abs(out[:m] - ref) <= tol * (1 + 1e-9))
    assert np.all(out[m:] == 0.0) and np.all(np.isfinite(out))


def test_row_major_scales_fail_the_token_contiguous_read():
    """The mistake the layout guards against: the quantizer's own [M, K/128]
    order handed over as if it were [K/128, m_pad] breaks the bound."""
    m, k, m_pad = 5, 5120, 16
    bits = workloads.normal_activation(m, k, 11, m)
    q, _ = oracle.group_quant_kmajor(bits, m, k, k, m_pad)
    _, s_row = oracle.group_quant(bits)
    wrong = np.zeros(k // 128 * m_pad, dtype=np.float32)
    wrong[:s_row.size] = s_row.reshape(-1)
    wrong = wrong.reshape(k // 128, m_pad)
    x = oracle.bf16_to_f32(bits).astype(np.float64).reshape(m, k // 128, 128)
    deq, sc = _dequant_with(lambda g, r: wrong[g, r], q, m, k)
    with np.errstate(divide="ignore", invalid="ignore"):
        bound = _ulp_bound(deq, x, np.where(sc == 0, 1.0, sc))
    assert np.any(np.abs(deq * sc - x) > bound)


def test_no_padding_is_a_plain_transpose():
    bits = workloads.prefill_quant(16, 1024)
    q, skm = oracle.group_quant_kmajor(bits, 16, 1024, 1024, 16)
    q0, s0 = oracle.group_quant(bits)
    assert np.array_equal(q, q0)
    assert np.array_equal(skm.view(np.uint32), s0.T.view(np.uint32))


def test_only_phantom_rows_and_degenerate_sizes():
    q, skm = oracle.group_quant_kmajor(np.zeros(0, dtype=np.uint16), 0, 384, 384, 16)
    assert q.shape == (16, 384) and not q.any()
    assert skm.shape == (3, 16) and not skm.view(np.uint32).any()
    q, skm = oracle.group_quant_kmajor(np.zeros(0, dtype=np.uint16), 0, 384, 384, 0)
    assert q.size == 0 and skm.shape == (3, 0)
    with pytest.raises(ValueError):
        oracle.group_quant_kmajor(workloads.decode_quant(2, 5120), 2, 5120, 5120, 1)
