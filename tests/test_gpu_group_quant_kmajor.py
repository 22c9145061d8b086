"""GPU parity of fp8_group_quant_kmajor against the oracle: codes of all
m_pad rows (phantom rows zero) and the K-major scale array [K/128, m_pad]
(pad columns zero) must be identical byte for byte.  Output buffers start
filled with NaN patterns, so a slot the kernel forgets to write shows up."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_group_b200 as fp8q
import workloads
from gpu_util import dev_bf16, f32_bits, first_mismatch, host

pytestmark = pytest.mark.gpu


def _assert_parity(bits, m, k, row_stride, m_pad):
    x = dev_bf16(bits).reshape(m, row_stride)[:, :k]
    q = torch.full((m_pad, k), 0x7F, dtype=torch.uint8, device="cuda")          # E4M3 NaN
    s = torch.full((k // 128, m_pad), float("nan"), dtype=torch.float32, device="cuda")
    fp8q.fp8_group_quant_kmajor(x, m_pad, q, s)
    q_ref, s_ref = oracle.group_quant_kmajor(bits, m, k, row_stride, m_pad)
    gq, gs = host(q), host(s)
    assert np.array_equal(gq, q_ref), first_mismatch(gq, q_ref)
    assert np.array_equal(f32_bits(gs), f32_bits(s_ref)), first_mismatch(f32_bits(gs),
                                                                          f32_bits(s_ref))


@pytest.mark.parametrize("m", workloads.DECODE_MS + (5, 11))
@pytest.mark.parametrize("k", workloads.DECODE_KS)
def test_decode_band_padded_to_16(m, k):
    _assert_parity(workloads.decode_quant(m, k), m, k, k, fp8q.ceil16(m))


@pytest.mark.parametrize("m,k,m_pad", [(1, 128, 16), (3, 384, 16), (17, 640, 32), (37, 1152, 48),
                                       (129, 640, 144), (7, 128 * 41, 9), (16, 256, 16),
                                       (20, 384, 61)])
def test_ragged_shapes_and_odd_pads(m, k, m_pad):
    # m_pad not a multiple of 8 leaves the last octet of rows partly outside
    _assert_parity(workloads.normal_activation(m, k, 92, m, k, std=3.0), m, k, k, m_pad)


@pytest.mark.parametrize("pad", [8, 72])
def test_strided_rows(pad):
    m, k = 13, 640
    bits = workloads.normal_activation(m, k + pad, 93, pad, 0)
    _assert_parity(bits, m, k, k + pad, 16)


def test_prefill_full_size():
    # 4593 x 5120 padded to 4608 rows: 23.6 M codes, 184,320 K-major scales
    bits = workloads.prefill_quant()
    m, k = bits.shape
    _assert_parity(bits, m, k, k, fp8q.ceil16(m))


def test_special_groups():
    # all-zero groups (floor scale), signed zeros, powers of two over the whole
    # bf16 range, subnormal bf16 and the largest finite bf16
    g = np.random.Generator(np.random.Philox(94))
    rows = [np.zeros(256, np.float32), -np.zeros(256, np.float32),
            np.ldexp(1.0, g.integers(-133, 127, 256)).astype(np.float32) *
            np.sign(g.standard_normal(256)).astype(np.float32),
            (g.standard_normal(256) * 1e-39).astype(np.float32),
            np.full(256, 3.3895314e38, np.float32)]
    bits = workloads.to_bf16_bits(np.stack(rows))
    _assert_parity(bits, 5, 256, 256, 16)


def test_only_phantom_rows():
    k, m_pad = 384, 16
    q = torch.full((m_pad, k), 0x7F, dtype=torch.uint8, device="cuda")
    s = torch.full((k // 128, m_pad), float("nan"), dtype=torch.float32, device="cuda")
    x = torch.empty((0, k), dtype=torch.bfloat16, device="cuda")
    fp8q.fp8_group_quant_kmajor(x, m_pad, q, s)
    assert not host(q).any() and not f32_bits(host(s)).any()


def test_rows_equal_the_row_major_quantizer():
    # the same codes as fp8_group_quant, and its scales transposed
    bits = workloads.decode_quant(16, 5120)
    x = dev_bf16(bits)
    q0, s0 = fp8q.fp8_group_quant(x)
    q1, s1 = fp8q.fp8_group_quant_kmajor(x)
    assert torch.equal(q0, q1) and torch.equal(s0.t().contiguous(), s1)


def test_rejects_m_pad_below_rows():
    x = dev_bf16(workloads.decode_quant(4, 5120))
    with pytest.raises(ValueError):
        fp8q.fp8_group_quant_kmajor(x, 3)
    st = fp8q.lib.fp8_group_quant_kmajor(x.data_ptr(), 5120, x.data_ptr(), x.data_ptr(), 4, 3,
                                         5120, None)
    assert st == -1
