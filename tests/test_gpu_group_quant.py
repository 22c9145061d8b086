"""GPU parity of fp8_group_quant against the CPU oracle: codes and scale bit
patterns must be identical, element by element."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_group_b200 as fp8q
import workloads
from gpu_util import dev_bf16, f32_bits, first_mismatch, host

pytestmark = pytest.mark.gpu


def _gpu_quant(bits: np.ndarray, row_stride: int | None = None, k: int | None = None):
    x = dev_bf16(bits)
    if row_stride is not None:
        x = x.reshape(bits.shape[0], row_stride)[:, :k]
    q, s = fp8q.fp8_group_quant(x)
    return host(q), host(s)


def _assert_parity(bits, row_stride=None, k=None):
    if row_stride is None:
        q_ref, s_ref = oracle.group_quant(bits)
    else:
        q_ref, s_ref = oracle.group_quant_strided(bits, bits.shape[0], k, row_stride)
    q, s = _gpu_quant(bits, row_stride, k)
    assert np.array_equal(q, q_ref), first_mismatch(q, q_ref)
    assert np.array_equal(f32_bits(s), f32_bits(s_ref)), first_mismatch(f32_bits(s), f32_bits(s_ref))


def test_tiny():
    _assert_parity(workloads.tiny_quant())


def test_prefill_full_size():
    # the 4593 x 5120 workload, all 23.5 M codes and 183,720 scales
    _assert_parity(workloads.prefill_quant())


@pytest.mark.parametrize("m", workloads.DECODE_MS)
@pytest.mark.parametrize("k", workloads.DECODE_KS)
def test_decode_widths(m, k):
    _assert_parity(workloads.decode_quant(m, k))


@pytest.mark.parametrize("m,k", [(1, 128), (3, 384), (37, 1152), (129, 640), (7, 128 * 41)])
def test_ragged_shapes(m, k):
    # odd group counts leave the last warp's eight groups partly empty
    _assert_parity(workloads.normal_activation(m, k, 90, m, k, std=3.0))


@pytest.mark.parametrize("pad", [8, 72, 1024])
def test_strided_rows(pad):
    m, k = 33, 640
    bits = workloads.normal_activation(m, k + pad, 91, pad, 0)
    _assert_parity(bits, row_stride=k + pad, k=k)


def test_more_rows_than_grid_y_limit():
    # M above 65535 (the reason M is never put on a 16-bit grid dimension)
    _assert_parity(workloads.normal_activation(70001, 128, 92, 0, 0))


def test_zero_rows_is_a_noop():
    x = torch.empty((0, 256), dtype=torch.bfloat16, device="cuda")
    q = torch.full((4,), 7, dtype=torch.uint8, device="cuda")
    s = torch.full((4,), 7.0, dtype=torch.float32, device="cuda")
    fp8q.fp8_group_quant(x, q, s)
    assert host(q).tolist() == [7] * 4 and host(s).tolist() == [7.0] * 4


def test_special_groups():
    # all-zero groups, signed zeros, the hand-worked amax-7 group, powers of two,
    # values spanning the whole bf16 range, subnormal bf16
    rows = []
    rows.append(np.zeros(256, np.float32))
    z = np.zeros(256, np.float32)
    z[3] = -0.0
    z[200] = -0.0
    rows.append(z)
    hw = np.zeros(256, np.float32)
    hw[:9] = [7, -7, 1, 0.5, 9 / 128, 17 / 64, 2.0 ** -16, 3 * 2.0 ** -16, -0.0]
    rows.append(hw)
    g = np.random.Generator(np.random.Philox(93))
    rows.append(np.ldexp(1.0, g.integers(-133, 127, 256)).astype(np.float32) *
                np.sign(g.standard_normal(256)).astype(np.float32))
    rows.append((g.standard_normal(256) * 1e-39).astype(np.float32))
    rows.append(np.full(256, 3.3895314e38, np.float32))
    bits = workloads.to_bf16_bits(np.stack(rows))
    _assert_parity(bits)


def _exhaustive_rows(a_lo: int, a_hi: int) -> np.ndarray:
    """Groups whose first element is the bf16 magnitude a (the group amax) and
    whose other 127 elements run through every bf16 pattern x with |x| <= a,
    both signs, for a in [a_lo, a_hi)."""
    groups = []
    for a in range(a_lo, a_hi):
        mags = np.arange(a + 1, dtype=np.uint16)
        xs = np.concatenate([mags, mags | np.uint16(0x8000)])
        n = -(-xs.size // 127)
        pad = np.zeros(n * 127 - xs.size, np.uint16)
        body = np.concatenate([xs, pad]).reshape(n, 127)
        head = np.full((n, 1), a, np.uint16)
        groups.append(np.concatenate([head, body], axis=1))
    return np.concatenate(groups)


def test_every_bf16_pair_of_value_and_group_max():
    """Exhaustive: for every finite positive bf16 group maximum a and every bf16
    x with |x| <= a, the GPU code equals the oracle's.  The code of an element
    depends only on (x, a), so this covers all inputs of the quantizer."""
    step = 2048
    total = 0
    for a_lo in range(0, 0x7F80, step):
        rows = _exhaustive_rows(a_lo, min(a_lo + step, 0x7F80))
        total += rows.size
        _assert_parity(rows.reshape(1, -1) if rows.shape[0] < 2 else rows.reshape(-1, 128))
    assert total > 1.0e9
