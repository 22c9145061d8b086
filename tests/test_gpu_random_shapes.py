"""Seeded random-shape parity: many small configurations of the quantizers and
the paged KV write drawn from one generator, each compared byte for byte with
the oracle (codes, scale bit patterns, whole pools with their sentinel bytes).

The draws cover what the fixed cases do not combine: head counts and head
dims (E from 8 to 2048, so 1 to 4 chunk rounds per warp), block sizes that are
and are not powers of two, padded row strides and block strides, padding and
out-of-range slots, tiny and large scales (the IEEE-division path beyond
[2^-64, 2^64] included), and activation widths and row counts with ragged
last warps, row-major and K-major.
"""
import numpy as np
import pytest

import oracle
import paged_kv_cache_group_b200 as fp8q
import workloads
from gpu_util import dev, dev_bf16, f32_bits, first_mismatch, host
from test_gpu_kv import _parity

pytestmark = pytest.mark.gpu

N_KV_CASES = 40
N_QUANT_CASES = 40


def _kv_case(i: int):
    g = workloads.generator(700, i, 0)
    heads = int(g.choice([1, 2, 4, 8]))
    dim = int(g.choice([8, 16, 64, 128, 256]))
    e = heads * dim
    block = int(g.choice([1, 3, 8, 16, 32]))
    num_blocks = int(g.integers(4, 64))
    spec = workloads.PoolSpec(num_blocks, block, heads, dim)
    t = int(g.integers(0, min(300, spec.num_slots) + 1))
    pad = int(g.choice([0, 8, 24]))
    scale_of = lambda: np.float32(np.exp(g.uniform(np.log(1e-3), np.log(20.0))))  # noqa: E731
    k = workloads.to_bf16_bits(g.standard_normal((t, e + pad)).astype(np.float32) *
                               np.float32(g.uniform(0.1, 30)))
    v = workloads.to_bf16_bits(g.standard_normal((t, e + pad)).astype(np.float32) *
                               np.float32(g.uniform(0.1, 30)))
    slots = g.permutation(spec.num_slots)[:t].astype(np.int64)
    if t:
        slots[g.random(t) < 0.05] = -1
    if t > 3 and i % 5 == 0:
        slots[2] = spec.num_slots + int(g.integers(0, 100))     # out of range: skipped, flagged
    ks, vs = scale_of(), scale_of()
    if i % 7 == 3:
        ks = np.float32(2.0 ** -70)                               # outside the reciprocal range
    if i % 11 == 5:
        vs = np.float32(2.0 ** 66)
    cache_pad = int(g.choice([0, 0, 8 * e]))
    b = workloads.KvBatchInput(k, v, slots, e + pad, e + pad)
    return spec, b, ks, vs, spec.cache_stride + cache_pad


@pytest.mark.parametrize("i", range(N_KV_CASES))
def test_random_kv_write(i):
    spec, b, ks, vs, cs = _kv_case(i)
    _parity(spec, b, ks, vs, cache_stride=cs)


def _quant_case(i: int):
    g = workloads.generator(701, i, 0)
    m = int(g.integers(0, 70))
    k = 128 * int(g.integers(1, 50))
    pad = int(g.choice([0, 8, 64]))
    x = g.standard_normal((m, k + pad)).astype(np.float32) * np.float32(g.uniform(1e-3, 100))
    if m and i % 4 == 0:
        x[g.integers(0, m), :128] = 0.0                           # a zero group: the floor scale
    return workloads.to_bf16_bits(x), m, k, k + pad


@pytest.mark.parametrize("i", range(N_QUANT_CASES))
def test_random_group_quant_both_layouts(i):
    bits, m, k, stride = _quant_case(i)
    x = dev_bf16(bits).reshape(m, stride)[:, :k] if m else dev_bf16(np.zeros((0, k), np.uint16))
    q_ref, s_ref = oracle.group_quant_strided(bits.reshape(-1), m, k, stride)
    q, s = fp8q.fp8_group_quant(x)
    gq, gs = host(q), host(s)
    assert np.array_equal(gq, q_ref), first_mismatch(gq, q_ref)
    assert np.array_equal(f32_bits(gs), f32_bits(s_ref)), first_mismatch(f32_bits(gs), f32_bits(s_ref))
    m_pad = fp8q.ceil16(m) + (8 if i % 3 == 0 else 0)
    qk, sk = fp8q.fp8_group_quant_kmajor(x, m_pad)
    qk_ref, sk_ref = oracle.group_quant_kmajor(bits.reshape(-1), m, k, stride, m_pad)
    gqk, gsk = host(qk), host(sk)
    assert np.array_equal(gqk, qk_ref), first_mismatch(gqk, qk_ref)
    assert np.array_equal(f32_bits(gsk), f32_bits(sk_ref)), first_mismatch(f32_bits(gsk),
                                                                           f32_bits(sk_ref))


N_CALIB_CASES = 24


def _calib_case(i: int):
    g = workloads.generator(702, i, 0)
    n = int(g.integers(2, 15))
    sizes = [int(g.integers(1, 65)) for _ in range(n)]
    nblk = [-(-t // 16) for t in sizes]
    recycle = {}
    for b in range(2, n + 1):
        if g.random() < 0.3:
            src = int(g.integers(1, b))
            recycle[b] = (src, int(g.integers(0, nblk[src - 1])))
    window = int(g.integers(1, sum(sizes) + 40))
    headroom = float(g.choice([0.5, 1.0, 1.0, 1.25, 2.0]))
    return tuple(sizes), recycle, window, headroom


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("i", range(N_CALIB_CASES))
def test_random_calibration_windows(i, fused):
    from test_gpu_calibration import _assert_frozen_state, _run_both
    sizes, recycle, window, headroom = _calib_case(i)
    spec, batches, _ = workloads.calib_window(batch_sizes=sizes, recycle=recycle)
    g, c, steps = _run_both(spec, batches, window, headroom, fused)
    if fp8q.STEP_FREEZE in steps:
        _assert_frozen_state(g, c)
    assert fp8q.fp8q_device_error(clear=True) == 0
