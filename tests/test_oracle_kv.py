"""Pins of the oracle's reshape_and_cache_fp8 and absmax (no GPU).

Brute force on small pools: every pool entry is predicted independently from
its last writer with exact arithmetic (tests/exact_ref.py); entries nobody
wrote must keep the sentinel; padding slots (-1) write nothing; out-of-range
slots are skipped and counted.  absmax is checked against numpy.
"""
import numpy as np

import oracle
import workloads
from exact_ref import tensor_codes_fast, tensor_codes_ref


def _expected_pools(spec, writes, k_scale, v_scale):
    """writes: list of (k_bits_row, v_bits_row, slot) in write order."""
    kp = spec.new_pool().reshape(-1)
    vp = spec.new_pool().reshape(-1)
    last = {}
    for k_row, v_row, slot in writes:
        if 0 <= slot < spec.num_slots:
            last[slot] = (k_row, v_row)
    e = spec.elems
    for slot, (k_row, v_row) in last.items():
        blk, off = divmod(slot, spec.block_size)
        base = blk * spec.cache_stride + off * e
        kp[base:base + e] = tensor_codes_ref(oracle.bf16_to_f32(k_row), k_scale)
        vp[base:base + e] = tensor_codes_ref(oracle.bf16_to_f32(v_row), v_scale)
    return kp, vp


def _run(spec, batch, k_scale, v_scale, kp=None, vp=None):
    kp = spec.new_pool().reshape(-1) if kp is None else kp
    vp = spec.new_pool().reshape(-1) if vp is None else vp
    oob = oracle.kv_write(batch.k, batch.v, batch.key_stride, batch.value_stride,
                          batch.slot_mapping, batch.num_tokens, spec.heads, spec.dim,
                          kp, vp, spec.block_size, spec.cache_stride, spec.num_blocks,
                          k_scale, v_scale)
    return kp, vp, oob


def test_tiny_write_matches_bruteforce():
    spec, b = workloads.tiny_kv()
    assert (b.slot_mapping == -1).sum() == 2
    kp, vp, oob = _run(spec, b, 2.0, 2.0)
    e = spec.elems
    writes = [(b.k[t, :e], b.v[t, :e], int(b.slot_mapping[t])) for t in range(b.num_tokens)]
    ek, ev = _expected_pools(spec, writes, 2.0, 2.0)
    assert oob == 0
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)
    touched = np.zeros(spec.num_slots, bool)
    touched[b.slot_mapping[b.slot_mapping >= 0]] = True
    untouched = ~np.repeat(touched, e)
    assert np.all(kp[untouched] == workloads.SENTINEL)


def test_strided_source_rows():
    spec, b = workloads.tiny_kv(row_pad=24)
    assert b.key_stride == spec.elems + 24
    kp, vp, _ = _run(spec, b, 1.25, 0.75)
    e = spec.elems
    writes = [(b.k[t, :e], b.v[t, :e], int(b.slot_mapping[t])) for t in range(b.num_tokens)]
    ek, ev = _expected_pools(spec, writes, 1.25, 0.75)
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def test_duplicate_slot_in_one_call_later_token_wins():
    spec = workloads.PoolSpec(4, 4, 2, 16)
    g = workloads.generator(500, 0, 0)
    k = workloads.to_bf16_bits(g.standard_normal((6, 32)).astype(np.float32))
    v = workloads.to_bf16_bits(g.standard_normal((6, 32)).astype(np.float32))
    slots = np.array([3, 7, 3, -1, 15, 7], dtype=np.int64)
    b = workloads.KvBatchInput(k, v, slots, 32, 32)
    kp, vp, _ = _run(spec, b, 0.5, 0.25)
    writes = [(k[t], v[t], int(slots[t])) for t in range(6)]
    ek, ev = _expected_pools(spec, writes, 0.5, 0.25)
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def test_provisional_scale_examples():
    # at scale 2.0: 896 is exactly 448 -> 0x7E; 1000 saturates; -3 -> -1.5 -> 0xBC
    spec = workloads.PoolSpec(1, 1, 1, 8)
    vals = np.array([896.0, 1000.0, -3.0, 1.0, -0.0, 0.0, 2.0 ** -9, 0.5], np.float32)
    bits = workloads.bf16_bits_of(vals).reshape(1, 8)
    b = workloads.KvBatchInput(bits, bits, np.array([0], np.int64), 8, 8)
    kp, _, _ = _run(spec, b, 2.0, 2.0)
    assert list(kp) == [0x7E, 0x7E, 0xBC, 0x30, 0x80, 0x00, 0x00, 0x28]


def test_out_of_range_slots_are_skipped_and_counted():
    spec, b = workloads.tiny_kv()
    slots = b.slot_mapping.copy()
    slots[0] = spec.num_slots          # one past the end
    slots[1] = 10 ** 12
    b2 = workloads.KvBatchInput(b.k, b.v, slots, b.key_stride, b.value_stride)
    kp, vp, oob = _run(spec, b2, 2.0, 2.0)
    assert oob == 2
    e = spec.elems
    writes = [(b.k[t, :e], b.v[t, :e], int(slots[t])) for t in range(b.num_tokens)]
    ek, ev = _expected_pools(spec, writes, 2.0, 2.0)
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def test_padded_cache_stride_leaves_pad_untouched():
    base = workloads.PoolSpec(8, 4, 2, 16)
    pad = 40
    cache_stride = base.cache_stride + pad
    g = workloads.generator(501, 0, 0)
    k = workloads.to_bf16_bits(g.standard_normal((32, 32)).astype(np.float32))
    slots = g.permutation(32).astype(np.int64)
    kp = np.full(base.num_blocks * cache_stride, 0x5A, np.uint8)
    vp = kp.copy()
    oracle.kv_write(k, k, 32, 32, slots, 32, 2, 16, kp, vp, 4, cache_stride, 8, 1.0, 1.0)
    pads = kp.reshape(8, cache_stride)[:, base.cache_stride:]
    assert np.all(pads == 0x5A)
    for t in range(32):
        blk, off = divmod(int(slots[t]), 4)
        got = kp[blk * cache_stride + off * 32: blk * cache_stride + off * 32 + 32]
        assert np.array_equal(got, tensor_codes_ref(oracle.bf16_to_f32(k[t]), 1.0))


def test_large_layer_sample_matches_exact_codes():
    b = workloads.large_kv_layer(0, tokens=300)
    spec = workloads.large_kv_spec()
    kp, vp, _ = _run(spec, b, 20.0 / 448.0, 0.03125)
    e = spec.elems
    for t in (0, 17, 150, 299):
        blk, off = divmod(int(b.slot_mapping[t]), spec.block_size)
        base = blk * spec.cache_stride + off * e
        assert np.array_equal(kp[base:base + e],
                              tensor_codes_fast(oracle.bf16_to_f32(b.k[t]), np.float32(20.0 / 448.0)))
        assert np.array_equal(vp[base:base + e],
                              tensor_codes_fast(oracle.bf16_to_f32(b.v[t]), 0.03125))


def test_absmax_matches_numpy_and_ignores_row_padding():
    spec, b = workloads.tiny_kv(row_pad=16)
    big = b.k.copy()
    big[:, spec.elems:] = 0x7F00          # 1.7e38 in the padding only
    got = oracle.absmax(big, b.num_tokens, spec.elems, b.key_stride)
    want = np.abs(oracle.bf16_to_f32(b.k[:, :spec.elems])).max()
    assert got == want
    assert oracle.absmax(big, 0, spec.elems, b.key_stride) == 0.0
