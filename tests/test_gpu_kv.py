"""GPU parity of fp8_kv_write and fp8_kv_amax_observe against the CPU oracle:
whole pools (sentinel bytes included) must be byte-identical; maxima must
match bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_group_b200 as fp8q
import workloads
from gpu_util import dev, dev_bf16, first_mismatch, host

pytestmark = pytest.mark.gpu


def _dev_rows(bits: np.ndarray, heads: int, dim: int) -> torch.Tensor:
    """[T, stride] bf16 bits -> device [T, heads, dim] view with that row stride."""
    t, stride = bits.shape
    base = dev_bf16(bits)
    return base.as_strided((t, heads, dim), (stride, dim, 1))


def _pools(spec, cache_stride=None):
    cs = spec.cache_stride if cache_stride is None else cache_stride
    flat = np.full(spec.num_blocks * cs, workloads.SENTINEL, np.uint8)
    return flat


def _dev_pool(flat: np.ndarray, spec, cache_stride=None):
    cs = spec.cache_stride if cache_stride is None else cache_stride
    t = dev(flat)
    return t.as_strided((spec.num_blocks, spec.block_size, spec.heads, spec.dim),
                        (cs, spec.elems, spec.dim, 1))


def _gpu_write(spec, b, ks, vs, cache_stride=None, scale_dev=None, pools=None):
    kp_h, vp_h = pools if pools is not None else (_pools(spec, cache_stride), _pools(spec, cache_stride))
    kp, vp = _dev_pool(kp_h, spec, cache_stride), _dev_pool(vp_h, spec, cache_stride)
    fp8q.fp8_kv_write(_dev_rows(b.k, spec.heads, spec.dim), _dev_rows(b.v, spec.heads, spec.dim),
                      dev(b.slot_mapping), kp, vp, ks, vs, scale_dev=scale_dev)
    n = spec.num_blocks * (spec.cache_stride if cache_stride is None else cache_stride)
    return host(kp.as_strided((n,), (1,))), host(vp.as_strided((n,), (1,)))


def _oracle_write(spec, b, ks, vs, cache_stride=None, pools=None):
    cs = spec.cache_stride if cache_stride is None else cache_stride
    kp, vp = (p.copy() for p in pools) if pools is not None else (_pools(spec, cs), _pools(spec, cs))
    oob = oracle.kv_write(b.k, b.v, b.key_stride, b.value_stride, b.slot_mapping, b.num_tokens,
                          spec.heads, spec.dim, kp, vp, spec.block_size, cs, spec.num_blocks, ks, vs)
    return kp, vp, oob


def _parity(spec, b, ks, vs, cache_stride=None, scale_dev=None):
    fp8q.fp8q_device_error(clear=True)
    gk, gv = _gpu_write(spec, b, ks, vs, cache_stride, scale_dev)
    ok, ov, oob = _oracle_write(spec, b, ks, vs, cache_stride)
    assert np.array_equal(gk, ok), first_mismatch(gk, ok)
    assert np.array_equal(gv, ov), first_mismatch(gv, ov)
    err = fp8q.fp8q_device_error(clear=True)
    assert bool(err & fp8q.DEVERR_SLOT_OUT_OF_RANGE) == (oob > 0)
    return err


def test_tiny_at_provisional_scale():
    spec, b = workloads.tiny_kv()
    assert _parity(spec, b, 2.0, 2.0) == 0


def test_strided_rows_and_distinct_scales():
    spec, b = workloads.tiny_kv(row_pad=24)
    _parity(spec, b, 600.0 / 448.0, 0.0123)


def test_large_layer_full_pool():
    spec = workloads.large_kv_spec()
    b = workloads.large_kv_layer(0)
    _parity(spec, b, np.float32(20.0) / np.float32(448.0), np.float32(2.0))


def test_batch_longer_than_two_tokens_per_warp_of_a_full_grid():
    # 20000 tokens: more than two per warp of the largest resident grid, so the
    # plain write's grid-stride loop runs after its two-token start
    spec = workloads.large_kv_spec()
    _parity(spec, workloads.large_kv_layer(11, tokens=20000), 0.05, 0.07)


def test_padded_cache_stride_and_wide_rows():
    spec = workloads.PoolSpec(24, 8, 8, 128)          # E = 1024: two chunk rounds per warp
    g = workloads.generator(600, 0, 0)
    t = 150
    k = workloads.to_bf16_bits(g.standard_normal((t, 1024 + 16)).astype(np.float32) * 3)
    v = workloads.to_bf16_bits(g.standard_normal((t, 1024 + 16)).astype(np.float32) * 3)
    slots = g.permutation(spec.num_slots)[:t].astype(np.int64)
    slots[::17] = -1
    b = workloads.KvBatchInput(k, v, slots, 1024 + 16, 1024 + 16)
    _parity(spec, b, 0.25, 0.75, cache_stride=spec.cache_stride + 64)


def test_narrow_rows():
    spec = workloads.PoolSpec(16, 4, 1, 64)           # E = 64: 8 of 32 lanes busy
    g = workloads.generator(601, 0, 0)
    t = 50
    k = workloads.to_bf16_bits(g.standard_normal((t, 64)).astype(np.float32))
    v = workloads.to_bf16_bits(g.standard_normal((t, 64)).astype(np.float32))
    slots = g.permutation(64)[:t].astype(np.int64)
    _parity(spec, workloads.KvBatchInput(k, v, slots, 64, 64), 0.01, 1.0 / 3.0)


def test_out_of_range_slots_are_skipped_and_flagged():
    spec, b = workloads.tiny_kv()
    slots = b.slot_mapping.copy()
    slots[0] = spec.num_slots
    slots[5] = 1 << 40
    b2 = workloads.KvBatchInput(b.k, b.v, slots, b.key_stride, b.value_stride)
    err = _parity(spec, b2, 2.0, 2.0)
    assert err & fp8q.DEVERR_SLOT_OUT_OF_RANGE


def test_every_bf16_value_at_many_scales():
    """All 65536 bf16 patterns (finite ones) at fast-path, boundary and
    slow-path scales, as one token each of 512 elements."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    finite = ((bits >> 7) & 0xFF) != 0xFF
    bits = bits[finite]
    bits = np.concatenate([bits, np.zeros((-bits.size) % 512, np.uint16)])
    t = bits.size // 512
    spec = workloads.PoolSpec(t, 1, 4, 128)
    g = workloads.generator(602, 0, 0)
    scales = [2.0, 600.0 / 448.0, 1.0 / 3.0, 1.0, 448.0, 2.0 ** -64, 2.0 ** 64,
              2.0 ** -64 * 1.5, 2.0 ** 63 * 1.99, 2.0 ** -70, 2.0 ** 70, 1e-30, 1e30,
              3.4e38, 1.2e-38, 1e-44]
    scales += list(np.exp(g.uniform(-40, 40, 16)))
    slots = np.arange(t, dtype=np.int64)
    rows = bits.reshape(t, 512)
    b = workloads.KvBatchInput(rows, rows[::-1].copy(), slots, 512, 512)
    for s in scales:
        s = float(np.float32(s))
        with np.errstate(over="ignore"):           # 2^120 * 7.3 overflows; the clip bounds it
            s2 = float(np.clip(np.float32(s) * np.float32(7.3), np.float32(1e-44),
                               np.float32(3e38)))
        _parity(spec, b, s, s2)


def test_device_scales_equal_host_scales():
    spec, b = workloads.tiny_kv()
    sd = torch.tensor([0.37, 5.5], dtype=torch.float32, device="cuda")
    gk, gv = _gpu_write(spec, b, 1.0, 1.0, scale_dev=sd)
    ok, ov, _ = _oracle_write(spec, b, np.float32(0.37), np.float32(5.5))
    assert np.array_equal(gk, ok) and np.array_equal(gv, ov)


def test_bad_device_scale_writes_nothing_and_flags():
    spec, b = workloads.tiny_kv()
    fp8q.fp8q_device_error(clear=True)
    sd = torch.tensor([float("nan"), -1.0], dtype=torch.float32, device="cuda")
    gk, gv = _gpu_write(spec, b, 1.0, 1.0, scale_dev=sd)
    assert np.all(gk == workloads.SENTINEL) and np.all(gv == workloads.SENTINEL)
    assert fp8q.fp8q_device_error(clear=True) & fp8q.DEVERR_BAD_SCALE


def test_zero_tokens_is_a_noop():
    spec, b = workloads.tiny_kv()
    empty = workloads.KvBatchInput(b.k[:0], b.v[:0], b.slot_mapping[:0], 512, 512)
    kp, vp = _pools(spec), _pools(spec)
    k = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    pk, pv = _dev_pool(kp, spec), _dev_pool(vp, spec)
    fp8q.fp8_kv_write(k, k, torch.empty(0, dtype=torch.int64, device="cuda"), pk, pv, 2.0, 2.0)
    assert np.all(host(pk) == workloads.SENTINEL)
    assert empty.num_tokens == 0


def test_later_call_wins_a_shared_slot():
    spec, b = workloads.tiny_kv()
    first = workloads.KvBatchInput(b.k, b.v, b.slot_mapping, 512, 512)
    second = workloads.KvBatchInput(b.v.copy(), b.k.copy(), b.slot_mapping, 512, 512)
    kp_h, vp_h = _pools(spec), _pools(spec)
    kp, vp = _dev_pool(kp_h, spec), _dev_pool(vp_h, spec)
    for bb, sc in ((first, 2.0), (second, 0.5)):
        fp8q.fp8_kv_write(_dev_rows(bb.k, 4, 128), _dev_rows(bb.v, 4, 128), dev(bb.slot_mapping),
                          kp, vp, sc, sc)
    ok, ov, _ = _oracle_write(spec, first, 2.0, 2.0)
    oracle.kv_write(second.k, second.v, 512, 512, second.slot_mapping, 16, 4, 128, ok, ov, 16,
                    spec.cache_stride, spec.num_blocks, 0.5, 0.5)
    assert np.array_equal(host(kp).reshape(-1), ok) and np.array_equal(host(vp).reshape(-1), ov)


@pytest.mark.parametrize("case", ["tiny", "strided", "large"])
def test_amax_matches_oracle_and_accumulates(case):
    if case == "large":
        b = workloads.large_kv_layer(1)
        heads, dim = 4, 128
    else:
        spec, b = workloads.tiny_kv(row_pad=24 if case == "strided" else 0)
        if case == "strided":
            b.k[:, 512:] = 0x7F00                      # huge values in the padding
        heads, dim = spec.heads, spec.dim
    e = heads * dim
    amax = torch.zeros(2, dtype=torch.float32, device="cuda")
    fp8q.fp8_kv_amax_observe(_dev_rows(b.k, heads, dim), _dev_rows(b.v, heads, dim), amax)
    got = host(amax)
    want = [oracle.absmax(b.k, b.num_tokens, e, b.key_stride),
            oracle.absmax(b.v, b.num_tokens, e, b.value_stride)]
    assert got.tolist() == [float(w) for w in want]
    # max-accumulation: a larger prior value survives, a smaller one is replaced
    amax2 = torch.tensor([1e30, 0.0], dtype=torch.float32, device="cuda")
    fp8q.fp8_kv_amax_observe(_dev_rows(b.k, heads, dim), _dev_rows(b.v, heads, dim), amax2)
    got2 = host(amax2)
    assert got2[0] == np.float32(1e30) and got2[1] == want[1]


def test_multi_layer_write_matches_the_oracle_per_layer():
    """fp8_kv_write_layers = fp8_kv_write applied to each layer: four layers
    with their own rows, slots (padding and an out-of-range slot in one), pools
    and scales (by value, and from the device for one layer)."""
    spec = workloads.large_kv_spec()
    layers = [workloads.large_kv_layer(l, tokens=700) for l in (2, 3, 4, 5)]
    layers[1].slot_mapping[::37] = -1
    layers[2].slot_mapping[5] = spec.num_slots + 3
    scales = [(0.05, 0.07), (2.0, 2.0), (600.0 / 448.0, 1e-30), (0.33, 0.44)]
    n = spec.num_blocks * spec.cache_stride
    kps = [torch.full((n,), workloads.SENTINEL, dtype=torch.uint8, device="cuda") for _ in layers]
    vps = [torch.full((n,), workloads.SENTINEL, dtype=torch.uint8, device="cuda") for _ in layers]
    shape = (spec.num_blocks, spec.block_size, spec.heads, spec.dim)
    sd = torch.tensor(scales[3], dtype=torch.float32, device="cuda")
    fp8q.fp8q_device_error(clear=True)
    fp8q.fp8_kv_write_layers(
        [_dev_rows(b.k, 4, 128) for b in layers], [_dev_rows(b.v, 4, 128) for b in layers],
        [dev(b.slot_mapping) for b in layers], [p.view(shape) for p in kps],
        [p.view(shape) for p in vps], k_scales=[s[0] for s in scales],
        v_scales=[s[1] for s in scales], scale_devs=[None, None, None, sd])
    err = fp8q.fp8q_device_error(clear=True)
    assert err & fp8q.DEVERR_SLOT_OUT_OF_RANGE
    for i, b in enumerate(layers):
        ok, ov, _ = _oracle_write(spec, b, np.float32(scales[i][0]), np.float32(scales[i][1]))
        assert np.array_equal(host(kps[i]), ok), f"layer {i} K: " + first_mismatch(host(kps[i]), ok)
        assert np.array_equal(host(vps[i]), ov), f"layer {i} V: " + first_mismatch(host(vps[i]), ov)


def test_multi_layer_write_zero_layers_and_tokens():
    spec, b = workloads.tiny_kv()
    fp8q.fp8_kv_write_layers([], [], [], [], [])
    k = torch.empty((0, 4, 128), dtype=torch.bfloat16, device="cuda")
    kp = _dev_pool(_pools(spec), spec)
    fp8q.fp8_kv_write_layers([k], [k], [torch.empty(0, dtype=torch.int64, device="cuda")], [kp],
                             [kp], k_scales=[1.0], v_scales=[1.0])
    assert np.all(host(kp) == workloads.SENTINEL)
