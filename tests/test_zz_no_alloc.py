"""The allocation-free calibration call (fp8_kv_calib_window_noalloc).

It exists for callers that cannot allocate device memory while the window
runs; its scratch is a fixed array inside the library.  Its pools and frozen
scales must equal, exactly, those of the CPU oracle fed the same batches and
those of the calibrator entry points with caller-provided staging
(fp8_kv_calib_create + observe_write), on consecutive calls that reuse the
array.  This file is collected last.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_group_b200 as fp8q
import workloads
from gpu_util import dev, dev_bf16, first_mismatch, host
from oracle import calibration as cal

pytestmark = pytest.mark.gpu


def _rows(bits, heads, dim):
    t, stride = bits.shape
    return dev_bf16(bits).as_strided((t, heads, dim), (stride, dim, 1))


def _pools(spec):
    n = spec.num_blocks * spec.cache_stride
    shape = (spec.num_blocks, spec.block_size, spec.heads, spec.dim)
    kp = torch.full((n,), workloads.SENTINEL, dtype=torch.uint8, device="cuda")
    vp = torch.full((n,), workloads.SENTINEL, dtype=torch.uint8, device="cuda")
    return kp, vp, kp.view(shape), vp.view(shape)


def _with_calibrator(spec, batches, window, headroom):
    kp, vp, kp4, vp4 = _pools(spec)
    cal = fp8q.KvCalibration(window, headroom, spec.heads, spec.dim, "cuda")
    for b in batches:
        cal.observe_write(_rows(b.k, spec.heads, spec.dim), _rows(b.v, spec.heads, spec.dim),
                          dev(b.slot_mapping), kp4, vp4)
    scales = cal.read_state()[2:]
    cal.close()
    return host(kp), host(vp), np.array(scales, np.float32)


def _with_oracle(spec, batches, window, headroom):
    c = cal.Fp8KvCalibration(0, window, headroom)
    kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
    cal.run_calibrated_writes(c, [cal.KvBatch(b.k, b.v, b.slot_mapping, b.key_stride,
                                              b.value_stride) for b in batches],
                              spec.heads, spec.dim, kp, vp, spec.block_size, spec.cache_stride,
                              spec.num_blocks)
    return kp, vp, np.array(c.scales(), np.float32)


def _without_allocation(spec, batches, window, headroom, launches=None):
    kp, vp, kp4, vp4 = _pools(spec)
    k = np.concatenate([b.k for b in batches])
    v = np.concatenate([b.v for b in batches])
    slots = np.concatenate([b.slot_mapping for b in batches])
    out = torch.full((2,), -1.0, dtype=torch.float32, device="cuda")
    k4, v4, s4 = _rows(k, spec.heads, spec.dim), _rows(v, spec.heads, spec.dim), dev(slots)
    before = fp8q.launch_count()
    fp8q.fp8_kv_calib_window_noalloc(k4, v4, s4, [b.num_tokens for b in batches], window,
                                     headroom, kp4, vp4, scales_out=out)
    if launches is not None:
        launches.append(fp8q.launch_count() - before)
    return host(kp), host(vp), host(out)


def _assert_same(a, b):
    assert np.array_equal(a[0].reshape(-1), b[0].reshape(-1)), \
        "K pools differ: " + first_mismatch(a[0], b[0])
    assert np.array_equal(a[1].reshape(-1), b[1].reshape(-1)), \
        "V pools differ: " + first_mismatch(a[1], b[1])
    assert np.array_equal(a[2].view(np.uint32), b[2].view(np.uint32)), (a[2], b[2])


def test_two_calls_in_a_row_match_the_oracle_and_the_calibrator():
    spec, batches, _ = workloads.calib_window()
    oracle_result = _with_oracle(spec, batches, workloads.CALIB_WINDOW, 1.0)
    want = _with_calibrator(spec, batches, workloads.CALIB_WINDOW, 1.0)
    _assert_same(want, oracle_result)
    for _ in range(2):
        got = _without_allocation(spec, batches, workloads.CALIB_WINDOW, 1.0)
        _assert_same(got, oracle_result)
        _assert_same(got, want)
    assert fp8q.fp8q_device_error(clear=True) == 0


def test_consecutive_calls_with_different_windows():
    spec, batches, _ = workloads.calib_window(row_pad=40)
    for window, headroom in ((100, 1.25), (300, 1.0), (1, 2.0)):
        want = _with_calibrator(spec, batches, window, headroom)
        _assert_same(_without_allocation(spec, batches, window, headroom), want)


def test_window_not_reached_leaves_the_provisional_scale():
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32))
    want = _with_calibrator(spec, batches, 256, 1.0)
    got = _without_allocation(spec, batches, 256, 1.0)
    _assert_same(got, want)
    _assert_same(got, _with_oracle(spec, batches, 256, 1.0))
    assert got[2].tolist() == [2.0, 2.0]


def test_one_staged_batch_replays_in_one_launch_with_the_crossing_batch():
    # window 20 over batches of 13 and 32: one staged batch, replayed in the
    # launch that also writes the crossing batch; a third batch is frozen
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32))
    launches = []
    got = _without_allocation(spec, batches, 20, 1.0, launches)
    # state set-up, one in-window pass, the crossing absmax, the merged
    # replay, the frozen write
    assert launches == [5]
    _assert_same(got, _with_oracle(spec, batches, 20, 1.0))
    _assert_same(got, _with_calibrator(spec, batches, 20, 1.0))


def test_staged_rows_and_a_large_crossing_batch_replay_batch_by_batch():
    # 77 staged rows in three batches plus a 2000-token crossing batch is more
    # than one whole-window launch takes: each staged batch replays in its own
    # launch, the last one together with the crossing batch
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32, 2000), num_blocks=256)
    launches = []
    got = _without_allocation(spec, batches, 100, 1.0, launches)
    # state set-up, three in-window passes, the crossing absmax, three replays
    assert launches == [8]
    _assert_same(got, _with_oracle(spec, batches, 100, 1.0))
    _assert_same(got, _with_calibrator(spec, batches, 100, 1.0))


def test_window_beyond_the_fixed_scratch_is_rejected():
    spec = workloads.large_kv_spec()
    full = workloads.large_kv_layer(0)
    kp, vp, kp4, vp4 = _pools(spec)
    with pytest.raises(fp8q.Fp8qError) as ei:
        fp8q.fp8_kv_calib_window_noalloc(
            _rows(full.k, 4, 128), _rows(full.v, 4, 128), dev(full.slot_mapping),
            list(workloads.LARGE_CHUNKS), workloads.LARGE_WINDOW_REQUEST, 1.0, kp4, vp4)
    assert ei.value.status == -5
    assert np.all(host(kp) == workloads.SENTINEL) and np.all(host(vp) == workloads.SENTINEL)
