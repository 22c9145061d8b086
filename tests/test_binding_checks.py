"""Argument checks of the Python binding that need no GPU.

K and V shapes are compared before anything touches a device, so a V with
fewer rows, narrower rows or another head layout than K is refused on any
machine; the library is never called with rows the kernels would read past."""
import pytest
import torch

import paged_kv_cache_group_b200 as fp8q

K = torch.zeros((16, 4, 128), dtype=torch.bfloat16)
BAD_V = [torch.zeros((15, 4, 128), dtype=torch.bfloat16),    # fewer rows
         torch.zeros((16, 4, 64), dtype=torch.bfloat16),     # narrower rows
         torch.zeros((16, 8, 64), dtype=torch.bfloat16),     # same width, other heads
         torch.zeros((16, 512), dtype=torch.bfloat16)]       # not [T, heads, dim]
SLOTS = torch.zeros(16, dtype=torch.int64)
POOL = torch.zeros((4, 16, 4, 128), dtype=torch.uint8)


def _calibrator_without_device():
    # the checks run before the handle is used, so no device state is needed
    return object.__new__(fp8q.KvCalibration)


@pytest.mark.parametrize("v", BAD_V, ids=["rows", "width", "heads", "rank"])
def test_mismatched_v_is_refused_everywhere(v):
    with pytest.raises(ValueError):
        fp8q.fp8_kv_write(K, v, SLOTS, POOL, POOL)
    with pytest.raises(ValueError):
        fp8q.fp8_kv_amax_observe(K, v, torch.zeros(2))
    with pytest.raises(ValueError):
        fp8q.fp8_kv_write_layers([K], [v], [SLOTS], [POOL], [POOL])
    with pytest.raises(ValueError):
        _calibrator_without_device().observe(K, v, SLOTS)
    with pytest.raises(ValueError):
        _calibrator_without_device().observe_write(K, v, SLOTS, POOL, POOL)
    with pytest.raises(ValueError):
        fp8q.fp8_kv_calib_window_noalloc(K, v, SLOTS, [16], 8, 1.0, POOL, POOL)


def test_matching_host_tensors_are_refused_as_not_cuda():
    with pytest.raises(TypeError):
        fp8q.fp8_kv_write(K, K.clone(), SLOTS, POOL, POOL)
    with pytest.raises(TypeError):
        fp8q.fp8_kv_calib_window_noalloc(K, K.clone(), SLOTS, [16], 8, 1.0, POOL, POOL)
