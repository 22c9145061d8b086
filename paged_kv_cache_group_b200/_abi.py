"""ctypes declarations of the C ABI in include/fp8q.h.

Loading fails loudly when libfp8q.so has not been built: there is no
fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfp8q.so")

# (name, restype, argtypes) of every exported function.
c = ctypes
_P = c.c_void_p
_I64 = c.c_int64
_I32 = c.c_int32
_F = c.c_float

STATUS = c.c_int32


class CalibStats(c.Structure):
    _fields_ = [
        ("requested_tokens", _I64),
        ("window_tokens", _I64),
        ("capacity_tokens", _I64),
        ("tokens_seen", _I64),
        ("staged_tokens", _I64),
        ("staged_batches", _I64),
        ("unstaged_tokens", _I64),
        ("freeze_tokens", _I64),
        ("replayed_tokens", _I64),
        ("replayed_batches", _I64),
        ("headroom", _F),
        ("state", _I32),
    ]


class KvLayer(c.Structure):
    _fields_ = [
        ("k", _P),
        ("v", _P),
        ("slot_mapping", _P),
        ("k_pool", _P),
        ("v_pool", _P),
        ("scale_dev", _P),
        ("k_scale", _F),
        ("v_scale", _F),
    ]


SIGNATURES = {
    "fp8_group_quant": (STATUS, [_P, _I64, _P, _P, _I64, _I64, _P]),
    "fp8_group_quant_kmajor": (STATUS, [_P, _I64, _P, _P, _I64, _I64, _I64, _P]),
    "fp8_kv_write": (STATUS, [_P, _P, _I64, _I64, _P, _I64, _I32, _I32, _P, _P, _I32, _I64,
                              _I64, _F, _F, _P, _P]),
    "fp8_kv_amax_observe": (STATUS, [_P, _P, _I64, _I64, _I64, _I32, _I32, _P, _P]),
    "fp8_kv_write_layers": (STATUS, [c.POINTER(KvLayer), _I32, _I64, _I64, _I64, _I32, _I32,
                                     _I32, _I64, _I64, _P]),
    "fp8_kv_calib_create": (STATUS, [_I64, _F, _I32, _I32, _P, _P, _P, _I64, _P, _P,
                                     c.POINTER(_P)]),
    "fp8_kv_calib_observe": (STATUS, [_P, _P, _P, _I64, _I64, _P, _I64, _I32, _I32, _P,
                                      c.POINTER(_I32)]),
    "fp8_kv_freeze_replay": (STATUS, [_P, _P, _P, _I32, _I64, _I64, _P, c.POINTER(_I64)]),
    "fp8_kv_calib_observe_write": (STATUS, [_P, _P, _P, _I64, _I64, _P, _I64, _I32, _I32, _P,
                                            _P, _I32, _I64, _I64, _P, c.POINTER(_I32)]),
    "fp8_kv_calib_scale_dev": (_P, [_P]),
    "fp8_kv_calib_restore": (STATUS, [_P, _F, _F, _P]),
    "fp8_kv_calib_stats_get": (STATUS, [_P, c.POINTER(CalibStats)]),
    "fp8_kv_calib_read_state": (STATUS, [_P, _P, c.POINTER(_F)]),
    "fp8_kv_calib_destroy": (None, [_P]),
    "fp8_kv_graphs_ready": (_I32, [_P, _I64]),
    "fp8_kv_calib_window_noalloc": (STATUS, [_P, _P, _I64, _I64, _P, _P, _I32, _I32, _I32, _I64,
                                             _F, _P, _P, _I32, _I64, _I64, _P, _P]),
    "fp8q_device_error": (STATUS, [c.POINTER(c.c_uint32), _I32]),
    "fp8q_status_string": (c.c_char_p, [STATUS]),
    "fp8q_version": (_I32, []),
    "fp8q_launch_count": (_I64, []),
}

OK, EINVAL, ECUDA, ESTATE, ENOMEM, ETOOBIG = 0, -1, -2, -3, -4, -5
STEP_STAGE, STEP_STAGE_DECLINED, STEP_FREEZE, STEP_FROZEN = 1, 2, 3, 4
DEVERR_SLOT_OUT_OF_RANGE, DEVERR_BAD_SCALE = 0x1, 0x2
MAX_STAGED_TOKENS = 4096
PROVISIONAL_SCALE = 2.0
CALIB_STATE_BYTES = 16
MAX_LAYERS = 128
NOALLOC_SCRATCH_BYTES = 1 << 20


class Fp8qError(RuntimeError):
    def __init__(self, name: str, status: int, text: str) -> None:
        super().__init__(f"{name} failed: {text} (status {status})")
        self.status = status


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python paged_kv_cache_group_b200/build.py` "
            "(there is no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
