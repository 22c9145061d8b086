"""The C-ABI library loads, exports every function include/fp8q.h declares,
and rejects bad arguments before touching a device (no GPU needed: every
call here returns before any CUDA call)."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_group_b200 as fp8q
from paged_kv_cache_group_b200 import _abi

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8q.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    text = "\n".join(l for l in text.splitlines() if not l.lstrip().startswith("#"))
    return sorted(set(re.findall(r"FP8Q_API\s+[\w\s\*]*?\b(\w+)\s*\(", text)))


def test_every_declared_function_is_exported_and_bound():
    names = declared_functions()
    assert len(names) >= 15
    raw = ctypes.CDLL(_abi.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
        assert n in _abi.SIGNATURES, f"{n} has no ctypes signature"
    assert set(_abi.SIGNATURES) == set(names)


def test_version_and_status_strings():
    assert fp8q.version() == 10100
    assert fp8q.lib.fp8q_status_string(0) == b"ok"
    assert fp8q.lib.fp8q_status_string(-1) == b"invalid argument"
    assert fp8q.lib.fp8q_status_string(-3) == b"calibration call out of order"


def test_group_quant_rejects_bad_sizes_without_a_device():
    L = fp8q.lib
    fake = 1 << 20   # never dereferenced: every call below fails validation
    assert L.fp8_group_quant(fake, 200, fake, fake, 4, 200, None) == _abi.EINVAL   # k % 128
    assert L.fp8_group_quant(fake, 100, fake, fake, 4, 128, None) == _abi.EINVAL   # stride < k
    assert L.fp8_group_quant(fake, 132, fake, fake, 4, 128, None) == _abi.EINVAL   # stride % 8
    assert L.fp8_group_quant(fake + 8, 128, fake, fake, 4, 128, None) == _abi.EINVAL  # x align
    assert L.fp8_group_quant(fake, 128, fake + 4, fake, 4, 128, None) == _abi.EINVAL  # q align
    assert L.fp8_group_quant(None, 128, None, None, 4, 128, None) == _abi.EINVAL
    assert L.fp8_group_quant(fake, 128, fake, fake, -1, 128, None) == _abi.EINVAL
    assert L.fp8_group_quant(None, 128, None, None, 0, 128, None) == _abi.OK        # empty


def test_kv_write_rejects_bad_arguments_without_a_device():
    L = fp8q.lib
    f = 1 << 20
    ok = dict(k=f, v=f, ks=512, vs=512, slots=f, t=4, h=4, d=128, kp=f, vp=f, bs=16,
              cs=16 * 512, nb=8, ksc=1.0, vsc=1.0, sd=None)

    def call(**kw):
        a = dict(ok, **kw)
        return L.fp8_kv_write(a["k"], a["v"], a["ks"], a["vs"], a["slots"], a["t"], a["h"],
                              a["d"], a["kp"], a["vp"], a["bs"], a["cs"], a["nb"], a["ksc"],
                              a["vsc"], a["sd"], None)

    assert call(t=0) == _abi.OK
    assert call(ks=500) == _abi.EINVAL            # stride < E
    assert call(vs=516) == _abi.EINVAL            # stride not a multiple of 8
    assert call(d=3, h=1) == _abi.EINVAL          # E % 8
    assert call(cs=100) == _abi.EINVAL            # cache_stride < block_size * E
    assert call(bs=0) == _abi.EINVAL
    assert call(ksc=0.0) == _abi.EINVAL
    assert call(vsc=-1.0) == _abi.EINVAL
    assert call(ksc=float("nan")) == _abi.EINVAL
    assert call(ksc=float("inf")) == _abi.EINVAL
    assert call(k=f + 8) == _abi.EINVAL           # 16-byte alignment
    assert call(kp=f + 4) == _abi.EINVAL          # pool alignment
    assert call(slots=None) == _abi.EINVAL
    assert call(sd=f + 4) == _abi.EINVAL          # device scale alignment


def test_calibration_create_rejects_bad_arguments_without_a_device():
    L = fp8q.lib
    f = 1 << 20
    h = ctypes.c_void_p()

    def create(window=256, head=1.0, heads=4, dim=128, sk=f, sv=f, ss=f, cap=256, state=f):
        return L.fp8_kv_calib_create(window, head, heads, dim, sk, sv, ss, cap, state, None,
                                     ctypes.byref(h))

    assert create(window=0) == _abi.EINVAL
    assert create(heads=0) == _abi.EINVAL
    assert create(dim=3, heads=1) == _abi.EINVAL
    assert create(cap=-1) == _abi.EINVAL
    assert create(sk=None) == _abi.EINVAL
    assert create(sk=f + 8) == _abi.EINVAL
    assert create(state=None) == _abi.EINVAL
    assert create(state=f + 8) == _abi.EINVAL
    assert h.value is None


def test_calibration_calls_reject_null_handles():
    L = fp8q.lib
    step = ctypes.c_int32()
    assert L.fp8_kv_calib_observe(None, None, None, 512, 512, None, 0, 4, 128, None,
                                  ctypes.byref(step)) == _abi.EINVAL
    assert L.fp8_kv_freeze_replay(None, None, None, 16, 8192, 1, None, None) == _abi.EINVAL
    assert L.fp8_kv_calib_stats_get(None, None) == _abi.EINVAL
    assert L.fp8_kv_calib_scale_dev(None) is None
    assert L.fp8_kv_calib_restore(None, 1.0, 1.0, None) == _abi.EINVAL
    L.fp8_kv_calib_destroy(None)


def test_graph_readiness_mirrors_the_pages():
    assert fp8q.fp8_kv_graphs_ready([])
    assert fp8q.fp8_kv_graphs_ready([None, None])
    assert fp8q.fp8_kv_graphs_ready([True, None, True])
    assert not fp8q.fp8_kv_graphs_ready([True, False])
    assert fp8q.lib.fp8_kv_graphs_ready(None, 3) == -1


def test_oracle_and_cuda_path_share_no_code():
    pkg = os.path.join(ROOT, "paged_kv_cache_group_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cpp", ".h", ".cuh")):
                text = open(os.path.join(dirpath, fn)).read()
                assert not re.search(r"^\s*(from|import)\s+oracle", text, re.M), fn
                assert "fp8q_oracle" not in text and "libfp8q_oracle" not in text, fn
    for fn in os.listdir(os.path.join(ROOT, "oracle")):
        if fn.endswith((".py", ".c", ".h")):
            text = open(os.path.join(ROOT, "oracle", fn)).read()
            assert "paged_kv_cache_group_b200" not in text, fn
            assert "fp8q.h" not in text and "csrc" not in text, fn


@pytest.mark.parametrize("name", ["fp8_group_quant", "fp8_kv_write", "fp8_kv_amax_observe",
                                  "fp8_kv_freeze_replay"])
def test_binding_exposes_the_abi_names(name):
    assert callable(getattr(fp8q, name))
