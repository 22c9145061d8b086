"""ctypes front end of the C oracle (``fp8q_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  Nothing here touches a
GPU or the CUDA library; arrays are numpy, bf16 tensors are carried as their
uint16 bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8q_oracle.c")
_LIB = os.path.join(_HERE, "libfp8q_oracle.so")
_lock = threading.Lock()
_lib = None

GROUP = 128

_CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/libfp8q_oracle.so``."""
    if force or not os.path.exists(_LIB) or \
            os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *_CFLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def lib() -> ctypes.CDLL:
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            c = ctypes
            P = c.c_void_p
            L.oracle_bf16_to_f32.argtypes = [c.c_uint16]
            L.oracle_bf16_to_f32.restype = c.c_float
            L.oracle_e4m3_encode.argtypes = [c.c_float]
            L.oracle_e4m3_encode.restype = c.c_uint8
            L.oracle_e4m3_encode_array.argtypes = [P, c.c_int64, P]
            L.oracle_e4m3_encode_array.restype = None
            L.oracle_group_scale.argtypes = [c.c_float]
            L.oracle_group_scale.restype = c.c_float
            L.oracle_group_quant.argtypes = [P, c.c_int64, c.c_int64, c.c_int64, P, P]
            L.oracle_group_quant.restype = c.c_int
            L.oracle_absmax.argtypes = [P, c.c_int64, c.c_int64, c.c_int64]
            L.oracle_absmax.restype = c.c_float
            L.oracle_kv_write.argtypes = [P, P, c.c_int64, c.c_int64, P, c.c_int64,
                                          c.c_int32, c.c_int32, P, P, c.c_int32,
                                          c.c_int64, c.c_int64, c.c_float, c.c_float]
            L.oracle_kv_write.restype = c.c_int64
            L.oracle_freeze_scale.argtypes = [c.c_float, c.c_float]
            L.oracle_freeze_scale.restype = c.c_float
            _lib = L
    return _lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (vectorised; same rule as the C)."""
    bits = np.asarray(bits, dtype=np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def e4m3_encode(y) -> np.ndarray:
    """E4M3 code of each fp32 value (RNE, saturating to +-448)."""
    y = np.ascontiguousarray(np.asarray(y, dtype=np.float32))
    out = np.empty(y.shape, dtype=np.uint8)
    lib().oracle_e4m3_encode_array(_ptr(y), y.size, _ptr(out))
    return out


def group_scale(amax: float) -> np.float32:
    return np.float32(lib().oracle_group_scale(float(np.float32(amax))))


def freeze_scale(amax: float, headroom: float) -> np.float32:
    return np.float32(lib().oracle_freeze_scale(float(np.float32(amax)),
                                                float(np.float32(headroom))))


def group_quant(x_bits: np.ndarray):
    """Per-token 1x128-group quantization of a packed ``[m, k]`` bf16 array.

    Returns ``(codes uint8 [m, k], scales float32 [m, k/128])``."""
    m, k = x_bits.shape
    return group_quant_strided(x_bits, m, k, k)


def group_quant_strided(x_bits: np.ndarray, m: int, k: int, row_stride: int):
    """Same, for an activation whose row ``r`` starts at element ``r * row_stride``
    of the flat buffer ``x_bits``."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    assert x_bits.size >= (m - 1) * row_stride + k if m > 0 else True
    q = np.empty((m, k), dtype=np.uint8)
    s = np.empty((m, k // GROUP if k % GROUP == 0 else 0), dtype=np.float32)
    rc = lib().oracle_group_quant(_ptr(x_bits), m, k, row_stride, _ptr(q), _ptr(s))
    if rc != 0:
        raise ValueError(f"oracle_group_quant rejected m={m} k={k} stride={row_stride}")
    return q, s


def group_quant_kmajor(x_bits: np.ndarray, m: int, k: int, row_stride: int, m_pad: int):
    """The activation quantized for a GEMM padded to ``m_pad`` rows, in the
    steps of decode_w8a8_quant_act ("spark_model/layers/ops/
    dispatch_proj_decode.rs"): quantize the m live rows; zero the codes of the
    phantom rows m..m_pad-1; write every slot of the K-major scale array
    ``[k/128, m_pad]``, the live rows' scales transposed and the pad rows 0.

    Returns ``(codes uint8 [m_pad, k], scales_km float32 [k/128, m_pad])``."""
    if m_pad < m:
        raise ValueError("m_pad must be >= m")
    q_live, s_live = group_quant_strided(x_bits, m, k, row_stride)
    q = np.zeros((m_pad, k), dtype=np.uint8)          # phantom rows: zero codes
    q[:m] = q_live
    scales_km = np.zeros((k // GROUP, m_pad), dtype=np.float32)   # pad rows: zero scales
    scales_km[:, :m] = s_live.T
    return q, scales_km


def absmax(x_bits: np.ndarray, rows: int, row_elems: int, row_stride: int) -> np.float32:
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    if rows > 0:
        assert x_bits.size >= (rows - 1) * row_stride + row_elems
    return np.float32(lib().oracle_absmax(_ptr(x_bits), rows, row_elems, row_stride))


def kv_write(k_bits, v_bits, key_stride, value_stride, slot_mapping, num_tokens,
             num_kv_heads, head_dim, k_pool, v_pool, block_size, cache_stride,
             num_blocks, k_scale, v_scale) -> int:
    """reshape_and_cache_fp8 into ``k_pool``/``v_pool`` (uint8 arrays, in place).

    Returns the number of out-of-range slots (skipped)."""
    k_bits = np.ascontiguousarray(k_bits, dtype=np.uint16)
    v_bits = np.ascontiguousarray(v_bits, dtype=np.uint16)
    slot_mapping = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    assert k_pool.dtype == np.uint8 and v_pool.dtype == np.uint8
    assert k_pool.flags["C_CONTIGUOUS"] and v_pool.flags["C_CONTIGUOUS"]
    elems = num_kv_heads * head_dim
    assert k_pool.size >= num_blocks * cache_stride and v_pool.size >= num_blocks * cache_stride
    if num_tokens > 0:
        assert k_bits.size >= (num_tokens - 1) * key_stride + elems
        assert v_bits.size >= (num_tokens - 1) * value_stride + elems
        assert slot_mapping.size >= num_tokens
    rc = lib().oracle_kv_write(_ptr(k_bits), _ptr(v_bits), key_stride, value_stride,
                               _ptr(slot_mapping), num_tokens, num_kv_heads, head_dim,
                               _ptr(k_pool), _ptr(v_pool), block_size, cache_stride,
                               num_blocks, float(np.float32(k_scale)),
                               float(np.float32(v_scale)))
    if rc < 0:
        raise ValueError("oracle_kv_write rejected its sizes")
    return int(rc)


def source_path() -> str:
    return _SRC
