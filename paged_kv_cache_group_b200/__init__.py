"""FP8 E4M3 quantization for B200: per-token 1x128-group activation
quantization, the paged KV-cache quantize-and-scatter, and online calibration
of the KV scales.

The compute is the CUDA library libfp8q.so (C ABI: include/fp8q.h).  This
module only marshals torch tensors (device memory) and streams into those
calls; every step runs in the library's kernels.  Function names match the C
ABI.  Importing fails if the library has not been built.
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import (CALIB_STATE_BYTES, DEVERR_BAD_SCALE, DEVERR_SLOT_OUT_OF_RANGE,  # noqa: F401
                   MAX_STAGED_TOKENS, PROVISIONAL_SCALE, STEP_FREEZE, STEP_FROZEN, STEP_STAGE,
                   STEP_STAGE_DECLINED, CalibStats, Fp8qError)

lib = _abi.load()

_BYTE_TYPES = (torch.uint8, torch.float8_e4m3fn)


def _check(name: str, status: int) -> None:
    if status != _abi.OK:
        raise Fp8qError(name, status, lib.fp8q_status_string(status).decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _bf16_rows(t: torch.Tensor, name: str):
    """``[T, ...]`` bf16 whose rows (all dimensions after the first) are
    contiguous; returns (rows, row stride in elements, elements per row)."""
    if t.dtype != torch.bfloat16 or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA bfloat16 tensor")
    if t.dim() < 2:
        raise ValueError(f"{name} must have a row dimension and at least one more")
    rows = t.shape[0]
    inner = 1
    for size in t.shape[1:]:
        inner *= size
    if t.numel() == 0:          # no data: any strides (an empty array may carry zeros)
        return rows, inner, inner
    expect = 1
    for size, stride in zip(reversed(t.shape[1:]), reversed(t.stride()[1:])):
        if size != 1 and stride != expect:
            raise ValueError(f"{name} rows must be contiguous")
        expect *= size
    return rows, (t.stride(0) if rows > 1 else inner), inner


def _kv_rows(k: torch.Tensor, v: torch.Tensor):
    """K and V ``[T, heads, dim]`` of the same shape (rows contiguous, row
    strides may differ); returns (T, key_stride, value_stride, heads, dim).
    The shapes are checked before anything else, so a mismatched V is refused
    whatever device it is on."""
    if k.dim() != 3 or v.dim() != 3:
        raise ValueError("k and v must both be [T, heads, dim]")
    if tuple(k.shape) != tuple(v.shape):
        raise ValueError(f"k and v must have the same shape, got {tuple(k.shape)} and "
                         f"{tuple(v.shape)}")
    t, ks, _ = _bf16_rows(k, "k")
    _, vs, _ = _bf16_rows(v, "v")
    return t, ks, vs, k.shape[1], k.shape[2]


def _check_slots(slot_mapping: torch.Tensor, t: int) -> None:
    if slot_mapping.dtype != torch.int64 or slot_mapping.numel() < t:
        raise ValueError("slot_mapping must be int64 with one entry per token")
    if t and (not slot_mapping.is_cuda or not slot_mapping.is_contiguous()):
        raise ValueError("slot_mapping must be a contiguous CUDA tensor")


def _check_scale_pair(t: torch.Tensor | None, name: str) -> None:
    """A device ``{k, v}`` fp32 pair the library reads or writes."""
    if t is None:
        return
    if t.dtype != torch.float32 or not t.is_cuda or not t.is_contiguous() or t.numel() < 2:
        raise ValueError(f"{name} must be a contiguous CUDA float32 tensor of 2 elements")


# ---------------------------------------------------------------------------
# activation quantization


def fp8_group_quant(x: torch.Tensor, q: torch.Tensor | None = None,
                    scales: torch.Tensor | None = None, stream=None):
    """Quantize a bf16 ``[m, k]`` activation (k % 128 == 0, rows may be
    strided) into E4M3 codes ``q [m, k]`` and fp32 ``scales [m, k/128]``."""
    m, stride, k = _bf16_rows(x, "x")
    if q is None:
        q = torch.empty((m, k), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((m, k // 128), dtype=torch.float32, device=x.device)
    if q.dtype not in _BYTE_TYPES or not q.is_contiguous() or q.numel() < m * k:
        raise ValueError("q must be a contiguous uint8/float8_e4m3fn tensor of m*k elements")
    if scales.dtype != torch.float32 or not scales.is_contiguous() or \
            scales.numel() < m * (k // 128):
        raise ValueError("scales must be a contiguous float32 tensor of m*(k/128) elements")
    _check("fp8_group_quant", lib.fp8_group_quant(
        _ptr(x), stride, _ptr(q), _ptr(scales), m, k, _stream(stream)))
    return q, scales


def ceil16(m: int) -> int:
    """Rows a GEMM padded to 16-row tiles is handed for an m-row activation."""
    return (m + 15) // 16 * 16


def fp8_group_quant_kmajor(x: torch.Tensor, m_pad: int | None = None,
                           q: torch.Tensor | None = None, scales_km: torch.Tensor | None = None,
                           stream=None):
    """Quantize a bf16 ``[m, k]`` activation for a padded FP8 GEMM: codes
    ``q [m_pad, k]`` with rows m..m_pad-1 zero, and fp32 scales K-major
    ``scales_km [k/128, m_pad]`` with the pad columns zero.  ``m_pad``
    defaults to ceil16(m)."""
    m, stride, k = _bf16_rows(x, "x")
    m_pad = ceil16(m) if m_pad is None else int(m_pad)
    if m_pad < m:
        raise ValueError("m_pad must be >= the number of rows")
    if q is None:
        q = torch.empty((m_pad, k), dtype=torch.uint8, device=x.device)
    if scales_km is None:
        scales_km = torch.empty((k // 128, m_pad), dtype=torch.float32, device=x.device)
    if q.dtype not in _BYTE_TYPES or not q.is_contiguous() or q.numel() < m_pad * k:
        raise ValueError("q must be a contiguous uint8/float8_e4m3fn tensor of m_pad*k elements")
    if scales_km.dtype != torch.float32 or not scales_km.is_contiguous() or \
            scales_km.numel() < m_pad * (k // 128):
        raise ValueError("scales_km must be a contiguous float32 tensor of (k/128)*m_pad elements")
    _check("fp8_group_quant_kmajor", lib.fp8_group_quant_kmajor(
        _ptr(x) if m else None, stride, _ptr(q), _ptr(scales_km), m, m_pad, k, _stream(stream)))
    return q, scales_km


# ---------------------------------------------------------------------------
# paged KV write


def _pool_geometry(k_pool: torch.Tensor, v_pool: torch.Tensor, elems: int):
    """Pools ``[num_blocks, block_size, heads, dim]`` (block stride may be padded)."""
    for name, p in (("k_pool", k_pool), ("v_pool", v_pool)):
        if p.dtype not in _BYTE_TYPES or not p.is_cuda:
            raise TypeError(f"{name} must be a CUDA uint8/float8_e4m3fn tensor")
    if k_pool.shape != v_pool.shape or k_pool.stride() != v_pool.stride():
        raise ValueError("k_pool and v_pool must have the same shape and strides")
    num_blocks, block_size = k_pool.shape[0], k_pool.shape[1]
    inner = k_pool[0].numel() if num_blocks else block_size * elems
    if inner != block_size * elems:
        raise ValueError("pool block does not hold block_size * num_kv_heads * head_dim codes")
    if num_blocks and not k_pool[0].is_contiguous():
        raise ValueError("each pool block must be contiguous")
    return num_blocks, block_size, k_pool.stride(0)


def fp8_kv_write(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                 k_pool: torch.Tensor, v_pool: torch.Tensor, k_scale: float = 1.0,
                 v_scale: float = 1.0, scale_dev: torch.Tensor | None = None, stream=None):
    """reshape_and_cache_fp8: K, V ``[T, heads, dim]`` bf16 into the pools at
    ``slot_mapping`` (int64, -1 skips), per-tensor scales by value or from the
    device ``scale_dev [2]``."""
    t, ks, vs, heads, dim = _kv_rows(k, v)
    _check_slots(slot_mapping, t)
    _check_scale_pair(scale_dev, "scale_dev")
    nb, bs, cs = _pool_geometry(k_pool, v_pool, heads * dim)
    _check("fp8_kv_write", lib.fp8_kv_write(
        _ptr(k), _ptr(v), ks, vs, _ptr(slot_mapping), t, heads, dim, _ptr(k_pool),
        _ptr(v_pool), bs, cs, nb, float(k_scale), float(v_scale), _ptr(scale_dev),
        _stream(stream)))


def fp8_kv_write_layers(ks, vs, slot_mappings, k_pools, v_pools, k_scales=None, v_scales=None,
                        scale_devs=None, stream=None):
    """reshape_and_cache_fp8 for several layers in one launch.  Per layer:
    K, V ``[T, heads, dim]`` (same shape and row strides for all layers), an
    int64 slot mapping and the layer's pools; scales by value (``k_scales``,
    ``v_scales``) or from device ``scale_devs[i]``."""
    n = len(ks)
    if not (len(vs) == len(slot_mappings) == len(k_pools) == len(v_pools) == n):
        raise ValueError("one k, v, slot_mapping, k_pool and v_pool per layer")
    if n > _abi.MAX_LAYERS:
        raise ValueError(f"at most {_abi.MAX_LAYERS} layers per launch")
    if n == 0:
        return
    t, kst, vst, heads, dim = _kv_rows(ks[0], vs[0])
    e = heads * dim
    nb, bs, cs = _pool_geometry(k_pools[0], v_pools[0], e)
    arr = (_abi.KvLayer * n)()
    for i in range(n):
        ti, ksi, vsi, hi, di = _kv_rows(ks[i], vs[i])
        if (ti, ksi, vsi, hi, di) != (t, kst, vst, heads, dim):
            raise ValueError("all layers must share the row shape and strides")
        _check_slots(slot_mappings[i], t)
        if _pool_geometry(k_pools[i], v_pools[i], e) != (nb, bs, cs):
            raise ValueError("all layers' pools must share one geometry")
        sd = None if scale_devs is None else scale_devs[i]
        _check_scale_pair(sd, "scale_devs[i]")
        arr[i] = _abi.KvLayer(_ptr(ks[i]), _ptr(vs[i]), _ptr(slot_mappings[i]), _ptr(k_pools[i]),
                              _ptr(v_pools[i]), _ptr(sd),
                              float(k_scales[i]) if k_scales is not None else 1.0,
                              float(v_scales[i]) if v_scales is not None else 1.0)
    _check("fp8_kv_write_layers", lib.fp8_kv_write_layers(
        arr, n, kst, vst, t, heads, dim, bs, cs, nb, _stream(stream)))


def fp8_kv_amax_observe(k: torch.Tensor, v: torch.Tensor, amax_dev: torch.Tensor, stream=None):
    """Max-accumulate max|K| and max|V| into the device fp32 ``amax_dev [2]``."""
    t, ks, vs, heads, dim = _kv_rows(k, v)
    _check_scale_pair(amax_dev, "amax_dev")
    _check("fp8_kv_amax_observe", lib.fp8_kv_amax_observe(
        _ptr(k), _ptr(v), ks, vs, t, heads, dim, _ptr(amax_dev), _stream(stream)))


# ---------------------------------------------------------------------------
# calibration


def fp8_kv_graphs_ready(states) -> bool:
    """``states``: per layer None (no calibrator), False (in window), True (frozen)."""
    arr = (ctypes.c_int8 * len(states))(*[-1 if s is None else int(bool(s)) for s in states])
    r = lib.fp8_kv_graphs_ready(arr, len(states))
    if r < 0:
        raise Fp8qError("fp8_kv_graphs_ready", r, "invalid argument")
    return bool(r)


class KvCalibration:
    """The calibrator of one attention layer (fp8_kv_calib_* of the C ABI).

    Device memory (staging for the window's bf16 K/V and slots, and the
    16-byte state) is allocated here with torch and handed to the library."""

    def __init__(self, window_tokens: int, headroom: float, num_kv_heads: int, head_dim: int,
                 device, stage_capacity: int | None = None, stream=None,
                 state: torch.Tensor | None = None) -> None:
        self.num_kv_heads = num_kv_heads
        self.head_dim = head_dim
        e = num_kv_heads * head_dim
        window = min(int(window_tokens), MAX_STAGED_TOKENS)
        cap = window if stage_capacity is None else int(stage_capacity)
        self.stage_k = torch.empty((max(cap, 1), e), dtype=torch.bfloat16, device=device)
        self.stage_v = torch.empty((max(cap, 1), e), dtype=torch.bfloat16, device=device)
        self.stage_slots = torch.empty(max(cap, 1), dtype=torch.int64, device=device)
        if state is None:
            state = torch.empty(4, dtype=torch.float32, device=device)
        if state.dtype != torch.float32 or state.numel() != 4 or not state.is_contiguous():
            raise ValueError("state must be a contiguous float32 tensor of 4 elements")
        self.state = state
        self._h = ctypes.c_void_p()
        self.handle = None
        _check("fp8_kv_calib_create", lib.fp8_kv_calib_create(
            int(window_tokens), float(headroom), num_kv_heads, head_dim, _ptr(self.stage_k),
            _ptr(self.stage_v), _ptr(self.stage_slots), cap, _ptr(self.state), _stream(stream),
            ctypes.byref(self._h)))
        self.handle = self._h.value

    def close(self) -> None:
        if self.handle:
            lib.fp8_kv_calib_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    @property
    def scale_dev(self) -> torch.Tensor:
        """Device ``{k_scale, v_scale}``: provisional until the freeze, frozen after."""
        return self.state[2:4]

    def observe(self, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                stream=None) -> int:
        t, ks, vs, heads, dim = _kv_rows(k, v)
        _check_slots(slot_mapping, t)
        step = ctypes.c_int32()
        _check("fp8_kv_calib_observe", lib.fp8_kv_calib_observe(
            self.handle, _ptr(k), _ptr(v), ks, vs, _ptr(slot_mapping), t, heads, dim,
            _stream(stream), ctypes.byref(step)))
        return step.value

    def freeze_replay(self, k_pool: torch.Tensor, v_pool: torch.Tensor, stream=None) -> int:
        nb, bs, cs = _pool_geometry(k_pool, v_pool, self.num_kv_heads * self.head_dim)
        n = ctypes.c_int64()
        _check("fp8_kv_freeze_replay", lib.fp8_kv_freeze_replay(
            self.handle, _ptr(k_pool), _ptr(v_pool), bs, cs, nb, _stream(stream),
            ctypes.byref(n)))
        return n.value

    def observe_write(self, k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                      k_pool: torch.Tensor, v_pool: torch.Tensor, stream=None) -> int:
        t, ks, vs, heads, dim = _kv_rows(k, v)
        _check_slots(slot_mapping, t)
        nb, bs, cs = _pool_geometry(k_pool, v_pool, heads * dim)
        step = ctypes.c_int32()
        _check("fp8_kv_calib_observe_write", lib.fp8_kv_calib_observe_write(
            self.handle, _ptr(k), _ptr(v), ks, vs, _ptr(slot_mapping), t, heads, dim,
            _ptr(k_pool), _ptr(v_pool), bs, cs, nb, _stream(stream), ctypes.byref(step)))
        return step.value

    def restore(self, k_scale: float, v_scale: float, stream=None) -> None:
        """Start frozen at saved scales (only before the first observe)."""
        _check("fp8_kv_calib_restore", lib.fp8_kv_calib_restore(
            self.handle, float(k_scale), float(v_scale), _stream(stream)))

    def saved_scales(self, stream=None) -> dict:
        """The frozen scales as exact hex floats, for save_scales()/restore()."""
        if self.stats()["state"] != 2:
            raise Fp8qError("saved_scales", _abi.ESTATE, "the calibrator has not frozen")
        _, _, ks, vs = self.read_state(stream)
        return {"k_scale": float(ks).hex(), "v_scale": float(vs).hex()}

    def stats(self) -> dict:
        s = CalibStats()
        _check("fp8_kv_calib_stats_get", lib.fp8_kv_calib_stats_get(self.handle, ctypes.byref(s)))
        return {name: getattr(s, name) for name, _ in CalibStats._fields_}

    def read_state(self, stream=None):
        """(k_amax, v_amax, k_scale, v_scale); synchronizes the stream."""
        out = (ctypes.c_float * 4)()
        _check("fp8_kv_calib_read_state", lib.fp8_kv_calib_read_state(
            self.handle, _stream(stream), out))
        return tuple(out)


def fp8_kv_calib_window_noalloc(k: torch.Tensor, v: torch.Tensor, slot_mapping: torch.Tensor,
                                batch_tokens, window_tokens: int, headroom: float,
                                k_pool: torch.Tensor, v_pool: torch.Tensor,
                                scales_out: torch.Tensor | None = None, stream=None) -> None:
    """One layer's calibration window in one call, with no device memory from
    the caller or the library's user: the scratch is a fixed array inside the
    library (see include/fp8q.h).  ``k``/``v`` hold every batch's rows back to
    back; ``batch_tokens`` lists each batch's token count."""
    t, ks, vs, heads, dim = _kv_rows(k, v)
    counts = [int(n) for n in batch_tokens]
    if sum(counts) != t:
        raise ValueError("batch_tokens must add up to the rows of k and v")
    _check_slots(slot_mapping, t)
    _check_scale_pair(scales_out, "scales_out")
    nb, bs, cs = _pool_geometry(k_pool, v_pool, heads * dim)
    arr = (ctypes.c_int64 * max(len(counts), 1))(*counts)
    _check("fp8_kv_calib_window_noalloc", lib.fp8_kv_calib_window_noalloc(
        _ptr(k), _ptr(v), ks, vs, _ptr(slot_mapping), arr, len(counts), heads, dim,
        int(window_tokens), float(headroom), _ptr(k_pool), _ptr(v_pool), bs, cs, nb,
        _ptr(scales_out), _stream(stream)))


def allreduce_kv_maxima(calibrator, group=None, stream=None) -> None:
    """KV heads sharded over ranks, one scale for all of them: after
    ``observe()`` returns STEP_FREEZE for the batch that reaches the window and
    before ``freeze_replay()``, make every rank's device |K| and |V| maxima the
    maximum over the group (one all-reduce of two fp32 values).  Every rank
    then freezes the same scales.  Pass the ``stream`` that ``observe()`` and
    ``freeze_replay()`` use (default: the current stream): the all-reduce is
    ordered after that stream's absmax kernels and before its replay."""
    import torch.distributed as dist
    if stream is None or isinstance(stream, int):
        dist.all_reduce(calibrator.state[0:2], op=dist.ReduceOp.MAX, group=group)
        return
    with torch.cuda.stream(stream):
        dist.all_reduce(calibrator.state[0:2], op=dist.ReduceOp.MAX, group=group)


def save_scales(calibrators, path: str) -> None:
    """Write every layer's frozen scales to a JSON file (exact hex floats)."""
    import json
    with open(path, "w") as fh:
        json.dump({"fp8_kv_scales": [c.saved_scales() for c in calibrators]}, fh, indent=1)


def load_scales(path: str) -> list[tuple[float, float]]:
    """Read scales written by save_scales(): [(k_scale, v_scale)] per layer."""
    import json
    with open(path) as fh:
        data = json.load(fh)["fp8_kv_scales"]
    return [(float.fromhex(d["k_scale"]), float.fromhex(d["v_scale"])) for d in data]


def fp8q_device_error(clear: bool = True) -> int:
    """Sticky device error bits of the current device (synchronizes)."""
    bits = ctypes.c_uint32()
    _check("fp8q_device_error", lib.fp8q_device_error(ctypes.byref(bits), int(clear)))
    return bits.value


def version() -> int:
    return lib.fp8q_version()


def launch_count() -> int:
    """Kernels the library has launched (or recorded into a graph) so far."""
    return lib.fp8q_launch_count()


# Module-level spellings of the calibrator entry points, with the C ABI's names.
def fp8_kv_calib_create(window_tokens: int, headroom: float, num_kv_heads: int, head_dim: int,
                        device, stage_capacity: int | None = None, stream=None) -> KvCalibration:
    return KvCalibration(window_tokens, headroom, num_kv_heads, head_dim, device,
                         stage_capacity, stream)


def fp8_kv_calib_observe(calib: KvCalibration, k, v, slot_mapping, stream=None) -> int:
    return calib.observe(k, v, slot_mapping, stream)


def fp8_kv_freeze_replay(calib: KvCalibration, k_pool, v_pool, stream=None) -> int:
    return calib.freeze_replay(k_pool, v_pool, stream)


def fp8_kv_calib_observe_write(calib: KvCalibration, k, v, slot_mapping, k_pool, v_pool,
                               stream=None) -> int:
    return calib.observe_write(k, v, slot_mapping, k_pool, v_pool, stream)
