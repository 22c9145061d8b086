"""Online FP8 KV scale calibration, restated as a host-side oracle.

TEST INFRASTRUCTURE ONLY (test suite, smoke check, benchmark CPU baseline).

Sources (page title, item):
  * "metrale_model_layers/layers/fp8_calibration.rs": module doc (running max of
    |K| and |V| over the first ``window_tokens`` observed tokens; the observe
    that reaches the window freezes ``scale = amax * headroom / 448`` over every
    observed token including its own batch; in-window entries are written at
    ``PROVISIONAL_SCALE`` and rewritten at the freeze), ``PROVISIONAL_SCALE``,
    ``Fp8KvCalibration::new`` (headroom clamp to >= 1, window clamp to
    ``MAX_STAGED_TOKENS``, window 1 freezes on the first observe, no calibrator
    for 0), ``Fp8KvCalibration::observe`` (Stage / Freeze / Frozen arms, the
    freeze log fields), ``graphs_ready_after_fp8_kv_cal`` and
    ``dtype_runs_online_fp8_kv_calibration``.
  * "spark_model/layers/fp8_calibration/staging.rs": ``MAX_STAGED_TOKENS``,
    ``KvStaging::stage`` (capacity reserved on first use, declines on an
    elements-per-token mismatch or overflow, strided rows packed, slots copied,
    batch recorded), ``KvStaging::replay_and_release`` (each staged batch, in
    the order staged, through reshape_and_cache_fp8 at the frozen scales with
    packed strides, then release).

The calibration state itself (``state.rs``) is not on the pages; its fields
and the freeze rule are taken from how the pages use them.  Readings:
  * ``record`` folds the batch maxima into the running maxima and adds the
    batch's tokens; it returns FREEZE when the running count first reaches the
    window, STAGE while below it, FROZEN afterwards;
  * the frozen scale is ``max(amax * headroom, 1e-12) / 448`` (fp32, product
    rounded first) -- see ``oracle_freeze_scale``;
  * ``staged_batches`` counts STAGE steps (whether or not staging accepted the
    batch), since it is a field of the state, which never sees the staging;
  * the opt-in EMA recalibration after the freeze is not built: after the
    freeze ``observe`` reduces nothing and the scales stay constant.

Everything is per-batch on the host: each batch's absmax is computed on its
own and folded into the running max here, and staging holds host copies.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

from . import core

MAX_STAGED_TOKENS = 4096
PROVISIONAL_SCALE = np.float32(2.0)

STAGE = "stage"
FREEZE = "freeze"
FROZEN = "frozen"


@dataclass
class Fp8KvWriteTarget:
    """Everything a replay needs to re-run reshape_and_cache_fp8 for one layer."""
    k_pool: np.ndarray          # uint8, flat, >= num_blocks * cache_stride
    v_pool: np.ndarray
    block_size: int
    cache_stride: int           # elements between blocks
    num_blocks: int
    key_stride: int             # source K row stride (elements) of the live write
    value_stride: int
    slot: np.ndarray            # int64 slot per token of this batch


@dataclass
class _StagedBatch:
    offset_tokens: int
    num_tokens: int


class KvStaging:
    """Host copies of the window's bf16 K/V rows and slot mappings."""

    def __init__(self) -> None:
        self._reset()

    def _reset(self) -> None:
        self.k = None
        self.v = None
        self.slots = None
        self.capacity_tokens = 0
        self.elems_per_token = 0
        self.used_tokens = 0
        self.batches: list[_StagedBatch] = []

    def stage(self, k_bits: np.ndarray, v_bits: np.ndarray, num_tokens: int,
              elems_per_token: int, target: Fp8KvWriteTarget,
              capacity_tokens: int) -> bool:
        if self.capacity_tokens == 0:
            self.k = np.zeros(capacity_tokens * elems_per_token, dtype=np.uint16)
            self.v = np.zeros(capacity_tokens * elems_per_token, dtype=np.uint16)
            self.slots = np.zeros(capacity_tokens, dtype=np.int64)
            self.capacity_tokens = capacity_tokens
            self.elems_per_token = elems_per_token
        n = num_tokens
        if elems_per_token != self.elems_per_token or \
                self.used_tokens + n > self.capacity_tokens:
            return False
        e = elems_per_token
        kf = np.asarray(k_bits, dtype=np.uint16).reshape(-1)
        vf = np.asarray(v_bits, dtype=np.uint16).reshape(-1)
        for t in range(n):
            dst = (self.used_tokens + t) * e
            self.k[dst:dst + e] = kf[t * target.key_stride:t * target.key_stride + e]
            self.v[dst:dst + e] = vf[t * target.value_stride:t * target.value_stride + e]
        self.slots[self.used_tokens:self.used_tokens + n] = \
            np.asarray(target.slot, dtype=np.int64)[:n]
        self.batches.append(_StagedBatch(self.used_tokens, n))
        self.used_tokens += n
        return True

    def replay_and_release(self, target: Fp8KvWriteTarget, num_kv_heads: int,
                           head_dim: int, k_scale, v_scale) -> int:
        rewritten = self.used_tokens
        e = self.elems_per_token
        for batch in self.batches:
            off = batch.offset_tokens
            core.kv_write(self.k[off * e:], self.v[off * e:], e, e,
                          self.slots[off:off + batch.num_tokens], batch.num_tokens,
                          num_kv_heads, head_dim, target.k_pool, target.v_pool,
                          target.block_size, target.cache_stride, target.num_blocks,
                          k_scale, v_scale)
        self._reset()
        return rewritten


class CalibrationState:
    def __init__(self, window_tokens: int, headroom: float, provisional) -> None:
        self.window_tokens = int(window_tokens)
        self.headroom = np.float32(headroom)
        self.k_running_max = np.float32(0.0)
        self.v_running_max = np.float32(0.0)
        self.tokens_seen = 0
        self.frozen = False
        self.k_scale = np.float32(provisional)
        self.v_scale = np.float32(provisional)
        self.staged_batches = 0

    def should_observe(self, num_tokens: int) -> bool:
        # Only the (unbuilt) EMA path observes after the freeze.
        return not self.frozen

    def record(self, k_max, v_max, num_tokens: int):
        self.k_running_max = np.float32(max(self.k_running_max, np.float32(k_max)))
        self.v_running_max = np.float32(max(self.v_running_max, np.float32(v_max)))
        self.tokens_seen += int(num_tokens)
        if self.frozen:
            return (FROZEN,)
        if self.tokens_seen >= self.window_tokens:
            self.frozen = True
            self.k_scale = core.freeze_scale(self.k_running_max, self.headroom)
            self.v_scale = core.freeze_scale(self.v_running_max, self.headroom)
            return (FREEZE, self.k_scale, self.v_scale, self.tokens_seen)
        self.staged_batches += 1
        return (STAGE,)


@dataclass
class FreezeLog:
    tokens_seen: int
    requested_tokens: int
    k_scale: np.float32
    k_amax: np.float32
    v_scale: np.float32
    v_amax: np.float32
    headroom: np.float32
    staged_tokens: int
    staged_batches: int
    unstaged_tokens: int


class Fp8KvCalibration:
    """Calibrator of one attention layer (oracle form)."""

    def __init__(self, attn_layer_idx: int, window_tokens: int, headroom: float,
                 staging_capacity: int | None = None) -> None:
        if window_tokens <= 0:
            raise ValueError("no calibrator is built for a window of 0 tokens")
        headroom = np.float32(headroom)
        if not headroom >= 1.0:
            headroom = np.float32(1.0)
        effective = min(int(window_tokens), MAX_STAGED_TOKENS)
        self.state = CalibrationState(effective, headroom, PROVISIONAL_SCALE)
        self.staging = KvStaging()
        self.unstaged_tokens = 0
        self.attn_layer_idx = attn_layer_idx
        self.requested_tokens = int(window_tokens)
        self.freeze_log: FreezeLog | None = None
        # The pages reserve staging for the whole (clamped) window.  A caller
        # that provides less staging gets min(provided, window): batches that
        # no longer fit are declined, exactly like an overflow.
        self.staging_capacity = effective if staging_capacity is None else \
            min(int(staging_capacity), effective)

    def is_calibrating(self) -> bool:
        return not self.state.frozen

    def scales(self):
        return (np.float32(self.state.k_scale), np.float32(self.state.v_scale))

    def restore(self, k_scale, v_scale) -> None:
        """Start frozen at scales saved from an earlier freeze.

        Not on the pages (they keep the state in memory only); this is the
        plainest extension of their state machine: a calibrator that has seen
        no batch takes the frozen branch with the given scales, which also
        stand in as the running maxima, and stages nothing."""
        if self.state.frozen or self.state.tokens_seen != 0 or self.staging.used_tokens != 0:
            raise RuntimeError("restore is only allowed before the first batch")
        k_scale, v_scale = np.float32(k_scale), np.float32(v_scale)
        if not (np.isfinite(k_scale) and np.isfinite(v_scale) and k_scale > 0 and v_scale > 0):
            raise ValueError("saved scales must be finite and positive")
        self.state.frozen = True
        self.state.k_scale, self.state.v_scale = k_scale, v_scale
        self.state.k_running_max, self.state.v_running_max = k_scale, v_scale

    def observe(self, k_bits, v_bits, num_tokens: int, num_kv_heads: int,
                head_dim: int, target: Fp8KvWriteTarget) -> str:
        if not self.state.should_observe(num_tokens):
            self.state.tokens_seen += int(num_tokens)
            return FROZEN
        e = num_kv_heads * head_dim
        k_max = core.absmax(k_bits, num_tokens, e, target.key_stride)
        v_max = core.absmax(v_bits, num_tokens, e, target.value_stride)
        step = self.state.record(k_max, v_max, num_tokens)
        if step[0] == STAGE:
            ok = self.staging.stage(k_bits, v_bits, num_tokens, e, target,
                                    self.staging_capacity)
            if not ok:
                self.unstaged_tokens += num_tokens
            return STAGE
        if step[0] == FREEZE:
            _, k_scale, v_scale, tokens_seen = step
            staged_tokens = self.staging.used_tokens
            self.staging.replay_and_release(target, num_kv_heads, head_dim,
                                            k_scale, v_scale)
            self.freeze_log = FreezeLog(
                tokens_seen=tokens_seen, requested_tokens=self.requested_tokens,
                k_scale=k_scale, k_amax=self.state.k_running_max,
                v_scale=v_scale, v_amax=self.state.v_running_max,
                headroom=self.state.headroom, staged_tokens=staged_tokens,
                staged_batches=self.state.staged_batches,
                unstaged_tokens=self.unstaged_tokens)
            return FREEZE
        return FROZEN


@dataclass
class KvBatch:
    """One batch of a layer's KV stream: bf16 bits ``[T, row_stride]`` and slots."""
    k: np.ndarray
    v: np.ndarray
    slot_mapping: np.ndarray
    key_stride: int
    value_stride: int

    @property
    def num_tokens(self) -> int:
        return int(self.slot_mapping.shape[0])


@dataclass
class CalibratedRun:
    steps: list = field(default_factory=list)
    scales_used: list = field(default_factory=list)
    out_of_range: int = 0


def run_calibrated_writes(cal: Fp8KvCalibration, batches, num_kv_heads: int,
                          head_dim: int, k_pool: np.ndarray, v_pool: np.ndarray,
                          block_size: int, cache_stride: int,
                          num_blocks: int) -> CalibratedRun:
    """The attention write path around the calibrator: observe each batch, then
    write it with reshape_and_cache_fp8 at ``scales()`` (provisional inside the
    window, frozen from the crossing batch on)."""
    run = CalibratedRun()
    for b in batches:
        target = Fp8KvWriteTarget(k_pool, v_pool, block_size, cache_stride,
                                  num_blocks, b.key_stride, b.value_stride,
                                  b.slot_mapping)
        step = cal.observe(b.k, b.v, b.num_tokens, num_kv_heads, head_dim, target)
        ks, vs = cal.scales()
        run.out_of_range += core.kv_write(b.k, b.v, b.key_stride, b.value_stride,
                                          b.slot_mapping, b.num_tokens, num_kv_heads,
                                          head_dim, k_pool, v_pool, block_size,
                                          cache_stride, num_blocks, ks, vs)
        run.steps.append(step)
        run.scales_used.append((ks, vs))
    return run


def graphs_ready_after_fp8_kv_cal(states) -> bool:
    """Per layer ``None`` (no calibrator), ``False`` (in the window) or ``True``
    (frozen); true when no layer is still inside its window."""
    return all(True if s is None else bool(s) for s in states)


def dtype_runs_online_fp8_kv_calibration(kv_dtype: str) -> bool:
    """Only an FP8 KV cache's write path observes."""
    return kv_dtype == "fp8"
