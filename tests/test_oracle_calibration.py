"""Pins of the calibration-window oracle (no GPU).

Closed forms (token counts of the 13 + 32k batch stream, window and headroom
clamps, window 1), the freeze invariant (frozen scale >= amax / 448 over every
observed token, up to the one fp32 rounding of the division), the freeze
formula in exact arithmetic, and brute-force
replay equivalence: after the crossing batch the pools must equal "every
window batch written in arrival order at the frozen scales", which is what
chronological replay promises even when a block was freed and reused inside
the window.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import workloads
from oracle import calibration as cal
from exact_ref import round_to_f32, tensor_codes_fast


def _as_oracle_batches(batches):
    return [cal.KvBatch(b.k, b.v, b.slot_mapping, b.key_stride, b.value_stride)
            for b in batches]


def _run_window(window, headroom, batches, spec, **kw):
    c = cal.Fp8KvCalibration(0, window, headroom, **kw)
    kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
    run = cal.run_calibrated_writes(c, _as_oracle_batches(batches), spec.heads, spec.dim,
                                    kp, vp, spec.block_size, spec.cache_stride,
                                    spec.num_blocks)
    return c, run, kp, vp


def test_window_token_counts_closed_form():
    spec, batches, _ = workloads.calib_window()
    c, run, _, _ = _run_window(workloads.CALIB_WINDOW, 1.0, batches, spec)
    assert run.steps == [cal.STAGE] * 8 + [cal.FREEZE] + [cal.FROZEN] * 2
    log = c.freeze_log
    assert log.tokens_seen == 13 + 8 * 32 == 269
    assert log.staged_tokens == 13 + 7 * 32 == 237
    assert log.staged_batches == 8 and log.unstaged_tokens == 0
    # in-window writes used the provisional scale, the crossing batch and
    # everything after it the frozen one
    assert all(s == (2.0, 2.0) for s in run.scales_used[:8])
    assert all(s == (log.k_scale, log.v_scale) for s in run.scales_used[8:])
    # the one exact 600 planted in batch 3 is the K maximum
    assert log.k_amax == np.float32(600.0)
    assert log.k_scale == np.float32(np.float32(600.0) / np.float32(448.0))


def test_clamps_and_degenerate_windows():
    c = cal.Fp8KvCalibration(0, 10_000, 1.0)
    assert c.state.window_tokens == cal.MAX_STAGED_TOKENS == 4096
    assert c.requested_tokens == 10_000
    assert cal.Fp8KvCalibration(0, 300, 0.5).state.headroom == np.float32(1.0)
    assert cal.Fp8KvCalibration(0, 300, float("nan")).state.headroom == np.float32(1.0)
    assert cal.Fp8KvCalibration(0, 300, 1.5).state.headroom == np.float32(1.5)
    with pytest.raises(ValueError):
        cal.Fp8KvCalibration(0, 0, 1.0)


def test_window_of_one_freezes_on_first_observe_with_nothing_staged():
    spec, batches, _ = workloads.calib_window()
    c, run, kp, vp = _run_window(1, 1.0, batches[:3], spec)
    assert run.steps == [cal.FREEZE, cal.FROZEN, cal.FROZEN]
    assert c.freeze_log.staged_tokens == 0 and c.freeze_log.tokens_seen == 13


def test_freeze_fires_when_the_count_reaches_the_window_exactly():
    # 13 + 32 = 45 tokens: the second observe reaches a 45-token window and
    # freezes (reaching is enough, exceeding is not required)
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32))
    c, run, _, _ = _run_window(45, 1.0, batches, spec)
    assert run.steps == [cal.STAGE, cal.FREEZE, cal.FROZEN]
    assert c.freeze_log.staged_tokens == 13 and c.freeze_log.tokens_seen == 45
    c, run, _, _ = _run_window(46, 1.0, batches, spec)
    assert run.steps == [cal.STAGE, cal.STAGE, cal.FREEZE]


@pytest.mark.parametrize("headroom", [1.0, 1.25, 3.0])
def test_freeze_invariant_and_formula(headroom):
    spec, batches, _ = workloads.calib_window()
    c, run, _, _ = _run_window(workloads.CALIB_WINDOW, headroom, batches, spec)
    seen = batches[:9]                                  # through the crossing batch
    kmax = max(np.abs(oracle.bf16_to_f32(b.k[:, :spec.elems])).max() for b in seen)
    vmax = max(np.abs(oracle.bf16_to_f32(b.v[:, :spec.elems])).max() for b in seen)
    ks, vs = c.scales()
    # The pages' invariant "frozen scale >= amax / 448" holds up to the one
    # fp32 rounding of the final division: with headroom 1 the scale can sit
    # half an ulp below the exact quotient (e.g. amax 592).  What must hold
    # exactly: the scale is never below the fp32 quotient amax/448 (headroom
    # >= 1 and rounding is monotone), never below the real quotient by more
    # than one rounding, and the largest observed element encodes inside the
    # finite range (to exactly 448 when headroom is 1).
    for scale, amax in ((ks, kmax), (vs, vmax)):
        assert scale >= np.float32(np.float32(amax) / np.float32(448.0))
        assert Fraction(float(scale)) * 448 >= Fraction(float(amax)) * (1 - Fraction(1, 2 ** 24))
        code = int(oracle.e4m3_encode([np.float32(amax) / scale])[0])
        assert code <= 0x7E
        if headroom == 1.0:
            assert code == 0x7E
    h = Fraction(float(np.float32(headroom)))
    want_k = round_to_f32(max(Fraction(float(round_to_f32(Fraction(float(kmax)) * h))),
                              Fraction(1, 10 ** 12)) / 448)
    assert ks == want_k


def _bruteforce_pools(spec, batches, write_seq):
    """Replay a sequence of whole-batch writes ``(batch index, (k_scale,
    v_scale))`` slot by slot: each slot ends with its last writer, encoded at
    that write's scales."""
    last = {}
    for bi, sc in write_seq:
        b = batches[bi]
        for t in range(b.num_tokens):
            s = int(b.slot_mapping[t])
            if 0 <= s < spec.num_slots:
                last[s] = (bi, t, sc)
    kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
    e = spec.elems
    for s, (bi, t, (ks, vs)) in last.items():
        blk, off = divmod(s, spec.block_size)
        base = blk * spec.cache_stride + off * e
        kp[base:base + e] = tensor_codes_fast(oracle.bf16_to_f32(batches[bi].k[t, :e]), ks)
        vp[base:base + e] = tensor_codes_fast(oracle.bf16_to_f32(batches[bi].v[t, :e]), vs)
    return kp, vp


def test_replay_equals_writing_the_window_in_order_at_the_frozen_scale():
    spec, batches, blocks = workloads.calib_window()
    shared = set(batches[1].slot_mapping) & set(batches[5].slot_mapping)
    assert len(shared) == 16, "batches 2 and 6 must share a reused block"
    c, run, kp, vp = _run_window(workloads.CALIB_WINDOW, 1.0, batches, spec)
    frozen = c.scales()
    ek, ev = _bruteforce_pools(spec, batches, [(i, frozen) for i in range(len(batches))])
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def test_replay_with_strided_sources():
    spec, batches, _ = workloads.calib_window(row_pad=40)
    c, run, kp, vp = _run_window(workloads.CALIB_WINDOW, 1.25, batches, spec)
    ek, ev = _bruteforce_pools(spec, batches, [(i, c.scales()) for i in range(len(batches))])
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)


def test_declined_batches_keep_their_provisional_codes():
    spec, batches, _ = workloads.calib_window()
    # staging capacity 60 tokens: batches 1 (13) and 2 (32) fit, 3..8 are
    # declined; declined entries stay at the provisional scale.  The replay at
    # the freeze still rewrites batches 1 and 2 in order, so where batch 6
    # (declined) reused batch 2's block, the replayed batch 2 ends up on top:
    # the write sequence is b1..b8 at 2.0, replay b1, b2 at the frozen scale,
    # then b9..b11 at the frozen scale.
    c, run, kp, vp = _run_window(workloads.CALIB_WINDOW, 1.0, batches, spec,
                                 staging_capacity=60)
    log = c.freeze_log
    assert log.staged_tokens == 45 and log.unstaged_tokens == 237 - 45
    frozen = c.scales()
    prov = (np.float32(2.0), np.float32(2.0))
    seq = [(i, prov) for i in range(8)] + [(0, frozen), (1, frozen)] + \
        [(i, frozen) for i in range(8, 11)]
    ek, ev = _bruteforce_pools(spec, batches, seq)
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)
    # the shared block holds replayed batch 2, not declined batch 6
    shared = sorted(set(batches[1].slot_mapping) & set(batches[5].slot_mapping))
    assert len(shared) == 16
    s0 = int(shared[0])
    t2 = int(np.flatnonzero(batches[1].slot_mapping == s0)[0])
    blk, off = divmod(s0, spec.block_size)
    base = blk * spec.cache_stride + off * spec.elems
    assert np.array_equal(kp[base:base + spec.elems],
                          tensor_codes_fast(oracle.bf16_to_f32(batches[1].k[t2, :spec.elems]),
                                            frozen[0]))


def test_elems_mismatch_declines():
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32))
    c = cal.Fp8KvCalibration(0, 100, 1.0)
    kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
    ob = _as_oracle_batches(batches)
    tgt = cal.Fp8KvWriteTarget(kp, vp, 16, spec.cache_stride, spec.num_blocks,
                               512, 512, ob[0].slot_mapping)
    assert c.observe(ob[0].k, ob[0].v, 13, 4, 128, tgt) == cal.STAGE
    tgt.slot = ob[1].slot_mapping
    # the same bytes seen as 2 heads x 128: a different row size, declined
    assert c.observe(ob[1].k, ob[1].v, 32, 2, 128, tgt) == cal.STAGE
    assert c.staging.used_tokens == 13 and c.unstaged_tokens == 32


def test_graph_readiness():
    assert cal.graphs_ready_after_fp8_kv_cal([])
    assert cal.graphs_ready_after_fp8_kv_cal([None, None])
    assert cal.graphs_ready_after_fp8_kv_cal([None, True, True])
    assert not cal.graphs_ready_after_fp8_kv_cal([True, False, None])
    assert cal.dtype_runs_online_fp8_kv_calibration("fp8")
    assert not cal.dtype_runs_online_fp8_kv_calibration("bf16")


def test_restored_calibrator_writes_like_brute_force_at_the_saved_scales():
    """A calibrator restored at saved scales is frozen from its first batch:
    every batch is written once, in order, at those scales (brute force), no
    batch is staged and the maxima read back as the scales."""
    spec, batches, _ = workloads.calib_window()
    done, _, _, _ = _run_window(workloads.CALIB_WINDOW, 1.0, batches, spec)
    saved = done.scales()
    c = cal.Fp8KvCalibration(0, workloads.CALIB_WINDOW, 1.0)
    c.restore(*saved)
    kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
    run = cal.run_calibrated_writes(c, _as_oracle_batches(batches), spec.heads, spec.dim,
                                    kp, vp, spec.block_size, spec.cache_stride, spec.num_blocks)
    assert run.steps == [cal.FROZEN] * len(batches)
    ek, ev = _bruteforce_pools(spec, batches, [(i, saved) for i in range(len(batches))])
    assert np.array_equal(kp, ek) and np.array_equal(vp, ev)
    assert c.staging.used_tokens == 0 and c.freeze_log is None
    assert (c.state.k_running_max, c.state.v_running_max) == saved


def test_restore_rejects_late_calls_and_bad_scales():
    spec, batches, _ = workloads.calib_window()
    c, _, _, _ = _run_window(workloads.CALIB_WINDOW, 1.0, batches[:1], spec)
    with pytest.raises(RuntimeError):
        c.restore(1.0, 1.0)
    for bad in ((0.0, 1.0), (1.0, -2.0), (float("inf"), 1.0), (1.0, float("nan"))):
        with pytest.raises(ValueError):
            cal.Fp8KvCalibration(0, 8, 1.0).restore(*bad)
