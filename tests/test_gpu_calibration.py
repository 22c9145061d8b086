"""GPU parity of the calibration window (observe, staging, freeze, replay,
crossing write) against the oracle's restatement of the pages' algorithm:
the pools after every batch, the steps, the frozen scales and the counters
must all agree exactly."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_group_b200 as fp8q
import workloads
from gpu_util import dev, dev_bf16, first_mismatch, host
from oracle import calibration as cal

pytestmark = pytest.mark.gpu

STEP_NAMES = {fp8q.STEP_STAGE: cal.STAGE, fp8q.STEP_STAGE_DECLINED: cal.STAGE,
              fp8q.STEP_FREEZE: cal.FREEZE, fp8q.STEP_FROZEN: cal.FROZEN}


def _rows(bits, heads, dim):
    t, stride = bits.shape
    return dev_bf16(bits).as_strided((t, heads, dim), (stride, dim, 1))


class GpuLayer:
    """One layer's pools on the device and the calibrator, driven the way the
    attention write path drives it."""

    def __init__(self, spec, window, headroom, fused, stage_capacity=None):
        self.spec = spec
        self.fused = fused
        n = spec.num_blocks * spec.cache_stride
        self.kp = torch.full((n,), workloads.SENTINEL, dtype=torch.uint8, device="cuda")
        self.vp = torch.full((n,), workloads.SENTINEL, dtype=torch.uint8, device="cuda")
        shape = (spec.num_blocks, spec.block_size, spec.heads, spec.dim)
        self.kp4, self.vp4 = self.kp.view(shape), self.vp.view(shape)
        self.cal = fp8q.KvCalibration(window, headroom, spec.heads, spec.dim, "cuda",
                                      stage_capacity=stage_capacity)

    def step(self, b):
        k, v = _rows(b.k, self.spec.heads, self.spec.dim), _rows(b.v, self.spec.heads, self.spec.dim)
        slots = dev(b.slot_mapping)
        if self.fused:
            return self.cal.observe_write(k, v, slots, self.kp4, self.vp4)
        step = self.cal.observe(k, v, slots)
        if step == fp8q.STEP_FREEZE:
            self.cal.freeze_replay(self.kp4, self.vp4)
        fp8q.fp8_kv_write(k, v, slots, self.kp4, self.vp4, scale_dev=self.cal.scale_dev)
        return step


def _oracle_layer(spec, window, headroom, stage_capacity=None):
    c = cal.Fp8KvCalibration(0, window, headroom, staging_capacity=stage_capacity)
    kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
    return c, kp, vp


def _run_both(spec, batches, window, headroom, fused, stage_capacity=None, check_every=True,
              launches=None):
    """Drive the GPU layer and the oracle with the same batches; the pools must
    agree after every batch (or after the last).  ``launches``, if a list,
    receives the number of kernels the library launched for each batch."""
    g = GpuLayer(spec, window, headroom, fused, stage_capacity)
    c, kp, vp = _oracle_layer(spec, window, headroom, stage_capacity)
    steps = []
    for i, b in enumerate(batches):
        before = fp8q.launch_count()
        gs = g.step(b)
        if launches is not None:
            launches.append(fp8q.launch_count() - before)
        run = cal.run_calibrated_writes(
            c, [cal.KvBatch(b.k, b.v, b.slot_mapping, b.key_stride, b.value_stride)],
            spec.heads, spec.dim, kp, vp, spec.block_size, spec.cache_stride, spec.num_blocks)
        assert STEP_NAMES[gs] == run.steps[0], (i, gs, run.steps[0])
        steps.append(gs)
        if check_every or i == len(batches) - 1:
            gk, gv = host(g.kp), host(g.vp)
            assert np.array_equal(gk, kp), f"batch {i}: " + first_mismatch(gk, kp)
            assert np.array_equal(gv, vp), f"batch {i}: " + first_mismatch(gv, vp)
    return g, c, steps


def _assert_frozen_state(g, c):
    ka, va, ks, vs = g.cal.read_state()
    assert np.float32(ka) == c.state.k_running_max and np.float32(va) == c.state.v_running_max
    assert (np.float32(ks), np.float32(vs)) == c.scales()
    st = g.cal.stats()
    log = c.freeze_log
    assert st["state"] == 2
    assert st["freeze_tokens"] == log.tokens_seen
    assert st["replayed_tokens"] == log.staged_tokens
    assert st["staged_batches"] == log.staged_batches
    assert st["unstaged_tokens"] == log.unstaged_tokens
    assert st["window_tokens"] == c.state.window_tokens
    assert st["requested_tokens"] == c.requested_tokens


@pytest.mark.parametrize("fused", [False, True])
def test_calibration_window_workload(fused):
    spec, batches, _ = workloads.calib_window()
    g, c, steps = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.0, fused)
    assert steps == [fp8q.STEP_STAGE] * 8 + [fp8q.STEP_FREEZE] + [fp8q.STEP_FROZEN] * 2
    _assert_frozen_state(g, c)
    assert g.cal.read_state()[2] == np.float32(np.float32(600.0) / np.float32(448.0))


@pytest.mark.parametrize("fused", [False, True])
def test_strided_sources_and_headroom(fused):
    spec, batches, _ = workloads.calib_window(row_pad=40)
    g, c, _ = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.25, fused)
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_declined_batches(fused):
    spec, batches, _ = workloads.calib_window()
    g, c, steps = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.0, fused, stage_capacity=60)
    assert steps[:8] == [fp8q.STEP_STAGE] * 2 + [fp8q.STEP_STAGE_DECLINED] * 6
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_whole_window_replay_with_the_crossing_batch_on_a_block_of_the_last_staged_batch(fused):
    # batch 9 reaches the window and receives batch 8's second block: the
    # replay of batch 8 and the crossing write touch the same 16 slots.  237
    # staged rows and 32 crossing rows fit one launch, which writes every slot
    # from its last writer (the crossing rows come last).
    spec, batches, _ = workloads.calib_window(recycle={6: (2, 1), 9: (8, 1)})
    shared = set(batches[7].slot_mapping) & set(batches[8].slot_mapping)
    assert len(shared) == 16
    launches = []
    g, c, steps = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.0, fused, launches=launches)
    assert steps[8] == fp8q.STEP_FREEZE
    # fused: absmax + the whole-window launch; unfused: absmax, whole-window
    # replay, then the crossing batch's own write
    assert launches[8] == (2 if fused else 3)
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_whole_window_replay_in_a_pool_above_the_bitmap_limit(fused):
    # the same window and block reuse in a pool of 19200 blocks (307200 slots,
    # above the 2^18 slots of a crossing bitmap); the whole-window launch keys
    # its last-writer table by slot whatever the pool size
    spec, batches, _ = workloads.calib_window(recycle={6: (2, 1), 9: (8, 1)})
    big = workloads.PoolSpec(19200, spec.block_size, spec.heads, spec.dim)
    assert big.num_slots > 2 ** 18
    shift = 19000 * spec.block_size
    moved = [workloads.KvBatchInput(b.k, b.v, b.slot_mapping + shift, b.key_stride,
                                    b.value_stride) for b in batches]
    launches = []
    g, c, steps = _run_both(big, moved, workloads.CALIB_WINDOW, 1.0, fused, check_every=False,
                            launches=launches)
    assert steps[8] == fp8q.STEP_FREEZE
    assert launches[8] == (2 if fused else 3)
    _assert_frozen_state(g, c)


def _large_window(num_blocks, crossing=2000):
    """Two staged batches of 1000 and 1500 tokens (2500 staged rows, more than
    one whole-window launch takes) and a batch of ``crossing`` tokens that
    reaches the 2501-token window; its first block is the sixth block of batch
    2, so the last staged batch and the crossing batch share 16 slots."""
    spec, batches, blocks = workloads.calib_window(batch_sizes=(1000, 1500, crossing),
                                                   recycle={3: (2, 5)}, num_blocks=num_blocks)
    shared = set(batches[1].slot_mapping) & set(batches[2].slot_mapping)
    assert len(shared) == 16
    return spec, batches


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("crossing", [500, 2000])
def test_merged_launch_skips_staged_rows_the_crossing_batch_rewrites(fused, crossing):
    """Per-batch replay with the crossing batch merged into the last staged
    batch's launch: the 16 staged rows whose slots the crossing batch writes
    must not land on top of it ("last writer wins", staging.rs module doc).
    500 crossing rows: each staged row's warp compares its slot with the
    crossing slots; 2000: the crossing slots as a bitmap over the 8192-slot
    pool."""
    spec, batches = _large_window(512, crossing)
    assert spec.num_slots <= 2 ** 18
    launches = []
    g, c, steps = _run_both(spec, batches, 2501, 1.0, fused, launches=launches)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_STAGE, fp8q.STEP_FREEZE]
    # fused: absmax, batch 1's replay, batch 2's replay merged with the
    # crossing batch; unfused: absmax, two replays, the crossing write
    assert launches[2] == (3 if fused else 4)
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_merged_launch_hash_set_in_a_pool_above_the_bitmap_limit(fused):
    """The same window in a pool of 19200 blocks (307200 slots): the merged
    launch keeps the crossing slots in its shared-memory hash set."""
    spec, batches = _large_window(19200)
    assert spec.num_slots > 2 ** 18
    launches = []
    g, c, steps = _run_both(spec, batches, 2501, 1.0, fused, check_every=False,
                            launches=launches)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_STAGE, fp8q.STEP_FREEZE]
    assert launches[2] == (3 if fused else 4)
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_window_of_4096_tokens_in_32_token_batches(fused):
    """A decode-like window: 127 staged batches of 32 tokens (4064 rows), the
    128th batch reaches 4096, two more follow at the frozen scale.  Batch 10's
    second block is freed and re-allocated to batch 64, and the crossing batch
    receives batch 127's first block.  The replay is one launch per staged
    batch, in arrival order, the last one merged with the crossing batch."""
    spec, batches, _ = workloads.calib_window(batch_sizes=(32,) * 130,
                                              recycle={64: (10, 1), 128: (127, 0)},
                                              num_blocks=512)
    assert len(set(batches[9].slot_mapping) & set(batches[63].slot_mapping)) == 16
    assert len(set(batches[126].slot_mapping) & set(batches[127].slot_mapping)) == 16
    launches = []
    g, c, steps = _run_both(spec, batches, 4096, 1.0, fused, launches=launches)
    assert steps == [fp8q.STEP_STAGE] * 127 + [fp8q.STEP_FREEZE] + [fp8q.STEP_FROZEN] * 2
    assert launches[127] == (1 + 127 if fused else 1 + 127 + 1)
    assert g.cal.stats()["replayed_batches"] == 127
    assert g.cal.stats()["replayed_tokens"] == 4064
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_whole_window_replay_with_a_block_written_four_times(fused):
    # batch 1's block goes to batch 4, then to batch 7, then to the crossing
    # batch 9: four writers of the same slots across the window.  The staged
    # batches and the crossing batch replay in one launch, where each slot must
    # end with its last writer.
    spec, batches, blocks = workloads.calib_window(recycle={4: (1, 0), 7: (4, 0), 9: (7, 0)})
    assert blocks[0][0] == blocks[3][0] == blocks[6][0] == blocks[8][0]
    launches = fp8q.launch_count()
    g, c, steps = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.0, fused)
    assert steps == [fp8q.STEP_STAGE] * 8 + [fp8q.STEP_FREEZE] + [fp8q.STEP_FROZEN] * 2
    if fused:   # init, 8 in-window passes, absmax + one replay, 2 frozen writes
        assert fp8q.launch_count() - launches == 1 + 8 + 2 + 2
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_whole_window_replay_then_a_crossing_batch_above_the_merge_limit(fused):
    # two staged batches of 1000 tokens replay in one launch (no crossing rows
    # in it); the 9000-token batch that reaches the 2048-token window is too
    # large to merge and gets its own launch after the scales are published
    spec = workloads.large_kv_spec()
    full = workloads.large_kv_layer(12, tokens=11000)
    chunks = workloads.split_batch(full, (1000, 1000, 9000))
    g, c, steps = _run_both(spec, chunks, 2048, 1.0, fused, check_every=False)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_STAGE, fp8q.STEP_FREEZE]
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_crossing_batch_larger_than_one_merged_launch(fused):
    # 9000 tokens reach a 1-token window at once: above the merge limit, the
    # crossing batch gets a launch of its own after the scales are published
    spec = workloads.large_kv_spec()
    big = workloads.large_kv_layer(5, tokens=9000)
    g, c, steps = _run_both(spec, [big], 1, 1.0, fused, check_every=True)
    assert steps == [fp8q.STEP_FREEZE]
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
def test_window_of_one_and_exact_window(fused):
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32))
    g, c, steps = _run_both(spec, batches, 1, 0.5, fused)
    assert steps == [fp8q.STEP_FREEZE, fp8q.STEP_FROZEN, fp8q.STEP_FROZEN]
    _assert_frozen_state(g, c)
    g, c, steps = _run_both(spec, batches, 45, 1.0, fused)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_FREEZE, fp8q.STEP_FROZEN]
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("layer", [0, 7])
def test_large_prefill_chunked_replay(fused, layer):
    """4095 staged tokens (the cap), then the 498-token crossing chunk."""
    spec = workloads.large_kv_spec()
    full = workloads.large_kv_layer(layer)
    chunks = workloads.split_batch(full, workloads.LARGE_CHUNKS)
    g, c, steps = _run_both(spec, chunks, workloads.LARGE_WINDOW_REQUEST, 1.0, fused,
                            check_every=False)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_FREEZE]
    _assert_frozen_state(g, c)
    assert g.cal.stats()["replayed_tokens"] == 4095
    assert g.cal.stats()["window_tokens"] == 4096


@pytest.mark.parametrize("fused", [False, True])
def test_large_prefill_single_chunk_freezes_at_once(fused):
    spec = workloads.large_kv_spec()
    full = workloads.large_kv_layer(3)
    g, c, steps = _run_both(spec, [full], workloads.LARGE_WINDOW_REQUEST, 1.0, fused)
    assert steps == [fp8q.STEP_FREEZE]
    assert g.cal.stats()["replayed_tokens"] == 0
    _assert_frozen_state(g, c)


@pytest.mark.parametrize("fused", [False, True])
@pytest.mark.parametrize("heads,dim", [(2, 64), (8, 128)])
def test_calibration_window_with_other_row_widths(fused, heads, dim):
    """Rows of 128 and 1024 elements take the general passes (the workload's
    512-element rows have kernels of their own): the in-window pass, the
    whole-window replay, and the merged launch of one staged batch with the
    crossing batch."""
    spec, batches, _ = workloads.calib_window(heads=heads, dim=dim)
    g, c, steps = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.0, fused)
    assert steps == [fp8q.STEP_STAGE] * 8 + [fp8q.STEP_FREEZE] + [fp8q.STEP_FROZEN] * 2
    _assert_frozen_state(g, c)
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32), heads=heads, dim=dim)
    launches = []
    g, c, steps = _run_both(spec, batches, 20, 1.0, fused, launches=launches)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_FREEZE, fp8q.STEP_FROZEN]
    # fused: absmax + the merged launch; unfused: absmax, replay, crossing write
    assert launches[1] == (2 if fused else 3)
    _assert_frozen_state(g, c)


def test_zero_token_observe_counts_a_stage_step():
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32))
    empty = workloads.KvBatchInput(batches[0].k[:0], batches[0].v[:0],
                                   batches[0].slot_mapping[:0], 512, 512)
    g, c, steps = _run_both(spec, [batches[0], empty, batches[1]], 40, 1.0, fused=False)
    assert steps == [fp8q.STEP_STAGE, fp8q.STEP_STAGE, fp8q.STEP_FREEZE]
    _assert_frozen_state(g, c)


def test_calls_out_of_order_are_rejected():
    spec, batches, _ = workloads.calib_window(batch_sizes=(13, 32, 32))
    g = GpuLayer(spec, 40, 1.0, fused=False)
    b0, b1 = batches[0], batches[1]
    with pytest.raises(fp8q.Fp8qError) as ei:
        g.cal.freeze_replay(g.kp4, g.vp4)          # nothing pending
    assert ei.value.status == -3
    k, v = _rows(b0.k, 4, 128), _rows(b0.v, 4, 128)
    assert g.cal.observe(k, v, dev(b0.slot_mapping)) == fp8q.STEP_STAGE
    k, v = _rows(b1.k, 4, 128), _rows(b1.v, 4, 128)
    assert g.cal.observe(k, v, dev(b1.slot_mapping)) == fp8q.STEP_FREEZE
    with pytest.raises(fp8q.Fp8qError) as ei:
        g.cal.observe(k, v, dev(b1.slot_mapping))   # replay still pending
    assert ei.value.status == -3
    assert g.cal.freeze_replay(g.kp4, g.vp4) == 13
    assert g.cal.observe(k, v, dev(b1.slot_mapping)) == fp8q.STEP_FROZEN


def test_post_freeze_write_in_a_cuda_graph():
    """After the freeze the write reads its scales from the device, so a graph
    captured once keeps writing at whatever the calibrator published."""
    spec, batches, _ = workloads.calib_window()
    g = GpuLayer(spec, workloads.CALIB_WINDOW, 1.0, fused=False)
    for b in batches[:9]:
        g.step(b)
    b = batches[9]
    k, v = _rows(b.k, 4, 128), _rows(b.v, 4, 128)
    slots = dev(b.slot_mapping)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        fp8q.fp8_kv_write(k, v, slots, g.kp4, g.vp4, scale_dev=g.cal.scale_dev, stream=s)
        torch.cuda.synchronize()
        with torch.cuda.graph(graph, stream=s):
            fp8q.fp8_kv_write(k, v, slots, g.kp4, g.vp4, scale_dev=g.cal.scale_dev, stream=s)
    eager = host(g.kp).copy()
    # replay the graph into pools reset to the sentinel: exactly batch 10's
    # entries come back, equal to the eager write
    g.kp.fill_(workloads.SENTINEL)
    g.vp.fill_(workloads.SENTINEL)
    graph.replay()
    torch.cuda.synchronize()
    got = host(g.kp)
    mask = np.zeros(got.size, bool)
    for slot in b.slot_mapping:
        blk, off = divmod(int(slot), spec.block_size)
        base = blk * spec.cache_stride + off * spec.elems
        mask[base:base + spec.elems] = True
    assert np.array_equal(got[mask], eager[mask])
    assert np.all(got[~mask] == workloads.SENTINEL)
    del graph


def test_saved_scales_restore_a_frozen_calibrator(tmp_path):
    """Calibrate, save the frozen scales to a file, restore them into a fresh
    calibrator (as after a restart) and write the whole window again: every
    batch is FROZEN and the pools equal the oracle's restored calibrator."""
    spec, batches, _ = workloads.calib_window()
    g, c, _ = _run_both(spec, batches, workloads.CALIB_WINDOW, 1.0, True, check_every=False)
    path = str(tmp_path / "scales.json")
    fp8q.save_scales([g.cal], path)
    (ks, vs), = fp8q.load_scales(path)
    assert (np.float32(ks), np.float32(vs)) == c.scales()

    fresh = GpuLayer(spec, workloads.CALIB_WINDOW, 1.0, fused=True)
    fresh.cal.restore(ks, vs)
    oc, kp, vp = _oracle_layer(spec, workloads.CALIB_WINDOW, 1.0)
    oc.restore(ks, vs)
    assert fresh.cal.stats()["state"] == 2
    assert [fresh.step(b) for b in batches] == [fp8q.STEP_FROZEN] * len(batches)
    cal.run_calibrated_writes(oc, [cal.KvBatch(b.k, b.v, b.slot_mapping, b.key_stride,
                                               b.value_stride) for b in batches],
                              spec.heads, spec.dim, kp, vp, spec.block_size, spec.cache_stride,
                              spec.num_blocks)
    gk, gv = host(fresh.kp), host(fresh.vp)
    assert np.array_equal(gk, kp), first_mismatch(gk, kp)
    assert np.array_equal(gv, vp), first_mismatch(gv, vp)
    ka, va, rks, rvs = fresh.cal.read_state()
    assert (np.float32(ka), np.float32(va)) == (oc.state.k_running_max, oc.state.v_running_max)
    assert (np.float32(rks), np.float32(rvs)) == oc.scales()
    # restoring is only allowed before the first observe
    with pytest.raises(fp8q.Fp8qError) as ei:
        g.cal.restore(ks, vs)
    assert ei.value.status == -3
    fresh.cal.close()


def test_unfused_freeze_with_the_maxima_allreduce_on_one_rank():
    """observe -> allreduce_kv_maxima (NCCL, one rank) -> freeze_replay, on the
    device state: the pools equal the oracle's, as without the all-reduce."""
    import socket
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1)
    try:
        spec, batches, _ = workloads.calib_window()
        g = GpuLayer(spec, workloads.CALIB_WINDOW, 1.0, fused=False)
        c, kp, vp = _oracle_layer(spec, workloads.CALIB_WINDOW, 1.0)
        for b in batches:
            k, v = _rows(b.k, spec.heads, spec.dim), _rows(b.v, spec.heads, spec.dim)
            slots = dev(b.slot_mapping)
            step = g.cal.observe(k, v, slots)
            if step == fp8q.STEP_FREEZE:
                fp8q.allreduce_kv_maxima(g.cal)
                g.cal.freeze_replay(g.kp4, g.vp4)
            fp8q.fp8_kv_write(k, v, slots, g.kp4, g.vp4, scale_dev=g.cal.scale_dev)
            cal.run_calibrated_writes(c, [cal.KvBatch(b.k, b.v, b.slot_mapping, b.key_stride,
                                                      b.value_stride)],
                                      spec.heads, spec.dim, kp, vp, spec.block_size,
                                      spec.cache_stride, spec.num_blocks)
        gk, gv = host(g.kp), host(g.vp)
        assert np.array_equal(gk, kp), first_mismatch(gk, kp)
        assert np.array_equal(gv, vp), first_mismatch(gv, vp)
        _assert_frozen_state(g, c)
    finally:
        dist.destroy_process_group()
