"""Host-side logic on CPU: bench.py's multi-rank aggregation (gloo, world
size 2), its reference arm's JSON contract, the per-launch slope fit and the
clock-sample window, and the all-reduce of the KV maxima for heads sharded
over ranks (gloo, world size 2)."""
import argparse
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    d = bench.Dist()
    d.init("gloo", timeout_s=60)
    d.barrier()
    seconds = 1.0 + rank          # rank 1 is the slow one
    units = 100.0 * (rank + 1)
    mx, total = bench.aggregate(d, seconds, units, torch.device("cpu"))
    out[rank] = (mx, total)
    d.close()


def test_aggregate_takes_max_time_and_total_units_over_ranks():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    assert res[0] == res[1] == (2.0, 300.0)


def test_single_process_aggregate_is_identity():
    d = bench.Dist()
    assert d.world == 1 or "WORLD_SIZE" in os.environ
    if d.world == 1:
        assert bench.aggregate(d, 3.5, 7.0, torch.device("cpu")) == (3.5, 7.0)


def test_reference_arm_only_rank_zero_reports(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    args = argparse.Namespace(steps=1, warmup=0)
    assert bench.run_reference(args) is None


def test_reference_arm_json_contract(monkeypatch):
    monkeypatch.setenv("RANK", "0")
    monkeypatch.delenv("WORLD_SIZE", raising=False)
    res = bench.run_reference(argparse.Namespace(steps=1, warmup=0))
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "cpu_baseline", "e2e", "config", "dtype"):
        assert key in res, key
    assert res["impl"] == "reference" and res["metric"] == bench.METRIC
    assert res["unit"] == "GB/s" and res["value"] > 0
    assert res["e2e"]["h2d_bytes_per_step"] == 0 and res["e2e"]["value"] == res["value"]
    assert res["cpu_baseline"]["kind"] == "oracle"


def test_algorithmic_bytes():
    assert bench.GROUP_QUANT_BYTES == 71_283_360
    assert bench.PER_TOKEN["kv_write"] == 3080
    assert bench.PER_TOKEN["observe_stage_write"] == 5136
    assert bench.launch_bytes("kv_write") == 4593 * 3080
    assert bench.launch_bytes("replay_crossing") == (4095 + 498) * 3080
    assert bench.step_bytes(16) == 71_283_360 + 16 * (4095 * 5136 + 498 * 2048 + 4095 * 3080 +
                                                      498 * 3080)
    assert len(bench.labels_of(16)) == 49


def test_launch_counts_cover_one_to_all_layers():
    assert bench.launch_counts(16) == [1, 2, 4, 8, 16]
    assert bench.launch_counts(2) == [1, 2]
    assert bench.launch_counts(1) == [1]
    assert bench.launch_counts(12) == [1, 2, 4, 8, 12]


def test_fit_line_recovers_slope_and_intercept():
    pts = {n: 5.1 + 3.25 * n for n in (1, 2, 4, 8, 16)}
    slope, icept = bench.fit_line(pts)
    assert slope == pytest.approx(3.25) and icept == pytest.approx(5.1)
    assert bench.fit_line({4: 12.0}) == (3.0, 0.0)
    # event deltas that snap up to a 2.048 us grid: over 1..16 launches the
    # slope stays within 2.048 / 15 of the true one
    tick = 2.048
    snapped = {n: tick * -(-(5.1 + 3.25 * n) // tick) for n in (1, 2, 4, 8, 16)}
    slope, _ = bench.fit_line(snapped)
    assert abs(slope - 3.25) < tick / 15


def test_clock_samples_outside_the_timed_region_are_dropped():
    smp = object.__new__(bench.NvmlClockSampler)
    smp.proc, smp.nv, smp.error, smp.max_mhz = None, object(), None, 1965
    smp.t0, smp.t1 = 10.0, 11.0
    smp.local = [(9.5, 900, 0x1, 90_000),          # before: idle clock, not counted
                 (10.2, 1965, 0x0, 600_000),
                 (10.7, 1900, 0x4, 980_000),       # sw_power_cap
                 (11.5, 800, 0x40, 100_000)]       # after: thermal, not counted
    info = smp.stop()
    assert info["samples"] == 2 and info["samples_in_process"] == 2
    assert info["sm_mhz"] == pytest.approx((1965 + 1900) / 2)
    assert info["sm_mhz_min"] == 1900 and info["power_w_max"] == 980.0
    assert info["reasons"] == ["sw_power_cap"]
    smp.local = [(9.0, 1965, 0, 1), (12.0, 1965, 0, 1)]
    assert smp.stop()["error"] == "no samples in the timed region"


def test_cli_rejects_short_warmup():
    with pytest.raises(SystemExit):
        bench.parse_args(["--warmup", "2"])


def _maxima_rank(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import types
    import torch.distributed as dist
    import paged_kv_cache_group_b200 as fp8q
    dist.init_process_group("gloo", rank=rank, world_size=world)
    # a calibrator's state layout {k_amax, v_amax, k_scale, v_scale} on the host
    cal = types.SimpleNamespace(state=torch.tensor([1.5 + rank, 7.0 - 3 * rank, 2.0, 2.0]))
    fp8q.allreduce_kv_maxima(cal)
    out[rank] = cal.state.tolist()
    dist.destroy_process_group()


def test_sharded_heads_share_the_maxima_before_the_freeze():
    world = 2
    port = _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_maxima_rank, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        res = dict(out)
    # maxima reduced, scales untouched
    assert res[0] == res[1] == [2.5, 7.0, 2.0, 2.0]
