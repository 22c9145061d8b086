"""Host-side logic on CPU: bench.py's multi-rank aggregation (gloo, world
size 2) and its reference arm's JSON contract, and the all-reduce of the KV
maxima for heads sharded over ranks (gloo, world size 2)."""
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
