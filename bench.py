#!/usr/bin/env python
"""Benchmark of the FP8 E4M3 quantization hot path on B200.

One step is one 4593-token prefill through every operation of the path:
  * fp8_group_quant of the 4593 x 5120 bf16 activation (1x128 groups);
  * for each of 16 layers (4 KV heads x 128 dims, 8192-block pools of 16
    slots), the calibrating KV write of that layer's 4593 tokens, arriving in
    two chunks through fp8_kv_calib_observe_write: 4095 tokens inside the
    window (one fused pass: absmax, staging copy, provisional-scale write),
    then 498 tokens that reach the 4096-token window (absmax, then one launch
    that freezes the scales, replays the 4095 staged tokens and writes the
    crossing chunk at the frozen scale).
That is 1 + 16 x 3 = 49 kernel launches, issued through the C ABI and
replayed as one CUDA graph.  Before every step L2 is flushed (a 2x-L2 write,
then a 2x-L2 read of a clean buffer) and the calibrators' device state is
reset, both outside the timed region.

`value` is effective HBM GB/s: the algorithmic bytes of the step (each
kernel's compulsory reads and writes) divided by the step time measured with
CUDA events.  Per-kernel times come from graphs of 1, 2, 4, 8 and 16 of each
kernel's launches as the step issues them (one per layer, back to back),
timed the same way: the per-launch time is the slope of graph time against
launches, which leaves out the fixed cost of timing a graph between events.
`--impl reference` times the CPU oracle on a bounded sample of the same step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "FP8 quant/KV-write effective HBM GB/s and % of B200 peak; tokens/s"
TOKENS = workloads.LARGE_TOKENS          # 4593
CHUNK1, CHUNK2 = workloads.LARGE_CHUNKS  # 4095, 498
E = workloads.KV_HEADS * workloads.HEAD_DIM
M, K = workloads.PREFILL_M, workloads.PREFILL_K

# Algorithmic bytes per launch (compulsory reads + writes of each kernel).
PER_TOKEN = {
    "observe_stage_write": 2 * E * 2 + 8 + 2 * E + 2 * E * 2 + 8,   # 5136
    "amax": 2 * E * 2,                                             # 2048
    "replay_crossing": 2 * E * 2 + 8 + 2 * E,                      # 3080, staged and crossing
    "kv_write": 2 * E * 2 + 8 + 2 * E,                             # 3080
}
STEP_KERNELS = ("observe_stage_write", "amax", "replay_crossing")
GROUP_QUANT_BYTES = M * K * 3 + M * (K // 128) * 4                 # 71,283,360


def launch_bytes(label: str) -> int:
    if label == "group_quant":
        return GROUP_QUANT_BYTES
    tokens = {"observe_stage_write": CHUNK1, "amax": CHUNK2, "replay_crossing": CHUNK1 + CHUNK2,
              "kv_write": TOKENS}[label]
    return PER_TOKEN[label] * tokens


def step_bytes(layers: int) -> int:
    per_layer = sum(launch_bytes(k) for k in STEP_KERNELS)
    return GROUP_QUANT_BYTES + layers * per_layer


# ---------------------------------------------------------------------------
# process group plumbing (one process per GPU; no data-path collective)


class Dist:
    def __init__(self) -> None:
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = False

    def init(self, backend: str, timeout_s: float = 120.0) -> None:
        if self.world > 1 and not torch.distributed.is_initialized():
            import datetime
            os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
            kw = {}
            if backend == "nccl":
                kw["device_id"] = torch.device("cuda", self.local_rank)
            torch.distributed.init_process_group(
                backend, rank=self.rank, world_size=self.world,
                timeout=datetime.timedelta(seconds=timeout_s), **kw)
            self.pg = True

    def barrier(self) -> None:
        if self.pg:
            torch.distributed.barrier()

    def reduce(self, value: float, op: str, device) -> float:
        if not self.pg:
            return value
        t = torch.tensor([value], dtype=torch.float64, device=device)
        torch.distributed.all_reduce(
            t, op=torch.distributed.ReduceOp.MAX if op == "max" else torch.distributed.ReduceOp.SUM)
        return float(t.item())

    def close(self) -> None:
        if self.pg:
            torch.distributed.destroy_process_group()
            self.pg = False


def aggregate(dist: Dist, seconds: float, units: float, device) -> tuple[float, float]:
    """Whole-job (max seconds over ranks, total units over ranks)."""
    return dist.reduce(seconds, "max", device), dist.reduce(units, "sum", device)


# ---------------------------------------------------------------------------
# clocks during the timed region


def smi_gpu_id(local_rank: int) -> str:
    """nvidia-smi's id of this rank's GPU (CUDA_VISIBLE_DEVICES may remap)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    ids = [v.strip() for v in vis.split(",") if v.strip()]
    return ids[local_rank] if local_rank < len(ids) else str(local_rank)


class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, gpu_index: str) -> None:
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        try:
            fd, self.path = tempfile.mkstemp(prefix="fp8q_clocks_", suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, ValueError):
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"error": "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as fh:
            for line in fh:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) != 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), parts[5:9]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return {"error": "no samples", "samples": 0}
        reasons = sorted({self.REASONS[i] for _, _, flags in rows
                          for i, f in enumerate(flags) if f.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows),
                "sm_max_mhz": max(r[1] for r in rows), "reasons": reasons,
                "samples": len(rows), "window": "warm-up and timed steps"}


NVML_POLLER = r"""
import signal, sys, time
import pynvml as nv
signal.signal(signal.SIGTERM, lambda *a: sys.exit(0))
nv.nvmlInit()
h = nv.nvmlDeviceGetHandleByUUID(sys.argv[1])
end = time.monotonic() + float(sys.argv[3])
with open(sys.argv[2], "w") as out:
    print("max", nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM), flush=True)
    while time.monotonic() < end:
        t = time.monotonic()
        try:
            out.write(f"{t} {nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)} "
                      f"{nv.nvmlDeviceGetCurrentClocksEventReasons(h)} "
                      f"{nv.nvmlDeviceGetPowerUsage(h)}\n")
        except nv.NVMLError as exc:
            print("nvml", exc, file=sys.stderr, flush=True)
        time.sleep(0.0002)
"""


class NvmlClockSampler:
    """SM clock, power and clock-event reasons of this rank's GPU, polled about
    every 0.2 ms by a separate process (so the polling never waits for this
    process's interpreter) and time-stamped on the host's monotonic clock; the
    samples inside [mark_start, mark_end] are the timed region's.  A timed
    region of a few milliseconds still gets samples, which a 100 ms
    nvidia-smi period misses.  sample_now() adds one query from this process;
    the timed loop calls it after enqueuing each step, while the GPU runs it,
    so the region has samples even when the poller is starved of CPU time."""

    REASONS = (("gpu_idle", 0x1), ("applications_clocks_setting", 0x2),
               ("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sync_boost", 0x10),
               ("sw_thermal_slowdown", 0x20), ("hw_thermal_slowdown", 0x40),
               ("hw_power_brake_slowdown", 0x80), ("display_clock_setting", 0x100))

    def __init__(self, device, max_seconds: float = 600.0) -> None:
        self.t0 = self.t1 = None
        self.proc = None
        self.error = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            fd, self.path = tempfile.mkstemp(prefix="fp8q_nvml_", suffix=".txt")
            os.close(fd)
            self.proc = subprocess.Popen(
                [sys.executable, "-c", NVML_POLLER, uuid, self.path, str(max_seconds)],
                stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True)
            first = self.proc.stdout.readline().split()   # waits until NVML is up
            if len(first) != 2 or first[0] != "max":
                raise RuntimeError("NVML poller did not start: " + self.proc.stderr.read()[-300:])
            self.max_mhz = int(first[1])
        except Exception as exc:
            self.error = f"{type(exc).__name__}: {exc}"
            if self.proc is not None:
                self.proc.kill()
            self.proc = None
        # the same query from this process, once per timed step while the GPU
        # works on it, so the region has samples even when the poller process
        # is not scheduled in time on a busy host
        self.local = []
        self.nv = self.handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByUUID(
                "GPU-" + str(torch.cuda.get_device_properties(device).uuid))
            if self.proc is None:
                self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as exc:
            self.nv = None
            self.error = (self.error or "") + f" in-process NVML: {type(exc).__name__}: {exc}"

    def sample_now(self) -> None:
        """One sample from this process (called while a timed step runs)."""
        if self.nv is None:
            return
        nv, h = self.nv, self.handle
        try:
            self.local.append((time.monotonic(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                               nv.nvmlDeviceGetCurrentClocksEventReasons(h),
                               nv.nvmlDeviceGetPowerUsage(h)))
        except Exception:
            pass

    def mark_start(self) -> None:
        self.t0 = time.monotonic()

    def mark_end(self) -> None:
        self.t1 = time.monotonic()

    def stop(self) -> dict:
        lines, stderr = [], ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                _, stderr = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                _, stderr = self.proc.communicate()
            with open(self.path) as fh:
                lines = fh.read().splitlines()
            os.unlink(self.path)
        if self.proc is None and self.nv is None:
            return {"error": self.error or "NVML unavailable"}

        def inside(t):
            return self.t0 is not None and self.t1 is not None and self.t0 <= t <= self.t1

        rows, poller_rows, poller_total = [], 0, 0
        for line in lines:
            parts = line.split()
            if len(parts) != 4:
                continue
            try:
                t, sm, r, pw = float(parts[0]), int(parts[1]), int(parts[2]), float(parts[3])
            except ValueError:
                continue
            poller_total += 1
            if inside(t):
                rows.append((sm, r, pw / 1e3))
                poller_rows += 1
        local_rows = 0
        for t, sm, r, pw in self.local:
            if inside(t):
                rows.append((sm, r, pw / 1e3))
                local_rows += 1
        if not rows:
            return {"error": "no samples in the timed region", "samples": 0,
                    "poller_samples_total": poller_total,
                    "poller_stderr": (stderr or "")[-300:], "note": self.error}
        mask = 0
        for _, r, _ in rows:
            mask |= r
        return {"sm_mhz": statistics.median(c for c, _, _ in rows), "sm_max_mhz": self.max_mhz,
                "sm_mhz_min": min(c for c, _, _ in rows),
                "power_w_max": round(max(p for _, _, p in rows), 1),
                "reasons": [name for name, bit in self.REASONS if mask & bit],
                "samples": len(rows), "samples_poller": poller_rows,
                "samples_in_process": local_rows,
                "timed_region_s": round(self.t1 - self.t0, 4),
                "window": ("timed steps only: NVML polled every ~0.2 ms by a separate process, "
                           "plus one in-process query per step while the GPU runs it")}


# ---------------------------------------------------------------------------
# the native step


class Workload:
    """Device-resident inputs, outputs, pools and calibrator state of one step."""

    def __init__(self, device, layers: int, flush: bool = True) -> None:
        import paged_kv_cache_group_b200 as fp8q
        self.fp8q = fp8q
        self.device = device
        self.layers = layers
        self.host_x = workloads.prefill_quant()
        self.host_kv = [workloads.large_kv_layer(l) for l in range(layers)]
        self.x = self._bf16(self.host_x)
        self.q = torch.empty((M, K), dtype=torch.uint8, device=device)
        self.s = torch.empty((M, K // 128), dtype=torch.float32, device=device)
        shape = (workloads.LARGE_NUM_BLOCKS, 16, workloads.KV_HEADS, workloads.HEAD_DIM)
        self.k, self.v, self.slots, self.k_pool, self.v_pool = [], [], [], [], []
        for b in self.host_kv:
            self.k.append(self._bf16(b.k).view(TOKENS, workloads.KV_HEADS, workloads.HEAD_DIM))
            self.v.append(self._bf16(b.v).view(TOKENS, workloads.KV_HEADS, workloads.HEAD_DIM))
            self.slots.append(torch.from_numpy(b.slot_mapping).to(device))
            self.k_pool.append(torch.full(shape, workloads.SENTINEL, dtype=torch.uint8, device=device))
            self.v_pool.append(torch.full(shape, workloads.SENTINEL, dtype=torch.uint8, device=device))
        self.states = torch.zeros((layers, 4), dtype=torch.float32, device=device)
        self.states_init = torch.tensor([0.0, 0.0, 2.0, 2.0], device=device).repeat(layers, 1)
        l2 = torch.cuda.get_device_properties(device).L2_cache_size if flush else 16
        self.flush_buf = torch.empty(2 * l2, dtype=torch.uint8, device=device)
        self.flush_read = torch.ones(2 * l2, dtype=torch.uint8, device=device)

    def _bf16(self, bits):
        t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
        return t.view(torch.bfloat16).to(self.device)

    def calibrators(self):
        fp8q = self.fp8q
        return [fp8q.KvCalibration(workloads.LARGE_WINDOW_REQUEST, 1.0, workloads.KV_HEADS,
                                   workloads.HEAD_DIM, self.device, state=self.states[l])
                for l in range(self.layers)]

    def flush(self, i: int) -> None:
        """Write 2x L2, then read another 2x L2 that is never written: L2 ends
        up holding only clean lines of a buffer no kernel uses, so the timed
        kernels neither hit in L2 nor pay for write-backs of dirty lines."""
        self.flush_buf.fill_(i & 0xFF)
        self._sink = torch.amax(self.flush_read)

    def reset(self, i: int) -> None:
        self.states.copy_(self.states_init)
        self.flush(i)

    def issue(self, calibs) -> None:
        fp8q = self.fp8q
        fp8q.fp8_group_quant(self.x, self.q, self.s)
        for l, c in enumerate(calibs):
            k, v, s = self.k[l], self.v[l], self.slots[l]
            kp, vp = self.k_pool[l], self.v_pool[l]
            st = c.observe_write(k[:CHUNK1], v[:CHUNK1], s[:CHUNK1], kp, vp)
            assert st == fp8q.STEP_STAGE, st
            st = c.observe_write(k[CHUNK1:], v[CHUNK1:], s[CHUNK1:], kp, vp)
            assert st == fp8q.STEP_FREEZE, st


def labels_of(layers: int) -> list[str]:
    return ["group_quant"] + list(STEP_KERNELS) * layers


def capture(w: Workload, stream):
    """Capture one step into a CUDA graph (no event nodes: they would break
    the programmatic overlap of consecutive launches)."""
    labels = labels_of(w.layers)
    with torch.cuda.stream(stream):
        calibs = w.calibrators()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    before = w.fp8q.launch_count()
    with torch.cuda.graph(graph, stream=stream):
        w.issue(calibs)
    launches = w.fp8q.launch_count() - before
    # The graph writes into these calibrators' staging tensors on every
    # replay: the caller keeps them alive as long as the graph.
    return graph, labels, launches, calibs


def time_graph(w: Workload, stream, graph, reps: int, reset_state: bool,
               during=None) -> list[float]:
    """Event time of each of reps replays, L2 flushed (and the calibrator
    state reset when reset_state) before each; during() runs on the host
    after each replay is enqueued, while the GPU works on it."""
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = []
    with torch.cuda.stream(stream):
        for i in range(reps):
            if reset_state:
                w.reset(i)
            else:
                w.flush(i)
            start.record()
            graph.replay()
            end.record()
            if during is not None:
                during()
            end.synchronize()
            out.append(start.elapsed_time(end))
    return out


def drained_step_ms(w: Workload, stream, graph, reps: int) -> float:
    """Step time with the write-back of its dirty L2 lines included.  The step
    leaves up to an L2's worth of written lines dirty; the untimed flush before
    the next step writes them back.  Here each step is followed, inside the
    timed region, by a read of a clean 2x-L2 buffer that evicts them, and the
    same read after a clean L2 (no dirty lines) is subtracted."""
    drain = torch.ones_like(w.flush_read)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with_wb, without = [], []
    with torch.cuda.stream(stream):
        for i in range(reps):
            w.reset(i)
            start.record()
            graph.replay()
            sink = torch.amax(drain)
            end.record()
            end.synchronize()
            with_wb.append(start.elapsed_time(end))
            w.reset(i)
            start.record()
            sink = torch.amax(drain)
            end.record()
            end.synchronize()
            without.append(start.elapsed_time(end))
    del drain, sink
    return statistics.median(with_wb) - statistics.median(without)


def launch_counts(layers: int) -> list[int]:
    """Graph sizes (launches per kernel) over which per-launch times are fitted."""
    return sorted({n for n in (1, 2, 4, 8, layers) if 1 <= n <= layers})


def fit_line(points: dict) -> tuple[float, float]:
    """Least-squares line through {n: t}: (slope, intercept)."""
    ns = list(points)
    if len(ns) == 1:
        return points[ns[0]] / ns[0], 0.0
    mn = statistics.fmean(ns)
    mt = statistics.fmean(points.values())
    slope = (sum((n - mn) * (points[n] - mt) for n in ns) /
             sum((n - mn) ** 2 for n in ns))
    return slope, mt - slope * mn


def kernel_sequences(w: Workload, stream, reps: int) -> dict:
    """Launch duration of each kernel of the step.  For each kernel, graphs of
    n of its launches (n = 1, 2, 4, 8 and all layers, one per layer, back to
    back as the step issues them, the state before them prepared eagerly;
    for group quant n = 1, 2, 4, 8 over four activations in turn) are timed
    between CUDA events (median over the repetitions), and the per-launch
    duration is the slope of graph time against n.  The intercept
    is the fixed cost of timing one graph after the L2 flush (about 5 us; a
    graph of one single-group launch shows the same), which belongs to no
    launch; graph time / launches at n = all layers is kept beside the slope.
    The merged freeze launch is only reachable together with the crossing
    chunk's absmax, so its times are the differences between that pair's
    graphs and the absmax-only graphs.
    Returns {label: {"us": slope, "intercept_us", "graph_us_per_launch",
    "graph_us": {n: us}}}."""
    fp8q = w.fp8q
    L = w.layers

    def stage_n(n):
        def body(calibs):
            for l in range(n):
                calibs[l].observe_write(w.k[l][:CHUNK1], w.v[l][:CHUNK1], w.slots[l][:CHUNK1],
                                        w.k_pool[l], w.v_pool[l])
        return body

    def amax_n(n):
        def body(calibs):
            for l in range(n):
                calibs[l].observe(w.k[l][CHUNK1:], w.v[l][CHUNK1:], w.slots[l][CHUNK1:])
        return body

    def freeze_n(n):
        def body(calibs):
            for l in range(n):
                calibs[l].observe_write(w.k[l][CHUNK1:], w.v[l][CHUNK1:], w.slots[l][CHUNK1:],
                                        w.k_pool[l], w.v_pool[l])
        return body

    def timed(prefix, body, n_launch):
        with torch.cuda.stream(stream):
            w.states.copy_(w.states_init)
            calibs = w.calibrators()
            for f in prefix:
                f(calibs)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        before = fp8q.launch_count()
        with torch.cuda.graph(g, stream=stream):
            body(calibs)
        assert fp8q.launch_count() - before == n_launch
        ts = time_graph(w, stream, g, reps, reset_state=False)
        del g
        for c in calibs:
            c.close()
        return 1e3 * statistics.median(ts)

    ns = launch_counts(L)
    xs = [w.x] + [w.x.clone() for _ in range(3)]
    qs = [w.q] + [torch.empty_like(w.q) for _ in range(3)]
    ss = [w.s] + [torch.empty_like(w.s) for _ in range(3)]

    def gq_n(n):
        # four distinct activations in turn (4 x 71 MB: a launch's input and
        # output have left L2 by the time they come round again)
        def body(calibs):
            for i in range(n):
                fp8q.fp8_group_quant(xs[i % 4], qs[i % 4], ss[i % 4])
        return body

    graphs = {
        "group_quant": {n: timed([], gq_n(n), n) for n in (1, 2, 4, 8)},
        "observe_stage_write": {n: timed([], stage_n(n), n) for n in ns},
        "amax": {n: timed([stage_n(L)], amax_n(n), n) for n in ns},
    }
    pair = {n: timed([stage_n(L)], freeze_n(n), 2 * n) for n in ns}
    graphs["replay_crossing"] = {n: max(pair[n] - graphs["amax"][n], 0.0) for n in ns}
    del xs, qs, ss
    out = {}
    for lab, pts in graphs.items():
        slope, icept = fit_line(pts)
        n_max = max(pts)
        out[lab] = {"us": slope, "intercept_us": icept,
                    "graph_us_per_launch": pts[n_max] / n_max,
                    "graph_us": {n: round(t, 3) for n, t in pts.items()}}
    return out


def run_native(args, dist: Dist) -> dict | None:
    import paged_kv_cache_group_b200 as fp8q
    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    w = Workload(device, args.layers)
    stream = torch.cuda.Stream(device)

    # eager warm-up: fills the library's launch-geometry caches, checks the flow
    with torch.cuda.stream(stream):
        for i in range(2):
            w.reset(i)
            w.issue(w.calibrators())
    torch.cuda.synchronize()
    assert fp8q.fp8q_device_error(clear=True) == 0

    graph, labels, launches, graph_calibs = capture(w, stream)
    assert launches == len(labels), (launches, len(labels))

    clocks = ClockSampler(smi_gpu_id(dist.local_rank)) if dist.rank == 0 else None
    nvml_clocks = NvmlClockSampler(device) if dist.rank == 0 else None
    time_graph(w, stream, graph, args.warmup, reset_state=True)
    torch.cuda.synchronize()

    dist.barrier()
    torch.cuda.synchronize()
    if nvml_clocks is not None:
        nvml_clocks.mark_start()
    step_ms = time_graph(w, stream, graph, args.steps, reset_state=True,
                         during=nvml_clocks.sample_now if nvml_clocks is not None else None)
    torch.cuda.synchronize()
    if nvml_clocks is not None:
        nvml_clocks.mark_end()
    dist.barrier()
    smi_info = clocks.stop() if clocks is not None else None
    clock_info = nvml_clocks.stop() if nvml_clocks is not None else None
    if clock_info is not None:
        clock_info["nvidia_smi_warmup_and_timed"] = smi_info
    gpu_launches = launches * args.steps

    total_s = sum(step_ms) / 1e3
    bytes_rank = step_bytes(args.layers) * args.steps
    max_s, total_bytes = aggregate(dist, total_s, bytes_rank, device)
    tokens_total = dist.reduce(TOKENS * args.steps, "sum", device)

    # correctness of the timed replays: the last step's pools and codes must be
    # those of a fresh eager step (identical inputs, deterministic kernels)
    q_graph = w.q.clone()
    pools_graph = (w.k_pool[-1].clone(), w.v_pool[-1].clone())
    with torch.cuda.stream(stream):
        w.reset(0)
        w.issue(w.calibrators())
    torch.cuda.synchronize()
    assert torch.equal(q_graph, w.q)
    assert torch.equal(pools_graph[0], w.k_pool[-1]) and torch.equal(pools_graph[1], w.v_pool[-1])
    del pools_graph
    assert fp8q.fp8q_device_error(clear=True) == 0

    # eager (no graph) step time through the Python binding, for context
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    eager_ms = []
    with torch.cuda.stream(stream):
        for i in range(min(args.steps, 20)):
            calibs = w.calibrators()
            w.reset(i)
            start.record()
            w.issue(calibs)
            end.record()
            end.synchronize()
            eager_ms.append(start.elapsed_time(end))

    drained_ms = drained_step_ms(w, stream, graph, reps=max(20, min(args.steps, 200)))
    seq = kernel_sequences(w, stream, reps=max(5, min(args.steps, 50)))
    targets = measure_targets(w, stream, args)
    sweep = calib = None
    if dist.rank == 0 and not args.no_configs:
        sweep = decode_sweep(device, stream)
        calib = calib_window(device, stream, warmup=args.warmup, windows=max(10, min(args.steps, 50)))
    e2e = None if args.no_e2e else measure_e2e(w, stream, args)
    del graph
    for c in graph_calibs:
        c.close()
    peaks = measured_peaks()
    result = None
    if dist.rank == 0:
        kernels = {}
        kernel_time = sum(v["us"] * labels.count(lab) for lab, v in seq.items())
        for lab, v in seq.items():
            n_per_step = labels.count(lab)
            b = launch_bytes(lab)
            gbs = b / (v["us"] * 1e-6) / 1e9
            graph_gbs = b / (v["graph_us_per_launch"] * 1e-6) / 1e9
            kernels[lab] = {"launches_per_step": n_per_step, "avg_us": round(v["us"], 3),
                            "bytes_per_launch": b, "gbs": round(gbs, 1),
                            "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
                            "share": round(n_per_step * v["us"] / kernel_time, 4),
                            "fit_intercept_us": round(v["intercept_us"], 3),
                            "graph_us_per_launch": round(v["graph_us_per_launch"], 3),
                            "graph_frac_of_hbm": round(graph_gbs / peaks["hbm_gbs"], 4),
                            "graph_us_by_launches": v["graph_us"]}
        dominant = max(kernels, key=lambda k: kernels[k]["launches_per_step"] * kernels[k]["avg_us"])
        dk = kernels[dominant]
        ms = 1e3 * max_s / args.steps
        result = {
            "metric": METRIC, "value": round(total_bytes / max_s / 1e9, 2), "unit": "GB/s",
            "n_gpus": dist.world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32",
            "data": "synthetic: seeded Philox draws rounded to bf16 (no weights, no dataset)",
            "config": {
                "workload": (f"prefill of {TOKENS} tokens: group quant {M}x{K} bf16 + "
                             f"{args.layers} layers x calibrating KV write "
                             f"({workloads.KV_HEADS} KV heads x {workloads.HEAD_DIM}, "
                             f"{workloads.LARGE_NUM_BLOCKS}-block pools of 16, window "
                             f"{workloads.LARGE_WINDOW_REQUEST}->4096, chunks {CHUNK1}+{CHUNK2}: "
                             "stage+write; absmax; freeze+replay+crossing write)"),
                "l2": "flushed before every step (2x L2 write, then 2x L2 read; untimed)",
                "timing": ("CUDA graph replay of the step's 49 launches (programmatic "
                           "dependent launch), CUDA events around each step; per-kernel "
                           "launch duration = slope of event-timed graph time against "
                           "launches (graphs of 1, 2, 4, 8 and all layers' launches of that "
                           "kernel in step order; group quant: 1, 2, 4, 8 launches over four "
                           "activations); graph time / launches kept beside it"),
                "bytes_per_step": step_bytes(args.layers),
                "parallelism": f"replicas x{dist.world} (one step per GPU, no collective)",
            },
            "tokens_per_s": round(tokens_total / max_s, 1),
            "roofline": {"bound": "hbm", "kernel": dominant, "achieved": dk["gbs"],
                         "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(dk["gbs"] / peaks["hbm_gbs"], 4),
                         "traffic": committed_traffic(dominant),
                         "peak_source": peaks["source"],
                         "algorithmic_bytes_per_launch": dk["bytes_per_launch"],
                         "launch_us": dk["avg_us"],
                         "launch_us_method": ("slope of event-timed graph time against the "
                                              "number of launches; the intercept, the fixed "
                                              "cost of timing a graph, is excluded"),
                         "graph_us_per_launch": dk["graph_us_per_launch"],
                         "graph_frac": dk["graph_frac_of_hbm"]},
            "kernels": kernels,
            "targets": targets,
            "eager_ms_per_step": round(statistics.median(eager_ms), 4),
            "writeback_drained": {
                "ms_per_step": round(drained_ms, 5),
                "value": round(step_bytes(args.layers) / (drained_ms * 1e-3) / 1e9, 2),
                "unit": "GB/s",
                "method": ("rank 0: (step + read of a clean 2x-L2 buffer) - (the same read on a "
                           "clean L2): the step with the write-back of the dirty L2 lines it "
                           "leaves behind counted in its time")},
            "gpu_launches": gpu_launches,
            "clocks": clock_info,
        }
        if e2e is not None:
            result["e2e"] = e2e
        if sweep is not None:
            result["sweep"] = sweep
        if calib is not None:
            result["calib_window"] = calib
        if not args.no_cpu_baseline and dist.world == 1:
            result["cpu_baseline"] = cpu_baseline(budget_s=args.cpu_budget)
    dist.close()
    return result


def measure_targets(w: Workload, stream, args) -> dict:
    """The stand-alone kernel figures the path is judged by: group quant of
    the 4593 x 5120 activation (one launch alone, and four back to back on
    distinct activations), the K-major variant, and the steady-state
    (post-freeze) KV write of 4593 tokens per layer, 16 layers back to back
    (one launch each) and as one multi-layer launch.

    Each figure is given twice (medians over the repetitions): the graph of
    the launches between CUDA events, and "drained": the same graph followed,
    inside the timed region, by a read of a clean 2x-L2 buffer that evicts
    every dirty line the launches left in L2, minus that read on a clean L2.  The drained figure
    counts the write-back of the codes to HBM, which the plain figure can
    leave to whatever runs next.  The chained figures (group quant, K-major,
    per-layer KV write) also carry the marginal duration: the slope of graph
    time against the number of launches, which leaves out the fixed cost of
    timing a graph between events (about 5 us after the L2 flush; a graph of
    one single-group launch shows the same) and, in a chain, counts the
    write-back of the previous launch's codes."""
    fp8q = w.fp8q
    peaks = measured_peaks()
    out = {}
    scale = torch.tensor([0.05, 0.05], dtype=torch.float32, device=w.device)
    reps = max(3, min(args.steps, 50))
    drain = torch.ones_like(w.flush_read)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def drained_us(g) -> float:
        with_wb, without = [], []
        with torch.cuda.stream(stream):
            for i in range(max(10, reps)):
                w.flush(i)
                ev0.record()
                g.replay()
                torch.amax(drain)
                ev1.record()
                ev1.synchronize()
                with_wb.append(ev0.elapsed_time(ev1))
                w.flush(i)
                ev0.record()
                torch.amax(drain)
                ev1.record()
                ev1.synchronize()
                without.append(ev0.elapsed_time(ev1))
        return 1e3 * (statistics.median(with_wb) - statistics.median(without))

    drained = {}

    def timed(fn, n_launch, name, drain_too=True):
        with torch.cuda.stream(stream):
            fn(lambda i: None)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn(lambda i: None)
        ts = time_graph(w, stream, g, reps, reset_state=False)
        if drain_too:
            drained[name] = drained_us(g) / n_launch
        del g
        return statistics.median(ts) * 1e3 / n_launch

    def marginal(entry, make_fn, ns, nbytes, unit_key):
        """Slope of graph time against launches (graphs of n launches for n in
        ns): the per-launch duration without the fixed cost of timing a graph."""
        pts = {n: timed(make_fn(n), n, f"fit{n}", drain_too=False) * n for n in ns}
        slope, icept = fit_line(pts)
        gbs = nbytes / (slope * 1e-6) / 1e9
        entry[unit_key] = round(slope, 3)
        entry["marginal_frac_of_hbm"] = round(gbs / peaks["hbm_gbs"], 4)
        entry["fit_intercept_us"] = round(icept, 3)
        entry["graph_us_by_launches"] = {n: round(t, 3) for n, t in pts.items()}
        return entry

    def with_drained(entry, name, nbytes):
        us = drained[name]
        gbs = nbytes / (us * 1e-6) / 1e9
        entry["drained_us"] = round(us, 3)
        entry["drained_frac_of_hbm"] = round(gbs / peaks["hbm_gbs"], 4)
        return entry

    def gq(mark):
        fp8q.fp8_group_quant(w.x, w.q, w.s)
        mark(0)

    us = timed(gq, 1, "gq")
    gbs = GROUP_QUANT_BYTES / (us * 1e-6) / 1e9
    out["group_quant_4593x5120"] = with_drained(
        {"us": round(us, 3), "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
         "tokens_per_s": round(M / (us * 1e-6), 1),
         "vs_pages_h100_636_gbs": round(gbs / 636.0, 2),
         "launch": "single launch in its own graph"}, "gq", GROUP_QUANT_BYTES)
    ncu_us = committed_ncu("group_quant", "gpu_time_us")
    if ncu_us is not None:
        kgbs = GROUP_QUANT_BYTES / (ncu_us * 1e-6) / 1e9
        out["group_quant_4593x5120"]["kernel_only"] = {
            "us": ncu_us, "frac_of_hbm": round(kgbs / peaks["hbm_gbs"], 4),
            "source": "ncu gpu__time_duration.sum of this launch (profiles/traffic.json)"}

    # the fixed cost of this way of timing one launch: the same quantizer on a
    # single 128-element group (one CTA), in its own graph, timed the same way
    x1 = w.x[:1, :128].contiguous()
    q1 = torch.empty((1, 128), dtype=torch.uint8, device=w.device)
    s1 = torch.empty((1, 1), dtype=torch.float32, device=w.device)

    def gq1(mark):
        fp8q.fp8_group_quant(x1, q1, s1)
        mark(0)

    out["launch_floor_1x128"] = {"us": round(timed(gq1, 1, "gq1"), 3),
                                 "launch": "single launch in its own graph, one 128-element group"}

    # back to back over four distinct activations (as consecutive layers
    # quantize theirs): inputs and outputs 4 x 71 MB, more than L2 holds
    xs = [w.x] + [w.x.clone() for _ in range(3)]
    qs = [w.q] + [torch.empty_like(w.q) for _ in range(3)]
    ss = [w.s] + [torch.empty_like(w.s) for _ in range(3)]

    def gq4(mark):
        for i in range(4):
            fp8q.fp8_group_quant(xs[i], qs[i], ss[i])
            mark(i)

    us4 = timed(gq4, 4, "gq4")
    gbs4 = GROUP_QUANT_BYTES / (us4 * 1e-6) / 1e9
    out["group_quant_4593x5120_seq4"] = with_drained(
        {"us": round(us4, 3), "gbs": round(gbs4, 1), "frac_of_hbm": round(gbs4 / peaks["hbm_gbs"], 4),
         "launch": "mean of 4 back-to-back launches"}, "gq4", GROUP_QUANT_BYTES)

    def gq_first(n):
        def fn(mark):
            for i in range(n):
                fp8q.fp8_group_quant(xs[i % 4], qs[i % 4], ss[i % 4])
                mark(i)
        return fn

    marginal(out["group_quant_4593x5120_seq4"], gq_first, (1, 2, 4, 8), GROUP_QUANT_BYTES,
             "marginal_us")
    del qs, ss

    # the same activation for a GEMM padded to ceil16(M) rows: K-major scales
    # and zeroed phantom rows in the same launch
    m_pad = fp8q.ceil16(M)
    qk = torch.empty((m_pad, K), dtype=torch.uint8, device=w.device)
    sk = torch.empty((K // 128, m_pad), dtype=torch.float32, device=w.device)

    def gqk(mark):
        fp8q.fp8_group_quant_kmajor(w.x, m_pad, qk, sk)
        mark(0)

    usk = timed(gqk, 1, "gqk")
    bk = M * K * 2 + m_pad * K + m_pad * (K // 128) * 4
    gbsk = bk / (usk * 1e-6) / 1e9
    out["group_quant_kmajor_4593x5120"] = with_drained(
        {"us": round(usk, 3), "gbs": round(gbsk, 1), "frac_of_hbm": round(gbsk / peaks["hbm_gbs"], 4),
         "m_pad": m_pad, "bytes": bk, "launch": "single launch in its own graph"}, "gqk", bk)
    qks = [qk] + [torch.empty_like(qk) for _ in range(3)]
    sks = [sk] + [torch.empty_like(sk) for _ in range(3)]

    def gqk_first(n):
        def fn(mark):
            for i in range(n):
                fp8q.fp8_group_quant_kmajor(xs[i % 4], m_pad, qks[i % 4], sks[i % 4])
                mark(i)
        return fn

    marginal(out["group_quant_kmajor_4593x5120"], gqk_first, (1, 2, 4, 8), bk, "marginal_us")
    del qk, sk, qks, sks, xs

    def kvw(mark):
        for l in range(w.layers):
            fp8q.fp8_kv_write(w.k[l], w.v[l], w.slots[l], w.k_pool[l], w.v_pool[l],
                              scale_dev=scale)
            mark(l)

    us = timed(kvw, w.layers, "kvw")
    b = PER_TOKEN["kv_write"] * TOKENS
    gbs = b / (us * 1e-6) / 1e9
    out["kv_write_4593"] = with_drained(
        {"us_per_layer": round(us, 3), "gbs": round(gbs, 1), "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4),
         "tokens_per_s": round(TOKENS / (us * 1e-6), 1), "bytes_per_layer": b,
         "launch": f"one launch per layer, {w.layers} back to back"}, "kvw", b)

    def kvw_first(n):
        def fn(mark):
            for l in range(n):
                fp8q.fp8_kv_write(w.k[l], w.v[l], w.slots[l], w.k_pool[l], w.v_pool[l],
                                  scale_dev=scale)
                mark(l)
        return fn

    marginal(out["kv_write_4593"], kvw_first, launch_counts(w.layers), b, "marginal_us_per_layer")

    def kvw_layers(mark):
        fp8q.fp8_kv_write_layers(w.k, w.v, w.slots, w.k_pool, w.v_pool,
                                 scale_devs=[scale] * w.layers)
        mark(0)

    us = timed(kvw_layers, 1, "kvl")
    gbs = b * w.layers / (us * 1e-6) / 1e9
    out["kv_write_4593_all_layers"] = with_drained(
        {"us": round(us, 3), "us_per_layer": round(us / w.layers, 3), "gbs": round(gbs, 1),
         "frac_of_hbm": round(gbs / peaks["hbm_gbs"], 4), "bytes": b * w.layers,
         "launch": f"fp8_kv_write_layers: {w.layers} layers, one launch"}, "kvl", b * w.layers)
    del drain
    return out


def measure_e2e(w: Workload, stream, args) -> dict:
    """The same step through the public API with host inputs: every step copies
    its inputs from pinned host memory and reads its results back.  The copies
    are pipelined with the compute the way a serving loop would issue them:
    inputs go up on a copy stream (the activation first, then layer by layer),
    each computation waits only for its own inputs, and the codes come back on
    a third stream as soon as they exist (PCIe is full duplex)."""
    fp8q = w.fp8q
    hx = torch.from_numpy(w.host_x.view(np.int16)).view(torch.bfloat16).pin_memory()
    hk = [torch.from_numpy(b.k.view(np.int16)).view(torch.bfloat16).pin_memory() for b in w.host_kv]
    hv = [torch.from_numpy(b.v.view(np.int16)).view(torch.bfloat16).pin_memory() for b in w.host_kv]
    hs = [torch.from_numpy(b.slot_mapping).pin_memory() for b in w.host_kv]
    oq = torch.empty((M, K), dtype=torch.uint8).pin_memory()
    os_ = torch.empty((M, K // 128), dtype=torch.float32).pin_memory()
    ost = torch.empty(tuple(w.states.shape), dtype=torch.float32).pin_memory()
    h2d = hx.numel() * 2 + sum(t.numel() * 2 for t in hk + hv) + sum(t.numel() * 8 for t in hs)
    d2h = oq.numel() + os_.numel() * 4 + ost.numel() * 4
    up, down = torch.cuda.Stream(w.device), torch.cuda.Stream(w.device)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    x_in, q_out = torch.cuda.Event(), torch.cuda.Event()
    layer_in = [torch.cuda.Event() for _ in range(w.layers)]
    times = []
    n = max(2, min(args.steps, 10))
    for i in range(n + 2):
        with torch.cuda.stream(stream):
            calibs = w.calibrators()
            w.reset(i)
            start.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        with torch.cuda.stream(up):
            w.x.copy_(hx, non_blocking=True)
            x_in.record(up)
            for l in range(w.layers):
                w.k[l].view(TOKENS, E).copy_(hk[l], non_blocking=True)
                w.v[l].view(TOKENS, E).copy_(hv[l], non_blocking=True)
                w.slots[l].copy_(hs[l], non_blocking=True)
                layer_in[l].record(up)
        with torch.cuda.stream(stream):
            stream.wait_event(x_in)
            fp8q.fp8_group_quant(w.x, w.q, w.s)
            q_out.record(stream)
            for l, c in enumerate(calibs):
                stream.wait_event(layer_in[l])
                k, v, sl = w.k[l], w.v[l], w.slots[l]
                c.observe_write(k[:CHUNK1], v[:CHUNK1], sl[:CHUNK1], w.k_pool[l], w.v_pool[l])
                c.observe_write(k[CHUNK1:], v[CHUNK1:], sl[CHUNK1:], w.k_pool[l], w.v_pool[l])
            ost.copy_(w.states, non_blocking=True)
        with torch.cuda.stream(down):
            down.wait_event(q_out)
            oq.copy_(w.q, non_blocking=True)
            os_.copy_(w.s, non_blocking=True)
        stream.wait_stream(down)
        stream.wait_stream(up)
        end.record(stream)
        end.synchronize()
        if i >= 2:
            times.append(start.elapsed_time(end))
        for c in calibs:
            c.close()
    ms = statistics.mean(times)
    assert fp8q.fp8q_device_error(clear=True) == 0
    assert torch.equal(oq, w.q.cpu()) and torch.equal(os_, w.s.cpu())
    return {"value": round(step_bytes(w.layers) / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
            "ms_per_step": round(ms, 4), "steps": n,
            "overlap": "inputs up on a copy stream layer by layer, codes down on a third stream"}


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            p = json.load(fh)
        return {"hbm_gbs": float(p["hbm_gbs"]), "source": "measured (MEASURED_PEAKS.json hbm_gbs)"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": 6650.0, "source": "fallback 6.65 TB/s"}


def _code_only(text: str) -> str:
    """C/C++ source without comments and whitespace (string literals kept)."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c == '"' or c == "'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        else:
            if not c.isspace():
                out.append(c)
            i += 1
    return "".join(out)


KERNEL_SOURCES = ("fp8q_kernels.cu", "fp8q_internal.h")   # device code and launch geometry


def source_hash() -> str:
    """Hash of the kernels' code (comments and whitespace ignored), the key
    under which ncu figures are recorded in profiles/traffic.json."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_group_b200", "csrc", name),
                  encoding="utf-8") as fh:
            h.update(_code_only(fh.read()).encode())
    return h.hexdigest()[:16]


# ncu kernel of each bench label (the launch list names kernels, not labels)
KERNEL_OF_LABEL = {
    "group_quant": "group_quant_kernel<1>",
    "observe_stage_write": "kv_stage512_kernel<0>",
    "amax": "kv_pass_kernel<1, 0, 0, 0, 64, 256>",
    "replay_crossing": "kv_freeze512_kernel<1>",
    "kv_write": "kv_write512_kernel<0>",
    "kv_write_layers": "kv_write_layers_kernel<64>",
    "group_quant_kmajor": "group_quant_kmajor_kernel",
}


def committed_ncu(label: str, key: str):
    """A figure of `label`'s launch from the committed ncu summary
    (profiles/traffic.json), or None when the kernels changed since it was
    taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            t = json.load(fh)
    except (OSError, ValueError):
        return None
    if t.get("source_hash") != source_hash():
        return None
    entry = t.get("kernels", {}).get(label)
    return None if entry is None else entry.get(key)


def committed_traffic(label: str):
    """DRAM bytes per launch of `label` (ncu), or None (see committed_ncu)."""
    return committed_ncu(label, "dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# the oracle on the host (CPU baseline and the reference arm)

SAMPLE_ROWS = 1148        # a quarter of the activation rows
SAMPLE_LAYERS = 2         # two of the sixteen layers


def reference_sample():
    x = workloads.prefill_quant()[:SAMPLE_ROWS]
    kv = [workloads.large_kv_layer(l) for l in range(SAMPLE_LAYERS)]
    return x, kv


def sample_bytes() -> int:
    gq = SAMPLE_ROWS * K * 3 + SAMPLE_ROWS * (K // 128) * 4
    per_layer = sum(launch_bytes(k) for k in STEP_KERNELS)
    return gq + SAMPLE_LAYERS * per_layer


def reference_step(x, kv) -> None:
    import oracle
    from oracle import calibration as cal
    oracle.group_quant(x)
    spec = workloads.large_kv_spec()
    for b in kv:
        c = cal.Fp8KvCalibration(0, workloads.LARGE_WINDOW_REQUEST, 1.0)
        kp, vp = spec.new_pool().reshape(-1), spec.new_pool().reshape(-1)
        chunks = [cal.KvBatch(p.k, p.v, p.slot_mapping, E, E)
                  for p in workloads.split_batch(b, workloads.LARGE_CHUNKS)]
        cal.run_calibrated_writes(c, chunks, workloads.KV_HEADS, workloads.HEAD_DIM, kp, vp, 16,
                                  spec.cache_stride, spec.num_blocks)


SAMPLE_DESC = (f"oracle (single-threaded C + Python calibration) on {SAMPLE_ROWS} of {M} "
               f"activation rows and {SAMPLE_LAYERS} of 16 layers of the step; bytes counted "
               "as for the GPU step")


def cpu_baseline(budget_s: float = 12.0) -> dict:
    x, kv = reference_sample()
    reference_step(x, kv)                     # warm (builds and loads the oracle)
    times = []
    t_end = time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 2:
        t0 = time.perf_counter()
        reference_step(x, kv)
        times.append(time.perf_counter() - t0)
    s = statistics.median(times)
    return {"value": round(sample_bytes() / s / 1e9, 4), "unit": "GB/s", "cores": 1,
            "kind": "oracle", "sample": SAMPLE_DESC, "repeats": len(times),
            "host_cores": os.cpu_count(), "cpu_model": cpu_model()}


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args) -> dict | None:
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    x, kv = reference_sample()
    for _ in range(args.warmup):
        reference_step(x, kv)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        reference_step(x, kv)
    s = (time.perf_counter() - t0) / args.steps
    value = round(sample_bytes() / s / 1e9, 4)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")), "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(s * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic: seeded Philox draws rounded to bf16 (no weights, no dataset)",
        "config": {"workload": SAMPLE_DESC, "bytes_per_step": sample_bytes()},
        "tokens_per_s": None,
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": SAMPLE_DESC},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def decode_sweep(dev, stream, n: int = 1000) -> dict:
    """Decode-width sweep: group quant at M in {1,2,4,8,16} x K in {5120,16384},
    1000 back-to-back launches per shape, timed as plain stream launches
    through the binding and as a CUDA graph of 1000 launches; once with the
    row-major scales and once K-major with the phantom rows up to ceil16(M)
    zeroed (the layout a padded FP8 GEMM reads).  Launch-bound by design;
    inputs stay in L2, as they do in a decode loop."""
    import paged_kv_cache_group_b200 as fp8q
    shapes = []
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for layout in ("row_major", "kmajor"):
        for m in workloads.DECODE_MS:
            for k in workloads.DECODE_KS:
                bits = workloads.decode_quant(m, k)
                x = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev)
                rows = m if layout == "row_major" else fp8q.ceil16(m)
                q = torch.empty((rows, k), dtype=torch.uint8, device=dev)
                if layout == "row_major":
                    sc = torch.empty((m, k // 128), dtype=torch.float32, device=dev)
                    call = lambda: fp8q.fp8_group_quant(x, q, sc)             # noqa: E731
                else:
                    sc = torch.empty((k // 128, rows), dtype=torch.float32, device=dev)
                    call = lambda: fp8q.fp8_group_quant_kmajor(x, rows, q, sc)  # noqa: E731
                with torch.cuda.stream(stream):
                    for _ in range(20):
                        call()
                    torch.cuda.synchronize()
                    plain = []
                    for _ in range(3):
                        start.record()
                        for _ in range(n):
                            call()
                        end.record()
                        end.synchronize()
                        plain.append(start.elapsed_time(end) * 1e3 / n)
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    for _ in range(n):
                        call()
                graph = []
                with torch.cuda.stream(stream):
                    for _ in range(5):
                        start.record()
                        g.replay()
                        end.record()
                        end.synchronize()
                        graph.append(start.elapsed_time(end) * 1e3 / n)
                del g
                # bytes read and written, phantom rows' zero codes and scales included
                b = m * k * 2 + rows * k + rows * (k // 128) * 4
                us_p, us_g = statistics.median(plain), statistics.median(graph)
                shapes.append({"layout": layout, "m": m, "m_pad": rows, "k": k, "bytes": b,
                               "plain_us_per_launch": round(us_p, 3),
                               "graph_us_per_launch": round(us_g, 3),
                               "graph_gbs": round(b / (us_g * 1e-6) / 1e9, 1),
                               "graph_tokens_per_s": round(m / (us_g * 1e-6), 1)})
    rm = [x["graph_us_per_launch"] for x in shapes if x["layout"] == "row_major"]
    return {"workload": ("decode-width group quant: M in {1,2,4,8,16} x K in {5120,16384} bf16 "
                         "N(0,1), groups of 128, 1000 back-to-back launches per shape"),
            "launches_per_shape": n, "l2": "inputs L2-resident (launch-bound by design)",
            "row_major_graph_us_per_launch": [min(rm), max(rm)], "shapes": shapes}


def calib_window(dev, stream, warmup: int = 5, windows: int = 20) -> dict:
    """The 256-token calibration window of one layer (13 + 32-token batches,
    freeze at batch 9, two batches after it) through fp8_kv_calib_observe_write,
    eager, with L2 flushed before each window; CUDA events around the window."""
    import paged_kv_cache_group_b200 as fp8q
    spec, batches, _ = workloads.calib_window()

    def rows(bits):
        t = bits.shape[0]
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(dev).view(t, 4, 128)
    ks = [rows(b.k) for b in batches]
    vs = [rows(b.v) for b in batches]
    ss = [torch.from_numpy(b.slot_mapping).to(dev) for b in batches]
    shape = (spec.num_blocks, spec.block_size, spec.heads, spec.dim)
    kp = torch.full(shape, workloads.SENTINEL, dtype=torch.uint8, device=dev)
    vp = torch.full(shape, workloads.SENTINEL, dtype=torch.uint8, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(2 * l2, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(2 * l2, dtype=torch.uint8, device=dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    times = []
    launches = 0
    with torch.cuda.stream(stream):
        for i in range(warmup + windows):
            cal = fp8q.KvCalibration(workloads.CALIB_WINDOW, 1.0, 4, 128, dev)
            flush_w.fill_(i & 0xFF)
            torch.amax(flush_r)
            torch.cuda._sleep(1_000_000)       # let the host queue the window ahead
            before = fp8q.launch_count()
            start.record()
            for k, v, s in zip(ks, vs, ss):
                cal.observe_write(k, v, s, kp, vp)
            end.record()
            launches = fp8q.launch_count() - before
            end.synchronize()
            if i >= warmup:
                times.append(start.elapsed_time(end) * 1e3)
            cal.close()
    staged = sum(b.num_tokens for b in batches[:8])
    seen = sum(b.num_tokens for b in batches)
    bytes_ = (staged * PER_TOKEN["observe_stage_write"] + batches[8].num_tokens * 2048 +
              (staged + batches[8].num_tokens) * 3080 +
              sum(b.num_tokens for b in batches[9:]) * 3080)
    us = statistics.median(times)
    return {"workload": ("calibration window: 256 tokens, 4 x 128, batches 13 + 10 x 32, freeze at "
                         "batch 9 (269 tokens), headroom 1.0"),
            "us_per_window": round(us, 2), "tokens": seen, "bytes": bytes_, "launches": launches,
            "gbs": round(bytes_ / (us * 1e-6) / 1e9, 1),
            "tokens_per_s": round(seen / (us * 1e-6), 1), "windows": len(times),
            "l2": "flushed before each window", "timing": "CUDA events around the window's calls"}


def run_profile(args) -> None:
    """A few eager steps on `--layers` layers for an ncu capture: each step is
    the bench step (group quant, then per layer the calibrating write) followed
    by the steady-state write of every layer one launch each, then the same as
    one fp8_kv_write_layers launch, then the activation quantized K-major for a
    GEMM padded to ceil16(M) rows.  Select kernels with ncu -k / -s / -c.
    ncu flushes caches itself, so no flush buffers are allocated."""
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = Workload(dev, args.layers, flush=False)
    scale = torch.tensor([0.05, 0.05], dtype=torch.float32, device=dev)
    m_pad = w.fp8q.ceil16(M)
    qk = torch.empty((m_pad, K), dtype=torch.uint8, device=dev)
    sk = torch.empty((K // 128, m_pad), dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        for i in range(args.warmup + args.steps):
            w.reset(i)
            w.issue(w.calibrators())
            for l in range(w.layers):
                w.fp8q.fp8_kv_write(w.k[l], w.v[l], w.slots[l], w.k_pool[l], w.v_pool[l],
                                    scale_dev=scale)
            w.fp8q.fp8_kv_write_layers(w.k, w.v, w.slots, w.k_pool, w.v_pool,
                                       scale_devs=[scale] * w.layers)
            w.fp8q.fp8_group_quant_kmajor(w.x, m_pad, qk, sk)
    torch.cuda.synchronize()
    assert w.fp8q.fp8q_device_error(clear=True) == 0
    print(json.dumps({"profile": "done", "layers": args.layers,
                      "steps": args.warmup + args.steps}))


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--layers", type=int, default=workloads.LARGE_LAYERS)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the decode-width sweep and the calibration window")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--profile", action="store_true",
                    help="run a few eager steps for an ncu capture and exit")
    ap.add_argument("--sweep", action="store_true",
                    help="decode-width sweep of the group quantizer (one JSON line per shape)")
    ap.add_argument("--calib", action="store_true",
                    help="time the 256-token calibration window end to end")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be at least 3")
    if a.steps < 1:
        ap.error("--steps must be at least 1")
    return a


def main(argv=None) -> int:
    args = parse_args(argv)
    if args.profile:
        run_profile(args)
        return 0
    if args.sweep or args.calib:
        torch.cuda.set_device(0)
        dev = torch.device("cuda", 0)
        stream = torch.cuda.Stream(dev)
        if args.sweep:
            for line in decode_sweep(dev, stream)["shapes"]:
                print(json.dumps(line), flush=True)
        if args.calib:
            print(json.dumps(calib_window(dev, stream, args.warmup, args.steps)), flush=True)
        return 0
    if args.impl == "reference":
        res = run_reference(args)
    else:
        res = run_native(args, Dist())
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
