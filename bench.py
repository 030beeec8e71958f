#!/usr/bin/env python
"""Benchmark of the LSE-weighted merge on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one merge of one batch of the large decode-merge workload
(R=16 partials, B=512, H=16, D=512, bf16 partials [B,H,R,D] -> fp32 output):
134.7 MB read and 16.8 MB written per step by the algorithmic count
R*B*H*(D*2+4) + B*H*(D*4+4).  Rank 0 prints one JSON line.

  value     device throughput (GB/s of algorithmic bytes, all ranks) with the
            inputs resident in HBM: W untimed launches, then 5 trials of K
            back-to-back launches, each timed with CUDA events on the launch
            stream; the median trial is reported (max over ranks for N > 1).
            Inputs and outputs rotate over enough buffer sets that each step
            misses L2.
  e2e       the same metric through the host-buffer call of the C ABI,
            lse_merge_host (via merge_host): each step copies its partials
            from pinned host memory to the GPU and the result back, in 8
            batch slices overlapped with the merge.
  roofline  the kernel's achieved GB/s against the measured HBM copy peak,
            and its DRAM traffic from the committed ncu summary.
  cpu_baseline  the fp64 CPU oracle on a bounded sample (rank 0, N = 1), on
            every host core and on one.
  state_update, decode_attention, cp_exchange_merge
            the rows built beside the merge.
  workloads (last key) every merge workload: eager and CUDA-graph-replayed
            us/call (median of 5 trials; eager 200 calls, graph 100 calls x
            50 replays), GB/s and fraction of peak from the graph time, and
            the largest error against the fp64 oracle over every output.

With --gpus N under torchrun every rank merges its own batch (the rows are
independent; no collective touches the data, NCCL only times the job).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "merge throughput GB/s (% of B200 HBM peak) and µs/call at 1 GPU"
FALLBACK_HBM_GBS = 6650.0
L2_FALLBACK = 126 * 1024 * 1024
BAD_REASONS = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown")
KERNEL_SOURCES = ("lse_weighted_merge_b200/csrc/lse_merge.cu",
                  "lse_weighted_merge_b200/csrc/device_common.cuh",
                  "lse_weighted_merge_b200/csrc/plan.cpp",
                  "lse_weighted_merge_b200/csrc/plan.h")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def parse_args(argv=None):
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=1000)
    p.add_argument("--warmup", type=int, default=50)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=None, help="workload name (default: the large merge)")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-extra", action="store_true", help="skip latency / per-workload lines")
    p.add_argument("--cpu-seconds", type=float, default=8.0)
    p.add_argument("--trials", type=int, default=5, help="timed trials per loop (median reported)")
    p.add_argument("--e2e-steps", type=int, default=10)
    p.add_argument("--decode-only", default=None, metavar="SHAPE",
                   help="only time the decode-attention shape SHAPE (for profiling)")
    p.add_argument("--cp-only", default=None, metavar="WORKLOAD",
                   help="only time the context-parallel exchange + merge WORKLOAD (for profiling)")
    p.add_argument("--state-only", action="store_true",
                   help="only time the in-place state update (for profiling)")
    return p.parse_args(argv)


# ------------------------------------------------------------------ distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def dist_init(world: int, backend: str = "nccl"):
    if world <= 1:
        return None
    import datetime

    import torch.distributed as dist
    dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device) -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device=None):
    if dist is not None:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------------------ clocks

class ClockSampler:
    """Polls the GPU's SM clock and clock-event (throttle) reasons through NVML."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x10: "sync_boost"}

    def __init__(self, device, period_s: float = 0.002):
        self.samples = []
        self.period = period_s
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        self.windows = []
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            props = torch.cuda.get_device_properties(device)
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                dom = getattr(props, "pci_domain_id", 0)
                devid = getattr(props, "pci_device_id", 0)
                bid = f"{dom:08x}:{bus:02x}:{devid:02x}.0".encode()
                self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bid)
            else:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as exc:  # no NVML: report why
            self.error = f"{type(exc).__name__}: {exc}"
            self.nv = None
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    bits = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, bits))
            except Exception as exc:
                self.error = f"{type(exc).__name__}: {exc}"
                return
            time.sleep(self.period)

    def start(self):
        if self.nv is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()

    def summary(self, t0: float, t1: float) -> dict:
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "error": self.error}
        win = [s for s in self.samples if t0 <= s[0] <= t1]
        where = "timed region"
        if len(win) < 3:   # a short timed region: widen to the samples around it
            mid = 0.5 * (t0 + t1)
            win = sorted(self.samples, key=lambda s: abs(s[0] - mid))[:25]
            where = "nearest 25 samples around the timed region (region shorter than the poll)"
        reasons = set()
        for _, _, bits in win:
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s[1] for s in win) if win else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(reasons), "samples": len(win),
                "window": where}


# ---------------------------------------------------------------- measurement

def kernel_source_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def profiled_traffic(workload: str):
    """DRAM bytes per launch from the committed ncu summary of this kernel and
    workload, or None when the kernel source changed since the capture."""
    path = os.path.join(ROOT, "profiles", f"lse_merge_{workload}.md")
    if not os.path.exists(path):
        return None, "no ncu summary for this workload"
    fields = {}
    with open(path) as fh:
        for line in fh:
            if ":" in line and line.startswith("- `"):
                k, v = line[3:].split("`", 1)
                fields[k.strip()] = v.split(":", 1)[1].strip().strip("`")
    if fields.get("source_sha256") != kernel_source_sha():
        return None, "kernel changed since the ncu capture"
    try:
        return int(fields["dram_bytes_per_launch"]), os.path.relpath(path, ROOT)
    except (KeyError, ValueError):
        return None, "summary has no dram_bytes_per_launch"


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or "unknown"."""
    try:
        with open("/proc/cpuinfo") as fh:
            for line in fh:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            return float(json.load(fh)["hbm_gbs"]), "measured (MEASURED_PEAKS.json hbm_gbs)"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback (no MEASURED_PEAKS.json)"


class DeviceSets:
    """`n` device copies of one workload's inputs and outputs, to rotate through
    so that consecutive steps touch different memory (no L2 reuse)."""

    def __init__(self, inp: dict, n: int, device):
        import numpy as np
        import torch
        from lse_weighted_merge_b200 import _native as nat
        from lse_weighted_merge_b200 import synth
        self.inp = inp
        self.R, self.B, self.H, self.D = inp["R"], inp["B"], inp["H"], inp["D"]
        o = inp["o"]
        host_o = torch.from_numpy(o.view(np.int16) if o.dtype == np.uint16 else o.view(np.int32))
        host_l = torch.from_numpy(inp["lse"])
        out_dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[inp["out_dtype"]]
        self.o = [host_o.to(device) for _ in range(n)]
        self.lse = [host_l.to(device) for _ in range(n)]
        self.out = [torch.empty((self.B, self.H, self.D), dtype=out_dt, device=device) for _ in range(n)]
        self.out_lse = [torch.empty((self.B, self.H), dtype=torch.float32, device=device) for _ in range(n)]
        self.strides = (*inp["o_strides"], *inp["lse_strides"])
        self.ind = synth.DTYPES[inp["in_dtype"]]
        self.outd = synth.DTYPES[inp["out_dtype"]]
        self.n = n
        self.args = [(self.o[i].data_ptr(), self.lse[i].data_ptr(), self.out[i].data_ptr(),
                      self.out_lse[i].data_ptr()) for i in range(n)]

    path = 0   # AUTO

    def launch(self, i: int, stream_handle: int):
        from lse_weighted_merge_b200 import _native as nat
        o, l, out, ol = self.args[i % self.n]
        rc = nat.merge_raw(o, l, self.R, self.B, self.H, self.D, self.strides, self.ind,
                           self.outd, out, ol, stream_handle, self.path, check=False)
        if rc != 0:
            raise RuntimeError(f"lse_merge returned {rc}: {nat.strerror(rc)}")


def n_sets(bytes_per_set: int, l2_bytes: int) -> int:
    return int(min(256, max(2, math.ceil(2 * l2_bytes / max(bytes_per_set, 1)) + 1)))


def time_eager(sets: DeviceSets, steps: int, warmup: int, device, trials: int = 1):
    """Run `warmup` launches, then `trials` times `steps` back-to-back launches
    on the current stream, each trial between two CUDA events; returns
    (list of region ms per trial, t0, t1) with t0/t1 the host times around all
    trials.  One kernel launch per step, so region/steps is the kernel's
    average launch duration; no event sits between launches (an event record
    between two launches would serialise them)."""
    import torch
    stream = torch.cuda.current_stream(device)
    sh = stream.cuda_stream
    for i in range(warmup):
        sets.launch(i, sh)
    torch.cuda.synchronize(device)
    regions = []
    t0 = time.perf_counter()
    k = warmup
    for _ in range(trials):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            sets.launch(k, sh)
            k += 1
        e1.record(stream)
        torch.cuda.synchronize(device)
        regions.append(e0.elapsed_time(e1))
    t1 = time.perf_counter()
    return regions, t0, t1


def time_graph(sets: DeviceSets, calls: int, replays: int, device, trials: int = 5):
    """us per call of `calls` merges captured in one CUDA graph and replayed
    `replays` times, median over `trials` timed rounds; returns
    (median us, host t0, host t1)."""
    import torch
    s = torch.cuda.Stream(device)
    s.wait_stream(torch.cuda.current_stream(device))
    with torch.cuda.stream(s):
        for i in range(3):
            sets.launch(i, s.cuda_stream)
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        h = torch.cuda.current_stream(device).cuda_stream
        for i in range(calls):
            sets.launch(i, h)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize(device)
    us = []
    t0 = time.perf_counter()
    for _ in range(trials):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(replays):
            g.replay()
        e1.record()
        torch.cuda.synchronize(device)
        us.append(e0.elapsed_time(e1) * 1000.0 / (calls * replays))
    t1 = time.perf_counter()
    del g
    return statistics.median(us), t0, t1


def time_e2e(inp: dict, steps: int, device, chunks: int = 8) -> dict:
    """The public host-buffer call (merge_host, pipelined as in a stream of
    batches): every step copies the step's partials from pinned host memory to
    the GPU, merges, and copies the result back to pinned host memory, the
    copies overlapped with the merge and with the neighbouring steps."""
    import numpy as np
    import torch
    from lse_weighted_merge_b200 import merge_host
    R, B, H, D = inp["R"], inp["B"], inp["H"], inp["D"]
    o = inp["o"]
    tdt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
    raw = torch.from_numpy(o.view(np.int16) if o.dtype == np.uint16 else o.view(np.int32))
    layout = inp["workload"].layout
    shape_o = (B, H, R, D) if layout == "bhrd" else (R, B, H, D)
    shape_l = (B, H, R) if layout == "bhrd" else (R, B, H)
    h_o = raw.view(tdt[inp["in_dtype"]]).reshape(shape_o).pin_memory()
    h_l = torch.from_numpy(inp["lse"]).reshape(shape_l).pin_memory()
    h_out = torch.empty((B, H, D), dtype=tdt[inp["out_dtype"]]).pin_memory()
    h_out_lse = torch.empty((B, H), dtype=torch.float32).pin_memory()

    def step():
        merge_host(h_o, h_l, layout=layout, out_dtype=tdt[inp["out_dtype"]], chunks=chunks,
                   device=device, out=h_out, out_lse=h_out_lse, sync=False, pipeline=True)

    for _ in range(2):
        step()
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    e0.record()
    for _ in range(steps):
        step()
    e1.record()
    torch.cuda.synchronize(device)
    t1 = time.perf_counter()
    ms = e0.elapsed_time(e1) / steps
    w = inp["workload"]
    return {"ms_per_step": ms, "gbs": w.bytes_total() / (ms * 1e-3) / 1e9,
            "h2d_bytes_per_step": int(h_o.numel() * h_o.element_size() + h_l.numel() * 4),
            "d2h_bytes_per_step": int(h_out.numel() * h_out.element_size() + h_out_lse.numel() * 4),
            "steps": steps, "chunks": chunks, "t0": t0, "t1": t1}


def sample_inputs(inp: dict, batches: int) -> dict:
    """The first `batches` batches of a [B,H,R,D] workload (a contiguous prefix)."""
    w = inp["workload"]
    if batches >= w.B:
        return inp
    assert w.layout == "bhrd"
    per_b_o = w.H * w.R * w.D
    per_b_l = w.H * w.R
    s = dict(inp)
    s["o"] = inp["o"][: batches * per_b_o]
    s["lse"] = inp["lse"][: batches * per_b_l]
    s["B"] = batches
    return s


def oracle_seconds(inp: dict, budget_s: float, threads: int = 1):
    """Run the fp64 oracle over `inp` repeatedly for at least budget_s, on
    `threads` host threads (0: one per core); returns (bytes/s, passes,
    seconds, threads used)."""
    import oracle
    from lse_weighted_merge_b200 import synth
    w = inp["workload"]
    byts = inp["R"] * inp["B"] * inp["H"] * (inp["D"] * synth.ELEM_BYTES[w.in_dtype] + 4) + \
        inp["B"] * inp["H"] * (inp["D"] * synth.ELEM_BYTES[w.out_dtype] + 4)
    lib = oracle.load()
    passes = 0
    st = {}
    t0 = time.perf_counter()
    while True:
        oracle.merge(inp["o"], inp["lse"], inp["R"], inp["B"], inp["H"], inp["D"], inp["o_strides"],
                     inp["lse_strides"], synth.DTYPES[w.in_dtype], lib=lib, threads=threads, stats=st)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    return byts * passes / dt, passes, dt, st.get("threads", 1)


def cpu_baselines(inp: dict, batches: int, seconds: float) -> dict:
    """The oracle on the first `batches` batches of the workload, on every
    host core (the reported value) and on one core; each leg runs for about
    `seconds`."""
    w = inp["workload"]
    smp = sample_inputs(inp, batches)
    what = f"first {batches} of {w.B} batches ({batches * w.H} of {w.rows} rows)"
    bps_n, passes_n, secs_n, used = oracle_seconds(smp, seconds, threads=0)
    bps_1, passes_1, secs_1, _ = oracle_seconds(smp, seconds, threads=1)
    return {"value": bps_n / 1e9, "unit": "GB/s", "cores": used, "kind": "oracle",
            "sample": (f"{what}, {passes_n} passes in {secs_n:.1f} s, fp64 C oracle, batches split "
                       f"over {used} host threads"),
            "single_thread": {"value": bps_1 / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
                              "sample": f"{what}, {passes_1} passes in {secs_1:.1f} s, one thread"},
            "cpu": cpu_model(), "host_cores": os.cpu_count()}


def oracle_errors(captured: dict) -> dict:
    """Largest error of each workload's GPU output (captured after its timing)
    against the fp64 oracle over every output element: |gpu - oracle| /
    (1 + |oracle|) and the merged-lse error over its bound max(1e-5, 2^-22
    |lse|); empty rows must give exactly 0 and -inf.  The oracle runs on every
    host core (the batches split over threads, each calling the unchanged
    oracle)."""
    import numpy as np
    import oracle
    from lse_weighted_merge_b200 import synth
    lib = oracle.load()
    tol = {"bf16": 4e-3, "f16": 4e-3, "f32": 1e-5}
    res = {}
    for name, (inp, got, got_lse) in captured.items():
        want, want_lse = oracle.merge(inp["o"], inp["lse"], inp["R"], inp["B"], inp["H"], inp["D"],
                                      inp["o_strides"], inp["lse_strides"],
                                      synth.DTYPES[inp["in_dtype"]], lib=lib, threads=0)
        err = float(np.max(np.abs(got - want) / (1.0 + np.abs(want))))
        empty = want_lse == -np.inf
        wl = want_lse[~empty]
        lerr = float(np.max(np.abs(got_lse[~empty] - wl) / np.maximum(1e-5, 2.0 ** -22 * np.abs(wl)))) \
            if wl.size else 0.0
        empty_ok = bool(np.array_equal(got_lse == -np.inf, empty) and np.all(got[empty] == 0.0))
        t = tol[inp["out_dtype"]]
        res[name] = {"max_scaled_err": err, "tol": t, "lse_err_over_bound": lerr,
                     "empty_rows": int(empty.sum()), "empty_rows_ok": empty_ok,
                     "nan": bool(np.isnan(got).any() or np.isnan(got_lse).any()),
                     "ok": bool(err <= t and lerr <= 1.0 and empty_ok)}
    return res


def _timed(fn, budget_s: float):
    """Call fn() repeatedly for at least budget_s; returns (calls, seconds)."""
    n, t0 = 0, time.perf_counter()
    while True:
        fn()
        n += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            return n, dt


def next_rows_cpu_baselines(extra: dict, budget_s: float = 1.0) -> None:
    """The fp64 oracle timed beside the state update, the decode attention and
    the exchange lines, on a bounded sample of each (single thread): adds a
    `cpu_baseline` entry to each row of `extra`."""
    import math
    import numpy as np
    import oracle
    from lse_weighted_merge_b200 import synth
    lib = oracle.load()
    rng = np.random.Generator(np.random.PCG64(7))
    if "state_update" in extra:
        # 8 of the 512 batches of the B=512 H=16 D=512 fold, fp32 accumulator, bf16 partial
        B, H, D = 8, 16, 512
        acc = rng.standard_normal(B * H * D, dtype=np.float32)
        new = synth.pack(rng.standard_normal(B * H * D, dtype=np.float32), "bf16")
        la = rng.uniform(0, 8, B * H).astype(np.float32)
        byts = B * H * (D * 10 + 12)
        n, dt = _timed(lambda: oracle.state_update(acc, la, oracle.F32, new, la, oracle.BF16,
                                                   B, H, D, lib=lib), budget_s)
        extra["state_update"]["cpu_baseline"] = {
            "value": byts * n / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"8 of 512 batches, {n} passes in {dt:.1f} s, fp64 C oracle, single thread"}
    for name, row in extra.get("decode_attention", {}).items():
        # one (b, query head) row of the shape: attention over all L keys, fp64
        L, D = (4096, 128) if "l4096" in name else (32768, 128)
        q = rng.standard_normal(D)
        k = rng.standard_normal((L, D))
        v = rng.standard_normal((L, D))
        n, dt = _timed(lambda: oracle.attention_shard(q, k, v, 1 / math.sqrt(D), 0, L, lib=lib),
                       budget_s)
        per_row = L * D * 2 * 2 // (4 if "hq32_hkv8" in name else 1)   # K and V bytes per query head
        row["cpu_baseline"] = {
            "value": per_row * n / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"one query head over all {L} keys, {n} passes in {dt:.1f} s, fp64 C oracle",
            "us_per_query_head": dt / n * 1e6}
    for name, row in extra.get("cp_exchange_merge", {}).items():
        w = synth.CP_WORKLOADS[name]
        inp = synth.make_inputs(w)
        n, dt = _timed(lambda: oracle.cp_exchange_merge(inp["o"], inp["lse"], w.R, w.B, w.H, w.D,
                                                        synth.DTYPES[w.in_dtype], lib=lib), budget_s)
        row["cpu_baseline"] = {"value": dt / n * 1e6, "unit": "us/call", "cores": 1, "kind": "oracle",
                               "sample": f"the whole workload, {n} calls in {dt:.1f} s, fp64 C oracle"}


# ------------------------------------------------------------------------- arms

def run_reference(args):
    """The fp64 CPU oracle as the reference arm: rank 0 only, host cores."""
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    from lse_weighted_merge_b200 import synth
    name = args.workload or synth.LARGE
    w = synth.WORKLOADS[name]
    inp = synth.make_inputs(w)
    batches = w.B   # the whole workload: one step of the oracle is one merge of the batch
    smp = sample_inputs(inp, batches)
    import oracle
    lib = oracle.load()
    sbytes = w.R * batches * w.H * (w.D * synth.ELEM_BYTES[w.in_dtype] + 4) + \
        batches * w.H * (w.D * synth.ELEM_BYTES[w.out_dtype] + 4)

    st = {}

    def one():
        oracle.merge(smp["o"], smp["lse"], w.R, batches, w.H, w.D, smp["o_strides"],
                     smp["lse_strides"], synth.DTYPES[w.in_dtype], lib=lib, threads=0, stats=st)

    for _ in range(args.warmup):
        one()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        one()
    dt = time.perf_counter() - t0
    ms = dt * 1e3 / args.steps
    gbs = sbytes * args.steps / dt / 1e9
    used = st.get("threads", 1)
    sample = (f"all {w.B} batches ({w.rows} rows) per step, fp64 C oracle, batches split over "
              f"{used} host threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(w, args.gpus, "no GPU (host cores)"),
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": used, "kind": "oracle",
                         "sample": sample, "cpu": cpu_model(), "host_cores": os.cpu_count()},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(w, n_gpus: int, l2: str) -> dict:
    return {"workload": w.name, "R": w.R, "B": w.B, "H": w.H, "D": w.D,
            "in_dtype": w.in_dtype, "out_dtype": w.out_dtype, "layout": w.layout,
            "bytes_per_step": w.bytes_total(), "global_batch": w.B * n_gpus, "l2": l2,
            "parallelism": f"replicas x{n_gpus} (independent rows, no collective)"}


def run_ours(args):
    import torch
    from lse_weighted_merge_b200 import _native as nat  # noqa: F401  (fails loudly without the library)
    from lse_weighted_merge_b200 import synth

    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        log(f"note: WORLD_SIZE={world} but --gpus {args.gpus}")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    dist = dist_init(world)

    name = args.workload or synth.LARGE
    w = synth.WORKLOADS[name]
    props = torch.cuda.get_device_properties(device)
    l2 = getattr(props, "L2_cache_size", 0) or L2_FALLBACK
    inp = synth.make_inputs(w, seed=w.seed + 7919 * rank)   # each rank its own batch
    nset = n_sets(w.bytes_total(), l2)
    sets = DeviceSets(inp, nset, device)
    l2_note = (f"rotating {nset} input/output sets ({nset * w.bytes_total() / 1e6:.0f} MB > 2 x L2 "
               f"{l2 / 2**20:.0f} MiB)")

    clock = ClockSampler(device)
    clock.start()
    attempts = []
    trials = max(1, args.trials)
    for attempt in range(2):
        barrier(dist, device)
        torch.cuda.synchronize(device)
        regions, t0, t1 = time_eager(sets, args.steps, args.warmup, device, trials)
        barrier(dist, device)
        # every rank takes the same collective steps: one max per trial
        regions = [max_over_ranks(r, dist, device) for r in regions]
        clk = clock.summary(t0, t1)
        attempts.append((regions, clk))
        bad = [r for r in clk.get("reasons", []) if r in BAD_REASONS]
        bad_flag = max_over_ranks(1.0 if bad else 0.0, dist, device)
        if bad_flag == 0.0:
            break
        log(f"clock reasons {bad} during the timed region: measuring once more")
    regions, clk = attempts[-1]
    region_ms = statistics.median(regions)
    launch_ms = region_ms / args.steps
    if len(attempts) > 1:
        clk["remeasured"] = True

    bytes_step = w.bytes_total()
    ms_per_step = region_ms / args.steps
    value = bytes_step * world * args.steps / (region_ms * 1e-3) / 1e9
    peak, peak_src = hbm_peak()
    achieved = bytes_step / (launch_ms * 1e-3) / 1e9
    traffic, traffic_src = profiled_traffic(name)

    e2e = None
    if not args.no_e2e:
        barrier(dist, device)
        r = time_e2e(inp, args.e2e_steps, device)
        ms_e2e = max_over_ranks(r["ms_per_step"], dist, device)
        e2e = {"value": bytes_step * world / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
               "h2d_bytes_per_step": r["h2d_bytes_per_step"],
               "d2h_bytes_per_step": r["d2h_bytes_per_step"], "ms_per_step": ms_e2e,
               "steps": r["steps"], "chunks": r["chunks"],
               "api": ("lse_merge_host (C ABI: chunked uploads, merges and copies back on its own "
                       "streams) through lse_weighted_merge_b200.merge_host(pipeline=True), pinned "
                       "host tensors in and out"),
               "clocks": clock.summary(r["t0"], r["t1"])}

    extra, captured = {}, {}
    if not args.no_extra:
        extra, captured = extra_workloads(device, l2, dist, clock, trials)
    clock.stop()
    del sets
    torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        if extra:
            next_rows_cpu_baselines(extra)
            errs = oracle_errors(captured)
            for wname, row in extra["workload_detail"].items():
                row["oracle"] = errs.get(wname)
            for wname, row in extra["workloads"].items():
                e = errs.get(wname)
                if e:
                    row.update({"err": _r(e["max_scaled_err"], 3), "tol": e["tol"],
                                "lse_over_bound": _r(e["lse_err_over_bound"], 3), "ok": e["ok"]})
        cpu = cpu_baselines(inp, max(1, w.B // 8), args.cpu_seconds)

    if dist is not None:
        barrier(dist, device)
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config_block(w, world, l2_note),
        "trials": {"count": trials, "steps_each": args.steps, "reported": "median",
                   "region_ms": regions},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": peak_src,
                     "traffic_source": traffic_src, "kernel_us": launch_ms * 1e3,
                     "algorithmic_bytes_per_launch": bytes_step,
                     "frac_of_nominal_8000": achieved / 8000.0},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": args.steps,
        "gpu_launches_note": "one merge kernel per step; each of the trials times exactly `steps` launches",
        "clocks": clk,
        "gpu": torch.cuda.get_device_name(device),
        **extra,
    }
    print(json.dumps(line), flush=True)
    return 0


def _r(x, digits: int = 4):
    """x rounded to `digits` significant digits (None stays None)."""
    return None if x is None else float(f"{x:.{digits}g}")


def extra_workloads(device, l2: int, dist, clock, trials: int = 5):
    """Every merge workload: eager us/call (200 back-to-back calls) and
    CUDA-graph-replayed us/call (100 calls x 50 replays), each the median of
    `trials` rounds, inputs rotated past L2 except for the two latency shapes
    (L2-resident, as a decode step's merge would be).  Returns (extra keys of
    the JSON line, {workload: (inputs, output, merged lse)} of one call for the
    oracle comparison).  The compact `workloads` block is placed last."""
    import numpy as np
    import torch
    from lse_weighted_merge_b200 import synth
    detail, compact, captured = {}, {}, {}
    peak, _ = hbm_peak()
    for name, w in synth.WORKLOADS.items():
        inp = synth.make_inputs(w)
        tiny = w.bytes_total() < 1 << 20
        nset = 4 if tiny else n_sets(w.bytes_total(), l2)
        sets = DeviceSets(inp, nset, device)
        # one call on set 0 for the comparison with the oracle
        sets.launch(0, torch.cuda.current_stream(device).cuda_stream)
        torch.cuda.synchronize(device)
        captured[name] = (inp, sets.out[0].double().cpu().numpy(),
                          sets.out_lse[0].double().cpu().numpy())
        regions, e_t0, e_t1 = time_eager(sets, 200, 20, device, trials)
        eager_us = statistics.median(regions) * 1e3 / 200
        graph_us, g_t0, g_t1 = time_graph(sets, 100, 50, device, trials)
        mhz = clock.summary(g_t0, g_t1).get("sm_mhz")
        gbs = w.bytes_total() / (graph_us * 1e-6) / 1e9
        detail[name] = {
            "eager_us_per_call": eager_us, "eager_trials_us": [r * 1e3 / 200 for r in regions],
            "graph_us_per_call": graph_us, "graph": "100 calls captured, 50 replays, median of trials",
            "gbs_graph": gbs, "gbs_eager": w.bytes_total() / (eager_us * 1e-6) / 1e9,
            "frac_of_measured_hbm_graph": gbs / peak, "bytes_per_call": w.bytes_total(),
            "sm_mhz_graph": mhz, "graph_kcycles": graph_us * mhz / 1e3 if mhz else None,
            "l2": "resident (latency shape)" if tiny else f"rotating {nset} sets"}
        compact[name] = {"eager_us": _r(eager_us), "graph_us": _r(graph_us), "gbs": _r(gbs),
                         "frac": _r(gbs / peak, 3), "mhz": mhz}
        del sets
        torch.cuda.empty_cache()
    extra = {"state_update": time_state_update(device, l2, peak, trials=trials),
             "many_partials": time_many_partials(device, l2, peak, trials=trials),
             "decode_attention": time_decode_attention(device, peak, trials=trials),
             "cp_exchange_merge": time_cp_exchange(device, peak, trials=trials),
             "workload_detail": detail,
             "workloads": compact}
    return extra, captured


def time_many_partials(device, l2: int, peak: float, trials: int = 5) -> dict:
    """A merge of R=32 partials (bf16 [B,H,R,D], B=256 H=16 D=512, 139 MB):
    graph-replayed us/call (100 calls x 50 replays, median of `trials`) of
    the AUTO choice (the persistent kernel's long form, chunks of 16 partials
    with a running max) and of the WIDE path forced, inputs rotated past L2."""
    import torch
    from lse_weighted_merge_b200 import _native as nat
    from lse_weighted_merge_b200 import synth
    w = synth.Workload("r32_b256_h16_d512", 32, 256, 16, 512, "bf16", "bf16", "bhrd", 1.0,
                       "normal", (8.0, 4.0), 1200)
    inp = synth.make_inputs(w)
    sets = DeviceSets(inp, n_sets(w.bytes_total(), l2), device)
    row = {"shape": "R=32 B=256 H=16 D=512, bf16 [B,H,R,D] -> bf16", "bytes_per_call": w.bytes_total()}
    for tag, path in (("auto", nat.PATH_AUTO), ("wide", nat.PATH_WIDE)):
        sets.path = path
        us, _, _ = time_graph(sets, 100, 50, device, trials)
        row[tag] = {"graph_us_per_call": us, "gbs": w.bytes_total() / (us * 1e-6) / 1e9,
                    "frac_of_measured_hbm": w.bytes_total() / (us * 1e-6) / 1e9 / peak}
    st = synth.strides(w.layout, w.R, w.B, w.H, w.D)
    rc, plan = nat.plan_query(sets.args[0][0], sets.args[0][1], w.R, w.B, w.H, w.D, st,
                              nat.BF16, nat.BF16, sets.args[0][2], sets.args[0][3])
    row["auto"]["path"] = plan["path_name"] + (" (long form)" if w.R > plan["rc"] else "")
    del sets
    torch.cuda.empty_cache()
    return row


def time_cp_exchange(device, peak: float, only: str | None = None, trials: int = 5) -> dict:
    """Context-parallel exchange + merge with every rank on this one GPU, all
    ranks played by one cooperative launch (lse_merge_cp_exchange_merge):
    us/call eager (a prepared CPMergeCall: one launch per call, 200 calls)
    and graph-replayed (20 calls captured, 50 replays), each the median of
    `trials` rounds.  Bytes per call on one GPU: every rank's partials read
    once, the (world-1)/world of them owned elsewhere written to and read back
    from the workspaces, the outputs written.  On world GPUs the same kernel
    would move the (world-1)/world share over NVLink instead; that cannot be
    measured here."""
    import torch
    from lse_weighted_merge_b200 import cp, synth
    res = {}
    for name, w in synth.CP_WORKLOADS.items():
        if only is not None and name != only:
            continue
        inp = synth.make_inputs(w)
        W, B, H, D = w.R, w.B, w.H, w.D
        dt = {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[w.in_dtype]
        raw = torch.from_numpy(inp["o"].view("int16") if w.in_dtype != "f32" else inp["o"])
        o = raw.to(device).view(dt).view(W, B, H, D)
        l = torch.from_numpy(inp["lse"]).to(device).view(W, B, H)
        lo = [o[r].contiguous() for r in range(W)]
        ll = [l[r].contiguous() for r in range(W)]
        ws = [cp.cp_workspace(W, B, H, D, dt, device) for _ in range(W)]
        call = cp.CPMergeCall(lo, ll, ws)
        eb = {"bf16": 2, "f16": 2, "f32": 4}[w.in_dtype]
        part = W * B * H * (D * eb + 4)
        byts = part + 2 * part * (W - 1) // W + W * B * (H // W) * (D * eb + 4)

        for _ in range(10):
            call()
        torch.cuda.synchronize(device)
        n = 200
        eager = []
        for _ in range(trials):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(n):
                call()
            e1.record()
            torch.cuda.synchronize(device)
            eager.append(e0.elapsed_time(e1) * 1e3 / n)
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream(device)
        side.wait_stream(torch.cuda.current_stream(device))
        reps = 20
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for _ in range(reps):
                    call()
        torch.cuda.synchronize(device)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize(device)
        graph = []
        for _ in range(trials):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(50):
                g.replay()
            e1.record()
            torch.cuda.synchronize(device)
            graph.append(e0.elapsed_time(e1) * 1e3 / (50 * reps))
        status = [cp.cp_status(x) for x in ws]
        gu = statistics.median(graph)
        res[name] = {"shape": f"world={W} B={B} H={H} D={D} {w.in_dtype}, all ranks in one launch",
                     "eager_us_per_call": statistics.median(eager), "graph_us_per_call": gu,
                     "bytes_per_call_one_gpu": byts,
                     "graph_gbs": byts / (gu * 1e-6) / 1e9,
                     "frac_of_measured_hbm_graph": byts / (gu * 1e-6) / 1e9 / peak,
                     "nvlink_bytes_per_rank_if_distributed": part // W * (W - 1) // W,
                     "timeouts": sum(1 for x in status if x)}
        del g, call, ws, lo, ll, o, l
        torch.cuda.empty_cache()
    return res


DECODE_SHAPES = (  # name, B, Hq, Hkv, L, D, R
    ("b64_hq32_hkv8_l4096_d128_r4", 64, 32, 8, 4096, 128, 4),
    ("b8_hq8_hkv8_l32768_d128_r8", 8, 8, 8, 32768, 128, 8),
)


def time_decode_attention(device, peak: float, only: str | None = None, trials: int = 5) -> dict:
    """Split-KV decode attention producing and merging the partials, three
    ways: fused (one launch; each split's partial goes to a workspace and the
    last split of each (b, KV head) merges them), cluster (one launch; the
    splits form a cluster and merge in distributed shared memory) and
    unfused (the partials kernel, then lse_merge).  Algorithmic bytes per call:
    K and V once (B*Hkv*L*D*2*2), q and the output once.  Two input/output
    sets alternate from call to call, so every call reads its 1.07 GB of K/V
    from HBM (the other set's 1.07 GB has passed through the 126 MB L2 in
    between).  50 calls per trial, median of `trials`."""
    import torch
    from lse_weighted_merge_b200 import _native as nat
    res = {}
    nsets = 2
    for name, B, Hq, Hkv, L, D, R in DECODE_SHAPES:
        if only is not None and name != only:
            continue
        gen = torch.Generator(device=device).manual_seed(7)
        sets = []
        for _ in range(nsets):
            q = torch.randn((B, Hq, D), generator=gen, device=device).to(torch.bfloat16)
            k = torch.randn((B, Hkv, L, D), generator=gen, device=device).to(torch.bfloat16)
            v = torch.randn((B, Hkv, L, D), generator=gen, device=device).to(torch.bfloat16)
            out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=device)
            lse = torch.empty((B, Hq), dtype=torch.float32, device=device)
            po = torch.empty((B, Hq, R, D), dtype=torch.float32, device=device)
            pl = torch.empty((B, Hq, R), dtype=torch.float32, device=device)
            ws = torch.zeros(nat.decode_workspace_bytes(B, Hq, Hkv, R, D), dtype=torch.uint8,
                             device=device)
            sets.append((q, k, v, out, lse, po, pl, ws))
        s = torch.cuda.current_stream(device).cuda_stream
        scale = 1.0 / math.sqrt(D)
        byts = B * Hkv * L * D * 2 * 2 + B * Hq * D * 2 * 2 + B * Hq * 4

        def fused(i):
            q, k, v, out, lse, _, _, ws = sets[i % nsets]
            nat.decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, B, Hq, Hkv, L, D, R,
                           scale, None, nat.BF16, out.data_ptr(), lse.data_ptr(), s, fused=True,
                           out_dtype=nat.BF16, workspace=ws.data_ptr(), workspace_bytes=ws.numel())

        def cluster(i):
            q, k, v, out, lse, _, _, _ = sets[i % nsets]
            nat.decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, B, Hq, Hkv, L, D, R,
                           scale, None, nat.BF16, out.data_ptr(), lse.data_ptr(), s, fused=True,
                           out_dtype=nat.BF16)

        def unfused(i):
            q, k, v, out, lse, po, pl, _ = sets[i % nsets]
            nat.decode_raw(q.data_ptr(), k.data_ptr(), v.data_ptr(), 0, B, Hq, Hkv, L, D, R,
                           scale, None, nat.BF16, po.data_ptr(), pl.data_ptr(), s, fused=False)
            nat.merge_raw(po.data_ptr(), pl.data_ptr(), R, B, Hq, D, None, nat.F32, nat.BF16,
                          out.data_ptr(), lse.data_ptr(), s)

        row = {"shape": f"B={B} Hq={Hq} Hkv={Hkv} L={L} D={D} splits={R}, bf16",
               "bytes_per_call": byts, "l2": f"{nsets} input sets alternating (K/V past L2)"}
        n = 50
        for tag, fn in (("fused", fused), ("cluster", cluster), ("unfused", unfused)):
            for i in range(4):
                fn(i)
            torch.cuda.synchronize(device)
            us = []
            for _ in range(trials):
                e0 = torch.cuda.Event(enable_timing=True)
                e1 = torch.cuda.Event(enable_timing=True)
                e0.record()
                for i in range(n):
                    fn(i)
                e1.record()
                torch.cuda.synchronize(device)
                us.append(e0.elapsed_time(e1) * 1e3 / n)
            u = statistics.median(us)
            row[tag] = {"us_per_call": u, "gbs": byts / (u * 1e-6) / 1e9,
                        "frac_of_measured_hbm": byts / (u * 1e-6) / 1e9 / peak,
                        "launches_per_call": 2 if tag == "unfused" else 1}
        row["fused_over_unfused"] = row["fused"]["us_per_call"] / row["unfused"]["us_per_call"]
        row["cluster_over_unfused"] = row["cluster"]["us_per_call"] / row["unfused"]["us_per_call"]
        res[name] = row
        del sets
        torch.cuda.empty_cache()
    return res


def time_state_update(device, l2: int, peak: float, B: int = 512, H: int = 16, D: int = 512,
                      trials: int = 5) -> dict:
    """In-place fold of one bf16 partial into an fp32 accumulator of B*H rows
    (lse_merge_state_update), eager, inputs rotated past L2, 200 calls per
    trial, median of `trials`.  Algorithmic bytes per call:
    B*H*(D*(4+2+4) + 12) (accumulator read and written, partial read, three
    lse values).  lse_new starts equal to lse_acc, so the new partial keeps a
    weight of about 1/k after k folds and is always read."""
    import torch
    from lse_weighted_merge_b200 import _native as nat
    per = B * H * (D * 10 + 12)
    nset = n_sets(per, l2)
    gen = torch.Generator(device=device).manual_seed(2024)
    accs = [torch.randn((B, H, D), generator=gen, device=device) for _ in range(nset)]
    news = [torch.randn((B, H, D), generator=gen, device=device).to(torch.bfloat16) for _ in range(nset)]
    las = [torch.rand((B, H), generator=gen, device=device) * 8 for _ in range(nset)]
    lns = [la.clone() for la in las]
    s = torch.cuda.current_stream(device).cuda_stream

    def launch(i):
        j = i % nset
        nat.state_update_raw(accs[j].data_ptr(), las[j].data_ptr(), news[j].data_ptr(),
                             lns[j].data_ptr(), B, H, D, None, nat.F32, nat.BF16, s)

    for i in range(20):
        launch(i)
    torch.cuda.synchronize(device)
    n = 200
    us = []
    k = 20
    for _ in range(trials):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(n):
            launch(k)
            k += 1
        e1.record()
        torch.cuda.synchronize(device)
        us.append(e0.elapsed_time(e1) * 1e3 / n)
    u = statistics.median(us)
    gbs = per / (u * 1e-6) / 1e9
    return {"shape": f"B={B} H={H} D={D}, fp32 accumulator, bf16 partial",
            "eager_us_per_call": u, "gbs": gbs, "frac_of_measured_hbm": gbs / peak,
            "bytes_per_call": per, "l2": f"rotating {nset} sets"}


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    if args.state_only:
        import torch
        device = torch.device("cuda", 0)
        peak, _ = hbm_peak()
        props = torch.cuda.get_device_properties(device)
        l2 = getattr(props, "L2_cache_size", 0) or L2_FALLBACK
        print(json.dumps({"state_update": time_state_update(device, l2, peak)}))
        return 0
    if args.cp_only:
        import torch
        device = torch.device("cuda", 0)
        peak, _ = hbm_peak()
        print(json.dumps({"cp_exchange_merge": time_cp_exchange(device, peak, args.cp_only)}))
        return 0
    if args.decode_only:
        import torch
        device = torch.device("cuda", 0)
        peak, _ = hbm_peak()
        print(json.dumps({"decode_attention": time_decode_attention(device, peak, args.decode_only)}))
        return 0
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
