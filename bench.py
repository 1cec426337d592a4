#!/usr/bin/env python
"""Benchmark of the multiresolution hash-grid encoding on B200: encoded points/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl b200|reference]
                    [--workload NAME] [--points N] [--min-timed-s S] [--skip-cpu-baseline]
                    [--skip-e2e] [--skip-legs] [--skip-peaks] [--skip-next-rows]

One step = one pass of the whole hot path over one batch resident in HBM: forward (voxel,
8 corner hashes, gathers, trilinear interpolation, level-major output rows), zero the table
gradient, backward (weighted scatter-add into the fp32 gradient table). The default
workload is the 16-level, F=2, T=2^19 grid (N 16->512) on 2^14 rays x 64 stratified
samples (2^20 points). W warm-up steps, then the K-step loop runs R times back to back so
that the timed region lasts at least --min-timed-s (all R*K steps timed with CUDA events,
L2 flushed before every step, outside its events: see L2Flush). Rank 0 prints one
JSON line with the rate, per-kernel rooflines (HBM basis, and the L2 basis against the
gather / reduction rates the probe kernels measure in the same run), clocks, the other
workloads as "legs" (forward-only grid on 2^18 uniform points, also under "fwd"; fp16
table; 1 GiB grid), "next_rows" (dL/dx, sparse Adam, encoding + MLP, 2-D / 4-D inputs,
fp16-gradient backward), an end-to-end figure through the C ABI from pinned host memory,
and the CPU oracle's rate.

Multi-GPU: one process per GPU (``--gpus N`` starts the N ranks through
torch.distributed.run when no launcher did); every rank encodes its own batch with its own
table replica (points are independent), there is no collective on the data path, and the
value is all ranks' points divided by the slowest rank's time (weak scaling).

``--impl reference`` times the CPU oracle (the only reference this method has) on a
bounded sample of the same workload, on rank 0 only.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads  # noqa: E402

METRIC = "encoded points/s fwd & fwd+bwd at L16 F2 T2^19; % of memory roofline"
UNIT = "points/s"
DEFAULT_WORKLOAD = "rays_L16F2T19"
FWD_WORKLOAD = "grid_L16F2T19"
FLUSH_BYTES = 256 << 20
CPU_SAMPLE_POINTS = 1 << 18
REFERENCE_SAMPLE_POINTS = 1 << 17
NEXT_ROWS_CPU_SAMPLE = 1 << 16
FALLBACK_HBM_GBS = 6650.0
GATHER_MODES = {"auto": 0, "corner": 1, "sector": 2, "pair": 3, "lanes": 4}  # HASHGRID_GATHER_*
SCHEDULES = {"auto": 0, "point": 1, "level": 2}             # HASHGRID_SCHEDULE_*
BACKWARD_MODES = {"auto": 0, "atomic": 1, "dedup": 2, "runs": 3, "dedup_adaptive": 4, "run_lanes": 5}  # HASHGRID_BACKWARD_*


# ---------------------------------------------------------------------------------------
# Roofline arithmetic (bytes the method must move, each counted once)
# ---------------------------------------------------------------------------------------

def algorithmic_bytes_per_point(w: workloads.Workload, kind: str) -> int:
    """fwd: 12 B of x + 8 corners x L*F table elements + 4 B per output element;
    bwd: 12 B of x + 4 B per upstream-gradient element + 8 corners x L*F fp32 reductions."""
    s = 2 if w.dtype == "f16" else 4
    LF = w.L * w.F
    fwd = 12 + 8 * LF * s + 4 * LF
    bwd = 12 + 4 * LF + 8 * LF * 4
    return {"fwd": fwd, "bwd": bwd, "fwdbwd": fwd + bwd}[kind]


def measured_peaks() -> tuple[float, str]:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------------------
# Memory-system peaks of the gather / reduction roofline, measured in the same run
# ---------------------------------------------------------------------------------------

PEAK_BUFFERS = {"32MiB": 32 << 20, "64MiB": 64 << 20}   # both stay in L2 (126 MB)
PEAK_OPS = 1 << 26               # lane operations per probe launch (~0.2-0.5 ms)
PROBE_PATTERNS = {"random": 0, "xpair": 1, "sector_pair": 2, "line_pair": 3, "stream": 4}


def probe_rate(kind: int, width: int, pattern: str, buf, sink, device, reps: int = 5) -> float:
    """Median lane operations per second of one probe (include/hashgrid_probe.h) over
    ``reps`` launches timed with CUDA events, after two untimed ones."""
    import torch
    import multiresolution_hash_grid_b200 as hg
    stream = torch.cuda.current_stream(device)
    nbytes = buf.numel() * buf.element_size()
    for _ in range(2):
        hg.hashgrid_probe(kind, width, PROBE_PATTERNS[pattern], buf, nbytes, PEAK_OPS, sink)
    ts, done = [], 0
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        done = hg.hashgrid_probe(kind, width, PROBE_PATTERNS[pattern], buf, nbytes, PEAK_OPS, sink)
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize(device)
    return done / (statistics.median(x.elapsed_time(y) for x, y in ts) * 1e-3)


def measure_l2_peaks(device) -> dict:
    """Rates of the encoding's own accesses on buffers that stay in L2 (32 and 64 MiB, the
    sizes of the fp16 and fp32 default tables and of one level of the 1 GiB grid), in lane
    operations per second: gathers of 4 to 16 bytes (a table entry of F*s bytes) and fp32 /
    fp16 reductions of 4 to 16 bytes (one corner's F-wide contribution), each with
    independent random units and with the hash's x-neighbour pairs (two lanes of an
    instruction on units v XOR K and (v + 1) XOR K: the access pattern of the lane-pair
    kernels); plus 32-byte random gathers and a coalesced sweep for context."""
    import torch
    import multiresolution_hash_grid_b200 as hg
    kinds = {"gather": hg.HASHGRID_PROBE_GATHER, "red": hg.HASHGRID_PROBE_RED, "red_f16": hg.HASHGRID_PROBE_RED_F16}
    out = {"ops_per_launch": PEAK_OPS, "unit": "G lane operations/s",
           "method": "hashgrid_probe kernels (8 blocks x 256 threads per SM, 8 independent operations in flight "
                     "per thread), median of 5 launches timed with CUDA events after 2 untimed ones",
           "buffers": {}}
    sink = torch.zeros(1, dtype=torch.float32, device=device)
    for key, nbytes in PEAK_BUFFERS.items():
        buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        b = {}
        for kname, kind in kinds.items():
            b[kname] = {}
            for w in (4, 8, 16):
                b[kname][str(w)] = {pat: round(probe_rate(kind, w, pat, buf, sink, device) / 1e9, 2)
                                    for pat in ("random", "xpair")}
        b["gather"]["32"] = {"random": round(probe_rate(kinds["gather"], 32, "random", buf, sink, device) / 1e9, 2)}
        b["stream_read_gbs"] = round(probe_rate(kinds["gather"], 16, "stream", buf, sink, device) * 16 / 1e9, 1)
        out["buffers"][key] = b
        del buf
    return out


def csrc_digest() -> str:
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "multiresolution_hash_grid_b200", "csrc", "*")))
    for f in files:
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode() + fh.read())
    return h.hexdigest()[:16]


def ncu_entry(kernel: str, workload: str) -> dict | None:
    """The committed ncu figures of ``kernel`` on ``workload`` (profiles/ncu_traffic.json),
    or None when the kernel sources changed since that capture."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    if d.get("csrc_sha") != csrc_digest():
        return None
    return d.get("kernels", {}).get(f"{kernel}@{workload}")


def ncu_traffic(kernel: str, workload: str) -> float | None:
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum), or None."""
    ent = ncu_entry(kernel, workload)
    return None if ent is None else float(ent["dram_bytes_per_launch"])


# ---------------------------------------------------------------------------------------
# Ranks (one process per GPU); helpers are backend-agnostic so gloo tests cover them
# ---------------------------------------------------------------------------------------

def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (independent units; weak scaling)."""
    return 1000 + rank


def max_over_ranks(value: float, device=None) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and getattr(device, "type", "cpu") == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def whole_job_rate(units_per_rank: int, world: int, max_seconds: float) -> float:
    return units_per_rank * world / max_seconds


# ---------------------------------------------------------------------------------------
# Clock sampling during the timed region (NVML polling thread; nvidia-smi as fallback)
# ---------------------------------------------------------------------------------------

REASON_BITS = {  # NVML clocks-event-reason bits
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
}


class ClockSampler:
    """Polls SM clock and clock-event reasons of the current GPU while active."""

    def __init__(self, device_index: int):
        self.samples: list[tuple[float, int]] = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hd = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hd)
                u = u.decode() if isinstance(u, bytes) else u
                if uuid.replace("GPU-", "") in u:
                    handle = hd
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self._handle = handle
            self._nvml = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: the JSON line records why
            self.error = f"nvml unavailable: {e}"

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
                self.samples.append((mhz, reasons))
            except Exception as e:
                self.error = str(e)
                return
            time.sleep(0.002)

    def __enter__(self):
        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.error or "no samples"}
        mhz = [m for m, _ in self.samples]
        bits = 0
        for _, r in self.samples:
            bits |= int(r)
        reasons = sorted(n for b, n in REASON_BITS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# ---------------------------------------------------------------------------------------
# Device timing
# ---------------------------------------------------------------------------------------

class Resident:
    """One workload's inputs and outputs resident in HBM, plus the library handle."""

    def __init__(self, w: workloads.Workload, seed: int, device, backward: bool,
                 gather: str = "auto", backward_mode: str = "auto", schedule: str = "auto", points: int | None = None):
        import torch

        import multiresolution_hash_grid_b200 as hg
        self.w, self.hg, self.backward = w, hg, backward
        inp = workloads.make_inputs(w, seed=seed, n_points=points, grads=backward)
        self.N = inp.x.shape[0]
        self.x = torch.from_numpy(inp.x).to(device)
        self.table = torch.from_numpy(inp.table).to(device)
        self.out = torch.empty((self.N, w.L * w.F), dtype=torch.float32, device=device)
        self.g = torch.from_numpy(inp.g).to(device) if backward else None
        self.dtable = torch.zeros((w.L, w.T, w.F), dtype=torch.float32, device=device) if backward else None
        dt = hg.HASHGRID_F16 if w.dtype == "f16" else hg.HASHGRID_F32
        self.handle = hg.hashgrid_create(w.L, w.F, w.log2T, w.N_min, w.N_max, dt)
        hg.hashgrid_set_option(self.handle, hg.HASHGRID_OPT_FORWARD_GATHER, GATHER_MODES[gather])
        hg.hashgrid_set_option(self.handle, hg.HASHGRID_OPT_BACKWARD_MODE, BACKWARD_MODES[backward_mode])
        hg.hashgrid_set_option(self.handle, hg.HASHGRID_OPT_SCHEDULE, SCHEDULES[schedule])
        self.host = inp

    def forward(self, stream):
        self.hg.hashgrid_forward(self.handle, self.x, self.N, self.table, self.out, stream)

    def backward_pass(self, stream):
        self.hg.hashgrid_backward(self.handle, self.x, self.g, self.N, self.dtable, stream)

    def close(self):
        self.hg.hashgrid_destroy(self.handle)


class L2Flush:
    """Evicts the workload's data from L2 before a timed launch, outside its events: writes
    a 256 MiB buffer (twice the L2), then reads a second 256 MiB buffer. The read evicts
    the write's dirty lines, so their write-back to HBM happens here rather than inside the
    next timed launch (measured: it added ~8 us to the 52 us sparse Adam step). L2 is left
    holding clean lines of the read buffer and none of the workload's data."""

    def __init__(self, device):
        import torch
        self.wbuf = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.rbuf = torch.ones(FLUSH_BYTES // 4, dtype=torch.int32, device=device)
        self()  # loads the two kernels now, so that no warm-up step pays for it
        torch.cuda.synchronize(device)

    def __call__(self):
        self.wbuf.fill_(1)
        self.rbuf.amax()


def loop_repeats(steps: int, step_s: float, min_timed_s: float) -> int:
    """How many times the K-step loop runs back to back in the timed region so that the
    region lasts at least ``min_timed_s`` (at least once)."""
    if min_timed_s <= 0 or step_s <= 0:
        return 1
    return max(1, int(-(-min_timed_s // (steps * step_s))))


def time_steps(res: Resident, steps: int, warmup: int, device, sampler=None, min_timed_s: float = 0.0) -> dict:
    """Times steps with CUDA events on the launching stream. Each step: forward, zero the
    gradient and backward (if backward). L2 is flushed before every step, outside the
    step's events. The timed region runs the K-step loop R times back to back (R from the
    warm-up's wall time so that the region lasts at least ``min_timed_s``; R is the same
    on every rank), and every one of the R * K steps is timed. Returns per-phase mean
    milliseconds, the max-over-ranks total and R."""
    import torch
    stream = torch.cuda.current_stream(device)
    sp = stream.cuda_stream
    flush = L2Flush(device)

    def one(evs=None):
        # forward, then zero the gradient, then backward: the zeroed gradient table is
        # still in L2 when the backward's reductions reach it (zeroing before the forward
        # lets the forward's output writes evict it; measured ~2% slower backward)
        flush()
        if evs:
            evs[0].record(stream)
        res.forward(sp)
        if evs:
            evs[1].record(stream)
        if res.backward:
            res.dtable.zero_()
        if evs:
            evs[2].record(stream)
        if res.backward:
            res.backward_pass(sp)
        if evs:
            evs[3].record(stream)

    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    for _ in range(warmup):
        one()
    torch.cuda.synchronize(device)
    step_s = (time.perf_counter() - t0) / max(warmup, 1)
    repeats = int(max_over_ranks(float(loop_repeats(steps, step_s, min_timed_s)), device))
    n = steps * repeats
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n)]
    torch.cuda.synchronize(device)
    barrier(device)
    torch.cuda.synchronize(device)
    if sampler is not None:
        sampler.__enter__()
    for k in range(n):
        one(events[k])
    torch.cuda.synchronize(device)
    if sampler is not None:
        sampler.__exit__(None, None, None)
    barrier(device)
    torch.cuda.synchronize(device)
    fwd = [e[0].elapsed_time(e[1]) for e in events]
    zero = [e[1].elapsed_time(e[2]) for e in events]
    bwd = [e[2].elapsed_time(e[3]) for e in events] if res.backward else [0.0] * n
    total = [e[0].elapsed_time(e[3]) for e in events]
    total_ms = sum(total)
    return {
        "total_ms": total_ms,
        "max_total_ms": max_over_ranks(total_ms, device),
        "zero_ms": statistics.mean(zero), "fwd_ms": statistics.mean(fwd), "bwd_ms": statistics.mean(bwd),
        "step_ms": statistics.mean(total),
        "repeats": repeats, "timed_steps": n,
        "launches": n * (2 if res.backward else 1),
    }


def time_e2e(res: Resident, steps: int, warmup: int, device, min_timed_s: float = 0.0) -> dict:
    """End to end through the C ABI from pinned host buffers: per step, copy x (and the
    upstream gradient) host->device, forward, zero the gradient, backward, and copy the
    encoding back to pinned host memory. The gradient table stays on the device for the
    optimizer. Steps are pipelined on three streams with double buffers: the upload of
    step k+1 and the download of step k-1 overlap step k's kernels (PCIe is full duplex).
    The timed run is R * K steps, R from the warm-up's wall time (the same on every rank)
    so that it lasts at least ``min_timed_s``: a stream of steps, whose rate the pipeline's
    fill and drain (about one upload and one download) distort less the longer it runs."""
    import torch
    hg = res.hg
    s_in, s_comp, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device), torch.cuda.Stream(device)
    xh = torch.from_numpy(res.host.x).pin_memory()
    gh = torch.from_numpy(res.host.g).pin_memory() if res.backward else None
    xd = [res.x, torch.empty_like(res.x)]
    gd = [res.g, torch.empty_like(res.g)] if res.backward else [None, None]
    od = [res.out, torch.empty_like(res.out)]
    oh = [torch.empty(res.out.shape, dtype=torch.float32).pin_memory() for _ in range(2)]
    h2d = xh.numel() * 4 + (gh.numel() * 4 if gh is not None else 0)
    d2h = oh[0].numel() * 4
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    for b in range(2):   # every buffer starts free
        ev_comp[b].record(s_comp)
        ev_out[b].record(s_out)

    def one(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[b])              # step k-2 no longer reads xd[b], gd[b]
            xd[b].copy_(xh, non_blocking=True)
            if gh is not None:
                gd[b].copy_(gh, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            s_comp.wait_event(ev_out[b])             # step k-2's download of od[b] is done
            sp = s_comp.cuda_stream
            hg.hashgrid_forward(res.handle, xd[b], res.N, res.table, od[b], sp)
            if res.backward:
                res.dtable.zero_()
                hg.hashgrid_backward(res.handle, xd[b], gd[b], res.N, res.dtable, sp)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            oh[b].copy_(od[b], non_blocking=True)
            ev_out[b].record(s_out)

    torch.cuda.synchronize(device)
    t0 = time.perf_counter()
    for k in range(warmup):
        one(k)
    torch.cuda.synchronize(device)
    step_s = (time.perf_counter() - t0) / max(warmup, 1)
    n = steps * int(max_over_ranks(float(loop_repeats(steps, step_s, min_timed_s)), device))
    barrier(device)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(n):
        one(warmup + k)
    e1.record(s_out)
    torch.cuda.synchronize(device)
    ms = max_over_ranks(e0.elapsed_time(e1), device)
    return {"ms": ms, "h2d": h2d, "d2h": d2h, "steps": n}


def time_launches(fn, steps: int, warmup: int, device, before=None) -> float:
    """Mean milliseconds of ``fn`` (one launch on the current stream) over ``steps`` timed
    calls, each after an L2 flush and the optional untimed ``before``."""
    import torch
    stream = torch.cuda.current_stream(device)
    flush = L2Flush(device)
    for _ in range(warmup):
        if before is not None:
            before()
        fn()
    ts = []
    for _ in range(steps):
        flush()
        if before is not None:
            before()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        fn()
        b.record(stream)
        ts.append((a, b))
    torch.cuda.synchronize(device)
    return statistics.mean(a.elapsed_time(b) for a, b in ts)


def time_next_rows(res: Resident, steps: int, warmup: int, device, l2peaks=None) -> tuple[dict, int]:
    """The operations beyond the forward/backward pair, on the same resident batch: the
    gradient w.r.t. x, one sparse Adam step over the table, the encoding fused with the
    3-layer MLP on the tensor cores, and the backward into an fp16 gradient table. Each is
    one launch, timed alone. Returns the JSON object and the number of timed launches."""
    import torch
    hg, w, N, sp = res.hg, res.w, res.N, torch.cuda.current_stream(device).cuda_stream
    peak, src = measured_peaks()
    s = 2 if w.dtype == "f16" else 4
    LF = w.L * w.F
    out, launches = {"workload": w.name, "peak_note": f"{src} HBM peak"}, 0

    def entry(ms, nbytes, kernel, **extra):
        gbs = nbytes / (ms * 1e-3) / 1e9
        return {"ms": round(ms, 5), "points_per_s": round(N / (ms * 1e-3), 1),
                "roofline": {"bound": "hbm", "kernel": kernel, "achieved": round(gbs, 1), "peak": peak,
                             "unit": "GB/s", "frac": round(gbs / peak, 4), "bytes_per_launch": int(nbytes),
                             "traffic": ncu_traffic(kernel, w.name)}, **extra}

    # dL/dx: x, upstream gradient and 8 corner gathers per level in; dL/dx out.
    dx = torch.empty((N, 3), dtype=torch.float32, device=device)
    ms = time_launches(lambda: hg.hashgrid_backward_input(res.handle, res.x, res.g, N, res.table, dx, sp),
                       steps, warmup, device)
    out["backward_input"] = entry(ms, N * (12 + 4 * LF + 8 * LF * s + 12), "backward_input_kernel")
    launches += steps

    # Sparse Adam over the table with the gradient of one backward pass: every gradient
    # element is read; parameter, m and v are read and written where the gradient is nonzero.
    if w.dtype == "f32":
        res.dtable.zero_()
        res.backward_pass(sp)
        nnz = int(torch.count_nonzero(res.dtable))
        table, m, v = res.table.clone(), torch.zeros_like(res.table), torch.zeros_like(res.table)
        step = [0]

        def adam():
            step[0] += 1
            hg.hashgrid_adam_step(res.handle, table, m, v, res.dtable, step[0], 1e-2, zero_grad=False, stream=sp)
        ms = time_launches(adam, steps, warmup, device)
        out["adam_step"] = entry(ms, 4 * res.dtable.numel() + 24 * nnz, "adam_kernel", elements=res.dtable.numel(),
                                 nonzero=nnz, elements_per_s=round(res.dtable.numel() / (ms * 1e-3), 1))
        out["adam_step"].pop("points_per_s")
        launches += steps
        del table, m, v

    # Encoding + MLP (LF -> 64 -> 64 -> 4, bf16 operands, fp32 accumulation): x and the
    # gathers in, 4 outputs per point out; the weights stay in shared memory.
    if LF in (16, 32, 48, 64):
        gen = torch.Generator(device="cpu").manual_seed(7)
        bf = lambda *shape: (torch.randn(*shape, generator=gen) * 0.1).to(torch.bfloat16).to(device)  # noqa: E731
        w1, w2, w3 = bf(64, LF), bf(64, 64), bf(4, 64)
        b1, b2, b3 = (torch.zeros(64, device=device), torch.zeros(64, device=device), torch.zeros(4, device=device))
        y = torch.empty((N, 4), dtype=torch.float32, device=device)
        ms = time_launches(lambda: hg.hashgrid_mlp_forward(res.handle, res.x, N, res.table, w1, b1, w2, b2, w3, b3, y,
                                                           stream=sp), steps, warmup, device)
        flops = 2 * N * (LF * 64 + 64 * 64 + 64 * 4)
        out["mlp_forward"] = entry(ms, N * (12 + 8 * LF * s + 16), "mlp_forward_kernel",
                                   tensor_tflops=round(flops / (ms * 1e-3) / 1e12, 2))
        launches += steps

    # D-dimensional inputs (D = 2, 4; 2^D corners, the 7-prime hash): forward and backward on
    # N uniform points of the same grid.
    nd = {}
    for D in (2, 4):
        gen = np.random.default_rng(1000 + D)
        xd = torch.from_numpy(gen.random((N, D), dtype=np.float32)).to(device)
        hd = hg.hashgrid_create_nd(D, w.L, w.F, w.log2T, w.N_min, w.N_max,
                                   hg.HASHGRID_F16 if w.dtype == "f16" else hg.HASHGRID_F32)
        outd = torch.empty((N, LF), dtype=torch.float32, device=device)
        dtd = torch.zeros((w.L, w.T, w.F), dtype=torch.float32, device=device)
        fms = time_launches(lambda: hg.hashgrid_forward(hd, xd, N, res.table, outd, sp), steps, warmup, device)
        bms = time_launches(lambda: hg.hashgrid_backward(hd, xd, res.g, N, dtd, sp), steps, warmup, device,
                            before=dtd.zero_)
        hg.hashgrid_destroy(hd)
        nd[f"D{D}"] = {"fwd_ms": round(fms, 5), "bwd_ms": round(bms, 5),
                       "fwd_points_per_s": round(N / (fms * 1e-3), 1), "bwd_points_per_s": round(N / (bms * 1e-3), 1),
                       "gathers_per_point": (1 << D) * w.L}
        launches += 2 * steps
        del xd, outd, dtd
    out["nd"] = {"workload": f"{w.name} grid, {N} uniform points in [0,1)^D", **nd}

    # Backward into an fp16 gradient table (packed f16x2 reductions), zeroed before each call.
    dh = torch.zeros((w.L, w.T, w.F), dtype=torch.float16, device=device)
    ms = time_launches(lambda: hg.hashgrid_backward_half(res.handle, res.x, res.g, N, dh, sp), steps, warmup,
                       device, before=dh.zero_)
    out["backward_half"] = {"ms": round(ms, 5), "points_per_s": round(N / (ms * 1e-3), 1),
                            "roofline": roofline(w, "bwd", N, ms, "backward_kernel_half", l2peaks, grad_dtype="f16")}
    launches += steps
    return out, launches


L2_RESIDENT_BYTES = 96 << 20   # a kernel's table (or gradient) working set that stays in L2


def stream_bytes_per_point(w: workloads.Workload, kind: str) -> int:
    """HBM-compulsory bytes of one point: x in, and the output (fwd) or the upstream
    gradient (bwd) rows."""
    return 12 + 4 * w.L * w.F


def roofline(w: workloads.Workload, kind: str, points: int, kernel_ms: float, kernel: str,
             l2peaks: dict | None, grad_dtype: str = "f32", level_major: bool | None = None) -> dict:
    """Roofline of one kernel launch over ``points`` points (kind "fwd" or "bwd").

    HBM (the primary fraction, bound "hbm"): the algorithmic bytes of the launch (x, the
    table gathers or fp32 reductions counted once each, the output or upstream-gradient
    rows) at the measured HBM copy bandwidth.
    L2 (the gather roofline of a table that fits in L2 is L2's, not HBM's): the 8 * L table
    gathers (fwd) or corner reductions (bwd) per point at the rate this device serves the
    hash's access pattern from an L2-resident buffer of the working set's size: x-neighbour
    pairs of F*s-byte entries (fwd) or F-wide fp32 / fp16 contributions (bwd), measured in
    the same run by the probe kernels. The working set is the table (fwd) or gradient
    (bwd), or one level of it under the level-major schedule (AUTO for tables above 96 MB;
    ``level_major`` says which schedule ran when it was chosen explicitly).
    bound_time is the larger of the L2 time and the time of the bytes that must cross HBM
    (all of them for a table larger than L2, else the x / output / upstream-gradient
    rows); frac_bound_time = bound_time / kernel time. Batches more coherent than the
    probe's independent random pairs (samples along rays share cache lines and voxels)
    can exceed 1 on the L2 basis. For the backward, the L2 reduction requests of the
    launch (counted once by ncu for the committed kernel sources) are also set against the
    rate at which the L2 serves independent random reductions of the same width, one
    request each: the request-rate ceiling that merging x-neighbours or run-walk faces
    does not move."""
    hbm, src = measured_peaks()
    s = 2 if w.dtype == "f16" else 4
    alg = algorithmic_bytes_per_point(w, kind) * points
    if kind == "bwd" and grad_dtype == "f16":
        alg = (12 + 4 * w.L * w.F + 8 * w.L * w.F * 2) * points
    hbm_gbs = alg / (kernel_ms * 1e-3) / 1e9
    elem = s if kind == "fwd" else (2 if grad_dtype == "f16" else 4)
    table_bytes = w.L * w.T * w.F * elem
    if level_major is None:
        level_major = w.L * w.T * w.F * s > L2_RESIDENT_BYTES
    working_set = table_bytes // w.L if level_major else table_bytes
    in_l2 = working_set <= L2_RESIDENT_BYTES
    out = {"bound": "hbm", "kernel": kernel, "kernel_ms": round(kernel_ms, 5), "unit": "GB/s",
           "achieved": round(hbm_gbs, 1), "peak": hbm, "frac": round(hbm_gbs / hbm, 4),
           "traffic": ncu_traffic(kernel, w.name), "algorithmic_bytes_per_launch": alg,
           "peak_source": f"hbm_gbs of {src} peaks"}
    # the table (or gradient) crosses HBM only when it does not fit in L2 as a whole
    t_stream = (alg if table_bytes > L2_RESIDENT_BYTES else stream_bytes_per_point(w, kind) * points) / (hbm * 1e9)
    t_l2 = 0.0
    if l2peaks is not None and in_l2:
        ops = 8 * w.L * points
        width = w.F * elem
        bkey = "32MiB" if working_set <= (32 << 20) else "64MiB"
        pk = "gather" if kind == "fwd" else ("red_f16" if grad_dtype == "f16" else "red")
        rates = l2peaks["buffers"][bkey][pk][str(width)]
        t_l2 = ops / (rates["xpair"] * 1e9)
        out["l2"] = {"access": (f"{width}-byte table gathers" if kind == "fwd" else
                                f"{width}-byte {grad_dtype} corner reductions") + ", 8 per point and level",
                     "ops_per_launch": ops, "achieved_g_ops_per_s": round(ops / (kernel_ms * 1e-3) / 1e9, 1),
                     "peak_g_ops_per_s": rates["xpair"], "frac": round(t_l2 / (kernel_ms * 1e-3), 4),
                     "frac_vs_random_units": round(ops / (rates["random"] * 1e9) / (kernel_ms * 1e-3), 4),
                     "peak_source": f"hashgrid_probe, x-neighbour pairs on a {bkey} L2-resident buffer, this run"}
    bound_s = max(t_stream, t_l2)
    out["bound_time_ms"] = round(bound_s * 1e3, 5)
    out["bound_by"] = "l2" if t_l2 >= t_stream else "hbm"
    out["frac_bound_time"] = round(bound_s / (kernel_ms * 1e-3), 4)
    ent = ncu_entry(kernel, w.name)
    if ent is not None and ent.get("l2_red_requests_per_launch"):
        reds = float(ent["l2_red_requests_per_launch"])
        g_per_s = reds / (kernel_ms * 1e-3) / 1e9
        out["l2_red_requests"] = {"per_launch": int(reds), "g_per_s": round(g_per_s, 1)}
        if "l2" in out:
            # one L2 request per operation when the units are independent and random
            peak = rates["random"]
            out["l2_red_requests"].update({"peak_g_per_s": peak, "frac": round(g_per_s / peak, 4),
                                           "peak_source": f"hashgrid_probe, random {width}-byte units on a "
                                                          f"{bkey} L2-resident buffer (one request each), this run"})
    return out


def cpu_baseline(w: workloads.Workload, sample: int, budget_s: float = 10.0) -> dict:
    """The oracle, as it stands, on the host cores: repeated fwd(+bwd) passes over a sample
    of the workload until about ``budget_s`` seconds of CPU time have elapsed."""
    import oracle
    threads = oracle.default_threads()
    inp = workloads.make_inputs(w, seed=rank_seed(0), n_points=sample, grads=w.backward)
    og = oracle.Grid(w.L, w.F, w.log2T, w.N_min, w.N_max, oracle.F16 if w.dtype == "f16" else oracle.F32)
    dtable = np.zeros((w.L, w.T, w.F)) if w.backward else None
    passes = 0
    t0 = time.perf_counter()
    while True:
        og.forward(inp.x, inp.table, nthreads=threads)
        if w.backward:
            og.backward(inp.x, inp.g, nthreads=threads, dtable=dtable)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= budget_s:
            break
    n = inp.x.shape[0]
    return {"value": round(n * passes / dt, 1), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{passes} passes over the first {n} points of {w.name} (seed {rank_seed(0)}), "
                      f"{'fwd+bwd' if w.backward else 'fwd'}; fwd parallel over points, "
                      f"bwd over the {w.L} levels; {dt:.1f} s"}


def cpu_next_rows(w: workloads.Workload, sample: int, budget_s: float = 3.0) -> dict:
    """The oracle's counterparts of the next-row kernels, as they stand, on the host cores:
    dL/dx and the encoding + MLP over a sample of the workload's points, and sparse Adam
    over the whole table with the oracle's own gradient of that sample (computed untimed),
    each repeated for about ``budget_s`` seconds."""
    import oracle
    threads = oracle.default_threads()
    inp = workloads.make_inputs(w, seed=rank_seed(0), n_points=sample, grads=True)
    og = oracle.Grid(w.L, w.F, w.log2T, w.N_min, w.N_max, oracle.F16 if w.dtype == "f16" else oracle.F32)
    n = inp.x.shape[0]

    def rate(fn):
        reps, t0 = 0, time.perf_counter()
        while True:
            fn()
            reps += 1
            dt = time.perf_counter() - t0
            if dt >= budget_s:
                return reps, dt

    out = {"cores": threads, "kind": "oracle"}
    reps, dt = rate(lambda: og.backward_x(inp.x, inp.table, inp.g, nthreads=threads))
    out["backward_input"] = {"value": round(n * reps / dt, 1), "unit": UNIT,
                             "sample": f"{reps} passes over the first {n} points, parallel over points"}
    LF = w.L * w.F
    if LF in (16, 32, 48, 64):
        rng = np.random.default_rng(7)
        bf = lambda *shape: (rng.standard_normal(shape).astype(np.float32) * 0.1).view(np.uint32) >> 16  # noqa: E731
        w1, w2, w3 = bf(64, LF).astype(np.uint16), bf(64, 64).astype(np.uint16), bf(4, 64).astype(np.uint16)
        b = np.zeros(64, dtype=np.float32)
        reps, dt = rate(lambda: og.mlp_forward(inp.x, inp.table, w1, b, w2, b, w3, b[:4], nthreads=threads))
        out["mlp_forward"] = {"value": round(n * reps / dt, 1), "unit": UNIT,
                              "sample": f"{reps} passes over the first {n} points, parallel over points"}
    if w.dtype == "f32":
        # one level's slice of the table (the oracle's step is elementwise, so its rate per
        # element does not depend on which slice)
        grad = og.backward(inp.x, inp.g, levels=(w.L - 1, w.L), nthreads=threads)[w.L - 1].astype(np.float32)
        table = inp.table[w.L - 1]
        m, v = np.zeros_like(grad), np.zeros_like(grad)
        step = [0]

        def adam():
            step[0] += 1
            oracle.adam_step(table, m, v, grad, step[0], 1e-2)
        reps, dt = rate(adam)
        out["adam_step"] = {"value": round(grad.size * reps / dt, 1), "unit": "elements/s",
                            "sample": f"{reps} steps over the finest level's {grad.size} elements with the "
                                      f"gradient of {n} points (single thread, fp64)"}
    return out


# ---------------------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------------------

def run_reference(args) -> None:
    """CPU oracle arm: rank 0 only (other ranks exit without work). Each step encodes a
    bounded sample of the workload, forward and backward, on the host cores."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    w = workloads.WORKLOADS[args.workload]
    threads = oracle.default_threads()
    inp = workloads.make_inputs(w, seed=rank_seed(0), n_points=REFERENCE_SAMPLE_POINTS, grads=True)
    og = oracle.Grid(w.L, w.F, w.log2T, w.N_min, w.N_max, oracle.F16 if w.dtype == "f16" else oracle.F32)

    dtable = np.zeros((w.L, w.T, w.F))

    def step():   # as in the GPU arm's step: forward, zero the gradient table, backward
        og.forward(inp.x, inp.table, nthreads=threads)
        dtable.fill(0.0)
        og.backward(inp.x, inp.g, nthreads=threads, dtable=dtable)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    n = inp.x.shape[0]
    value = n * args.steps / dt
    sample = (f"{n} points of {w.name} per step (seed {rank_seed(0)}), fwd + zeroing of the fp64 gradient "
              f"table + bwd; fwd parallel over points, bwd over the {w.L} levels")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": w.name, "description": w.describe(),
                                        "sample_points_per_step": n},
        "cpu_baseline": {"value": round(value, 1), "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 1), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


LEGS = ("grid_L16F2T19", "half_L16F2T19", "large_L16F4T22")   # timed besides the step's workload


def time_level_major(res: Resident, args, device, l2peaks) -> tuple[dict, int]:
    """The forward of a table that fits in L2, run level-major (one pass per group of
    levels whose reachable entries fit in 32 MB: the group's slices are the live working
    set) instead of point by point (the whole table live): if the point-major forward were
    losing to L2 capacity, this would be the faster one. Returns the JSON object and the
    number of timed launches."""
    import torch
    hg = res.hg
    sp = torch.cuda.current_stream(device).cuda_stream
    steps = min(args.steps, 20)
    hg.hashgrid_set_option(res.handle, hg.HASHGRID_OPT_SCHEDULE, SCHEDULES["level"])
    try:
        ms = time_launches(lambda: res.forward(sp), steps, min(args.warmup, 3), device)
    finally:
        hg.hashgrid_set_option(res.handle, hg.HASHGRID_OPT_SCHEDULE, SCHEDULES[args.schedule])
    return {"schedule": "level", "fwd_ms": round(ms, 5),
            "rooflines": {"fwd": roofline(res.w, "fwd", res.N, ms, "forward_kernel_levels", l2peaks, level_major=True)},
            "note": "the same forward with the level-major schedule: a group of levels (at most 32 MB of entries "
                    "reachable) live instead of the whole table; if the point-major forward lost to L2 capacity, "
                    "this one would be faster"}, steps


def time_workload(w: workloads.Workload, args, device, rank: int, world: int, l2peaks, min_timed_s: float,
                  sampler=None) -> tuple[dict, Resident, int]:
    """Times one workload's step (forward, or forward + zero + backward) and returns its
    JSON object (rate, phases, a roofline per kernel), the resident inputs and the number
    of timed launches."""
    res = Resident(w, rank_seed(rank), device, backward=w.backward, gather=args.forward_gather,
                   backward_mode=args.backward_mode, schedule=args.schedule,
                   points=args.points if w.name == args.workload else None)
    t = time_steps(res, args.steps, args.warmup, device, sampler, min_timed_s=min_timed_s)
    n = t["timed_steps"]
    seconds = t["max_total_ms"] * 1e-3
    obj = {"workload": w.name, "description": w.describe(), "value": round(whole_job_rate(res.N * n, world, seconds), 1),
           "unit": UNIT, "ms_per_step": round(t["max_total_ms"] / n, 5), "points_per_rank": res.N,
           "timed_steps": n, "loop_repeats": t["repeats"],
           "phase_ms": {"fwd": round(t["fwd_ms"], 5), "zero": round(t["zero_ms"], 5), "bwd": round(t["bwd_ms"], 5)},
           "rooflines": {"fwd": roofline(w, "fwd", res.N, t["fwd_ms"], "forward_kernel", l2peaks)}}
    if w.backward:
        obj["rooflines"]["bwd"] = roofline(w, "bwd", res.N, t["bwd_ms"], "backward_kernel", l2peaks)
        hbm, src = measured_peaks()
        step_bytes = algorithmic_bytes_per_point(w, "fwdbwd") * res.N
        step_gbs = step_bytes / (t["step_ms"] * 1e-3) / 1e9
        bound_ms = obj["rooflines"]["fwd"]["bound_time_ms"] + obj["rooflines"]["bwd"]["bound_time_ms"]
        obj["roofline_step"] = {"achieved": round(step_gbs, 1), "peak": hbm, "unit": "GB/s",
                                "frac": round(step_gbs / hbm, 4),
                                "bound_time_ms": round(bound_ms, 5),
                                "frac_bound_time": round(bound_ms / t["step_ms"], 4),
                                "note": f"whole step incl. gradient zeroing; frac against the {src} HBM peak, "
                                        "frac_bound_time = (fwd + bwd bound times) / step time"}
    return obj, res, t["launches"]


def run_b200(args) -> None:
    import torch
    rank, world, local = dist_env()
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=timedelta(seconds=180), device_id=torch.device("cuda", local))
    device = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(device)
    w = workloads.WORKLOADS[args.workload]
    l2peaks = None if args.skip_peaks else measure_l2_peaks(device)

    sampler = ClockSampler(device.index)
    main, res, launches = time_workload(w, args, device, rank, world, l2peaks, args.min_timed_s, sampler)
    rl = main["rooflines"]
    kind = "bwd" if w.backward and main["phase_ms"]["bwd"] >= main["phase_ms"]["fwd"] else "fwd"
    line = {
        "metric": METRIC, "value": main["value"], "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": main["ms_per_step"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16" if w.dtype == "f16" else "f32",
        "data": "synthetic (seeded NeRF-like ray samples; random table)",
        "config": {"workload": w.name, "description": w.describe(), "points_per_rank": res.N,
                   "global_points": res.N * world, "parallelism": f"dp{world}: points sharded, no collective",
                   "step": "forward + zero dL_dtable + backward" if w.backward else "forward",
                   "modes": {"forward_gather": args.forward_gather, "backward": args.backward_mode,
                             "schedule": args.schedule},
                   "l2": "flushed before every timed step, outside the events: a 256 MiB write, then a 256 MiB read "
                         "that evicts the write's dirty lines",
                   "timed_region": f"the {args.steps}-step loop run {main['loop_repeats']} times back to back "
                                   f"({main['timed_steps']} steps, all timed) so that it lasts >= {args.min_timed_s} s",
                   "phase_ms": main["phase_ms"]},
        "roofline": rl[kind],
        "roofline_step": main.get("roofline_step"),
        "rooflines": rl,
        "clocks": sampler.summary(),
    }
    if l2peaks is not None:
        line["peaks"] = {"l2": l2peaks}

    if not args.skip_legs:
        legs = {}
        for name in LEGS:
            if name == w.name:
                continue
            lw = workloads.WORKLOADS[name]
            obj, lres, n = time_workload(lw, args, device, rank, world, l2peaks, 0.0)
            if name == FWD_WORKLOAD and args.schedule == "auto":
                obj["level_major"], m = time_level_major(lres, args, device, l2peaks)
                n += m
            lres.close()
            del lres
            torch.cuda.empty_cache()
            legs[name] = obj
            launches += n
        line["legs"] = legs
        if "grid_L16F2T19" in legs:          # the metric's forward-only figure
            line["fwd"] = legs["grid_L16F2T19"]

    if not args.skip_next_rows and w.backward:
        line["next_rows"], n = time_next_rows(res, min(args.steps, 20), min(args.warmup, 3), device, l2peaks)
        launches += n
        if rank == 0 and world == 1 and not args.skip_cpu_baseline:
            line["next_rows"]["cpu_oracle"] = cpu_next_rows(w, min(NEXT_ROWS_CPU_SAMPLE, res.N))

    if not args.skip_e2e:
        e = time_e2e(res, args.steps, min(args.warmup, 3), device, args.min_timed_s)
        launches += e["steps"] * (2 if w.backward else 1)
        line["e2e"] = {"value": round(res.N * world * e["steps"] / (e["ms"] * 1e-3), 1), "unit": UNIT,
                       "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"], "timed_steps": e["steps"],
                       "note": "pinned host x (and upstream grads) -> device, fwd + zero + bwd through "
                               "the C ABI, encoding -> pinned host; the gradient table stays on the device"}
    line["gpu_launches"] = launches
    if rank == 0 and world == 1 and not args.skip_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, min(CPU_SAMPLE_POINTS, res.N))
    res.close()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        barrier(device)
        dist.destroy_process_group()


def free_port() -> int:
    import socket
    sk = socket.socket()
    sk.bind(("127.0.0.1", 0))
    port = sk.getsockname()[1]
    sk.close()
    return port


def spawn_ranks(gpus: int, argv: list[str]) -> int:
    """``--gpus N`` (N > 1) without a launcher: start N ranks of this script on this node
    with torch.distributed.run (one process per GPU, rendezvous on 127.0.0.1) and return
    its exit status. The ranks find WORLD_SIZE set and do not spawn again."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(free_port()), os.path.abspath(__file__), *argv]
    return subprocess.run(cmd).returncode


def run_stub(args) -> None:
    """The rank plumbing without a GPU (gloo, CPU): each rank sleeps a fixed time per step
    in place of the GPU step, and rank 0 prints a line marked ``"impl": "stub"`` with the
    world size, the max-over-ranks time and the whole-job rate. Tests use it to check that
    ``--gpus N`` starts N ranks and that they agree on one line."""
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1:
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    units = 1 << 20
    barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        time.sleep(0.002 * (1 + rank))
    dt = max_over_ranks(time.perf_counter() - t0)
    barrier()
    if rank == 0:
        print(json.dumps({"impl": "stub", "metric": METRIC, "value": round(whole_job_rate(units * args.steps, world, dt), 1),
                          "unit": UNIT, "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                          "ms_per_step": round(dt / args.steps * 1e3, 3), "scaling": "weak"}), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main(argv=None) -> None:
    argv = list(sys.argv[1:] if argv is None else argv)
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--workload", choices=sorted(workloads.WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--forward-gather", choices=sorted(GATHER_MODES), default="auto")
    ap.add_argument("--backward-mode", choices=sorted(BACKWARD_MODES), default="auto")
    ap.add_argument("--schedule", choices=sorted(SCHEDULES), default="auto")
    ap.add_argument("--skip-cpu-baseline", action="store_true")
    ap.add_argument("--skip-e2e", action="store_true")
    ap.add_argument("--skip-legs", "--skip-fwd-leg", dest="skip_legs", action="store_true",
                    help="skip timing the other workloads (forward-only grid, fp16 table, 1 GiB grid)")
    ap.add_argument("--skip-peaks", action="store_true", help="skip measuring the L2 gather / reduction peaks")
    ap.add_argument("--skip-next-rows", action="store_true",
                    help="skip timing dL/dx, Adam, the fused MLP and the fp16-gradient backward")
    ap.add_argument("--points", type=int, default=None,
                    help="encode this many points of the workload instead of all (profiling captures on a "
                         "reduced batch; the reported line then names a smaller workload than the config's)")
    ap.add_argument("--min-timed-s", type=float, default=1.0,
                    help="repeat the K-step loop inside the timed region until it lasts at least this long")
    ap.add_argument("--stub-step", action="store_true",
                    help="test the rank plumbing on CPU (gloo, a sleep in place of the GPU step; prints impl=stub)")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "b200":
        print("note: fewer than 3 warm-up steps; the timing rules want at least 3", file=sys.stderr)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(spawn_ranks(args.gpus, argv))
    _, world, _ = dist_env()
    if world != args.gpus:
        print(f"note: --gpus {args.gpus} but WORLD_SIZE={world}; using WORLD_SIZE", file=sys.stderr)
    if args.stub_step:
        run_stub(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_b200(args)


if __name__ == "__main__":
    main()
