"""Benchmark: Swish forward + save-input-only backward, bf16 storage / fp32
math, on the transformer-scale activation [8, 2048, 4096] (67,108,864
elements), the configuration the headline metric is quoted on.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = mea_act_fwd (read x, write y) + mea_act_bwd (read x and dy,
write dx) over one batch: 10 algorithmic bytes per element, 671,088,640 bytes
per step.  Each rank processes its own full-size batch (weak scaling, no
data-path collective); under torchrun the elapsed time is the max over ranks.
Inputs are resident in HBM when the timed region starts; the per-step working
set (x, y, dy, dx = 536 MB) is larger than the 126 MB L2, so no flush is
needed between steps.

Rank 0 prints one JSON line.  Besides the device-timed value it reports the
end-to-end number through the same public API with host buffers (pinned
host -> device copies of x and dy, device -> host copies of y and dx inside
the timed region), the dominant kernel's roofline fraction from CUDA events
on its own stream, the SM clocks sampled during the timed region, and the
CPU oracle's throughput on a bounded sample (the baseline, not the target).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import memory_efficient_activation_b200 as mea  # noqa: E402
from memory_efficient_activation_b200 import accounting, synthetic  # noqa: E402

METRIC = "Swish fwd+bwd GB/s and % of B200 HBM roofline at 67M bf16 elements"
WORKLOAD = "swish_bf16_8x2048x4096"
SHAPE = (8, 2048, 4096)
DTYPE = "bf16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0        # the B200's nominal HBM3e bandwidth (8 TB/s per GPU, DGX figure)
DOMINANT_KERNEL = "act_kernel<Swish, Bf16, MODE 1> (mea_act_bwd)"


# ----------------------------------------------------------------- helpers

def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws <= 1:
        return 0, 1, 0
    import datetime
    import torch.distributed as dist
    rank = int(os.environ["RANK"])
    local = int(os.environ.get("LOCAL_RANK", rank))
    torch.cuda.set_device(local)
    dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                            device_id=torch.device("cuda", local))
    if dist.get_world_size() != ws:
        raise SystemExit(f"process group formed {dist.get_world_size()} ranks, WORLD_SIZE says {ws}")
    return rank, ws, local


def _relaunch(nproc: int, argv, script: str | None = None) -> int:
    """Runs `script` (this file by default) as nproc ranks of one node under
    torch.distributed.run (rendezvous on 127.0.0.1, a free port), passing
    argv to every rank; returns the launcher's exit code.  NCCL's init log is
    switched on (to stderr, so that stdout carries only rank 0's JSON line),
    which shows how many ranks the communicator formed."""
    import socket
    import subprocess
    with socket.socket() as so:
        so.bind(("127.0.0.1", 0))
        port = so.getsockname()[1]
    env = dict(os.environ)
    env.setdefault("NCCL_DEBUG", "INFO")
    env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    env.setdefault("NCCL_DEBUG_FILE", "/dev/stderr")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={nproc}",
           "--master-addr", "127.0.0.1", f"--master-port={port}", script or os.path.abspath(__file__), *argv]
    return subprocess.run(cmd, env=env).returncode


def _barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(v: float, ws: int) -> float:
    if ws <= 1:
        return v
    from memory_efficient_activation_b200 import dist as mdist
    return mdist.max_over_ranks(v, device="cuda")


def _bf16_peak():
    """(TFLOP/s, kind): the measured burst bf16 matmul rate, else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured burst"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# Sources that define the streaming kernels; a committed ncu traffic figure
# is used only while these files are unchanged since it was taken.
KERNEL_SOURCES = ("mea_act.cu", "mea_math.cuh", "mea_device.cuh", "mea_internal.h")


def source_hash(files=KERNEL_SOURCES) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "memory_efficient_activation_b200", "csrc")
    for name in sorted(files):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel_key: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            d = json.load(f)
        e = d[kernel_key]
        if e.get("source_hash") != source_hash(e.get("sources", KERNEL_SOURCES)):
            return None
        return int(e["dram_bytes_per_launch"])
    except Exception:
        return None


class _ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = [(0x1, "gpu_idle"), (0x2, "applications_clocks_setting"), (0x4, "sw_power_cap"),
               (0x8, "hw_slowdown"), (0x10, "sync_boost"), (0x20, "sw_thermal_slowdown"),
               (0x40, "hw_thermal_slowdown"), (0x80, "hw_power_brake_slowdown"),
               (0x100, "display_clock_setting")]

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = device_index
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].isdigit():
                    idx = int(ids[device_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self._nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            pass

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                try:
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                except AttributeError:
                    r = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self._h)
                for bit, name in self.REASONS:
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ------------------------------------------------------------ our arm

def _inputs(rank: int):
    w = synthetic.swish_bf16_transformer(seed=1 + 1000 * rank, shape=SHAPE)
    return w


def run_ours(args, rank, ws, local):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = _inputs(rank)
    n = w.n
    x = w.x.to(dev)
    dy = w.dy.to(dev)
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    stream = torch.cuda.current_stream(dev)

    def step():
        mea.act_fwd("swish", x, 1.0, out=y)
        mea.act_bwd("swish", x, dy, 1.0, out=dx)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # Timed region: K steps, no events between the kernels (an event between
    # two kernels costs the overlap of the second kernel's launch with the
    # first one's drain).
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    _barrier(ws)
    torch.cuda.synchronize()
    with _ClockSampler(local) as clk:
        start.record(stream)
        for _ in range(args.steps):
            step()
        end.record(stream)
        torch.cuda.synchronize()
        _barrier(ws)
        elapsed_ms = _max_over_ranks(start.elapsed_time(end), ws)
        # Kernel-timing pass (the roofline), right after the timed region:
        # each kernel timed over back-to-back launches of itself (5 rounds of
        # `per` forwards, then `per` backwards, CUDA events at the round
        # boundaries on the launching stream), so that every launch overlaps
        # its neighbours' ramp and drain as it does in the timed steps; 3
        # unbracketed steps first refill the launch queue.  Median over rounds.
        rounds = 5
        per = max(10, max(50, args.steps) // rounds)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(rounds)]
        for _ in range(3):
            step()
        for e3 in ev:
            e3[0].record(stream)
            for _ in range(per):
                mea.act_fwd("swish", x, 1.0, out=y)
            e3[1].record(stream)
            for _ in range(per):
                mea.act_bwd("swish", x, dy, 1.0, out=dx)
            e3[2].record(stream)
        torch.cuda.synchronize()
    _barrier(ws)
    fwd_ms = _max_over_ranks(statistics.median(e[0].elapsed_time(e[1]) / per for e in ev), ws)
    bwd_ms = _max_over_ranks(statistics.median(e[1].elapsed_time(e[2]) / per for e in ev), ws)

    step_bytes = accounting.step_bytes(n, DTYPE)
    ms_per_step = elapsed_ms / args.steps
    value = ws * step_bytes * args.steps / (elapsed_ms * 1e-3) / 1e9

    # End to end through the public API with host buffers.
    e2e = run_e2e(args, rank, ws, local, w)

    peak, peak_kind = _peaks()
    bwd_bytes = accounting.bwd_bytes(n, DTYPE)
    achieved = bwd_bytes / (bwd_ms * 1e-3) / 1e9
    roofline = {
        "kernel": DOMINANT_KERNEL,
        "bound": "hbm",
        "achieved": round(achieved, 1),
        "peak": peak,
        "peak_kind": f"{peak_kind} (copy bandwidth, burst)",
        "unit": "GB/s",
        "frac": round(achieved / peak, 4),
        "traffic": _traffic("swish_bf16_bwd"),
        "algorithmic_bytes_per_launch": bwd_bytes,
        "fwd_ms": round(fwd_ms, 5),
        "bwd_ms": round(bwd_ms, 5),
        "fwd_plus_bwd_ms": round(fwd_ms + bwd_ms, 5),
        "ms_per_step": round(ms_per_step, 5),
        "launches_timed": 2 * rounds * per,
        "timing": f"after the timed region: {rounds} rounds of {per} back-to-back launches of each kernel, CUDA "
                  "events at the round boundaries on the launching stream; median per launch",
        "fwd_frac": round(accounting.fwd_bytes(n, DTYPE) / (fwd_ms * 1e-3) / 1e9 / peak, 4),
        "step_frac": round(step_bytes / (ms_per_step * 1e-3) / 1e9 / peak, 4),
        "step_frac_of_nominal_8tbs": round(step_bytes / (ms_per_step * 1e-3) / 1e9 / NOMINAL_HBM_GBS, 4),
    }

    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": DTYPE,
        "data": "synthetic",
        "config": {
            "workload": WORKLOAD,
            "shape": list(SHAPE),
            "elements_per_gpu": n,
            "alpha": 1.0,
            "bytes_per_step_per_gpu": step_bytes,
            "x_dist": "N(0,1)", "dy_dist": "N(0,1)",
            "l2": "inputs larger than L2 (536 MB working set per step vs 126 MB L2); no flush",
            "parallelism": f"replicas x{ws} (independent shards, no data-path collective)",
            "process_group": ({"backend": "nccl", "ranks": ws} if ws > 1 else None),
            "pct_of_hbm_roofline": round(100 * value / ws / peak, 2),
            "saved_bytes_per_layer": accounting.saved_bytes_per_layer(n, DTYPE),
            "saved_bytes_per_layer_naive": accounting.saved_bytes_per_layer(n, DTYPE, naive=True),
        },
        "roofline": roofline,
        "e2e": e2e,
        "gpu_launches": 2 * args.steps,
        "clocks": clk.summary(),
    }
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_seconds)
    return out


def run_e2e(args, rank, ws, local, w):
    """The metric through the public API on host data: act_fwd_bwd_host copies
    the step's inputs from pinned host memory and its results back, pipelined
    over eight pieces on three streams; the timed region holds all of it."""
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    hx = w.x.contiguous().pin_memory()
    hdy = w.dy.contiguous().pin_memory()
    hy = torch.empty_like(hx).pin_memory()
    hdx = torch.empty_like(hx).pin_memory()
    steps = max(1, min(args.steps, args.e2e_steps))

    def step():
        mea.act_fwd_bwd_host("swish", hx, hdy, 1.0, hy=hy, hdx=hdx, chunks=8, device=dev)

    for _ in range(max(1, min(args.warmup, 3))):
        step()
    torch.cuda.synchronize()
    _barrier(ws)
    s = torch.cuda.Event(enable_timing=True)
    e = torch.cuda.Event(enable_timing=True)
    s.record(stream)
    for _ in range(steps):
        step()
    e.record(stream)
    torch.cuda.synchronize()
    _barrier(ws)
    ms = _max_over_ranks(s.elapsed_time(e), ws)
    nbytes = accounting.step_bytes(w.n, DTYPE)
    link = _copy_bound(hx, hdy, hy, hdx, dev)
    return {
        "value": round(ws * nbytes * steps / (ms * 1e-3) / 1e9, 2),
        "unit": "GB/s",
        "h2d_bytes_per_step": 2 * accounting.tensor_bytes(w.n, DTYPE),
        "d2h_bytes_per_step": 2 * accounting.tensor_bytes(w.n, DTYPE),
        "steps": steps,
        "ms_per_step": round(ms / steps, 4),
        "pipelining": "8 pieces over 3 streams (copy in, kernels, copy out)",
        "host_link": link,
        "frac_of_copy_bound": round(link["both_ms"] / (ms / steps), 4),
    }


def _copy_bound(hx, hdy, hy, hdx, dev, reps: int = 3):
    """The host link's floor for one end-to-end step: the time to copy the
    step's inputs to the device and its results back, pinned host memory,
    the two directions at once on two streams (no kernels); also each
    direction alone.  Min over reps."""
    dx_, ddy = torch.empty_like(hx, device=dev), torch.empty_like(hdy, device=dev)
    dy_, ddx = torch.empty_like(hy, device=dev), torch.empty_like(hdx, device=dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)
    res = {"h2d_ms": [], "d2h_ms": [], "both_ms": []}
    for _ in range(reps):
        for key in ("h2d_ms", "d2h_ms", "both_ms"):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            torch.cuda.synchronize()
            a.record(cur)
            s_in.wait_stream(cur)
            s_out.wait_stream(cur)
            if key != "d2h_ms":
                with torch.cuda.stream(s_in):
                    dx_.copy_(hx, non_blocking=True)
                    ddy.copy_(hdy, non_blocking=True)
            if key != "h2d_ms":
                with torch.cuda.stream(s_out):
                    hy.copy_(dy_, non_blocking=True)
                    hdx.copy_(ddx, non_blocking=True)
            cur.wait_stream(s_in)
            cur.wait_stream(s_out)
            b.record(cur)
            torch.cuda.synchronize()
            res[key].append(a.elapsed_time(b))
    nb = hx.numel() * hx.element_size() + hdy.numel() * hdy.element_size()
    out = {k: round(min(v), 4) for k, v in res.items()}
    out["h2d_GB/s"] = round(nb / (out["h2d_ms"] * 1e-3) / 1e9, 1)
    out["d2h_GB/s"] = round(nb / (out["d2h_ms"] * 1e-3) / 1e9, 1)
    out["note"] = "pinned copies of the step's 2 input and 2 output tensors, no kernels; both_ms is the floor"
    return out


# ------------------------------------------------- oracle (CPU) baseline

def _oracle_step(oracle, xd, gd):
    y = oracle.act_fwd("swish", xd, 1.0)
    dx = oracle.act_bwd("swish", xd, gd, 1.0)
    oracle.round_bf16(y)
    oracle.round_bf16(dx)


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline(w, budget_s: float = 12.0):
    """The double-precision oracle (as it stands, OpenMP over the host cores)
    on the same workload: forward + backward + rounding of y and dx to bf16,
    repeated over the full 67M-element batch until about budget_s seconds of
    work; GB/s under the same 10 bytes/element accounting.  Then the same on
    one core, over the first 1/16 of the batch for about budget_s / 3 s."""
    import oracle
    xd = w.x.reshape(-1).double().numpy()
    gd = w.dy.reshape(-1).double().numpy()
    reps, t_total = 0, 0.0
    while t_total < budget_s and reps < 50:
        t0 = time.perf_counter()
        _oracle_step(oracle, xd, gd)
        t_total += time.perf_counter() - t0
        reps += 1
    n = w.n
    cores = oracle.num_threads()
    m = n // 16
    xs, gs = xd[:m], gd[:m]
    oracle.set_num_threads(1)
    try:
        reps1, t1 = 0, 0.0
        while t1 < budget_s / 3 and reps1 < 50:
            t0 = time.perf_counter()
            _oracle_step(oracle, xs, gs)
            t1 += time.perf_counter() - t0
            reps1 += 1
    finally:
        oracle.set_num_threads(cores)
    return {
        "value": round(reps * accounting.step_bytes(n, DTYPE) / t_total / 1e9, 3),
        "unit": "GB/s",
        "cores": cores,
        "kind": "oracle",
        "sample": f"{reps} x full {n}-element batch (fwd + bwd + bf16 rounding), {t_total:.1f} s",
        "cpu_model": _cpu_model(),
        "single_core": {"value": round(reps1 * accounting.step_bytes(m, DTYPE) / t1 / 1e9, 4), "unit": "GB/s",
                        "cores": 1, "sample": f"{reps1} x first {m} elements, {t1:.1f} s"},
    }


def run_reference(args, rank, ws):
    """The reference arm: the CPU oracle on bounded samples of the same
    workload, one sample per step, sized so warm-up plus steps take about
    args.ref_seconds."""
    if rank != 0:
        return None
    import numpy as np
    import oracle
    w = _inputs(0)
    xs = w.x.reshape(-1)
    gs = w.dy.reshape(-1)
    probe = 1 << 20
    xd, gd = xs[:probe].double().numpy(), gs[:probe].double().numpy()
    t0 = time.perf_counter()
    _oracle_step(oracle, xd, gd)
    per_elem = (time.perf_counter() - t0) / probe
    total_steps = args.steps + args.warmup
    sample = int(args.ref_seconds / max(total_steps, 1) / max(per_elem, 1e-12))
    sample = max(1 << 12, min(sample, w.n))
    xd, gd = xs[:sample].double().numpy(), gs[:sample].double().numpy()
    for _ in range(args.warmup):
        _oracle_step(oracle, xd, gd)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_step(oracle, xd, gd)
    dt = time.perf_counter() - t0
    nbytes = accounting.step_bytes(sample, DTYPE)
    value = round(args.steps * nbytes / dt / 1e9, 4)
    cb = {"value": value, "unit": "GB/s", "cores": oracle.num_threads(), "kind": "oracle",
          "sample": f"first {sample} of {w.n} elements per step (fwd + bwd + bf16 rounding)"}
    del np
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(1e3 * dt / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "shape": list(SHAPE), "sample_elements": sample},
        "cpu_baseline": cb,
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# --------------------------------------- secondary workloads (not the headline)

L2_BYTES = 126 * 1024 * 1024


def _time_ops(ops, steps, warmup, stream, reps: int = 24):
    """ops: list of (name, launchers, algorithmic_bytes) where launchers is a
    list of callables, one per buffer set.  Each op is captured once in a
    CUDA graph of `reps` back-to-back launches that rotate over its buffer
    sets (so consecutive launches touch different memory and, with more than
    the L2's worth of sets, find none of it in L2), the graphs are replayed
    in op order `steps` times with CUDA events around every replay on the
    launching stream, and the mean device time of one launch is returned per
    op, together with the total elapsed ms of one launch of every op."""
    graphs = []
    for _, launchers, _ in ops:
        for _ in range(max(1, warmup)):
            for fn in launchers:
                fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for r in range(reps):
                launchers[r % len(launchers)]()
        graphs.append(g)
    torch.cuda.synchronize()
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(ops) + 1)] for _ in range(steps)]
    for k in range(steps):
        ev[k][0].record(stream)
        for j, g in enumerate(graphs):
            g.replay()
            ev[k][j + 1].record(stream)
    torch.cuda.synchronize()
    per = {name: statistics.mean(ev[k][j].elapsed_time(ev[k][j + 1]) for k in range(steps)) / reps
           for j, (name, _, _) in enumerate(ops)}
    total = sum(per.values())
    return per, total


def _sets_for(nbytes: int) -> int:
    """Buffer sets to rotate over: at least 2, and together over 3x the L2."""
    return max(2, -(-3 * L2_BYTES // max(nbytes, 1)))


def _ops_for(wl, dev, args):
    """The launchers of one workload's kernels, each over buffer sets that
    together exceed the L2 (the 1M fp32 case excepted): a list of (name,
    launchers, algorithmic bytes or FLOPs).  Sets args._flop_ops for the
    workloads whose ops are contractions."""
    ops = []

    def clones(ts, k):
        return [[t.to(dev).clone() for t in ts] for _ in range(k)]

    if wl == "family_bf16":
        w = synthetic.family_bf16("swish")
        n = w.n
        k = _sets_for(accounting.bwd_bytes(n, "bf16"))
        sets = clones([w.x, w.dy, w.x, w.x], k)      # x, dy, y, dx
        for act in synthetic.ACTIVATIONS:
            p = 0.01 if act == "leaky_relu" else 1.0
            ops.append((f"{act}_fwd", [lambda a=act, p=p, b=b: mea.act_fwd(a, b[0], p, out=b[2]) for b in sets],
                        accounting.fwd_bytes(n, "bf16")))
            ops.append((f"{act}_bwd", [lambda a=act, p=p, b=b: mea.act_bwd(a, b[0], b[1], p, out=b[3]) for b in sets],
                        accounting.bwd_bytes(n, "bf16")))
    elif wl == "effnet_f32_dalpha":
        for i in range(len(synthetic.EFFNET_B0_SHAPES)):
            w = synthetic.effnet_swish_f32(i)
            k = _sets_for(accounting.bwd_bytes(w.n, "f32"))
            a = torch.tensor([w.param], dtype=torch.float32, device=dev)
            sets = clones([w.x, w.dy, w.x, w.x], k)
            ds = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(k)]
            wss = [torch.zeros(mea.act_bwd_workspace_bytes("swish", w.n, True), dtype=torch.uint8, device=dev)
                   for _ in range(k)]
            tag = "x".join(map(str, w.x.shape))
            ops.append((f"{tag}_fwd", [lambda b=b, a=a: mea.act_fwd("swish", b[0], 0.0, param_dev=a, out=b[2])
                                       for b in sets], accounting.fwd_bytes(w.n, "f32")))
            ops.append((f"{tag}_bwd_dalpha",
                        [lambda b=b, d=d, ws=ws, a=a: mea.act_bwd("swish", b[0], b[1], 0.0, param_dev=a, dparam=d,
                                                                  out=b[3], workspace=ws)
                         for b, d, ws in zip(sets, ds, wss)], accounting.bwd_bytes(w.n, "f32")))
    elif wl == "effnet_f32_dalpha_grouped":
        # the same six maps, each direction one grouped launch over all six
        wls = [synthetic.effnet_swish_f32(i) for i in range(len(synthetic.EFFNET_B0_SHAPES))]
        fwd_b = sum(accounting.fwd_bytes(w.n, "f32") for w in wls)
        bwd_b = sum(accounting.bwd_bytes(w.n, "f32") for w in wls)
        k = _sets_for(bwd_b)
        alphas = [w.param for w in wls]
        sets = [[clones([w.x, w.dy, w.x, w.x], 1)[0] for w in wls] for _ in range(k)]
        ds = [[torch.empty(1, dtype=torch.float32, device=dev) for _ in wls] for _ in range(k)]
        need = mea.act_bwd_grouped_workspace_bytes("swish", [w.n for w in wls], True)
        wss = [torch.zeros(need, dtype=torch.uint8, device=dev) for _ in range(k)]
        ops.append(("grouped_fwd", [lambda b=b: mea.act_fwd_grouped("swish", [t[0] for t in b], alphas,
                                                                    outs=[t[2] for t in b]) for b in sets], fwd_b))
        ops.append(("grouped_bwd_dalpha",
                    [lambda b=b, d=d, w_=w_: mea.act_bwd_grouped("swish", [t[0] for t in b], [t[1] for t in b], alphas,
                                                                 dparams=d, outs=[t[3] for t in b], workspace=w_)
                     for b, d, w_ in zip(sets, ds, wss)], bwd_b))
    elif wl == "affine_nhwc_bf16":
        w = synthetic.affine_swish_nhwc()
        C = w.extra["gamma"].numel()
        k = _sets_for(accounting.affine_bwd_bytes(w.n, "bf16", C))
        g, b_ = w.extra["gamma"].to(dev), w.extra["beta"].to(dev)
        sets = clones([w.x, w.dy, w.x, w.x], k)
        gr = [(torch.empty(C, device=dev), torch.empty(C, device=dev)) for _ in range(k)]
        need = mea.affine_swish_bwd_workspace_bytes(torch.bfloat16, "nhwc", w.extra["nchw_shape"])
        wss = [torch.zeros(need, dtype=torch.uint8, device=dev) for _ in range(k)]
        ops.append(("affine_fwd", [lambda s=s: mea.affine_swish_fwd(s[0], g, b_, "nhwc", out=s[2]) for s in sets],
                    accounting.affine_fwd_bytes(w.n, "bf16", C)))
        ops.append(("affine_bwd", [lambda s=s, q=q, ws=ws: mea.affine_swish_bwd(s[0], s[1], g, b_, "nhwc", out=s[3],
                                                                               dgamma=q[0], dbeta=q[1], workspace=ws)
                                   for s, q, ws in zip(sets, gr, wss)],
                    accounting.affine_bwd_bytes(w.n, "bf16", C)))
    elif wl == "affine_family_nhwc_bf16":
        w = synthetic.affine_act_nhwc("swish")
        C = w.extra["gamma"].numel()
        k = _sets_for(accounting.affine_bwd_bytes(w.n, "bf16", C))
        g, b_ = w.extra["gamma"].to(dev), w.extra["beta"].to(dev)
        sets = clones([w.x, w.dy, w.x, w.x], k)
        gr = [(torch.empty(C, device=dev), torch.empty(C, device=dev)) for _ in range(k)]
        need = mea.affine_act_bwd_workspace_bytes(torch.bfloat16, "nhwc", w.extra["nchw_shape"])
        wss = [torch.zeros(need, dtype=torch.uint8, device=dev) for _ in range(k)]
        for act in synthetic.ACTIVATIONS:
            p = 0.01 if act == "leaky_relu" else 1.0
            ops.append((f"{act}_fwd", [lambda a=act, p=p, s=s: mea.affine_act_fwd(a, s[0], g, b_, p, "nhwc", out=s[2])
                                       for s in sets], accounting.affine_fwd_bytes(w.n, "bf16", C)))
            ops.append((f"{act}_bwd", [lambda a=act, p=p, s=s, q=q, ws=ws:
                                       mea.affine_act_bwd(a, s[0], s[1], g, b_, p, "nhwc", out=s[3], dgamma=q[0],
                                                          dbeta=q[1], workspace=ws)
                                       for s, q, ws in zip(sets, gr, wss)],
                        accounting.affine_bwd_bytes(w.n, "bf16", C)))
    elif wl == "swish_channel_f32":
        for i in range(len(synthetic.EFFNET_B0_SHAPES)):
            w = synthetic.swish_channel_nchw(seed=8 + i, shape=synthetic.EFFNET_B0_SHAPES[i])
            C = w.extra["alpha"].numel()
            k = _sets_for(accounting.channel_swish_bwd_bytes(w.n, "f32", C))
            a = w.extra["alpha"].to(dev)
            sets = clones([w.x, w.dy, w.x, w.x], k)
            ds = [torch.empty(C, dtype=torch.float32, device=dev) for _ in range(k)]
            need = mea.swish_channel_bwd_workspace_bytes(torch.float32, "nchw", w.extra["nchw_shape"])
            wss = [torch.zeros(need, dtype=torch.uint8, device=dev) for _ in range(k)]
            tag = "x".join(map(str, w.x.shape))
            ops.append((f"{tag}_fwd", [lambda b=b, a=a: mea.swish_channel_fwd(b[0], a, "nchw", out=b[2])
                                       for b in sets], accounting.channel_swish_fwd_bytes(w.n, "f32", C)))
            ops.append((f"{tag}_bwd_dalpha",
                        [lambda b=b, d=d, ws=ws, a=a: mea.swish_channel_bwd(b[0], b[1], a, "nchw", out=b[3], dalpha=d,
                                                                            workspace=ws)
                         for b, d, ws in zip(sets, ds, wss)], accounting.channel_swish_bwd_bytes(w.n, "f32", C)))
    elif wl == "swish_channel_f32_grouped":
        # Swish with alpha per channel on the six maps: the three small stages
        # (28 x 28, 14 x 14, 7 x 7) as one grouped launch per direction, then
        # all six in one grouped call (the three large maps are launched alone
        # inside it)
        all_ws = [synthetic.swish_channel_nchw(seed=8 + i, shape=synthetic.EFFNET_B0_SHAPES[i])
                  for i in range(len(synthetic.EFFNET_B0_SHAPES))]
        for tag, wls in (("small3", all_ws[3:]), ("all6", all_ws)):
            fwd_b = sum(accounting.channel_swish_fwd_bytes(w.n, "f32", w.extra["alpha"].numel()) for w in wls)
            bwd_b = sum(accounting.channel_swish_bwd_bytes(w.n, "f32", w.extra["alpha"].numel()) for w in wls)
            k = _sets_for(bwd_b)
            alphas = [w.extra["alpha"].to(dev) for w in wls]
            sets = [[clones([w.x, w.dy, w.x, w.x], 1)[0] for w in wls] for _ in range(k)]
            ds = [[torch.empty(a.numel(), dtype=torch.float32, device=dev) for a in alphas] for _ in range(k)]
            need = mea.swish_channel_bwd_grouped_workspace_bytes(torch.float32, [tuple(w.x.shape) for w in wls])
            wss = [torch.zeros(need, dtype=torch.uint8, device=dev) for _ in range(k)]
            ops.append((f"{tag}_grouped_fwd",
                        [lambda b=b, a=alphas: mea.swish_channel_fwd_grouped([t[0] for t in b], a,
                                                                             outs=[t[2] for t in b])
                         for b in sets], fwd_b))
            ops.append((f"{tag}_grouped_bwd_dalpha",
                        [lambda b=b, d=d, w_=w_, a=alphas: mea.swish_channel_bwd_grouped(
                            [t[0] for t in b], [t[1] for t in b], a, outs=[t[3] for t in b], dalphas=d, workspace=w_)
                         for b, d, w_ in zip(sets, ds, wss)], bwd_b))
            del sets
    elif wl == "matmul_act_bf16":
        # the d x d matmul of problem B07 ([8 x 2048, 4096] x [4096, 4096]) with
        # the activation in its epilogue, and the same work unfused (cuBLAS
        # through torch.matmul, then the streaming activation kernels)
        M, N, K = 16384, 4096, 4096
        flops = 2 * M * N * K
        tf_peak = _bf16_peak()
        x = synthetic.normal(M * K, 1.0, 41, synthetic.STREAM_X, "bf16").view(M, K)
        w = synthetic.normal(N * K, K ** -0.5, 41, synthetic.STREAM_PARAM, "bf16").view(N, K)
        nbytes = (2 * M * K + N * K + 2 * M * N) * 2
        k = _sets_for(nbytes)
        sets = [[x.to(dev), w.to(dev), x.to(dev),
                 torch.empty(M, N, dtype=torch.bfloat16, device=dev),
                 torch.empty(M, N, dtype=torch.bfloat16, device=dev)] for _ in range(k)]   # x, w, g, z, out
        for act in ("relu", "swish", "gelu_erf"):
            ops.append((f"fused_fwd_{act}", [lambda a=act, b=b: mea.matmul_act_fwd(a, b[0], b[1], 1.0, z=b[3], y=b[4])
                                             for b in sets], flops))
            ops.append((f"fused_bwd_{act}", [lambda a=act, b=b: mea.matmul_act_bwd(a, b[2], b[1], b[3], 1.0, out=b[4])
                                             for b in sets], flops))
        ops.append(("cublas_matmul", [lambda b=b: torch.matmul(b[0], b[1].t(), out=b[3]) for b in sets], flops))
        ops.append(("act_fwd_gelu_erf_on_z", [lambda b=b: mea.act_fwd("gelu_erf", b[3], out=b[4]) for b in sets],
                    accounting.fwd_bytes(M * N, "bf16")))
        ops.append(("act_bwd_gelu_erf_on_z", [lambda b=b: mea.act_bwd("gelu_erf", b[3], b[4], out=b[4]) for b in sets],
                    accounting.bwd_bytes(M * N, "bf16")))
        args._flop_ops = {name for name, _, _ in ops if not name.startswith("act_")}
        args._tf_peak = tf_peak
    elif wl == "swish_f32_1m":
        w = synthetic.swish_f32_1m()
        sets = clones([w.x, w.dy, w.x, w.x], 1)       # L2-resident on purpose
        ops.append(("fwd", [lambda b=sets[0]: mea.act_fwd("swish", b[0], out=b[2])], accounting.fwd_bytes(w.n, "f32")))
        ops.append(("bwd", [lambda b=sets[0]: mea.act_bwd("swish", b[0], b[1], out=b[3])],
                    accounting.bwd_bytes(w.n, "f32")))
    else:
        raise SystemExit(f"unknown workload {wl}")
    return ops


def run_secondary(args):
    """Per-kernel GB/s and roofline fractions for the other configurations
    (activation family, EfficientNet-like fp32 maps with d alpha, fused
    affine + Swish NHWC, fused affine + every activation NHWC, Swish with a
    per-channel alpha on EfficientNet-like maps, the L2-resident 1M fp32
    case, the fused matmul).  Diagnostics: the headline line is the default
    run, which carries the configurations' figures in its "configs" block."""
    wl = args.workload
    if wl == "mlp_bf16":
        return run_mlp(args)
    if wl == "densenet_bn_bf16":
        return run_densenet_bn(args)
    if wl == "memory_study":
        return run_memory_study(args)
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = _peaks()
    ops = _ops_for(wl, dev, args)
    # capture on a side stream (graphs cannot be captured on the legacy stream)
    cap = torch.cuda.Stream(dev)
    cap.wait_stream(stream)
    with torch.cuda.stream(cap), _ClockSampler(0) as clk:
        per, total = _time_ops(ops, args.steps, args.warmup, cap)
    stream.wait_stream(cap)
    tot_bytes = sum(b for name, _, b in ops if name not in getattr(args, "_flop_ops", ()))
    out = {
        "workload": wl,
        "value": round(tot_bytes / (total * 1e-3) / 1e9, 2) if not getattr(args, "_flop_ops", None) else None,
        "unit": "GB/s",
        "steps": args.steps,
        "warmup": args.warmup,
        "peak": peak,
        "peak_kind": peak_kind,
        "timing": "mean device time per launch from CUDA-graph replays of 24 back-to-back launches rotating over "
                  "buffer sets that together exceed 3x L2",
        "ops": {name: ({"ms": round(per[name], 5), "TFLOP/s": round(b / (per[name] * 1e-3) / 1e12, 1),
                        "frac": round(b / (per[name] * 1e-3) / 1e12 / args._tf_peak[0], 4),
                        "peak": args._tf_peak, "flops": b, "sets": len(fns)}
                       if name in getattr(args, "_flop_ops", ()) else
                       {"ms": round(per[name], 5), "GB/s": round(b / (per[name] * 1e-3) / 1e9, 1),
                        "frac": round(b / (per[name] * 1e-3) / 1e9 / peak, 4), "bytes": b, "sets": len(fns)})
                for name, fns, b in ops},
        "clocks": clk.summary(),
    }
    if wl == "swish_f32_1m":
        out["note"] = "21 MB of traffic per step fits in the 126 MB L2: an L2-resident figure, not HBM bandwidth"
    return out


# The other configurations of the metric's workload list, timed in the
# default run after the headline (N = 1): key -> _ops_for workload.
CONFIG_WORKLOADS = (
    ("c1_swish_f32_1m", "swish_f32_1m"),
    ("c3_family_bf16_8x2048x4096", "family_bf16"),
    ("c4_effnet_b0_f32_dalpha", "effnet_f32_dalpha"),
    ("c4_effnet_b0_f32_dalpha_grouped", "effnet_f32_dalpha_grouped"),
    ("c5_affine_swish_nhwc_bf16_128x56x56x144", "affine_nhwc_bf16"),
)


def run_configs(args):
    """Per-kernel device time, GB/s and fraction of the HBM peak for
    configurations 1 and 3-5, each kernel captured in a CUDA graph of 24
    launches that rotate over buffer sets together larger than 3x the L2
    (configuration 1, 21 MB of traffic, fits in L2 and is reported as such),
    replayed args.config_steps times with events around every replay; the
    configuration's figure is its total algorithmic bytes over the total
    device time of one launch of each of its kernels."""
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = _peaks()
    res = {}
    t0 = time.perf_counter()
    for key, wl in CONFIG_WORKLOADS:
        ops = _ops_for(wl, dev, args)
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            per, total = _time_ops(ops, args.config_steps, 3, cap)
        stream.wait_stream(cap)
        tot_bytes = sum(b for _, _, b in ops)
        res[key] = {
            "GB/s": round(tot_bytes / (total * 1e-3) / 1e9, 1),
            "frac": round(tot_bytes / (total * 1e-3) / 1e9 / peak, 4),
            "bytes": tot_bytes,
            "us": round(total * 1e3, 2),
            "kernels": {name: {"us": round(per[name] * 1e3, 2), "bytes": b,
                               "GB/s": round(b / (per[name] * 1e-3) / 1e9, 1),
                               "frac": round(b / (per[name] * 1e-3) / 1e9 / peak, 4)} for name, _, b in ops},
        }
        if wl == "swish_f32_1m":
            res[key]["note"] = "21 MB of traffic per step stays in the 126 MB L2: an L2 figure, not HBM"
        del ops
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
    return {"peak": peak, "peak_kind": peak_kind, "steps": args.config_steps,
            "timing": "CUDA-graph replays of 24 launches per kernel rotating over buffer sets > 3x L2; mean per launch",
            "wall_s": round(time.perf_counter() - t0, 1), **res}


def run_mlp(args, M: int = 16384, d: int = 4096, h: int = 4096, act: str = "gelu_tanh"):
    """One MLP block (Linear d -> h, activation, Linear h -> d; bf16, no bias)
    at the d x d size of problem B07, forward + backward: the memory-efficient
    block (fused matmul epilogues, keeps x and z) against the same block in
    plain PyTorch autograd (F.linear, F.gelu, F.linear).  Reports time per
    step, matmul throughput (6 matmuls of 2 M d h FLOPs), the activation
    memory held between forward and backward, and the peak during a step."""
    import torch.nn.functional as F
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    m = mea.MemoryEfficientMLP(d, h, act).to(dev)
    x = synthetic.normal(M * d, 1.0, 43, synthetic.STREAM_X, "bf16").view(M, d).to(dev).requires_grad_(True)
    dout = synthetic.normal(M * d, 1.0, 43, synthetic.STREAM_DY, "bf16").view(M, d).to(dev)

    def ours():
        return m(x)

    def plain():
        return F.linear(F.gelu(F.linear(x, m.w1), approximate="tanh"), m.w2)

    flops = 6 * 2 * M * d * h
    res = {}
    with _ClockSampler(0) as clk:
        for name, fwd in (("memory_efficient", ours), ("plain_pytorch", plain)):
            for _ in range(max(3, args.warmup)):
                fwd().backward(dout)
            x.grad = None
            m.w1.grad = None
            m.w2.grad = None
            torch.cuda.synchronize()
            base = torch.cuda.memory_allocated()
            out = fwd()
            torch.cuda.synchronize()
            held = torch.cuda.memory_allocated() - base - out.numel() * out.element_size()
            torch.cuda.reset_peak_memory_stats()
            out.backward(dout)
            torch.cuda.synchronize()
            peak = torch.cuda.max_memory_allocated() - base
            del out
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            for _ in range(args.steps):
                fwd().backward(dout)
            e.record()
            torch.cuda.synchronize()
            ms = s.elapsed_time(e) / args.steps
            res[name] = {"ms_per_step": round(ms, 4), "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1),
                         "activation_bytes_held": int(held), "backward_peak_bytes": int(peak)}
    return {"workload": "mlp_bf16", "shape": {"tokens": M, "d_model": d, "d_hidden": h}, "act": act,
            "steps": args.steps, "warmup": args.warmup, "bf16_peak": _bf16_peak(), "results": res,
            "speedup": round(res["plain_pytorch"]["ms_per_step"] / res["memory_efficient"]["ms_per_step"], 4),
            "clocks": clk.summary()}


def run_densenet_bn(args, N: int = 64, ks=(64, 32, 32, 32, 32, 32), spatial=(56, 56)):
    """Concatenation + batch normalization + ReLU of one DenseNet-121 layer
    (first dense block, sixth layer: 224 channels at 56 x 56, batch 64, bf16)
    over one training step (forward, the backward's re-population of the
    output, backward): the kernels that never form the concatenation and keep
    only the statistics, against torch.cat + F.batch_norm + relu under
    autograd.  Reports time per step, the bytes each path moves per step
    (algorithmic: the tensors each kernel must read and write), and the
    activation memory held between forward and backward."""
    import torch.nn.functional as F
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    HW = spatial[0] * spatial[1]
    C = sum(ks)
    pieces = [synthetic.normal(N * k * HW, 1.5, 70 + i, synthetic.STREAM_X, "bf16").view((N, k) + spatial).to(dev)
              for i, k in enumerate(ks)]
    g = torch.from_numpy(synthetic.uniform_f64(C, 0.5, 1.5, 71, synthetic.STREAM_GAMMA)).float().to(dev)
    b = torch.from_numpy(synthetic.normal_f64(C, 0.3, 71, synthetic.STREAM_BETA)).float().to(dev)
    dy = synthetic.normal(N * C * HW, 1.0, 72, synthetic.STREAM_DY, "bf16").view((N, C) + spatial).to(dev)
    y = torch.empty((N, C) + spatial, dtype=torch.bfloat16, device=dev)
    dps = [torch.empty_like(p) for p in pieces]
    rmean = torch.zeros(C, device=dev)
    rvar = torch.ones(C, device=dev)
    ws = torch.zeros(int(mea._capi.lib().mea_concat_bn_relu_workspace_bytes(N, C)), dtype=torch.uint8, device=dev)
    T = N * C * HW * 2
    ours_bytes = 10 * T       # fwd: stats read x, apply read x + write y; re-populate: read x + write y;
    #                           bwd: reduce read x + dy, dx read x + dy + write dx

    def ours():
        _, mean, invstd = mea.concat_bn_relu_fwd(pieces, g, b, 1e-5, 0.1, rmean, rvar, out=y, workspace=ws)
        mea.concat_bn_relu_apply(pieces, g, b, mean, invstd, out=y)
        mea.concat_bn_relu_bwd(pieces, dy, g, b, mean, invstd, dpieces=dps, workspace=ws)

    pr = [p.detach().clone().requires_grad_(True) for p in pieces]
    gr = g.clone().requires_grad_(True)
    br = b.clone().requires_grad_(True)

    def plain_fwd():
        return torch.relu(F.batch_norm(torch.cat(pr, 1), rmean, rvar, gr, br, training=True, momentum=0.1, eps=1e-5))

    def plain():
        plain_fwd().backward(dy)

    res = {}
    with _ClockSampler(0) as clk:
        for name, fn in (("memory_efficient", ours), ("plain_pytorch", plain)):
            for _ in range(max(3, args.warmup)):
                fn()
            torch.cuda.synchronize()
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            for _ in range(args.steps):
                fn()
            e.record()
            torch.cuda.synchronize()
            res[name] = {"ms_per_step": round(s.elapsed_time(e) / args.steps, 4)}
    # activation memory held between forward and backward
    base = torch.cuda.memory_allocated()
    out = plain_fwd()
    torch.cuda.synchronize()
    res["plain_pytorch"]["activation_bytes_held"] = int(torch.cuda.memory_allocated() - base
                                                        - out.numel() * out.element_size())
    del out
    res["memory_efficient"]["activation_bytes_held"] = 2 * C * 4      # mean and invstd
    res["memory_efficient"]["GB/s"] = round(ours_bytes / (res["memory_efficient"]["ms_per_step"] * 1e-3) / 1e9, 1)
    res["memory_efficient"]["frac"] = round(res["memory_efficient"]["GB/s"] / _peaks()[0], 4)
    return {"workload": "densenet_bn_bf16", "shape": {"N": N, "pieces": list(ks), "H": spatial[0], "W": spatial[1]},
            "steps": args.steps, "warmup": args.warmup, "algorithmic_bytes_per_step": ours_bytes,
            "peak_hbm_gbs": _peaks(), "results": res,
            "speedup": round(res["plain_pytorch"]["ms_per_step"] / res["memory_efficient"]["ms_per_step"], 4),
            "clocks": clk.summary()}


class _PlainSwish(torch.nn.Module):
    """The plain autograd Swish of the pages' first listing: x * sigmoid(alpha x)
    built from PyTorch ops, which keeps every intermediate for the backward.
    Comparator only."""

    def __init__(self, alpha=1.0):
        super().__init__()
        self.alpha = alpha

    def forward(self, x):
        return x * torch.sigmoid(self.alpha * x)


def run_memory_study(args, layers: int = 32, shape=SHAPE):
    """Peak memory and step time of an L-layer stack at [8, 2048, 4096] bf16 with
    the plain autograd Swish versus the save-input-only Swish, in two stacks:
    activations only, and Linear(d, d) + Swish blocks (a transformer-style MLP
    path).  Re-measures, on synthetic data, the memory the Swish page's
    "How much GPU memory is saved?" section reports for EfficientNets."""
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    d = shape[-1]
    x0 = synthetic.normal(accounting.elements(shape), 1.0, 7, synthetic.STREAM_X, "bf16").view(shape).to(dev)
    res = {}
    for stack in ("activations", "linear_swish"):
        for impl in ("plain", "save_input_only"):
            torch.manual_seed(0)
            mods = []
            for _ in range(layers):
                if stack == "linear_swish":
                    mods.append(torch.nn.Linear(d, d, bias=False, device=dev, dtype=torch.bfloat16))
                mods.append(_PlainSwish() if impl == "plain" else mea.MemoryEfficientSwish())
            net = torch.nn.Sequential(*mods)
            for p in net.parameters():
                p.requires_grad_(True)

            def step():
                x = x0.detach().requires_grad_(True)
                y = net(x)
                y.backward(torch.ones_like(y))
                return x.grad

            step()
            torch.cuda.synchronize()
            for p in net.parameters():
                p.grad = None
            torch.cuda.empty_cache()
            torch.cuda.reset_peak_memory_stats(dev)
            base = torch.cuda.memory_allocated(dev)
            s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record()
            reps = max(1, min(args.steps, 5))
            for _ in range(reps):
                step()
                for p in net.parameters():
                    p.grad = None
            s1.record()
            torch.cuda.synchronize()
            res[f"{stack}/{impl}"] = {
                "peak_GB": round((torch.cuda.max_memory_allocated(dev) - base) / 1e9, 3),
                "ms_per_fwd_bwd": round(s0.elapsed_time(s1) / reps, 3),
            }
            del net, mods
            torch.cuda.empty_cache()
    for stack in ("activations", "linear_swish"):
        a, b = res[f"{stack}/plain"], res[f"{stack}/save_input_only"]
        res[f"{stack}/saved_GB"] = round(a["peak_GB"] - b["peak_GB"], 3)
        res[f"{stack}/saved_fraction"] = round(1 - b["peak_GB"] / a["peak_GB"], 4)
    return {"workload": "memory_study", "layers": layers, "shape": list(shape), "dtype": "bf16",
            "per_layer_tensor_MB": round(accounting.tensor_bytes(accounting.elements(shape), "bf16") / 1e6, 1),
            "note": "peak = max_memory_allocated above the memory held before the step (inputs, weights)",
            "results": res}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--ref-seconds", type=float, default=90.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="leave out the configs block (configurations 1, 3-5 timed after the headline)")
    ap.add_argument("--config-steps", type=int, default=10)
    ap.add_argument("--workload", default="swish_bf16",
                    choices=["swish_bf16", "family_bf16", "effnet_f32_dalpha", "effnet_f32_dalpha_grouped",
                             "affine_nhwc_bf16",
                             "affine_family_nhwc_bf16", "swish_channel_f32", "swish_channel_f32_grouped",
                             "matmul_act_bf16", "mlp_bf16",
                             "densenet_bn_bf16", "swish_f32_1m", "memory_study"],
                    help="swish_bf16 (default) is the headline; the others print per-kernel diagnostics")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.gpus < 1:
        ap.error("--gpus must be at least 1")
    env_ws = os.environ.get("WORLD_SIZE")
    if env_ws is None:
        if args.gpus > 1:
            # one process per GPU: start args.gpus ranks of this script
            return _relaunch(args.gpus, sys.argv[1:] if argv is None else list(argv))
    elif int(env_ws) != args.gpus:
        ap.error(f"--gpus {args.gpus} but WORLD_SIZE={env_ws}: launch one rank per GPU")

    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        ws = int(os.environ.get("WORLD_SIZE", "1"))
        out = run_reference(args, rank, ws)
        if out is not None:
            print(json.dumps(out), flush=True)
        return 0

    if args.workload != "swish_bf16":
        print(json.dumps(run_secondary(args)), flush=True)
        return 0

    rank, ws, local = _dist()
    out = run_ours(args, rank, ws, local)
    if rank == 0 and ws == 1 and not args.no_configs:
        out["configs"] = run_configs(args)
    if rank == 0:
        print(json.dumps(out), flush=True)
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
