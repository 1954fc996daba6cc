"""Benchmark of the fused DyT forward + backward on B200.

One step = one forward and one backward (dx, dgamma, dbeta, dalpha) of the
workload over one batch of synthetic input. Prints ONE JSON line on rank 0.
The headline workload is the largest configuration (32768 x 8192 bf16); the
line's `shapes` block times every other workload and layout variant the same
way, each with its roofline entry, replay percentiles, clocks and the oracle's
CPU time next to it.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one process per GPU): each rank runs the whole workload
on its own batch of rows (weak scaling); the parameter gradients are summed
across ranks inside the finalize, which reads every rank's binary64 partials
through peer pointers after a one-element NCCL all-reduce (or, where the
workspaces cannot be mapped, by one NCCL all-reduce of the 2N+1 rounded
gradients): the exchange that row sharding of the column sums requires.

Device timing: CUDA events around K steps on the launching stream (one GPU: a
CUDA graph of them; several: launched directly, so that no NCCL collective is
captured into a graph), barrier + synchronize on both sides, max over ranks.
The steps cycle
through enough buffer sets that the data touched between two uses of a set
is more than twice the L2 size, so no step reads another's data from L2.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "DyT fwd+bwd achieved HBM GB/s (and % of B200 peak), rows/s per shape"
FALLBACK_HBM_GBS = 6650.0
PROFILES = os.path.join(ROOT, "profiles")
KERNEL_SOURCES = [os.path.join(ROOT, "elementwise_reduction_b200", "csrc", f)
                  for f in ("dyt_kernels.cuh", "dyt_math.cuh", "dyt_async.cuh", "dyt_finalize.cuh", "dyt_select.cuh",
                            "dyt_select_impl.cuh", "dyt_api.cu")]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=50)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default=None)
    p.add_argument("--e2e-steps", type=int, default=None)
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-clocks", action="store_true")
    p.add_argument("--no-shapes", action="store_true", help="skip the per-shape table of the other workloads")
    p.add_argument("--no-latency", action="store_true", help="skip the per-call cold-L2 latency percentiles")
    p.add_argument("--no-sustained", action="store_true", help="skip the 1 s back-to-back replay of the step")
    p.add_argument("--record-traffic", metavar="NCU_CSV", default=None,
                   help="store DRAM bytes per launch from an ncu --csv capture of dram__bytes_read.sum and "
                        "dram__bytes_write.sum into profiles/dram_traffic.json for --workload, then exit")
    p.add_argument("--ncu-command", default="", help="the ncu command line that wrote --record-traffic's CSV")
    return p.parse_args()


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash(read=None) -> str:
    """Hash of the kernel sources with comments and blank space removed, so that
    only a change of the code itself invalidates the recorded traffic.
    read(path) -> text (default: the file on disk)."""
    import re
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        if read is None:
            with open(p, encoding="utf-8") as f:
                text = f.read()
        else:
            text = read(p)
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"(?m)//.*$", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def committed_traffic(workload: str, kernel: str):
    """dram read+write bytes per launch from a committed ncu summary, or None when the
    kernel sources changed since it was taken."""
    path = os.path.join(PROFILES, "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        return None
    e = d.get(workload, {}).get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


def record_traffic(csv_path: str, workload: str, command: str) -> None:
    """DRAM bytes per launch of each DyT kernel from an ncu CSV, stored with the hash of
    the kernel sources they were taken on."""
    import csv
    import re

    per = {}
    with open(csv_path) as f:
        rows = [r for r in csv.reader(f) if len(r) > 5]
    hdr = rows[0]
    ki, mi, vi, ui = (hdr.index(k) for k in ("Kernel Name", "Metric Name", "Metric Value", "Metric Unit"))
    idi = hdr.index("ID")
    scale = {"byte": 1, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9}
    launches = {}
    for r in rows[1:]:
        m = re.search(r"(dyt_\w+)", r[ki])
        if not m or not r[mi].startswith("dram__bytes_"):
            continue
        kernel = "dyt_bwd_kernel" if "bwd" in m.group(1) else "dyt_fwd_kernel" if "fwd" in m.group(1) \
            else "dyt_finalize_kernel"
        per.setdefault(kernel, 0.0)
        per[kernel] += float(r[vi].replace(",", "")) * scale.get(r[ui], 1)
        launches.setdefault(kernel, set()).add(r[idi])
    path = os.path.join(PROFILES, "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except Exception:
        d = {}
    entry = {k: {"bytes_per_launch": v / len(launches[k]), "launches": len(launches[k]),
                 "source_hash": kernel_source_hash(), "command": command} for k, v in per.items()}
    if "dyt_bwd_kernel" in entry and "dyt_finalize_kernel" in entry:
        # one backward call: its stage-1 launches (one per phase of a strided
        # call whose pitches are not whole vectors, else one) and its finalize
        calls = len(launches["dyt_finalize_kernel"])
        entry["dyt_backward"] = {
            "bytes_per_launch": (per["dyt_bwd_kernel"] + per["dyt_finalize_kernel"]) / calls,
            "stage1_launches_per_call": len(launches["dyt_bwd_kernel"]) / calls,
            "source_hash": kernel_source_hash(), "command": command}
    d[workload] = entry
    with open(path, "w") as f:
        json.dump(d, f, indent=1, sort_keys=True)
    print(json.dumps(entry, indent=1))


# ---- clocks sampled during the timed region ---------------------------------------------------

class ClockSampler:
    """SM clock, power and throttle reasons of one GPU, sampled every few ms while
    the `with` block runs: through NVML (the GPU matched by UUID), else by
    polling nvidia-smi every 100 ms."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown"}
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int, enabled: bool = True, period_s: float = 0.005):
        self.index, self.enabled, self.period = index, enabled, period_s
        self.rows = []  # (host time, sm MHz, max sm MHz, watts, [reasons])
        self.proc, self.thread, self._stop = None, None, threading.Event()

    def _nvml_handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        uuid = str(torch.cuda.get_device_properties(self.index).uuid)
        if not uuid.startswith("GPU-"):
            uuid = "GPU-" + uuid
        return pynvml, pynvml.nvmlDeviceGetHandleByUUID(uuid)

    def __enter__(self):
        if not self.enabled:
            return self
        try:
            nv, h = self._nvml_handle()
            mx = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            reasons_of = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons

            def poll():
                while not self._stop.is_set():
                    try:
                        sm = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                        w = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                        bits = reasons_of(h)
                        self.rows.append((time.time(), float(sm), float(mx), w,
                                          [n for b, n in self.REASONS.items() if bits & b]))
                    except Exception:
                        pass
                    time.sleep(self.period)

            self.thread = threading.Thread(target=poll, daemon=True)
            self.thread.start()
        except Exception:
            try:
                self.proc = subprocess.Popen(
                    ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                     "--format=csv,noheader,nounits", "-lms", "100"],
                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
                self.thread = threading.Thread(target=self._read_smi, daemon=True)
                self.thread.start()
            except Exception:
                self.proc = None
        return self

    def _read_smi(self):
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.proc.stdout:
            r = [c.strip() for c in line.split(",")]
            try:
                self.rows.append((time.time(), float(r[1]), float(r[2]), float(r[3]),
                                  [n for n, v in zip(names, r[5:9]) if v.lower() == "active"]))
            except (ValueError, IndexError):
                pass

    def __exit__(self, *exc):
        self._stop.set()
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0: float | None = None, t1: float | None = None):
        rows = [r for r in self.rows if (t0 is None or r[0] >= t0) and (t1 is None or r[0] <= t1)]
        if not rows:
            return None
        sm = [r[1] for r in rows]
        return {"sm_mhz": statistics.median(sm), "sm_min_mhz": min(sm), "sm_max_mhz": max(r[2] for r in rows),
                "power_w": statistics.median(r[3] for r in rows),
                "reasons": sorted({n for r in rows for n in r[4]}), "samples": len(rows)}


# ---- CPU baseline: the oracle on a bounded sample ---------------------------------------------

def oracle_sample_rows(w, seconds_budget: float) -> int:
    # about 50 ns per element for forward + backward in binary64 with libm tanh/cosh
    rows = int(seconds_budget / (50e-9 * max(1, w.N)))
    return max(1, min(w.M, rows))


def run_oracle_sample(w, rows: int, min_seconds: float = 0.0):
    """Oracle forward + backward on the first `rows` rows of the workload, repeated until
    `min_seconds` have elapsed (at least once); returns (seconds, algorithmic bytes, passes)."""
    import oracle
    from synth import workloads

    ws = dataclasses.replace(w, M=rows)
    inp = workloads.make_inputs(ws)
    passes, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(inp["x"], inp["alpha"], inp["gamma"], inp["beta"], rows, w.N, w.x_dtype, w.p_dtype)
        oracle.backward(inp["x"], inp["dy"], inp["alpha"], inp["gamma"], rows, w.N, w.x_dtype, w.p_dtype)
        passes += 1
        dt = time.perf_counter() - t0
        if dt >= min_seconds:
            return dt, passes * (ws.fwd_bytes() + ws.bwd_bytes()), passes


def cpu_baseline(w, seconds_budget=10.0):
    rows = oracle_sample_rows(w, seconds_budget)
    dt, nbytes, passes = run_oracle_sample(w, rows, min_seconds=seconds_budget)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {rows} of {w.M} rows (x {w.N} columns), forward + backward, {passes} pass(es), "
                      f"single-threaded binary64 C oracle, {dt:.2f} s",
            "rows_per_s": passes * rows / dt}


def cpu_baseline_threads(w, seconds_budget=5.0):
    """The same oracle fanned out over row blocks, one thread per host core in
    this process's affinity set (its C calls release the interpreter lock).
    Only the timing harness is parallel: each block is an ordinary oracle call
    on its rows, and the blocks' parameter-gradient sums would be added
    afterwards (N values, not timed). Repeated full passes until the budget
    has elapsed."""
    import concurrent.futures

    import oracle
    from synth import workloads

    cores = len(os.sched_getaffinity(0))
    rows = oracle_sample_rows(w, seconds_budget * cores)
    ws = dataclasses.replace(w, M=rows)
    inp = workloads.make_inputs(ws)
    N = w.N
    edges = [rows * i // cores for i in range(cores + 1)]
    blocks = [(a, b) for a, b in zip(edges[:-1], edges[1:]) if b > a]

    def run(block):
        a, b = block
        x, dy = inp["x"][a * N:b * N], inp["dy"][a * N:b * N]
        oracle.forward(x, inp["alpha"], inp["gamma"], inp["beta"], b - a, N, w.x_dtype, w.p_dtype)
        oracle.backward(x, dy, inp["alpha"], inp["gamma"], b - a, N, w.x_dtype, w.p_dtype)

    with concurrent.futures.ThreadPoolExecutor(max_workers=len(blocks)) as ex:
        passes, t0 = 0, time.perf_counter()
        while True:
            list(ex.map(run, blocks))
            passes += 1
            dt = time.perf_counter() - t0
            if dt >= seconds_budget:
                break
    nbytes = passes * (ws.fwd_bytes() + ws.bwd_bytes())
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": len(blocks), "kind": "oracle, row blocks on threads",
            "sample": f"first {rows} of {w.M} rows (x {N} columns) in {len(blocks)} row blocks, forward + backward, "
                      f"{passes} pass(es), {dt:.2f} s",
            "rows_per_s": passes * rows / dt}


# ---- the reference arm: the oracle as it stands ------------------------------------------------

def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    per_step_budget = min(10.0, 120.0 / max(1, args.steps + args.warmup))
    rows = oracle_sample_rows(w, per_step_budget)
    for _ in range(args.warmup):
        run_oracle_sample(w, max(1, rows // 8))
    times, nbytes = [], 0
    for _ in range(args.steps):
        dt, nbytes, _ = run_oracle_sample(w, rows)
        times.append(dt)
    total = sum(times)
    value = nbytes * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, args.gpus),
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"first {rows} of {w.M} rows per step, forward + backward, "
                                   "single-threaded binary64 C oracle"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config(w, gpus: int):
    """The workload as both arms name it (the same dict in both)."""
    return {"workload": w.name, "M": w.M, "N": w.N, "x_dtype": w.x_dtype, "param_dtype": w.p_dtype,
            "alpha": w.alpha, "x_std": w.x_std, "dy_std": w.dy_std, "gamma": f"N({w.gamma_mean},{w.gamma_std})",
            "beta": f"N({w.beta_mean},{w.beta_std})", "seed": w.seed, "parallelism": f"rows{gpus}"}


# ---- device buffers and timing -------------------------------------------------------------------

def _to_torch(a, dtype, device):
    import torch
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if dtype == "bf16" else torch.from_numpy(a)
    return t if str(device) == "cpu" else t.to(device)


def _matrix(src, w, dev, off):
    """An M x N device matrix holding src, starting `off` elements past a 16-byte
    boundary (0 for the workloads themselves), rows w.pitch elements apart."""
    t = _to_torch(src, w.x_dtype, "cpu")
    m = _empty_like_matrix(t, w, off, dev)
    m.copy_(t.view(w.M, w.N))
    return m


def _empty_like_matrix(m, w, off, dev=None):
    import torch
    ld = w.pitch or w.N
    buf = torch.empty(w.M * ld + off + 8, dtype=m.dtype, device=dev or m.device)
    return buf[off:off + w.M * ld].view(w.M, ld)[:, :w.N]


def _sets(w, inp, dev, L2):
    """Buffer sets for back-to-back calls: enough that the data touched between two
    uses of one set exceeds 3x the L2 size, so no call reads another's data from L2."""
    import torch
    from synth import workloads
    set_bytes = 4 * w.M * w.N * workloads.ITEMSIZE[w.x_dtype]  # x, dy, y, dx
    nsets = int(min(64, max(1, -(-3 * L2 // set_bytes))))
    x0, dy0 = _matrix(inp["x"], w, dev, w.x_off), _matrix(inp["dy"], w, dev, w.offset)
    ad, gd, bd = w.param_dtypes
    a, g, b = _to_torch(inp["alpha"], ad, dev), _to_torch(inp["gamma"], gd, dev), _to_torch(inp["beta"], bd, dev)
    sets = []
    for i in range(nsets):
        x = x0 if i == 0 else _empty_like_matrix(x0, w, w.x_off).copy_(x0)
        d = dy0 if i == 0 else _empty_like_matrix(dy0, w, w.offset).copy_(dy0)
        sets.append({"x": x, "dy": d, "y": _empty_like_matrix(x0, w, w.offset),
                     "dx": _empty_like_matrix(x0, w, w.offset),
                     "dg": torch.empty_like(g), "db": torch.empty_like(b), "da": torch.empty_like(a)})
    return sets, (a, g, b), set_bytes, nsets


def _graph(stream, fn, n):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(n):
            fn(i)
    return g


class _Eager:
    """The n calls fn(0) .. fn(n - 1) launched directly on the current stream at
    each replay(): the multi-rank steps, whose NCCL collectives (the exchange's
    barrier, or the all-reduce of the gradients) are not captured into graphs."""

    def __init__(self, fn, n):
        self.fn, self.n = fn, n

    def replay(self):
        for i in range(self.n):
            self.fn(i)


def _time_replays(g, stream, dev, K, clock_index, clocks=True, idle_s=0.4, min_seconds=0.6, min_replays=7,
                  max_replays=2000):
    """Per-call device time (us) of a K-call graph over repeated replays (CUDA events
    on the launching stream), after `idle_s` without load so that the GPU starts
    below its power limit. `burst`: the median of the first three replays;
    `sustained`: the median over the second half of the window, when a kernel that
    draws the power limit has reached its capped clock. p10 / p50 / p90 over all.
    Clocks, power and throttle reasons are sampled throughout."""
    import torch
    g.replay()
    torch.cuda.synchronize(dev)
    time.sleep(idle_s)
    rec = []
    with ClockSampler(clock_index, enabled=clocks) as clk:
        t_start = time.time()
        t_end = time.perf_counter() + min_seconds
        while len(rec) < min_replays or (time.perf_counter() < t_end and len(rec) < max_replays):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            t = time.time()
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            rec.append((t, e0.elapsed_time(e1) * 1e3 / K))
        while time.perf_counter() < t_end:  # keep the load on for the whole window
            g.replay()
            torch.cuda.synchronize(dev)
        t_stop = time.time()
    per = np.array([r[1] for r in rec])
    q = np.percentile(per, [10, 50, 90])
    t_half = rec[len(rec) // 2][0]
    return {"us_p10": float(q[0]), "us_p50": float(q[1]), "us_p90": float(q[2]), "replays": len(per),
            "burst_us": float(np.median(per[:3])), "sustained_us": float(np.median(per[len(per) // 2:])),
            "clocks": clk.summary(t_start, t_stop), "clocks_burst": clk.summary(t_start, t_start + 0.05),
            "clocks_sustained": clk.summary(t_half, t_stop)}


def _roofline(nbytes, us, peak, peak_kind, traffic):
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
            "peak_kind": peak_kind, "traffic": traffic, "algorithmic_bytes_per_launch": nbytes}


# ---- our arm ------------------------------------------------------------------------------------

def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import elementwise_reduction_b200 as dyt
    from synth import workloads

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    M, N = w.M, w.N
    inp = workloads.make_inputs(w)
    L2 = torch.cuda.get_device_properties(dev).L2_cache_size
    sets, (alpha, gamma, beta), set_bytes, nsets = _sets(w, inp, dev, L2)
    ws = dyt.workspace(sets[0]["x"], gamma, sets[0]["dy"], sets[0]["dx"])
    grads = torch.empty(2 * N + 1, dtype=torch.float32, device=dev)
    from elementwise_reduction_b200.dist import FusedGradientSum, allreduce_param_grads

    def make_exchange(x, dy, dx):
        """The fused cross-rank gradient sum, or None (every rank then falls back to the
        all-reduce of the rounded gradients): the ranks decide together."""
        if world == 1:
            return None, None
        ex = FusedGradientSum(x, dy, dx, gamma)  # records a local failure in ex.error
        ok = torch.tensor([1 if ex.error is None else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(ok, op=dist.ReduceOp.MIN)
        if int(ok.item()) == 0:
            ex.close()
            return None, ex.error or "another rank could not map the peer workspaces"
        return ex, None

    exchange, exchange_note = make_exchange(sets[0]["x"], sets[0]["dy"], sets[0]["dx"])
    sched = FusedGradientSum.schedule(max(2, args.steps)) if exchange is not None else None

    def fwd(s):
        dyt.forward(s["x"], alpha, gamma, beta, out=s["y"])

    default = object()  # bwd's ex: the run's exchange unless a lane passes its own (None: the all-reduce)

    def bwd(s, ws_=None, i=None, ex=default, gbuf=None):
        ex = exchange if ex is default else ex
        if ex is not None:  # stage 1, barrier, finalize over every rank's partials
            ex(s["x"], s["dy"], alpha, gamma, beta, s["dx"], s["dg"], s["db"], s["da"],
               buffer=None if i is None else sched[i % len(sched)])
            return
        dyt.backward(s["x"], s["dy"], alpha, gamma, beta, dx=s["dx"], dgamma=s["dg"], dbeta=s["db"],
                     dalpha=s["da"], ws=ws if ws_ is None else ws_)
        if world > 1:
            allreduce_param_grads(s["dg"], s["db"], s["da"], buf=grads if gbuf is None else gbuf)

    def step(i):
        s = sets[i % nsets]
        fwd(s)
        bwd(s, i=i)

    stream = torch.cuda.Stream(dev)
    torch.cuda.synchronize(dev)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
        # the launch records of one forward and one backward (the backward with
        # the next buffer of the exchange's schedule, as a further warm-up step)
        fwd(sets[0])
        launch_info_fwd = dyt.dyt_last_launch_info()
        bwd(sets[0], i=args.warmup)
        launch_info_bwd = dyt.dyt_last_launch_info()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()  # every rank's eager calls are done before any replay reuses a workspace
        # One rank: CUDA graphs of K calls. Several: the same calls launched
        # eagerly (no NCCL collective inside a graph).
        steps_of = (lambda fn: _graph(stream, fn, args.steps)) if world == 1 else (lambda fn: _Eager(fn, args.steps))
        g_step = steps_of(step)
        g_fwd = steps_of(lambda i: fwd(sets[i % nsets]))
        g_bwd = steps_of(lambda i: bwd(sets[i % nsets], i=i))
        for g in (g_step, g_fwd, g_bwd):  # untimed replay: first-launch costs
            g.replay()
        torch.cuda.synchronize(dev)

        def timed(g):
            if world > 1:
                dist.barrier()
            torch.cuda.synchronize(dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            torch.cuda.synchronize(dev)
            if world > 1:
                dist.barrier()
            ms = e0.elapsed_time(e1)
            if world > 1:
                t = torch.tensor([ms], device=dev)
                dist.all_reduce(t, op=dist.ReduceOp.MAX)
                ms = float(t.item())
            return ms

        with ClockSampler(local, enabled=not args.no_clocks) as clk:
            t0 = time.time()
            ms_step = timed(g_step)  # the timed region: K steps, clocks sampled every 5 ms
            t1 = time.time()
            ms_fwd = timed(g_fwd)
            ms_bwd = timed(g_bwd)
        clocks = clk.summary(t0, t1) or clk.summary()
        # The same step graph replayed back to back for about a second: what a long
        # run of this layer alone gets once the GPU sits at its power limit.
        sustained = _time_replays(g_step, stream, dev, args.steps, local, clocks=not args.no_clocks, idle_s=0.0,
                                  min_seconds=1.0) if world == 1 and not args.no_sustained else None
        del g_step, g_fwd, g_bwd
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()

    # ---- end to end through the public API: pinned host buffers in, results out ----
    # Consecutive steps alternate between two streams, each with its own device
    # buffers, workspace and host result buffers, so that one step's copies out
    # overlap the next step's copies in (the link's two directions are
    # independent). Every step still copies in its own inputs and copies out
    # its own results.
    # enough steps that the pipeline's fill and drain (one step's copies in, the
    # last step's copies out) do not dominate; a c5 step is ~20-30 ms of copies
    e2e_steps = args.e2e_steps or max(3, min(args.steps, 16))
    hx = _to_torch(inp["x"], w.x_dtype, "cpu").view(M, N).pin_memory()
    hdy = _to_torch(inp["dy"], w.x_dtype, "cpu").view(M, N).pin_memory()
    lanes = []
    for j in range(2):
        x0 = sets[0]["x"]
        d = sets[j] if j < nsets else {"x": _empty_like_matrix(x0, w, w.x_off), "dy": _empty_like_matrix(x0, w, w.offset),
                                       "y": _empty_like_matrix(x0, w, w.offset),
                                       "dx": _empty_like_matrix(x0, w, w.offset),
                                       "dg": torch.empty_like(gamma), "db": torch.empty_like(beta),
                                       "da": torch.empty_like(alpha)}
        lanes.append({"dev": d, "ws": dyt.workspace(x0, gamma, d["dy"], d["dx"]),
                      "stream": stream if j == 0 else torch.cuda.Stream(dev),
                      "ex": exchange if j == 0 or exchange is None else make_exchange(x0, x0, x0)[0],
                      "grads": torch.empty(2 * N + 1, dtype=torch.float32, device=dev),
                      "hy": torch.empty_like(hx).pin_memory(), "hdx": torch.empty_like(hx).pin_memory(),
                      "hdg": torch.empty(N, dtype=gamma.dtype).pin_memory(),
                      "hdb": torch.empty(N, dtype=beta.dtype).pin_memory(),
                      "hda": torch.empty(1, dtype=alpha.dtype).pin_memory()})

    # Copies in one direction run one step after another (each step's copies in
    # wait for the previous step's, likewise out), so that the link carries one
    # step's inputs while it returns the previous step's results instead of
    # splitting one direction between two steps.
    link = {"in": None, "out": None}

    def e2e_step(i):
        ln = lanes[i % 2]
        d = ln["dev"]
        st = ln["stream"]
        with torch.cuda.stream(st):
            if link["in"] is not None:
                st.wait_event(link["in"])
            d["x"].copy_(hx, non_blocking=True)
            d["dy"].copy_(hdy, non_blocking=True)
            link["in"] = torch.cuda.Event()
            link["in"].record(st)
            fwd(d)
            bwd(d, ln["ws"], ex=ln["ex"], gbuf=ln["grads"])
            if link["out"] is not None:
                st.wait_event(link["out"])
            ln["hy"].copy_(d["y"], non_blocking=True)
            ln["hdx"].copy_(d["dx"], non_blocking=True)
            ln["hdg"].copy_(d["dg"], non_blocking=True)
            ln["hdb"].copy_(d["db"], non_blocking=True)
            ln["hda"].copy_(d["da"], non_blocking=True)
            link["out"] = torch.cuda.Event()
            link["out"].record(st)

    e2e_step(0)
    e2e_step(1)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    lanes[1]["stream"].wait_stream(stream)  # nothing of the timed region starts before e0
    for i in range(e2e_steps):
        e2e_step(i)
    stream.wait_stream(lanes[1]["stream"])  # e1 after both streams' work
    e1.record(stream)
    torch.cuda.synchronize(dev)
    ms_e2e = e0.elapsed_time(e1)
    if world > 1:
        t = torch.tensor([ms_e2e], device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_e2e = float(t.item())
    sx = workloads.ITEMSIZE[w.x_dtype]
    sa, sg, sb = (workloads.ITEMSIZE[d] for d in w.param_dtypes)
    h2d = 2 * M * N * sx
    d2h = 2 * M * N * sx + N * (sg + sb) + sa
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()  # no rank still reads a peer's workspace
    for ln in lanes:
        if ln["ex"] is not None and ln["ex"] is not exchange:
            ln["ex"].close()
    if exchange is not None:
        exchange.close()
    del lanes, sets, ws
    torch.cuda.empty_cache()

    # ---- numbers ----
    fb, bb = w.fwd_bytes(), w.bwd_bytes()
    step_bytes = (fb + bb) * world
    ms_per_step = ms_step / args.steps
    value = step_bytes / (ms_per_step * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()
    t_fwd, t_bwd = ms_fwd / args.steps * 1e-3, ms_bwd / args.steps * 1e-3
    bw_fwd, bw_bwd = fb / t_fwd / 1e9, bb / t_bwd / 1e9
    dominant = "bwd" if t_bwd >= t_fwd else "fwd"
    traffic = committed_traffic(w.name, "dyt_backward" if dominant == "bwd" else "dyt_fwd_kernel")
    roofline = _roofline(bb if dominant == "bwd" else fb, (t_bwd if dominant == "bwd" else t_fwd) * 1e6, peak,
                         peak_kind, traffic)
    roofline["kernel"] = "dyt_backward (stage 1 + finalize)" if dominant == "bwd" else "dyt_forward"
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": workload_config(w, world),
        "l2": f"{nsets} rotating buffer set(s), {nsets * set_bytes / 2**20:.0f} MiB touched per cycle vs L2 "
              f"{L2 / 2**20:.0f} MiB (inputs larger than L2)" if set_bytes > L2 else
              f"{nsets} rotating buffer sets, {nsets * set_bytes / 2**20:.0f} MiB touched per cycle vs L2 "
              f"{L2 / 2**20:.0f} MiB",
        "pct_of_peak": 100.0 * value / world / peak,
        "rows_per_s": M * world / (ms_per_step * 1e-3),
        "fwd": {"us": t_fwd * 1e6, "GB_s": bw_fwd, "frac": bw_fwd / peak, "rows_per_s": M / t_fwd,
                "launch": launch_info_fwd},
        "bwd": {"us": t_bwd * 1e6, "GB_s": bw_bwd, "frac": bw_bwd / peak, "rows_per_s": M / t_bwd,
                "launch": launch_info_bwd},
        "roofline": roofline,
        "e2e": {"value": (fb + bb) * world * e2e_steps / (ms_e2e * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                "ms_per_step": ms_e2e / e2e_steps},
        "gpu_launches": args.steps * (launch_info_fwd["kernels"] + (2 if world > 1 and exchange is not None
                                                                     else launch_info_bwd["kernels"])),
        "grad_exchange": None if world == 1 else (
            "finalize over every rank's partials through peer pointers, after a one-element NCCL all-reduce"
            if exchange is not None else f"NCCL all-reduce of the rounded gradients ({exchange_note})"),
        "clocks": clocks,
    }
    if sustained is not None:
        ms_s = sustained["sustained_us"] * 1e-3
        line["sustained"] = {"ms_per_step": ms_s, "value": step_bytes / (ms_s * 1e-3) / 1e9, "unit": "GB/s",
                             "clocks": sustained["clocks_sustained"],
                             "note": "the step graph replayed back to back for 1 s; second half"}
    if world > 1:
        dist.destroy_process_group()
    if world == 1 and not args.no_shapes:
        line["shapes"] = shape_table(args, dev, local, cpu=not args.no_cpu_baseline)
    if world == 1 and not args.no_latency:
        line["latency_us"] = call_latency(args, dev)
    if world == 1 and not args.no_cpu_baseline:  # the oracle's baseline belongs to the 1-GPU line
        line["cpu_baseline"] = cpu_baseline(w)
        line["cpu_baseline_threads"] = cpu_baseline_threads(w)
    print(json.dumps(line), flush=True)


def call_latency(args, dev, calls=30):
    """Per-call device time of one forward and one backward call (both backward
    kernels), each with L2 flushed just before it, as p10 / p50 / p90 over
    `calls` calls; forward and backward alternate, and the workloads are visited
    in rotation. This is the latency of one isolated call, next to the graph
    throughput figures."""
    import torch

    import elementwise_reduction_b200 as dyt
    from synth import workloads

    L2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(2 * L2, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(dev)
    state = {}
    for name, w in {**workloads.WORKLOADS, **workloads.VARIANTS}.items():
        inp = workloads.make_inputs(w)
        x = _matrix(inp["x"], w, dev, w.x_off)
        ad, gd, bd = w.param_dtypes
        st = {"x": x, "dy": _matrix(inp["dy"], w, dev, w.offset), "y": _empty_like_matrix(x, w, w.offset),
              "dx": _empty_like_matrix(x, w, w.offset),
              "p": [_to_torch(inp[k], dt, dev) for k, dt in zip(("alpha", "gamma", "beta"), (ad, gd, bd))],
              "ws": None, "t": {"fwd": [], "bwd": []}}
        st["ws"] = dyt.workspace(x, st["p"][1], st["dy"], st["dx"])
        state[name] = st
    with torch.cuda.stream(stream):
        for i in range(calls + 2):  # the first two rounds are warm-up
            for name, st in state.items():
                a, g, b = st["p"]
                for op in ("fwd", "bwd"):
                    flush.fill_(i & 0xFF)
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(stream)
                    if op == "fwd":
                        dyt.forward(st["x"], a, g, b, out=st["y"])
                    else:
                        dyt.backward(st["x"], st["dy"], a, g, b, dx=st["dx"], ws=st["ws"])
                    e1.record(stream)
                    e1.synchronize()
                    if i >= 2:
                        st["t"][op].append(e0.elapsed_time(e1) * 1e3)
    out = {}
    for name, st in state.items():
        out[name] = {op: {q: round(float(np.percentile(v, p)), 2) for q, p in (("p10", 10), ("p50", 50), ("p90", 90))}
                     for op, v in st["t"].items()}
    del state, flush
    torch.cuda.empty_cache()
    return out


def shape_table(args, dev, clock_index, cpu=True):
    """Every workload and layout variant, forward and backward, each timed like the
    headline: a CUDA graph of K calls over rotating buffer sets that exceed L2,
    replayed for 0.6 s after an idle gap (burst: the first replays; sustained:
    the second half, once a power-hungry kernel sits at its power limit; p10 /
    p50 / p90 over all) with the SM clocks, power and throttle reasons sampled
    during the replays. Each line carries its roofline entry (burst, and
    sustained) and, next to it, the oracle on the host cores on a bounded sample
    of the same workload. A plain PyTorch copy (the forward's bytes) and a
    three-operand add (the backward's bytes), timed the same way, give what a
    library kernel moving the same bytes meets in this setting."""
    import torch

    import elementwise_reduction_b200 as dyt
    from synth import workloads

    out = {}
    peak, peak_kind = hbm_peak()
    L2 = torch.cuda.get_device_properties(dev).L2_cache_size
    K = args.steps
    for name, w in {**workloads.WORKLOADS, **workloads.VARIANTS}.items():
        inp = workloads.make_inputs(w)
        sets, (a, g, b), _, nsets = _sets(w, inp, dev, L2)
        ws = dyt.workspace(sets[0]["x"], g, sets[0]["dy"], sets[0]["dx"])
        stream = torch.cuda.Stream(dev)
        res = {}
        with torch.cuda.stream(stream):
            calls = {
                "fwd": lambda i: dyt.forward(sets[i % nsets]["x"], a, g, b, out=sets[i % nsets]["y"]),
                "bwd": lambda i: dyt.backward(sets[i % nsets]["x"], sets[i % nsets]["dy"], a, g, b,
                                              dx=sets[i % nsets]["dx"], dgamma=sets[i % nsets]["dg"],
                                              dbeta=sets[i % nsets]["db"], dalpha=sets[i % nsets]["da"], ws=ws),
            }
            # library floors: the same bytes moved by a PyTorch copy and a three-operand add
            calls["copy_floor"] = lambda i: sets[i % nsets]["y"].copy_(sets[i % nsets]["x"])
            calls["add3_floor"] = lambda i: torch.add(sets[i % nsets]["x"], sets[i % nsets]["dy"],
                                                      out=sets[i % nsets]["dx"])
            for op, call in calls.items():
                for i in range(3):
                    call(i)
                info = dyt.dyt_last_launch_info() if op in ("fwd", "bwd") else None
                graph = _graph(stream, call, K)
                t = _time_replays(graph, stream, dev, K, clock_index, clocks=not args.no_clocks)
                del graph
                nbytes = w.fwd_bytes() if op in ("fwd", "copy_floor") else w.bwd_bytes()
                kernel = {"fwd": "dyt_fwd_kernel", "bwd": "dyt_backward"}.get(op)
                t["roofline"] = _roofline(nbytes, t["burst_us"], peak, peak_kind,
                                          committed_traffic(name, kernel) if kernel else None)
                t["roofline_sustained"] = _roofline(nbytes, t["sustained_us"], peak, peak_kind, None)
                t["rows_per_s"] = w.M / (t["burst_us"] * 1e-6)
                if info is not None:
                    t["launch"] = {k: info[k] for k in ("path", "vec", "grid", "row_lanes", "row_groups",
                                                        "pack_rows", "kernels")}
                res[op] = t
        if cpu:
            res["cpu_baseline"] = cpu_baseline(w, seconds_budget=2.0)
            res["cpu_baseline_threads"] = cpu_baseline_threads(w, seconds_budget=1.5)
        out[name] = res
        del sets, ws
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    from synth import workloads

    name = args.workload or workloads.DEFAULT_BENCH
    w = {**workloads.WORKLOADS, **workloads.VARIANTS}[name]
    if args.record_traffic:
        record_traffic(args.record_traffic, w.name, args.ncu_command)
        return
    if args.impl == "reference":
        run_reference(args, w)
    else:
        run_ours(args, w)


if __name__ == "__main__":
    main()
