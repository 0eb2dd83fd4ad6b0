"""Benchmark of exact attention (forward + backward, bf16, causal) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole hot path over one batch: fa_fwd (O, LSE) then fa_bwd
(dQ, dK, dV).  The headline workload is the long wide shape (B=1, H=96,
N=8192, d=128, causal), the largest causal d=128 configuration that fits one
GPU; the training shape (B=2, H=16, N=2048, d=128, causal) is measured
alongside it under ``extra``.  FLOPs follow the metric: forward 4*B*H*N^2*d,
halved when causal; forward+backward = 3.5x forward.

Timing: W untimed warm-up steps, then K steps, each bracketed by CUDA events
on the launching stream, with L2 flushed between steps outside the events (a
256 MiB write, then a 256 MiB read so the lines left in L2 are clean); barrier + synchronize around the loop; with N > 1
processes (torchrun) every rank runs its own batch (weak scaling, no
collective on the data path) and the time is the max over ranks.  Rank 0
prints one JSON line.

``--impl reference`` times the fp64 CPU oracle (the reference arm) on a
bounded sample of the same workload on the host cores.
"""
import argparse
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

METRIC = "attention TFLOP/s fwd & fwd+bwd (bf16, causal) and % of B200 dense BF16 peak"
DENSE_PEAK_TFLOPS = 2250.0  # NVIDIA B200 dense BF16 datasheet figure

WORKLOADS = {
    "train": dict(name="training-shape attention B=2 H=16 N=2048 d=128 causal fwd+bwd",
                  B=2, N=2048, H=16, Hkv=16, d=128, causal=True, window=(-1, -1), seed=1002),
    "wide": dict(name="long wide attention B=1 H=96 N=8192 d=128 causal fwd+bwd",
                 B=1, N=8192, H=96, Hkv=96, d=128, causal=True, window=(-1, -1), seed=1005),
    # a third of the wide shape: inputs still larger than L2, small enough for a
    # full profiler capture of single launches
    "mid": dict(name="attention B=1 H=32 N=8192 d=128 causal fwd+bwd",
                B=1, N=8192, H=32, Hkv=32, d=128, causal=True, window=(-1, -1), seed=1006),
}


# DRAM traffic (dram__bytes_read.sum + dram__bytes_write.sum) of one launch,
# from the ncu captures summarised under profiles/; the table itself lives in
# profiles/traffic.json (workload key, kernel kind, bytes, the capture's
# summary file, and a sha256 of the kernel sources that were profiled).  A
# figure is reported only while the current sources hash to that value: a
# changed kernel reports null until it is captured again.
TRAFFIC_TABLE = os.path.join(ROOT, "profiles", "traffic.json")


def load_traffic():
    try:
        with open(TRAFFIC_TABLE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return "", {}
    rows = {(r["workload"], r["kernel"]): dict(bytes=float(r["bytes"]), profile=r["profile"])
            for r in t.get("captures", [])}
    return t.get("sources_sha256", ""), rows


def sources_sha256():
    """sha256 over the kernel sources (csrc/*.cu, *.cuh and include/fa.h)."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "exact_io_aware_89_b200", "csrc")
    files = sorted(os.path.join(csrc, f) for f in os.listdir(csrc) if f.endswith((".cu", ".cuh")))
    files.append(os.path.join(ROOT, "include", "fa.h"))
    for f in files:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def ncu_traffic(workload_key, kernel, table=None):
    sha, rows = table if table is not None else load_traffic()
    t = rows.get((workload_key, kernel))
    if t is None or not sha or sources_sha256() != sha:
        return None, None
    return t["bytes"], t["profile"]


def fwd_flops(w):
    f = 4.0 * w["B"] * w["H"] * w["N"] * w["N"] * w["d"]
    return f / 2 if w["causal"] else f


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p["bf16_tflops_sustained"]), source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


class L2Flush:
    """Evicts the step's inputs from the 126 MB L2 between timed calls: a
    256 MiB write, then a 256 MiB read of another buffer.  The read leaves L2
    holding clean lines, as it would after ordinary work; after the write
    alone, L2 is full of dirty lines whose write-back (about 15 us of HBM
    time) would land inside the next timed call."""

    def __init__(self, dev):
        import torch
        self.dirty = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.clean = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def __call__(self):
        self.dirty.zero_()
        self.clean.sum()


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """SM clock and clock-event (throttle) reasons sampled through NVML (read
    only) every ``period_s`` while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, device, period_s=0.002):
        self.device = device
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.error = None
        self._stop = threading.Event()
        self._thread = None

    def _handle(self):
        import pynvml
        import torch
        pynvml.nvmlInit()
        try:
            uuid = "GPU-%s" % torch.cuda.get_device_properties(self.device).uuid
            return pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
        except Exception:
            return pynvml.nvmlDeviceGetHandleByIndex(self.device.index or 0)

    def _run(self, h):
        import pynvml
        get_reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                     int(get_reasons(h))))
            except Exception as e:  # pragma: no cover
                self.error = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        try:
            import pynvml
            h = self._handle()
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self._thread = threading.Thread(target=self._run, args=(h,), daemon=True)
            self._thread.start()
        except Exception as e:
            self.error = str(e)
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=5)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz,
                    "reasons": ["no samples" + (": " + self.error if self.error else "")]}
        reasons = set()
        for _, bits in self.samples:
            for bit, name in self.REASONS.items():
                if bits & bit:
                    reasons.add(name)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(reasons), "source": "nvml"}


# ------------------------------------------------------------ distributed

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus %d needs torchrun with %d processes" % (args.gpus, args.gpus))
    return world, rank, local


def max_over_ranks(value, world):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64,
                     device="cuda" if dist.get_backend() == "nccl" else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(flops_per_step, steps, t_ms_local, world):
    """Whole-job TFLOP/s under weak scaling: every rank ran `steps` steps of
    `flops_per_step` on its own batch; the job's time is the slowest rank's."""
    t_max = max_over_ranks(t_ms_local, world)
    return flops_per_step * steps * world / (t_max * 1e-3) / 1e12


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ GPU arm

def make_device_inputs(w, rank, dev, dtype="bf16"):
    import torch
    from seeded_inputs import make_inputs
    inp = make_inputs(w["B"], w["N"], w["N"], w["H"], w["Hkv"], w["d"], w["seed"] + 7919 * rank,
                      dtype=dtype)
    return {n: t.to(dev) for n, t in inp.items()}, inp


def time_gpu(w, steps, warmup, world, rank, dev, with_e2e=True, with_trace=True):
    import torch
    import exact_io_aware_89_b200 as fa

    x, host = make_device_inputs(w, rank, dev)
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    B, N, H, Hkv, d = w["B"], w["N"], w["H"], w["Hkv"], w["d"]
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, fa.fa_bwd_workspace_size(B, N, H, d)), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    stream = torch.cuda.current_stream()
    sp = stream.cuda_stream
    scale = 1.0 / math.sqrt(d)
    c, (wl, wr) = int(w["causal"]), w["window"]

    def step(q_, k_, v_, do_):
        st = fa.fa_fwd(q_.data_ptr(), k_.data_ptr(), v_.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       B, N, N, H, Hkv, d, scale, c, wl, wr, sp)
        if st:
            raise fa.FAError("fa_fwd", st)
        st = fa.fa_bwd(q_.data_ptr(), k_.data_ptr(), v_.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       do_.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, N, H, Hkv,
                       d, scale, c, wl, wr, ws.data_ptr(), ws.numel(), sp)
        if st:
            raise fa.FAError("fa_bwd", st)

    def fwd_only():
        st = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       B, N, N, H, Hkv, d, scale, c, wl, wr, sp)
        if st:
            raise fa.FAError("fa_fwd", st)

    for _ in range(warmup):
        step(q, k, v, do)
    torch.cuda.synchronize()
    if fa.fa_get_device_status(None) != 0:
        raise RuntimeError("device status reports a timed-out wait")

    # --- device-timed loop (inputs resident in HBM)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    if with_trace:
        fa.fa_trace_enable(1)
        fa.fa_trace_read()
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev) as clocks:
        for i in range(steps):
            flush()
            ev[i][0].record(stream)
            step(q, k, v, do)
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    trace_ms, trace_n = (fa.fa_trace_read() if with_trace else ({}, {}))
    if with_trace:
        fa.fa_trace_enable(0)

    # --- forward alone (for the fwd TFLOP/s the metric also names)
    fev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(steps)]
    for i in range(steps):
        flush()
        fev[i][0].record(stream)
        fwd_only()
        fev[i][1].record(stream)
    torch.cuda.synchronize()
    fwd_ms = [a.elapsed_time(b) for a, b in fev]

    out = dict(step_ms=step_ms, fwd_ms=fwd_ms, trace_ms=trace_ms, trace_n=trace_n,
               clocks=clocks.summary())

    # --- end to end through the public API: pinned host inputs in, results
    # out.  Every step copies its inputs from pinned host memory and reads O,
    # LSE, dQ, dK and dV back; the copies run on their own streams (host to
    # device and device to host use separate copy engines), so step i's
    # kernels overlap step i+1's upload and step i-1's download, with three
    # device buffer sets taking turns (with two, each set's upload, kernels and
    # download would form one serial chain).
    if with_e2e:
        hin = {n: t.pin_memory() for n, t in host.items()}
        names_out = ("o", "lse", "dq", "dk", "dv")
        shapes_out = {"o": o, "lse": lse, "dq": dq, "dk": dk, "dv": dv}
        hout = {n: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for n, t in shapes_out.items()}
        NSETS = 3
        sets = []
        for _ in range(NSETS):
            dbuf = {n: torch.empty_like(x[n]) for n in ("q", "k", "v", "do")}
            dbuf.update({n: torch.empty_like(t) for n, t in shapes_out.items()})
            sets.append(dbuf)
        h2d = sum(t.numel() * t.element_size() for t in hin.values())
        d2h = sum(t.numel() * t.element_size() for t in hout.values())
        e_steps = max(6, min(steps, 12))
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev = lambda: torch.cuda.Event()
        in_done = [ev() for _ in range(e_steps)]
        comp_done = [ev() for _ in range(e_steps)]
        out_done = [ev() for _ in range(e_steps)]
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

        def e2e_step(b, out_b):
            st = fa.fa_fwd(b["q"].data_ptr(), b["k"].data_ptr(), b["v"].data_ptr(), out_b["o"].data_ptr(),
                           out_b["lse"].data_ptr(), B, N, N, H, Hkv, d, scale, c, wl, wr, sp)
            if st:
                raise fa.FAError("fa_fwd", st)
            st = fa.fa_bwd(b["q"].data_ptr(), b["k"].data_ptr(), b["v"].data_ptr(), out_b["o"].data_ptr(),
                           out_b["lse"].data_ptr(), b["do"].data_ptr(), out_b["dq"].data_ptr(),
                           out_b["dk"].data_ptr(), out_b["dv"].data_ptr(), B, N, N, H, Hkv, d, scale, c, wl, wr,
                           ws.data_ptr(), ws.numel(), sp)
            if st:
                raise fa.FAError("fa_bwd", st)

        barrier(world)
        torch.cuda.synchronize()
        t_start.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(e_steps):
            b = sets[i % NSETS]
            if i >= NSETS:  # the set's previous step has been computed and read back
                s_in.wait_event(out_done[i - NSETS])
            with torch.cuda.stream(s_in):
                for n in ("q", "k", "v", "do"):
                    b[n].copy_(hin[n], non_blocking=True)
                in_done[i].record(s_in)
            stream.wait_event(in_done[i])
            e2e_step(b, b)
            comp_done[i].record(stream)
            s_out.wait_event(comp_done[i])
            with torch.cuda.stream(s_out):
                for n in names_out:
                    hout[n].copy_(b[n], non_blocking=True)
                out_done[i].record(s_out)
        stream.wait_event(out_done[e_steps - 1])
        t_end.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        out["e2e_ms"] = [t_start.elapsed_time(t_end) / e_steps] * e_steps
        out["h2d"], out["d2h"] = h2d, d2h
        del sets
    if fa.fa_get_device_status(None) != 0:
        raise RuntimeError("device status reports a timed-out wait")
    del flush
    return out


def kernel_algorithmic(w):
    """Algorithmic work per launch of each kernel kind (FLOPs for the tensor-core
    kernels, bytes for the preprocess).  The backward's five contractions
    (S, dP, dV, dK, dQ; 2.5x forward) are split between the dK/dV kernel (S,
    dP, dV, dK = 2x forward) and the dQ kernel (dQ = 0.5x forward; its own
    recomputation of S and dP is not algorithmic work)."""
    F = fwd_flops(w)
    rows = w["B"] * w["H"] * w["N"]
    return {
        "fwd": ("tensor", F),
        "bwd_dkdv": ("tensor", 2.0 * F),
        "bwd_dq": ("tensor", 0.5 * F),
        "bwd_prep": ("hbm", rows * (2 * w["d"] * 2 + 4 + 8)),
        # a whole backward call: the preprocess, then dQ and dK/dV at the same
        # time on two streams; the backward's algorithmic work, 2.5x forward
        "bwd_call": ("tensor", 2.5 * F),
    }


# The step's units for the roofline: the forward kernel and the whole
# backward call.  dQ and dK/dV overlap in time, so their own event spans
# include each other's share of the GPU and are reported only as detail.
STEP_UNITS = ("fwd", "bwd_call")
SPAN_KINDS = ("bwd_call",)  # traced spans that are not kernels


def tensor_peak(peaks, clocks):
    """The measured bf16 peak that applies to a kernel timed in this run, by
    the clock it ran at: the burst figure when the median SM clock sampled
    over the timed region stayed within 5% of its maximum (the cuBLAS burst
    ran at full clock), whether or not the power cap was reported; else the
    sustained figure, measured with the clock pulled down by the power cap.
    Returns (TFLOP/s, label)."""
    mhz, mx = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if mhz and mx and mhz >= 0.95 * mx:
        return peaks["bf16"], "burst"
    return peaks["bf16_sustained"], "sustained"


def roofline(w, res, peaks):
    alg = kernel_algorithmic(w)
    tpeak, tlabel = tensor_peak(peaks, res.get("clocks") or {})
    per = {}
    for kind, (bound, work) in alg.items():
        n = res["trace_n"].get(kind, 0)
        if not n:
            continue
        avg_ms = res["trace_ms"][kind] / n
        if bound == "tensor":
            ach = work / (avg_ms * 1e-3) / 1e12
            peak, label = tpeak, tlabel
            unit = "TFLOP/s"
        else:
            ach = work / (avg_ms * 1e-3) / 1e9
            peak, label = peaks["hbm_gbs"], "copy"
            unit = "GB/s"
        per[kind] = dict(bound=bound, achieved=round(ach, 2), peak=peak, peak_kind=label, unit=unit,
                         frac=round(ach / peak, 4), avg_ms=round(avg_ms, 4), launches=n,
                         share=None)
    units = [k for k in STEP_UNITS if k in per]
    total = sum(res["trace_ms"].get(k, 0.0) for k in units)
    for k in per:
        per[k]["share"] = round(res["trace_ms"][k] / total, 4) if total else None
        if k in ("bwd_dq", "bwd_dkdv") and "bwd_dq" in per and "bwd_dkdv" in per:
            per[k]["note"] = "runs concurrently with the other backward kernel; span includes its share"
    dom = max(units, key=lambda k: res["trace_ms"][k]) if units else None
    return dom, per


# ------------------------------------------------------------ CPU oracle arm

_ORACLE_INPUTS = {}


def oracle_sample(w, max_heads=None, budget_s=20.0):
    """Time the fp64 oracle's forward + backward on whole heads of the workload
    (full N) until about budget_s has passed; return (TFLOP/s by the metric's
    count, heads timed, seconds, threads)."""
    import numpy as np
    import oracle
    from seeded_inputs import make_inputs
    if w["name"] not in _ORACLE_INPUTS:
        inp = make_inputs(w["B"], w["N"], w["N"], w["H"], w["Hkv"], w["d"], w["seed"])
        _ORACLE_INPUTS[w["name"]] = {n: t.double().numpy() for n, t in inp.items()}
    f64 = _ORACLE_INPUTS[w["name"]]
    scale = 1.0 / math.sqrt(w["d"])
    per_head = fwd_flops(w) / (w["B"] * w["H"]) * 3.5
    nthreads = oracle.default_threads()
    heads, t_total = 0, 0.0
    total_heads = w["B"] * w["H"]
    G = w["H"] // w["Hkv"]
    while heads < (max_heads or total_heads):
        b, h = divmod(heads, w["H"])
        hk = h // G
        sl = lambda a, hh: np.ascontiguousarray(a[b:b + 1, :, hh:hh + 1])
        q, k, v, do = sl(f64["q"], h), sl(f64["k"], hk), sl(f64["v"], hk), sl(f64["do"], h)
        t0 = time.perf_counter()
        oracle.attn_fwd(q, k, v, scale=scale, causal=w["causal"], window=w["window"],
                        nthreads=nthreads)
        oracle.attn_bwd(q, k, v, do, scale=scale, causal=w["causal"], window=w["window"],
                        nthreads=nthreads)
        t_total += time.perf_counter() - t0
        heads += 1
        if t_total >= budget_s:
            break
    return per_head * heads / t_total / 1e12, heads, t_total, nthreads


def run_reference(args, world, rank):
    """The reference arm: the fp64 oracle as it stands, on the host cores.  Each
    step is a bounded sample of the workload (one whole head at full N, forward
    and backward); the batch time is extrapolated from the per-head median."""
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    for _ in range(args.warmup):
        oracle_sample(w, max_heads=1, budget_s=0.0)
    samples, threads = [], 1
    for _ in range(args.steps):
        _, h_s, s_s, threads = oracle_sample(w, max_heads=1, budget_s=0.0)
        samples.append(s_s / h_s)
    per_head = fwd_flops(w) / (w["B"] * w["H"]) * 3.5
    step_s = statistics.median(samples) * w["B"] * w["H"]
    value = per_head * w["B"] * w["H"] / step_s / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(step_s * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded N(0,1), bf16-rounded)",
        "config": {"workload": w["name"], "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"],
                   "causal": w["causal"]},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": threads,
                         "kind": "oracle",
                         "sample": "1 of %d heads per step (full N, fwd+bwd), batch time "
                                   "extrapolated from the per-head median" % (w["B"] * w["H"])},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------ sweep

def sweep_workloads():
    """The sequence-length sweep (N in 512..16k, d in {64, 128}, hidden 2048 so
    H = 2048 / d, batch 16384 / N, causal and not), then the GQA + window and
    the d = 256 workloads."""
    from seeded_inputs import config_seed, sweep_seed
    out = []
    for d in (64, 128):
        for N in (512, 1024, 2048, 4096, 8192, 16384):
            for causal in (False, True):
                out.append(dict(name="sweep N=%d d=%d %s" % (N, d, "causal" if causal else "non-causal"),
                                B=16384 // N, N=N, H=2048 // d, Hkv=2048 // d, d=d, causal=causal,
                                window=(-1, -1), seed=sweep_seed(N, d)))
    out.append(dict(name="GQA + window B=1 Hq=32 Hkv=8 N=8192 d=128 causal window (4096, 0)",
                    B=1, N=8192, H=32, Hkv=8, d=128, causal=True, window=(4096, 0), seed=config_seed(4)))
    out.append(dict(name="long wide d=256 B=1 H=16 N=16384 causal", B=1, N=16384, H=16, Hkv=16, d=256,
                    causal=True, window=(-1, -1), seed=config_seed(5) + 50))
    return out


def visible_pairs(w):
    """Number of visible (query, key) pairs per (batch, head) under the mask."""
    N = w["N"]
    wl, wr = w["window"]
    wr = 0 if w["causal"] else wr
    i = range(N)
    hi = [N - 1 if wr < 0 else min(N - 1, r + wr) for r in i]
    lo = [0 if wl < 0 else max(0, r - wl) for r in i]
    return sum(max(0, h - l + 1) for h, l in zip(hi, lo))


def time_modes(w, steps, warmup, dev, dtype="bf16"):
    """Median ms of fa_fwd alone, fa_bwd alone and fa_fwd + fa_bwd (L2 flushed
    before every timed call, CUDA events on the launching stream)."""
    import torch
    import exact_io_aware_89_b200 as fa
    x, _ = make_device_inputs(w, 0, dev, dtype)
    q, k, v, do = x["q"], x["k"], x["v"], x["do"]
    B, N, H, Hkv, d = w["B"], w["N"], w["H"], w["Hkv"], w["d"]
    fa_fwd, fa_bwd = (fa.fa_fwd_f16, fa.fa_bwd_f16) if dtype == "fp16" else (fa.fa_fwd, fa.fa_bwd)
    o = torch.empty_like(q)
    lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    ws = torch.empty(max(16, fa.fa_bwd_workspace_size(B, N, H, d)), dtype=torch.uint8, device=dev)
    flush = L2Flush(dev)
    sp = torch.cuda.current_stream().cuda_stream
    scale = 1.0 / math.sqrt(d)
    c, (wl, wr) = int(w["causal"]), w["window"]

    def fwd():
        st = fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       B, N, N, H, Hkv, d, scale, c, wl, wr, sp)
        if st:
            raise fa.FAError("fa_fwd", st)

    def bwd():
        st = fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                       do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, N, H, Hkv,
                       d, scale, c, wl, wr, ws.data_ptr(), ws.numel(), sp)
        if st:
            raise fa.FAError("fa_bwd", st)

    def both():
        fwd()
        bwd()

    out = {}
    for mode, fn in (("fwd", fwd), ("bwd", bwd), ("fwd_bwd", both)):
        for _ in range(warmup):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(steps)]
        for i in range(steps):
            flush()
            ev[i][0].record()
            fn()
            ev[i][1].record()
        torch.cuda.synchronize()
        out[mode] = statistics.median(a.elapsed_time(b) for a, b in ev)
    if fa.fa_get_device_status(None) != 0:
        raise RuntimeError("device status reports a timed-out wait")
    del flush, x
    torch.cuda.empty_cache()
    return out


def run_sweep(args, local):
    """One JSON line per workload of the sweep: fwd, bwd and fwd+bwd timed
    separately, TFLOP/s by the metric's formula (forward 4 B H N^2 d, halved
    when causal; backward 2.5x; fwd+bwd 3.5x), and, for a window, also by the
    visible pairs (4 B H pairs d)."""
    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    for w in sweep_workloads():
        if args.sweep_filter and args.sweep_filter not in w["name"]:
            continue
        t = time_modes(w, args.steps, args.warmup, dev, args.dtype)
        F = fwd_flops(w)
        line = {"sweep": w["name"], "dtype": args.dtype, "B": w["B"], "H": w["H"], "Hkv": w["Hkv"], "N": w["N"], "d": w["d"],
                "causal": w["causal"], "window": list(w["window"]),
                "ms": {m: round(v, 4) for m, v in t.items()},
                "tflops": {"fwd": round(F / t["fwd"] / 1e9, 1), "bwd": round(2.5 * F / t["bwd"] / 1e9, 1),
                           "fwd_bwd": round(3.5 * F / t["fwd_bwd"] / 1e9, 1)}}
        line["pct_dense_peak"] = {m: round(100 * v / DENSE_PEAK_TFLOPS, 2) for m, v in line["tflops"].items()}
        if w["window"] != (-1, -1):
            Fv = 4.0 * w["B"] * w["H"] * visible_pairs(w) * w["d"]
            line["tflops_visible_pairs"] = {"fwd": round(Fv / t["fwd"] / 1e9, 1),
                                            "bwd": round(2.5 * Fv / t["bwd"] / 1e9, 1),
                                            "fwd_bwd": round(3.5 * Fv / t["fwd_bwd"] / 1e9, 1)}
        print(json.dumps(line), flush=True)


# ------------------------------------------------------------ decode (split-KV)

def decode_workloads():
    """Decoding steps with a KV cache (few query rows, many cached keys,
    causal bottom-right): GQA shapes of common model families, long context,
    MHA, and a 4-token speculative step."""
    return [
        dict(name="decode GQA B=8 Hq=32 Hkv=8 Nq=1 Nk=32768 d=128", B=8, Nq=1, Nk=32768, Hq=32, Hkv=8, d=128),
        dict(name="decode GQA B=1 Hq=32 Hkv=8 Nq=1 Nk=131072 d=128", B=1, Nq=1, Nk=131072, Hq=32, Hkv=8, d=128),
        dict(name="decode GQA B=64 Hq=64 Hkv=8 Nq=1 Nk=8192 d=128", B=64, Nq=1, Nk=8192, Hq=64, Hkv=8, d=128),
        dict(name="decode MHA B=16 H=32 Nq=1 Nk=8192 d=128", B=16, Nq=1, Nk=8192, Hq=32, Hkv=32, d=128),
        dict(name="decode GQA B=8 Hq=32 Hkv=8 Nq=4 Nk=32768 d=128 (speculative)", B=8, Nq=4, Nk=32768,
             Hq=32, Hkv=8, d=128),
        dict(name="decode GQA B=8 Hq=16 Hkv=2 Nq=1 Nk=32768 d=64", B=8, Nq=1, Nk=32768, Hq=16, Hkv=2, d=64),
        dict(name="decode GQA B=4 Hq=16 Hkv=4 Nq=1 Nk=32768 d=256", B=4, Nq=1, Nk=32768, Hq=16, Hkv=4, d=256),
        dict(name="decode GQA B=16 Hq=32 Hkv=8 Nq=1 d=128, KV cache of 32768 keys with ragged lengths "
                   "(seeded uniform), one new key/value appended in place", B=16, Nq=1, Nk=32768, Hq=32,
             Hkv=8, d=128, ragged=True),
    ]


def decode_lengths(w):
    """Cached keys per sequence of a ragged decoding workload (seeded)."""
    import numpy as np
    rng = np.random.default_rng(4321)
    return rng.integers(1, w["Nk"], w["B"]).tolist()


def decode_bytes(w):
    """Algorithmic HBM bytes of one decoding step (causal, so every cached key
    is visible): read K, V, Q; write O (bf16) and LSE (fp32).  With ragged
    lengths, K and V of each sequence's own keys (its cached ones plus the
    new one), and the new key/value read once and written into the cache."""
    row = w["Hkv"] * w["d"] * 2
    if w.get("ragged"):
        kv = 2 * row * sum(min(w["Nk"], n + 1) for n in decode_lengths(w)) + 2 * 2 * w["B"] * row
    else:
        kv = 2 * w["B"] * w["Nk"] * row
    qo = 2 * w["B"] * w["Nq"] * w["Hq"] * w["d"] * 2
    return kv + qo + 4 * w["B"] * w["Hq"] * w["Nq"]


def run_decode(args, local):
    """One JSON line per decoding workload: fa_fwd_splitkv (the library's split
    count) timed with CUDA events on the launching stream, L2 flushed before
    every call, median over the steps; algorithmic bytes / time against the
    measured HBM copy bandwidth; fa_fwd on the same inputs for comparison."""
    import torch
    import exact_io_aware_89_b200 as fa
    from seeded_inputs import make_inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    flush = L2Flush(dev)
    sp = torch.cuda.current_stream().cuda_stream
    for n, w in enumerate(decode_workloads()):
        if args.decode_case is not None and n != args.decode_case:
            continue
        B, Nq, Nk, Hq, Hkv, d = w["B"], w["Nq"], w["Nk"], w["Hq"], w["Hkv"], w["d"]
        inp = make_inputs(B, Nq, Nk, Hq, Hkv, d, 4000 + n, with_dout=False)
        q, k, v = (inp[x].to(dev) for x in ("q", "k", "v"))
        del inp
        ragged = bool(w.get("ragged"))
        if ragged:
            lens = torch.tensor(decode_lengths(w), dtype=torch.int32, device=dev)
            new = make_inputs(B, 1, 1, Hkv, Hkv, d, 5000 + n, with_dout=False)
            k_new, v_new = new["k"].to(dev), new["v"].to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, Hq, Nq), dtype=torch.float32, device=dev)
        scale = 1.0 / math.sqrt(d)
        wsb = (fa.fa_fwd_kvcache_workspace_size(B, Nq, Nk, Hq, Hkv, d, 1, -1, -1, 0, 1) if ragged else
               fa.fa_fwd_splitkv_workspace_size(B, Nq, Nk, Hq, Hkv, d, 1, -1, -1, 0))
        ws = torch.empty(max(16, wsb), dtype=torch.uint8, device=dev)

        def split():
            if ragged:
                st = fa.fa_fwd_kvcache(q.data_ptr(), k.data_ptr(), v.data_ptr(), k_new.data_ptr(),
                                       v_new.data_ptr(), lens.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                       B, Nq, Nk, 1, Hq, Hkv, d, scale, 1, -1, -1, 0, ws.data_ptr(),
                                       ws.numel(), sp)
                if st:
                    raise fa.FAError("fa_fwd_kvcache", st)
                return
            st = fa.fa_fwd_splitkv(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                   lse.data_ptr(), B, Nq, Nk, Hq, Hkv, d, scale, 1, -1, -1, 0,
                                   ws.data_ptr(), ws.numel(), sp)
            if st:
                raise fa.FAError("fa_fwd_splitkv", st)

        def plain():
            st = fa.fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                           B, Nq, Nk, Hq, Hkv, d, scale, 1, -1, -1, sp)
            if st:
                raise fa.FAError("fa_fwd", st)

        def timed(fn, trace=False):
            for _ in range(args.warmup):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            if trace:
                fa.fa_trace_enable(1)
                fa.fa_trace_read()
            torch.cuda.synchronize()
            with ClockSampler(dev) as clocks:
                for i in range(args.steps):
                    flush()
                    ev[i][0].record()
                    fn()
                    ev[i][1].record()
                torch.cuda.synchronize()
            tr = fa.fa_trace_read() if trace else None
            if trace:
                fa.fa_trace_enable(0)
            return statistics.median(a.elapsed_time(b) for a, b in ev), tr, clocks.summary()

        t_split, (tms, tn), clk = timed(split, trace=True)
        t_plain = None if ragged else timed(plain)[0]
        if fa.fa_get_device_status(None) != 0:
            raise RuntimeError("device status reports a timed-out wait")
        nbytes = decode_bytes(w)
        gbs = nbytes / (t_split * 1e-3) / 1e9
        main_ms = tms["decode"] / max(1, tn["decode"])
        G = Hq // Hkv
        qpt = min(Nq, 128 // G)
        units = B * Hkv * (-(-Nq // qpt))
        n_splits = (wsb - 8 * units) // (4 * (d + 1)) // (units * qpt * G) if wsb else 1
        line = {"decode": w["name"], "B": B, "Nq": Nq, "Nk": Nk, "Hq": Hq, "Hkv": Hkv, "d": d,
                "causal": True, "ms": round(t_split, 4),
                "fa_fwd_ms": None if t_plain is None else round(t_plain, 4),
                "speedup_vs_fa_fwd": None if t_plain is None else round(t_plain / t_split, 2),
                "n_splits": n_splits, "workspace_bytes": wsb,
                "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"],
                             "unit": "GB/s", "frac": round(gbs / peaks["hbm_gbs"], 4),
                             "algorithmic_bytes": nbytes,
                             "traffic": ncu_traffic("decode%d" % n, "decode")[0],
                             "traffic_profile": ncu_traffic("decode%d" % n, "decode")[1],
                             "kernel_ms": round(main_ms, 4),
                             "kernel_frac": round(nbytes / (main_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
                             "peak_source": peaks["source"] + ", copy"},
                "clocks": clk}
        if ragged:
            lens_h = decode_lengths(w)
            line["cache_lengths"] = {"min": min(lens_h), "max": max(lens_h),
                                     "mean": round(sum(lens_h) / B, 1)}
            line["append_kernel_ms"] = round(tms["kvcache_append"] / max(1, tn["kvcache_append"]), 4)
            # the whole call is two launches (append, then attention)
            line["roofline"]["kernel_ms"] = round(main_ms + line["append_kernel_ms"], 4)
            line["roofline"]["kernel_frac"] = round(
                nbytes / (line["roofline"]["kernel_ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)
        print(json.dumps(line), flush=True)
        del q, k, v, o, lse, ws
        torch.cuda.empty_cache()
    del flush


# ------------------------------------------------------------ packed sequences

def varlen_workloads():
    """Packed variable-length training batches: sequence lengths drawn
    (seeded) uniformly from a range until the token budget is filled."""
    return [
        dict(name="packed causal H=16 d=128, 32768 tokens, lengths uniform in [256, 4096]",
             tokens=32768, lo=256, hi=4096, H=16, Hkv=16, d=128, causal=True, seed=6001),
        dict(name="packed causal GQA Hq=32 Hkv=8 d=128, 65536 tokens, lengths uniform in [1024, 8192]",
             tokens=65536, lo=1024, hi=8192, H=32, Hkv=8, d=128, causal=True, seed=6002),
    ]


def varlen_lengths(w):
    import numpy as np
    rng = np.random.default_rng(w["seed"])
    lens, total = [], 0
    while total < w["tokens"]:
        n = int(rng.integers(w["lo"], w["hi"] + 1))
        n = min(n, w["tokens"] - total)
        lens.append(n)
        total += n
    return lens


def varlen_fwd_flops(w, lens):
    """4 d flop per visible (query, key) pair and head: the metric's count
    applied per sequence (causal: L (L + 1) / 2 pairs)."""
    pairs = sum(n * (n + 1) // 2 if w["causal"] else n * n for n in lens)
    return 4.0 * w["H"] * pairs * w["d"]


def run_varlen(args, local):
    """One JSON line per packed workload: fa_fwd_varlen, fa_bwd_varlen and both
    timed separately (L2 flushed before each call, median of the steps)."""
    import numpy as np
    import torch
    import exact_io_aware_89_b200 as fa
    from seeded_inputs import make_inputs
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    for w in varlen_workloads():
        lens = varlen_lengths(w)
        T, H, Hkv, d = sum(lens), w["H"], w["Hkv"], w["d"]
        inp = make_inputs(1, T, T, H, Hkv, d, w["seed"])
        q, k, v, do = (inp[n][0].to(dev) for n in ("q", "k", "v", "do"))
        del inp
        cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device=dev)
        mx = max(lens)
        scale = 1.0 / math.sqrt(d)
        o = torch.empty_like(q)
        lse = torch.empty((H, T), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(16, fa.fa_bwd_workspace_size(len(lens), mx, H, d)), dtype=torch.uint8,
                         device=dev)
        sp = torch.cuda.current_stream().cuda_stream
        c = int(w["causal"])

        def fwd():
            st = fa.fa_fwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  cu.data_ptr(), cu.data_ptr(), len(lens), mx, mx, T, T, H, Hkv, d, scale,
                                  c, -1, -1, sp)
            if st:
                raise fa.FAError("fa_fwd_varlen", st)

        def bwd():
            st = fa.fa_bwd_varlen(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(),
                                  do.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), cu.data_ptr(),
                                  cu.data_ptr(), len(lens), mx, mx, T, T, H, Hkv, d, scale, c, -1, -1,
                                  ws.data_ptr(), ws.numel(), sp)
            if st:
                raise fa.FAError("fa_bwd_varlen", st)

        def both():
            fwd()
            bwd()

        ms = {}
        for mode, fn in (("fwd", fwd), ("bwd", bwd), ("fwd_bwd", both)):
            for _ in range(args.warmup):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for i in range(args.steps):
                flush()
                ev[i][0].record()
                fn()
                ev[i][1].record()
            torch.cuda.synchronize()
            ms[mode] = statistics.median(a.elapsed_time(b) for a, b in ev)
        if fa.fa_get_device_status(None) != 0:
            raise RuntimeError("device status reports a timed-out wait")
        F = varlen_fwd_flops(w, lens)
        tf = {"fwd": F / ms["fwd"] / 1e9, "bwd": 2.5 * F / ms["bwd"] / 1e9,
              "fwd_bwd": 3.5 * F / ms["fwd_bwd"] / 1e9}
        line = {"varlen": w["name"], "sequences": len(lens), "tokens": T, "max_seqlen": mx,
                "H": H, "Hkv": Hkv, "d": d, "causal": w["causal"],
                "ms": {m: round(x, 4) for m, x in ms.items()},
                "tflops": {m: round(x, 1) for m, x in tf.items()},
                "pct_dense_peak": {m: round(100 * x / DENSE_PEAK_TFLOPS, 2) for m, x in tf.items()}}
        print(json.dumps(line), flush=True)
        del q, k, v, do, o, lse, dq, dk, dv, ws
        torch.cuda.empty_cache()


# ------------------------------------------------------------ block-sparse

def blocksparse_workloads():
    """Block-sparse patterns over 128 x 128 tiles at long sequence lengths:
    a band of local blocks plus global first blocks (local + global sparse
    attention), and random blocks at a fixed density (seeded)."""
    return [
        dict(name="block-sparse local (4 blocks) + global (first block) B=2 H=16 N=8192 d=128",
             B=2, N=8192, H=16, d=128, pattern="local_global", band=4, causal=False, seed=7001),
        dict(name="block-sparse random 25% of blocks B=2 H=16 N=8192 d=128",
             B=2, N=8192, H=16, d=128, pattern="random", density=0.25, causal=False, seed=7002),
    ]


def blocksparse_mask(w):
    import numpy as np
    nb = -(-w["N"] // 128)
    if w["pattern"] == "local_global":
        m = np.zeros((nb, nb), dtype=bool)
        for i in range(nb):
            m[i, max(0, i - w["band"] + 1):i + 1] = True
            m[i, 0] = True
            m[0, i] = True
        return m[None, None]
    rng = np.random.default_rng(w["seed"])
    return rng.random((1, w["H"], nb, nb)) < w["density"]


def run_blocksparse(args, local):
    """One JSON line per block-sparse workload: fa_fwd_blocksparse,
    fa_bwd_blocksparse and both, L2 flushed before every call; TFLOP/s
    counted on the computed blocks (4 d flop per (query, key) pair inside
    them, backward 2.5x), and the dense kernels on the same inputs."""
    import numpy as np
    import torch
    import exact_io_aware_89_b200 as fa
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    flush = L2Flush(dev)
    for w in blocksparse_workloads():
        B, N, H, d = w["B"], w["N"], w["H"], w["d"]
        x, _ = make_device_inputs(dict(B=B, N=N, H=H, Hkv=H, d=d, seed=w["seed"]), 0, dev)
        q, k, v, do = x["q"], x["k"], x["v"], x["do"]
        mask_np = blocksparse_mask(w)
        m = torch.from_numpy(mask_np.astype(np.uint8)).to(dev)
        o = torch.empty_like(q)
        lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        ws = torch.empty(max(16, fa.fa_bwd_workspace_size(B, N, H, d)), dtype=torch.uint8, device=dev)
        c = w["causal"]
        fns = {
            "fwd": lambda: fa.attention_forward_blocksparse(q, k, v, m, causal=c, out=o, lse=lse),
            "bwd": lambda: fa.attention_backward_blocksparse(q, k, v, o, lse, do, m, causal=c, dq=dq,
                                                             dk=dk, dv=dv, workspace=ws),
            "dense_fwd": lambda: fa.attention_forward(q, k, v, causal=c, out=o, lse=lse),
            "dense_bwd": lambda: fa.attention_backward(q, k, v, o, lse, do, causal=c, dq=dq, dk=dk,
                                                       dv=dv, workspace=ws),
        }
        ms = {}
        for mode, fn in fns.items():
            for _ in range(args.warmup):
                fn()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
            for i in range(args.steps):
                flush()
                ev[i][0].record()
                fn()
                ev[i][1].record()
            torch.cuda.synchronize()
            ms[mode] = statistics.median(a.elapsed_time(b) for a, b in ev)
        if fa.fa_get_device_status(None) != 0:
            raise RuntimeError("device status reports a timed-out wait")
        density = float(np.broadcast_to(mask_np, (B, H) + mask_np.shape[2:]).mean())
        F = 4.0 * B * H * N * N * d * density
        line = {"blocksparse": w["name"], "block_density": round(density, 4),
                "ms": {k2: round(x2, 4) for k2, x2 in ms.items()},
                "tflops_on_computed_blocks": {"fwd": round(F / ms["fwd"] / 1e9, 1),
                                              "bwd": round(2.5 * F / ms["bwd"] / 1e9, 1)},
                "speedup_vs_dense": {"fwd": round(ms["dense_fwd"] / ms["fwd"], 2),
                                     "bwd": round(ms["dense_bwd"] / ms["bwd"], 2)}}
        print(json.dumps(line), flush=True)
        del q, k, v, do, o, lse, dq, dk, dv, ws, m
        torch.cuda.empty_cache()


def run_ring(args, world, rank, local):
    """Ring (context-parallel) attention on the long wide workload: the one
    sequence split into equal slices, fwd+bwd of the whole sequence per step.
    Under torchrun (N ranks, NCCL) each rank holds one slice and the slices
    travel between GPUs (strong scaling; time = max over ranks); on one GPU,
    --ring R emulates R ranks (each with its own buffers, the exchange a device
    copy), which measures what the split itself costs next to the plain call.
    One JSON line (rank 0)."""
    import torch
    import exact_io_aware_89_b200 as fa
    from exact_io_aware_89_b200 import ring
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    w = WORKLOADS["wide"]
    R = world if world > 1 else args.ring
    layout = args.ring_layout
    n_chunks = R if layout == "contiguous" else 2 * R
    if w["N"] % n_chunks:
        raise SystemExit("the sequence does not split into %d equal chunks" % n_chunks)
    c = w["N"] // n_chunks
    n = w["N"] // R
    x, _ = make_device_inputs(w, 0, dev)  # the same sequence on every rank; each takes its rows
    sl = lambda t, r: torch.cat([t[:, i * c:(i + 1) * c] for i in ring.rank_chunks(r, R, layout)],
                                dim=1).contiguous()
    causal = w["causal"]
    flush = L2Flush(dev)
    if world > 1:
        q, k, v, do = (sl(x[name], rank) for name in ("q", "k", "v", "do"))

        def step():
            o, lse = ring.ring_attention_forward(q, k, v, causal=causal, layout=layout)
            ring.ring_attention_backward(q, k, v, o, lse, do, causal=causal, layout=layout)
    else:
        qs, ks, vs, dos = ([sl(x[name], r) for r in range(R)] for name in ("q", "k", "v", "do"))
        timers = []

        def step(timed=False):
            tf, tb = (RankStepTimer(R), RankStepTimer(R)) if timed else (None, None)
            os_, lses = ring.local_ring_forward(qs, ks, vs, causal=causal, layout=layout, timer=tf)
            ring.local_ring_backward(qs, ks, vs, os_, lses, dos, causal=causal, layout=layout, timer=tb)
            if timed:
                timers.append((tf, tb))
    del x
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    barrier(world)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        ev[i][0].record()
        step()
        ev[i][1].record()
    torch.cuda.synchronize()
    barrier(world)
    if fa.fa_get_device_status(None) != 0:
        raise RuntimeError("device status reports a timed-out wait")
    t_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ev), world)
    crit = None
    if world == 1:
        # a second set of steps with events around every emulated rank's work
        # at every ring step (kept apart, so the run above times the plain calls)
        for _ in range(args.steps):
            flush()
            step(timed=True)
        torch.cuda.synchronize()
        crit = sum(tf.critical_path_ms() + tb.critical_path_ms() for tf, tb in timers) / args.steps
    F = fwd_flops(w)
    if rank == 0:
        line = {"ring": w["name"], "ranks": R, "layout": layout, "emulated_on_one_gpu": world == 1,
                "scaling": "strong (one sequence split over the ranks)",
                "ms_per_step": round(t_ms / args.steps, 4),
                "fwd_bwd_tflops": round(3.5 * F * args.steps / (t_ms * 1e-3) / 1e12, 2),
                "slice_rows": n}
        if crit is not None:
            line["critical_path_ms"] = round(crit, 4)
            line["critical_path_note"] = ("sum over ring steps of the slowest emulated rank's kernel time at "
                                          "that step, forward and backward: the step time R GPUs would "
                                          "need if every exchange hid behind the kernels (not measured on "
                                          "R GPUs)")
        print(json.dumps(line), flush=True)


class RankStepTimer:
    """CUDA events around each emulated rank's work at each ring step."""

    def __init__(self, R):
        import torch
        self.R = R
        self.ev = {(t, r): (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for t in range(R) for r in range(R)}

    def start(self, t, r):
        self.ev[(t, r)][0].record()

    def stop(self, t, r):
        self.ev[(t, r)][1].record()

    def critical_path_ms(self):
        return sum(max(a.elapsed_time(b) for a, b in (self.ev[(t, r)] for r in range(self.R)))
                   for t in range(self.R))


def run_ours(args, world, rank, local):
    import torch
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    peaks = load_peaks()
    w = WORKLOADS[args.workload]
    res = time_gpu(w, args.steps, args.warmup, world, rank, dev)
    F = fwd_flops(w)
    value = job_throughput(3.5 * F, args.steps, sum(res["step_ms"]), world)
    fwd_tf = job_throughput(F, args.steps, sum(res["fwd_ms"]), world)
    e2e_val = job_throughput(3.5 * F, len(res["e2e_ms"]), sum(res["e2e_ms"]), world)
    dom, per = roofline(w, res, peaks)
    launches = int(sum(n for k, n in res["trace_n"].items() if k not in SPAN_KINDS))

    extra = []
    if args.extra:
        for key in ("wide", "train"):
            if key == args.workload:
                continue
            we = WORKLOADS[key]
            r2 = time_gpu(we, max(3, args.steps // 2), max(3, args.warmup), world, rank, dev,
                          with_e2e=False)
            F2 = fwd_flops(we)
            tf2 = job_throughput(3.5 * F2, len(r2["step_ms"]), sum(r2["step_ms"]), world)
            ff2 = job_throughput(F2, len(r2["fwd_ms"]), sum(r2["fwd_ms"]), world)
            d2, per2 = roofline(we, r2, peaks)
            extra.append({"workload": we["name"], "fwd_bwd_tflops": round(tf2, 2),
                          "fwd_tflops": round(ff2, 2),
                          "fwd_bwd_pct_dense_peak": round(100 * tf2 / (world * DENSE_PEAK_TFLOPS), 2),
                          "fwd_pct_dense_peak": round(100 * ff2 / (world * DENSE_PEAK_TFLOPS), 2),
                          "ms_per_step": round(statistics.mean(r2["step_ms"]), 4),
                          "dominant": d2, "kernels": per2, "clocks": r2["clocks"]})

    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        tf_c, heads, secs, threads = oracle_sample(w, budget_s=args.oracle_budget)
        total = w["B"] * w["H"]
        cpu = {"value": round(tf_c, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
               "sample": "%d of %d heads, full N, fwd+bwd, %.1f s%s" % (
                   heads, total, secs,
                   "; batch throughput extrapolated from the sampled heads" if heads < total else "")}
    dk = per.get(dom, {}) if dom else {}
    traffic, traffic_profile = ncu_traffic(args.workload, dom)
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(statistics.mean(res["step_ms"]), 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1), bf16)",
        "config": {"workload": w["name"], "B": w["B"], "H": w["H"], "N": w["N"], "d": w["d"],
                   "causal": w["causal"], "global_batch": w["B"] * world,
                   "parallelism": "dp%d" % world,
                   "l2": "flushed between steps outside the timed events (256 MiB write, then a "
                         "256 MiB read so the evicted lines are clean)"},
        "fwd_tflops": round(fwd_tf, 3),
        "fwd_bwd_pct_dense_peak": round(100 * value / (world * DENSE_PEAK_TFLOPS), 2),
        "fwd_pct_dense_peak": round(100 * fwd_tf / (world * DENSE_PEAK_TFLOPS), 2),
        "roofline": {"kernel": dom, "bound": dk.get("bound"), "achieved": dk.get("achieved"),
                     "peak": dk.get("peak"), "unit": dk.get("unit"), "frac": dk.get("frac"),
                     "traffic": traffic, "traffic_profile": traffic_profile,
                     "peak_source": "%s, %s" % (peaks["source"], dk.get("peak_kind"))},
        "kernels": per,
        "gpu_launches": launches,
        "e2e": {"value": round(e2e_val, 3), "unit": "TFLOP/s", "h2d_bytes_per_step": res["h2d"],
                "d2h_bytes_per_step": res["d2h"]},
        "clocks": res["clocks"],
        "cpu_baseline": cpu,
        "extra": extra,
    }
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="wide")
    ap.add_argument("--no-extra", dest="extra", action="store_false")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--oracle-budget", type=float, default=15.0,
                    help="seconds of oracle time for the CPU baseline sample")
    ap.add_argument("--decode", action="store_true",
                    help="instead of the benchmark line: the KV-cache decoding workloads through "
                         "fa_fwd_splitkv, one JSON line each")
    ap.add_argument("--blocksparse", action="store_true",
                    help="instead of the benchmark line: block-sparse workloads through "
                         "fa_fwd_blocksparse / fa_bwd_blocksparse, one JSON line each")
    ap.add_argument("--varlen", action="store_true",
                    help="instead of the benchmark line: packed variable-length workloads through "
                         "fa_fwd_varlen / fa_bwd_varlen, one JSON line each")
    ap.add_argument("--decode-case", type=int, default=None,
                    help="with --decode: only this workload (index into the list)")
    ap.add_argument("--dtype", choices=["bf16", "fp16"], default="bf16",
                    help="with --sweep: the element type of the inputs (bf16 or fp16 entry points)")
    ap.add_argument("--sweep-filter", default=None,
                    help="with --sweep: only workloads whose name contains this text")
    ap.add_argument("--ring", type=int, default=0,
                    help="instead of the benchmark line: ring (context-parallel) attention on the long wide "
                         "workload, over the torchrun ranks, or with N emulated ranks on one GPU")
    ap.add_argument("--ring-layout", choices=["contiguous", "zigzag"], default="zigzag",
                    help="with --ring: each rank's chunk of the sequence ('contiguous') or two chunks, one "
                         "from each end ('zigzag', the same causal work on every rank)")
    ap.add_argument("--sweep", action="store_true",
                    help="instead of the benchmark line: the sequence-length sweep and the GQA/window "
                         "and d=256 workloads, fwd / bwd / fwd+bwd timed separately, one JSON line each")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    if args.ring:
        if world > 1:
            import datetime
            import torch
            import torch.distributed as dist
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        try:
            run_ring(args, world, rank, local)
        finally:
            if world > 1:
                import torch.distributed as dist
                dist.destroy_process_group()
        return
    if args.sweep or args.decode or args.varlen or args.blocksparse:
        if world > 1:
            raise SystemExit("--sweep, --decode, --varlen and --blocksparse run on one GPU")
        fn = (run_sweep if args.sweep else run_decode if args.decode else
              run_varlen if args.varlen else run_blocksparse)
        fn(args, local)
        return
    if args.impl == "reference":
        run_reference(args, world, rank)  # rank 0 alone; no process group
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
