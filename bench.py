"""Benchmark of the selective scan (S6) forward on B200: achieved HBM GB/s, fraction of the
measured HBM peak, and state-updates/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload m130] [--impl ours|reference]

One step is one call of selective_scan_fwd over the whole workload (every launch the call
makes), with inputs resident in HBM; L2 is flushed (a 256 MiB write) before every timed step,
outside the step's events.  value = algorithmic bytes of the step (u, delta_raw, z, B, C read
once, out written once, parameters and last_state) / device time, summed over ranks.  Under
torchrun every rank runs the whole workload on its own GPU (independent problems, weak
scaling, no collective on the data path); the step time is the max over ranks.

The JSON line also carries: roofline (the HBM roofline of the scan pipeline: algorithmic bytes
over the pipeline's event time against the measured copy bandwidth; beside it the FP32, MUFU and
instruction-issue fractions against ceilings measured live by the probes of libss_probe.so; DRAM
traffic and warp instructions per step come from the committed ncu record while the kernel
sources match it), e2e (the C entry point selective_scan_fwd_host from pinned host buffers to
pinned host buffers, copies included), clocks (NVML during the timed region), gpu_launches and
cpu_baseline (the oracle on the host cores).

--impl reference runs the fp64 CPU oracle on a bounded sample of the same workload on the host
cores (there is no other implementation of this path to compare with).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from selective_state_space_13_b200 import workloads as wl  # noqa: E402

METRIC = "selective-scan achieved HBM GB/s and % of peak; state-updates/s at 1 B200"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "long"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 7700.0  # the specification figure, stated beside the measured peak
FLUSH_BYTES = 256 << 20
# FP32 operations of one state update in the form the kernels compute: the power-chain multiply
# that gives exp(Delta*A[d,n]), the state multiply-add and the readout multiply-add
FP32_OPS_PER_UPDATE = 3
# MUFU operations per step and channel: ex2 and lg2 of the softplus, ex2 of exp(Delta*A[d,0]),
# the reciprocal of the normalisation, and tanh of the silu gate (with z)
MUFU_PER_STEP = 4
MUFU_PER_STEP_GATE = 5
CPU_SECONDS = 10.0  # CPU work the cpu_baseline sample runs (repeating a small sample)
# workloads whose description states that last_state is returned
RETURNS_LAST_STATE = {"tiny", "long"}


# ----------------------------------------------------------------------------- helpers (CPU-testable)

def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def max_over_ranks(value: float, world: int, device=None) -> float:
    """Max of a float over all ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value: float, world: int, device=None) -> float:
    """Sum of a float over all ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            pk = json.load(fh)
        return float(pk["hbm_gbs"]), "measured (MEASURED_PEAKS.json: STREAM-style copy)", pk
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback (6.65 TB/s earlier pool measurement)", {}


def code_without_comments(text: str) -> str:
    """C/C++/CUDA source with comments, trailing spaces and blank lines removed (string and
    character literals kept), so that edits to comments alone keep the digest."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = [ln.rstrip() for ln in "".join(out).splitlines()]
    return "\n".join(ln for ln in lines if ln)


def kernel_source_digest() -> str:
    """Digest of the CUDA library's code (sources and headers, comments ignored): the ncu
    record in profiles/traffic.json applies only while it matches."""
    from selective_state_space_13_b200 import build as b
    h = hashlib.sha256()
    for f in b.SOURCES + b.HEADERS:
        with open(f, encoding="utf-8") as fh:
            h.update(os.path.basename(f).encode())
            h.update(code_without_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def recorded_counters(workload: str) -> dict:
    """The committed ncu record of the scan pipeline for this workload (DRAM bytes and warp
    instructions per step), or {} when the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as fh:
            rec = json.load(fh).get(workload)
    except (OSError, ValueError):
        return {}
    if not rec or rec.get("source_digest") != kernel_source_digest():
        return {}
    return rec


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, index: int, period_s: float = 0.0005):
        self.index, self.period = index, period_s
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:  # noqa: BLE001 - no NVML: clocks reported as null
            self.ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            # the sampler thread needs the interpreter lock every period: shorten the switch
            # interval while it runs (the timed region of a small workload lasts milliseconds),
            # and return once it is sampling
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
            t0 = time.time()
            while not self.samples and time.time() - t0 < 1.0:
                time.sleep(1e-4)
            self._first = len(self.samples)

    def stop(self):
        if self._thr:
            self._stop.set()
            self._thr.join()
            sys.setswitchinterval(self._switch)

    def report(self):
        if not self.ok:
            return None
        # the sample taken before the first step was enqueued is not part of the region
        during = self.samples[getattr(self, "_first", 0):] or self.samples
        return {"sm_mhz": statistics.median(during) if during else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(during), "period_ms": self.period * 1e3,
                "source": "NVML during the timed region"}


def workload_of(args) -> wl.Workload:
    w = wl.WORKLOADS[args.workload]
    if args.seqlen:
        if w.H:
            raise SystemExit("--seqlen does not apply to image workloads")
        w = wl.variant(w.name, seqlen=args.seqlen)
    if args.conv or args.delta_int8:
        w = wl.variant(w.name, seqlen=w.seqlen, conv=args.conv, delta_int8=args.delta_int8)
    return w


def describe(w: wl.Workload) -> str:
    text = wl.DESCRIPTIONS[w.name]
    if w.conv:
        text += ", causal depthwise conv1d (%d taps) + SiLU fused before the scan" % w.conv
    if w.delta_int8:
        text += ", int8 Delta codes with per-channel scales"
    return text


def workload_bytes(w: wl.Workload) -> int:
    return w.algorithmic_bytes(with_last_state=w.name in RETURNS_LAST_STATE)


def config_of(w: wl.Workload, args, world: int) -> dict:
    """The workload description both arms print (identical keys and values)."""
    return {"workload": describe(w) + (" (seqlen overridden to %d)" % w.seqlen if args.seqlen else ""),
            "name": w.name, "batch": w.batch, "seqlen": w.seqlen, "dim": w.dim,
            "dstate": w.dstate, "directions": w.K, "gate": w.gate,
            "returns_last_state": w.name in RETURNS_LAST_STATE, "conv": w.conv,
            "delta_int8": w.delta_int8,
            "parallelism": ("1 GPU" if world <= 1 else
                            "%d ranks, one workload each" % world if args.shard == "replica" else
                            "%d ranks, one workload split by %s" % (world, args.shard)),
            "l2": "flushed (256 MiB write) before every timed step"}


def probe_ceilings() -> dict:
    """FP32, MUFU and issue ceilings measured on this GPU by the probes of libss_probe.so."""
    import ctypes
    from selective_state_space_13_b200 import build as b
    lib = ctypes.CDLL(b.build_probe())
    out = {}
    for name in ("ffma2", "ffma", "ex2", "issue"):
        fn = getattr(lib, "ss_probe_" + name)
        fn.restype = ctypes.c_int
        fn.argtypes = [ctypes.POINTER(ctypes.c_double)]
        v = ctypes.c_double(0.0)
        if fn(ctypes.byref(v)) != 0:
            raise RuntimeError("probe %s failed" % name)
        out[name] = v.value
    return out


# ----------------------------------------------------------------------------- CPU baseline

def oracle_sample_plan(w: wl.Workload, target_updates: float):
    """Channels of the workload (all batch rows, all steps) whose updates add up to about
    target_updates; the oracle runs on those."""
    per_channel = w.K * w.batch * w.seqlen * w.dstate
    nch = max(1, min(w.dim, int(target_updates // per_channel)))
    return list(range(nch))


def time_oracle(inp, channels, threads):
    import oracle
    w = inp["workload"]
    f = wl.inputs_f64(inp, channels=channels)
    t0 = time.perf_counter()
    oracle.selective_scan(f["u"], f["delta"], f["A"], f["B"], f["C"], Dskip=f["Dskip"], z=f["z"],
                          delta_bias=f["delta_bias"], softplus=w.softplus, dirs=w.dirs, H=w.H,
                          W=w.W, threads=threads, conv_weight=f["conv_weight"],
                          conv_bias=f["conv_bias"], delta_scale=f["delta_scale"])
    return time.perf_counter() - t0


def sample_fraction(w: wl.Workload, channels) -> float:
    return len(channels) / float(w.dim)


# ----------------------------------------------------------------------------- reference arm

def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    w = workload_of(args)
    inp = wl.make_inputs(w)
    threads = oracle.max_threads()
    # each step: the oracle on a channel sample worth about 2e7 state updates
    channels = oracle_sample_plan(w, 2e7)
    frac = sample_fraction(w, channels)
    for _ in range(args.warmup):
        time_oracle(inp, channels, threads)
    times = [time_oracle(inp, channels, threads) for _ in range(args.steps)]
    step_s = sum(times) / len(times)
    nbytes = workload_bytes(w) * frac
    value = nbytes / step_s / 1e9
    sample = "%d of %d channels (all batch rows, all steps, all directions) per step" % (
        len(channels), w.dim)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic (seeded, %s)" % describe(w),
            "config": config_of(w, args, world),
            "updates_per_s": w.updates() * frac / step_s,
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    from selective_state_space_13_b200 import scan

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)
    w_full = workload_of(args)
    w = w_full
    inp = wl.make_inputs(w_full)
    shard_info = None
    if args.shard != "replica" and world > 1:
        # this rank scans its slice of the one workload (batch rows or channels); the slices
        # are independent, so no data crosses between ranks
        from selective_state_space_13_b200 import shard
        try:
            axis, lo, hi, w = shard.plan(w_full, world, rank,
                                         None if args.shard == "auto" else args.shard)
        except ValueError as e:  # raised on every rank alike: all stop together
            raise SystemExit("--shard: %s; use fewer ranks" % e)
        inp = shard.shard_inputs(inp, axis, lo, hi)
        shard_info = {"axis": axis, "lo": lo, "hi": hi}
    t = wl.to_device(inp, device)
    want_last = w.name in RETURNS_LAST_STATE
    out = torch.empty((w.batch, w.seqlen, w.dim), dtype=t["u"].dtype, device=device)
    last = torch.empty((w.K, w.batch, w.dim, w.dstate), dtype=torch.float32, device=device) \
        if want_last else None
    stream = torch.cuda.current_stream(device)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device)

    def call(events=None):
        scan.selective_scan_fwd(t["u"], t["delta"], t["A"], t["B"], t["C"], D=t["D"], z=t["z"],
                                delta_bias=t["delta_bias"], softplus=w.softplus, dirs=w.dirs,
                                H=w.H, W=w.W, out=out, last_state=last, segments=args.segments,
                                flags=args.flags, events=events, conv_weight=t["conv_weight"],
                                conv_bias=t["conv_bias"], delta_scale=t["delta_scale"])

    # plan facts for the report
    shape = scan.make_shape(w.batch, w.seqlen, w.dim, w.dstate,
                            scan.SS_BF16 if w.dtype == wl.BF16 else scan.SS_F32)
    dmap = scan.make_dirmap(w.dirs, w.H, w.W)
    ws_bytes = scan.selective_scan_workspace_size(shape, dmap, scan.make_opts(args.segments,
                                                                              args.flags))
    launches_per_step = 1 + (1 if w.K > 1 else 0)
    # a second launch (segment aggregates) exists exactly when the plan has carries
    seg_probe = scan.selective_scan_workspace_size(shape, None, scan.make_opts(args.segments,
                                                                               args.flags))
    if seg_probe > 0:
        launches_per_step += 1

    kb = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sb = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    se = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in kb + ke:
        e.record(stream)  # create the CUDA events the library records into
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        call()
    torch.cuda.synchronize(device)
    if scan.selective_scan_device_status(clear=True) != scan.SS_OK:
        raise RuntimeError("device timeout during warm-up")

    sampler = ClockSampler(torch.cuda.current_device())
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    for i in range(args.steps):
        flush.zero_()
        sb[i].record(stream)
        call(events=(kb[i], ke[i]))
        se[i].record(stream)
    torch.cuda.synchronize(device)
    if world > 1:
        dist.barrier()
    sampler.stop()
    step_ms = sum(sb[i].elapsed_time(se[i]) for i in range(args.steps)) / args.steps
    kern_ms = sum(kb[i].elapsed_time(ke[i]) for i in range(args.steps)) / args.steps
    step_ms = max_over_ranks(step_ms, world, device)
    kern_ms = max_over_ranks(kern_ms, world, device)
    if scan.selective_scan_device_status(clear=True) != scan.SS_OK:
        raise RuntimeError("device timeout during the timed region")

    nbytes = workload_bytes(w)
    # the whole job's bytes and updates: every rank's own (a replica or a slice), summed
    job_bytes = sum_over_ranks(float(nbytes), world, device)
    job_updates = sum_over_ranks(float(w.updates()), world, device)
    value = job_bytes / (step_ms * 1e-3) / 1e9
    updates_s = job_updates / (step_ms * 1e-3)
    peak, peak_src, peaks = load_peaks()
    achieved = nbytes / (kern_ms * 1e-3) / 1e9
    # the FP32, MUFU and issue ceilings of this GPU, measured now (libss_probe.so)
    ceil = probe_ceilings()

    # ---- end to end: pinned host inputs -> device, scan, out -> pinned host, every step
    e2e = None
    if not args.no_e2e:
        host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in t.items()}
        h2d_keys = ["u", "delta", "B", "C"] + (["z"] if t["z"] is not None else [])
        h2d_bytes = sum(host[k].numel() * host[k].element_size() for k in h2d_keys)
        out_host = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
        d2h_bytes = out_host.numel() * out_host.element_size()
        if last is not None:
            last_host = torch.empty(last.shape, dtype=last.dtype, pin_memory=True)
            d2h_bytes += last_host.numel() * last_host.element_size()
        n_e2e = max(1, min(args.steps, 20))
        ea = [torch.cuda.Event(enable_timing=True) for _ in range(n_e2e)]
        eb = [torch.cuda.Event(enable_timing=True) for _ in range(n_e2e)]

        def e2e_step():
            # the C entry point selective_scan_fwd_host: pinned host inputs in, host outputs
            # back, the copies and the scans of successive pieces pipelined by the library
            scan.selective_scan_fwd_host(
                host["u"], host["delta"], t["A"], host["B"], host["C"], D=t["D"], z=host["z"],
                delta_bias=t["delta_bias"], softplus=w.softplus, dirs=w.dirs, H=w.H, W=w.W,
                out=out_host, last_state=last_host if last is not None else None,
                flags=args.flags, conv_weight=t["conv_weight"], conv_bias=t["conv_bias"],
                delta_scale=t["delta_scale"], chunks=args.e2e_pieces)

        e2e_step()
        torch.cuda.synchronize(device)
        for i in range(n_e2e):
            ea[i].record(stream)
            e2e_step()
            eb[i].record(stream)
        torch.cuda.synchronize(device)
        e2e_ms = sum(ea[i].elapsed_time(eb[i]) for i in range(n_e2e)) / n_e2e
        e2e_ms = max_over_ranks(e2e_ms, world, device)
        e2e = {"value": job_bytes / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes,
               "ms_per_step": e2e_ms, "steps": n_e2e,
               "path": "C entry point selective_scan_fwd_host: pinned host inputs -> device, "
                       "scan, device -> pinned host, %d pieces pipelined on the library's three "
                       "streams" % args.e2e_pieces}

    # ---- CPU baseline: the oracle on a bounded sample (rank 0 at N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        threads = oracle.max_threads()
        channels = oracle_sample_plan(w, args.cpu_updates)
        # repeat the sample until about CPU_SECONDS of CPU work have run (a small workload is
        # sampled whole and then repeated), and report the mean pass
        runs = []
        while not runs or (sum(runs) < CPU_SECONDS and len(runs) < 30):
            runs.append(time_oracle(inp, channels, threads))
        secs = sum(runs) / len(runs)
        frac = sample_fraction(w, channels)
        cpu = {"value": workload_bytes(w) * frac / secs / 1e9, "unit": UNIT, "cores": threads,
               "kind": "oracle", "seconds": secs, "repeats": len(runs),
               "updates_per_s": w.updates() * frac / secs,
               "sample": "%d of %d channels, all batch rows, all %d steps, all %d directions "
                         "(%.3g state updates), timed %d times (%.1f s of CPU work)"
                         % (len(channels), w.dim, w.seqlen, w.K, w.updates() * frac, len(runs),
                            sum(runs))}
        if threads > 1:
            # the same oracle on one core, on a sample sized for a few seconds
            ch1 = channels[:max(1, len(channels) * 2 // threads)]
            s1 = time_oracle(inp, ch1, 1)
            f1 = sample_fraction(w, ch1)
            cpu["single_core"] = {"value": workload_bytes(w) * f1 / s1 / 1e9, "unit": UNIT,
                                  "updates_per_s": w.updates() * f1 / s1, "seconds": s1,
                                  "sample": "%d channels, all batch rows and steps" % len(ch1)}

    counters = {} if args.seqlen else recorded_counters(
        w.name + ("_conv%d" % w.conv if w.conv else "") + ("_int8" if w.delta_int8 else ""))
    traffic = counters.get("dram_bytes_per_launch")
    # beside the HBM roofline: the scan pipeline's FP32 work (3 operations per state update),
    # MUFU work (per step and channel) and, from the committed ncu record, its warp instructions,
    # each against the ceiling the probes measured on this GPU just now
    fp32_ach = FP32_OPS_PER_UPDATE * w.updates() / (kern_ms * 1e-3)
    mufu_ops = (MUFU_PER_STEP_GATE if w.gate and w.K == 1 else MUFU_PER_STEP) * w.updates() / w.dstate
    mufu_ach = mufu_ops / (kern_ms * 1e-3)
    alu = {"fp32": {"achieved": fp32_ach / 1e12, "peak": ceil["ffma2"] / 1e12,
                    "unit": "T fp32 lane-ops/s", "frac": fp32_ach / ceil["ffma2"],
                    "ops_per_update": FP32_OPS_PER_UPDATE,
                    "peak_source": "measured: packed fma.rn.f32x2 probe (scalar fma: %.1f T/s)"
                                   % (ceil["ffma"] / 1e12)},
           "mufu": {"achieved": mufu_ach / 1e12, "peak": ceil["ex2"] / 1e12,
                    "unit": "T MUFU ops/s", "frac": mufu_ach / ceil["ex2"],
                    "ops_per_step_and_channel": mufu_ops / (w.updates() / w.dstate),
                    "peak_source": "measured: ex2.approx probe"}}
    if counters.get("warp_instructions_per_launch"):
        issue_ach = counters["warp_instructions_per_launch"] / (kern_ms * 1e-3)
        alu["issue"] = {"achieved": issue_ach / 1e12, "peak": ceil["issue"] / 1e12,
                        "unit": "T warp-instructions/s", "frac": issue_ach / ceil["issue"],
                        "warp_instructions_per_launch": counters["warp_instructions_per_launch"],
                        "peak_source": "measured: fp32 + integer issue probe; instructions from "
                                       "ncu smsp__inst_executed.sum (profiles/traffic.json)"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True,
        "scaling": "strong" if shard_info else "weak", "vs_baseline": None,
        "dtype": "bf16" if w.dtype == wl.BF16 else "f32",
        "data": "synthetic (seeded N(0,1) inputs, A=-(n+1), log-uniform Delta bias)",
        "config": config_of(w_full, args, world),
        "plan": {"segments": args.segments or "auto", "workspace_bytes": ws_bytes,
                 "shard": shard_info or args.shard},
        "hbm_frac_of_peak": value / world / peak,
        "updates_per_s": updates_s,
        "roofline": {"bound": "hbm",
                     "kernel": "scan pipeline: the segment-aggregate launch (if any) and the scan "
                               "launch, timed with CUDA events the library records around them "
                               "(the direction merge excluded)",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": traffic, "peak_source": peak_src,
                     "algorithmic_bytes_per_launch": nbytes, "kernel_ms": kern_ms,
                     "nominal": {"peak": NOMINAL_HBM_GBS, "frac": achieved / NOMINAL_HBM_GBS,
                                 "source": "B200 HBM3e specification (HGX)"},
                     "alu": alu},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": sampler.report(),
        "e2e": e2e,
        "cpu_baseline": cpu,
    }
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def parse(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(wl.WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--segments", type=int, default=0, help="0 = the library's choice")
    ap.add_argument("--shard", choices=["replica", "batch", "channels", "auto"], default="replica",
                    help="with several ranks: 'replica' = every rank scans the whole workload "
                         "(weak scaling); 'batch' / 'channels' / 'auto' = every rank scans its "
                         "slice of one workload (strong scaling, no collective on the data path)")
    ap.add_argument("--flags", type=int, default=0, help="SS_FLAG_* bits (1 = generic A)")
    ap.add_argument("--seqlen", type=int, default=0,
                    help="override the workload's sequence length (smaller cases for profiling)")
    ap.add_argument("--conv", type=int, default=0,
                    help="taps of a causal depthwise conv1d + SiLU fused before the scan (0 = none)")
    ap.add_argument("--delta-int8", action="store_true",
                    help="Delta as int8 codes with one scale per channel")
    ap.add_argument("--e2e-pieces", type=int, default=8,
                    help="pieces of the end-to-end host-buffer pipeline")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-updates", type=float, default=4e9,
                    help="state updates the CPU-baseline sample covers")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    return args


def main(argv=None):
    args = parse(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
