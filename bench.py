#!/usr/bin/env python
"""Benchmark of the selective-scan forward (libselscan) on B200.

One step = one ss_fwd over the whole workload (every (b, d, l, n) state
update).  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference]

Metric: state updates per second, B*D*L*N / t.  Timing: CUDA events on the
launching stream around each ss_fwd call; L2 is flushed (a write larger than
L2) before every timed step, outside the events.  ``value`` sums all ranks'
updates over the slowest rank's time (ranks run independent problems: weak
scaling, no data-path collective).  ``e2e`` is the same metric through the
host-buffer entry point ss_fwd_hostio: pinned host inputs copied in, the
forward, y copied back, per step.  The roofline of the scan kernel is its
exp count against the SFU rate (16 ex2 per clock per SM at the maximum SM
clock); its HBM side (compulsory bytes over measured copy bandwidth) is
reported beside it.  ``per_config`` adds, in the same line, the forward of
every other configuration at full size (device time with L2 flushed per step,
fewer steps each, clocks sampled over the warm-ups and timed steps) and its
backward (ss_bwd, all gradients, 3 timed steps).  ``train_step`` (headline
layer and each configuration) times forward + backward both ways: ss_fwd +
ss_bwd, and ss_fwd_ckpt + ss_bwd_ckpt (the forward keeps the checkpoints the
backward would otherwise recompute).
``--impl reference`` times the fp64 CPU oracle on the host cores instead (a
bounded sample of rows per step).
"""
import argparse
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_41_b200 import gen, selscan, workloads as W  # noqa: E402

DEFAULT_WORKLOAD = W.MAMBA130M
METRIC = "selective-scan state-updates/s (B·D·L·N) & HBM GB/s vs roofline, 1×B200"
SFU_EX2_PER_CLK_PER_SM = 16  # MUFU.EX2 results per clock per SM (compute capability 10.0)
FALLBACK_HBM_GBS = 6650.0
FALLBACK_SM_MHZ = 1965.0

# NVML clock-event reason bits
_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
            0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "sm_max_mhz": FALLBACK_SM_MHZ}, "fallback"


def kernel_source_digest() -> str:
    """sha256 of the kernel source (csrc/ss_fwd_kernel.cuh) with its // comments
    and blank lines removed: identifies the kernel code a recorded ncu traffic
    figure belongs to (editing a comment does not change the kernel)."""
    import hashlib
    import re
    path = os.path.join(ROOT, "selective_state_space_41_b200", "csrc", "ss_fwd_kernel.cuh")
    with open(path, encoding="utf-8") as fh:
        lines = [re.sub(r"//.*$", "", line).rstrip() for line in fh.read().splitlines()]
    code = "\n".join(line for line in lines if line.strip())
    return hashlib.sha256(code.encode()).hexdigest()


def recorded_traffic(workload: str, shape):
    """DRAM bytes per launch of the scan kernel from the committed ncu record
    (profiles/traffic.json), or None if there is none for this workload and
    launch shape, or the kernel source changed since it was taken."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f).get(workload)
    except (OSError, ValueError):
        return None
    if (not rec or rec.get("kernel_sha256") != kernel_source_digest()
            or list(rec.get("launch_shape", [])) != list(shape)):
        return None
    return rec.get("dram_bytes_per_launch")


def algorithmic_bytes(w: W.Workload) -> int:
    """Compulsory HBM bytes of one forward: u, delta, (z) read and y written
    once per (b, d, l); B and C read once per (b, n, l); A, D, bias per
    channel; last_state written once per (b, d, n)."""
    ein = 2 if w.dtype == torch.bfloat16 else 4
    eout = 2 if (w.out_dtype or w.dtype) == torch.bfloat16 else 4
    bdl = w.batch * w.dim * w.seqlen
    per_bdl = (2 + (1 if w.has_z else 0)) * ein + eout
    bc = 2 * w.batch * w.dstate * w.seqlen * ein
    params = w.dim * w.dstate * 4 + w.dim * 4 * ((w.D_kind != "none") + (w.bias_kind != "none"))
    last = w.batch * w.dim * w.dstate * 4 if w.return_last_state else 0
    return bdl * per_bdl + bc + params + last


class ClockSampler:
    """Polls NVML (SM clock, max clock, clock-event reasons) in a thread."""

    def __init__(self, index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples, self.reasons = [], 0
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # no NVML: report no clocks
            self.nv = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(nv.nvmlDeviceGetCurrentClocksEventReasons(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if self.nv is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        names = [n for bit, n in _REASONS.items() if self.reasons & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(w: W.Workload, rank: int) -> W.Workload:
    """Each rank runs its own problem of the same shape (its own seed)."""
    return W.with_shape(w, seed=w.seed + 1000003 * rank)


def cpu_model() -> str:
    """The host CPU's model name (Linux /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cpu_oracle_one_core(w: W.Workload, inp: dict, target_s: float = 2.0):
    """The oracle on one thread over the first rows of the workload (about
    ``target_s`` seconds).  Returns (updates/s, description)."""
    import oracle

    def run(nrows):
        sl = lambda t: None if t is None else t[0:1, :nrows]  # noqa: E731
        pd = lambda t: None if t is None else t[:nrows]  # noqa: E731
        t0 = time.perf_counter()
        oracle.selective_scan(sl(inp["u"]), sl(inp["delta"]), inp["A"][:nrows], inp["B"][0:1], inp["C"][0:1],
                              D=pd(inp["D"]), z=sl(inp["z"]), delta_bias=pd(inp["delta_bias"]),
                              delta_softplus=w.delta_softplus, return_last_state=w.return_last_state, nthreads=1)
        return time.perf_counter() - t0

    per_row = run(1)
    rows = int(max(1, min(w.dim, target_s / max(per_row, 1e-9))))
    dt = run(rows)
    updates = rows * w.seqlen * w.dstate
    return updates / dt, f"the first {rows} (b, d) rows, all {w.seqlen} steps, N={w.dstate}, 1 thread"


def cpu_oracle_sample(w: W.Workload, inp: dict = None, target_s: float = 10.0):
    """The oracle, as it stands, on all host cores over a bounded sample of the
    same workload (about ``target_s`` seconds): the whole workload, repeated,
    when one pass is shorter than that, else its first rows in (b, d) order,
    every step.  Returns (updates/s, threads, description)."""
    import oracle
    if inp is None:
        inp = W.make_inputs(w)
    threads = oracle.max_threads()
    total = w.batch * w.dim

    def run_rows(nrows):
        t0 = time.perf_counter()
        done, b = 0, 0
        while done < nrows:
            take = min(w.dim, nrows - done)
            sl = lambda t: None if t is None else t[b:b + 1, :take]  # noqa: E731
            pd = lambda t: None if t is None else t[:take]  # noqa: E731
            oracle.selective_scan(sl(inp["u"]), sl(inp["delta"]), inp["A"][:take],
                                  inp["B"][b:b + 1], inp["C"][b:b + 1], D=pd(inp["D"]),
                                  z=sl(inp["z"]), delta_bias=pd(inp["delta_bias"]),
                                  delta_softplus=w.delta_softplus,
                                  return_last_state=w.return_last_state, nthreads=threads)
            done += take
            b += 1
        return time.perf_counter() - t0

    probe = min(total, 2 * threads)
    per_row = run_rows(probe) / probe
    want = target_s / max(per_row, 1e-12)
    if want >= total:
        # one whole pass, then as many more as fill target_s at its measured rate
        # (the probe's few rows overstate the per-row time)
        dt = run_rows(total)
        reps = 1 + int(min(49, max(0, round((target_s - dt) / max(dt, 1e-9)))))
        dt += sum(run_rows(total) for _ in range(reps - 1))
        updates = reps * w.updates
        desc = (f"the whole workload ({total} rows x {w.seqlen} steps x N={w.dstate}), "
                f"{reps} pass(es): {updates:.3e} updates in {dt:.2f} s")
    else:
        rows = max(1, int(want))
        dt = run_rows(rows)
        updates = rows * w.seqlen * w.dstate
        desc = (f"the first {rows} of {total} (b, d) rows, all {w.seqlen} steps, N={w.dstate}: "
                f"{updates:.3e} updates in {dt:.2f} s")
    return updates / dt, threads, desc


def bench_reference(args, w, world, rank):
    """--impl reference: the fp64 oracle on the host cores (rank 0 only)."""
    if rank != 0:
        return None
    import oracle
    inp = W.make_inputs(W.with_shape(w, batch=1))
    threads = oracle.max_threads()
    # rows per step so that warm-up + timed steps take about a minute
    probe_rows = min(w.dim, threads)
    t0 = time.perf_counter()
    oracle.selective_scan(inp["u"][:, :probe_rows], inp["delta"][:, :probe_rows],
                          inp["A"][:probe_rows], inp["B"], inp["C"], delta_softplus=True,
                          nthreads=threads)
    per_row = (time.perf_counter() - t0) / probe_rows
    budget = 60.0 / max(1, args.steps + args.warmup)
    rows = int(max(1, min(w.dim, budget / max(per_row, 1e-9))))
    sl = lambda t: None if t is None else t[:, :rows]  # noqa: E731
    pd = lambda t: None if t is None else t[:rows]  # noqa: E731

    def step():
        oracle.selective_scan(sl(inp["u"]), sl(inp["delta"]), inp["A"][:rows], inp["B"], inp["C"],
                              D=pd(inp["D"]), z=sl(inp["z"]), delta_bias=pd(inp["delta_bias"]),
                              delta_softplus=w.delta_softplus,
                              return_last_state=w.return_last_state, nthreads=threads)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = (time.perf_counter() - t0) / max(args.steps, 1)
    updates = rows * w.seqlen * w.dstate
    value = updates / dt
    sample = (f"each step: {rows} of {w.batch * w.dim} (b, d) rows (batch entry 0), all "
              f"{w.seqlen} steps, N={w.dstate} ({updates:.3e} updates)")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": "updates/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded Philox4x32-10)",
            "config": dict(w.describe(), sample=sample),
            "cpu_baseline": {"value": value, "unit": "updates/s", "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "updates/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def bench_ours(args, w, world, rank, local):
    peaks, peak_src = measured_peaks()
    dev = torch.device("cuda", local)
    wr = rank_workload(w, rank)
    host = W.make_inputs(wr, pin=True)
    names_in = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
    d = {k: (host[k].to(dev, non_blocking=True) if host[k] is not None else None) for k in names_in}
    out_dtype = host["out_dtype"]
    y = torch.empty(host["u"].shape, dtype=out_dtype, device=dev)
    last = (torch.empty((wr.batch, wr.dim, wr.dstate), dtype=torch.float32, device=dev)
            if wr.return_last_state else None)
    ws = selscan.workspace_for(wr.batch, wr.dim, wr.seqlen, wr.dstate, wr.dtype, out_dtype,
                               device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def launch():
        selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"],
                       delta_bias=d["delta_bias"], delta_softplus=wr.delta_softplus,
                       last_state=last, stream=stream, workspace=ws)

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    # Clocks are sampled over the whole forward leg: warm-ups and timed steps.
    with ClockSampler(local, period_s=0.001) as clocks:
        for _ in range(args.warmup):
            flush.zero_()
            launch()
        torch.cuda.synchronize(dev)
        barrier(world)
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            launch()
            ends[i].record(stream)
        torch.cuda.synchronize(dev)
    barrier(world)
    kernel_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    my_ms = sum(kernel_ms) / len(kernel_ms)
    ms = max_over_ranks(my_ms, world)
    updates = w.updates * world
    value = updates / (ms * 1e-3)

    # end to end through the host-buffer entry point: pinned inputs in, y out
    host["y"] = torch.empty(y.shape, dtype=out_dtype).pin_memory()
    host["last_state"] = (torch.empty(last.shape, dtype=torch.float32).pin_memory()
                          if last is not None else None)
    dd = dict(d, y=y, last_state=last)
    h2d = sum(host[k].numel() * host[k].element_size() for k in names_in if host[k] is not None)
    d2h = host["y"].numel() * host["y"].element_size() + (
        host["last_state"].numel() * 4 if last is not None else 0)
    e2e_steps = max(1, min(args.steps, 20))
    # Pipelined over the caller's stream and two more (ss_fwd_hostio_streams):
    # each call first waits for everything already queued on the three.
    e2e_streams = [stream, torch.cuda.Stream(dev), torch.cuda.Stream(dev)]
    e2e_ws = torch.empty(3 * (ws.numel() if ws is not None else 0) + 256, dtype=torch.uint8, device=dev)

    def e2e_call():
        selscan.ss_fwd_hostio(host, dd, delta_softplus=wr.delta_softplus, workspace=e2e_ws,
                              streams=e2e_streams)
        for st in e2e_streams[1:]:
            stream.wait_stream(st)   # the step ends when every range's outputs are back

    for _ in range(2):
        e2e_call()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_call()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, world)
    barrier(world)

    # roofline of the scan kernel: exps at the SFU rate; bytes at HBM bandwidth
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    sm_max = float(peaks.get("sm_max_mhz") or FALLBACK_SM_MHZ)
    sfu_peak = SFU_EX2_PER_CLK_PER_SM * sms * sm_max * 1e6           # ex2/s
    achieved_ex2 = w.updates / (my_ms * 1e-3)
    nbytes = algorithmic_bytes(w)
    hbm_gbs = nbytes / (my_ms * 1e-3) / 1e9
    hbm_peak = float(peaks.get("hbm_gbs") or FALLBACK_HBM_GBS)
    t_sfu = w.updates / sfu_peak
    t_hbm = nbytes / (hbm_peak * 1e9)
    roofline_ms = max(t_sfu, t_hbm) * 1e3
    shape = selscan.ss_fwd_heuristic(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype,
                                     workspace_bytes=ws.numel() if ws is not None else 0)
    traffic = (args.traffic_bytes if args.traffic_bytes
               else recorded_traffic(w.name, [shape["lanes_per_row"], int(shape["split_states"]),
                                              shape["warps_per_block"], shape["segments"]]))

    line = {
        "metric": METRIC, "value": value, "unit": "updates/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f32",  # the arithmetic; the inputs' and outputs' dtype is in config
        "data": "synthetic (seeded Philox4x32-10 + Box-Muller)",
        "config": dict(w.describe(), parallelism=f"{world} independent problem(s), one per GPU",
                       l2="flushed before every timed step (write of %d MB)" % (flush.numel() >> 20),
                       launch=shape),
        "roofline": {"bound": "alu", "achieved": achieved_ex2 / 1e12, "peak": sfu_peak / 1e12,
                     "unit": "T ex2/s", "frac": achieved_ex2 / sfu_peak, "traffic": traffic,
                     "peak_source": f"derived: {SFU_EX2_PER_CLK_PER_SM} ex2/clk/SM x {sms} SMs x "
                                    f"{sm_max:.0f} MHz ({peak_src} max SM clock)",
                     "roofline_ms": roofline_ms, "frac_of_roofline_time": roofline_ms / ms},
        "hbm": {"achieved_gbs": hbm_gbs, "peak_gbs": hbm_peak, "frac": hbm_gbs / hbm_peak,
                "algorithmic_bytes": nbytes, "peak_source": peak_src},
        "e2e": {"value": updates / (e2e_ms * 1e-3), "unit": "updates/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "api": "ss_fwd_hostio_streams (pinned host buffers, batch ranges pipelined over 3 streams)"},
        "gpu_launches": args.steps * (3 if shape["segments"] > 1 else 1),  # segments: + carry fold + fix-up
        "clocks": clocks.summary(),
        "kernel_ms": {"min": min(kernel_ms), "median": statistics.median(kernel_ms),
                      "max": max(kernel_ms)},
    }
    clk = line["clocks"]
    if clk.get("sm_mhz"):
        line["clocks"]["ms_x_median_sm_mhz"] = my_ms * clk["sm_mhz"]
    line["decode"] = bench_decode(wr, d, out_dtype, stream, world)
    if not args.no_bwd:
        line["backward"] = bench_backward(args, wr, d, host, out_dtype, flush, stream, sfu_peak, world)
        dy = gen.fill(tuple(host["u"].shape), out_dtype, wr.seed, 9).to(dev)
        line["train_step"] = _time_train_step(wr, d, dy, out_dtype, flush, stream, steps=max(3, min(args.steps, 20)),
                                              warmup=3)
        del dy
    if w.dtype == torch.bfloat16 and not args.no_per_config:
        line["fused_dtproj"] = bench_dtproj(wr, dev, stream, flush, steps=max(3, min(args.steps, 20)), warmup=3,
                                            sfu_peak=sfu_peak, unfused_ms=statistics.median(kernel_ms))
    if not args.no_per_config:
        # Every other configuration at full size, forward only, fewer steps
        # each (the headline value stays the workload above).
        per = {}
        for name in W.WORKLOADS:
            if name == w.name:
                continue
            wn = rank_workload(W.WORKLOADS[name], rank)
            per[name] = bench_forward_config(wn, dev, stream, flush, steps=max(3, min(args.steps, 10)), warmup=3,
                                             sfu_peak=sfu_peak, hbm_peak=hbm_peak)
            if not args.no_bwd:
                per[name]["backward"] = bench_backward_config(wn, dev, stream, flush, steps=3, warmup=3,
                                                              sfu_peak=sfu_peak)
        line["per_config"] = per
    del flush
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample = cpu_oracle_sample(w, host)
        v1, sample1 = cpu_oracle_one_core(w, host)
        line["cpu_baseline"] = {"value": v, "unit": "updates/s", "cores": cores, "kind": "oracle",
                                "sample": sample, "cpu_model": cpu_model(),
                                "one_core": {"value": v1, "unit": "updates/s", "sample": sample1}}
    return line if rank == 0 else None


def bench_forward_config(w: W.Workload, dev, stream, flush, steps: int, warmup: int, sfu_peak: float,
                         hbm_peak: float):
    """Device time of one full forward of workload ``w`` (every kernel the
    heuristic launches for it, with the workspace that enables the
    sequence-segmented shape), L2 flushed before each step, clocks sampled
    over warm-ups and timed steps.  Used for the configurations beside the
    headline one."""
    host = W.make_inputs(w)
    names_in = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
    d = {k: (host[k].to(dev) if host[k] is not None else None) for k in names_in}
    del host
    out_dtype = w.out_dtype or w.dtype
    y = torch.empty(d["u"].shape, dtype=out_dtype, device=dev)
    last = (torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev)
            if w.return_last_state else None)
    ws = selscan.workspace_for(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype, device=dev)

    def launch():
        selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"],
                       delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus,
                       last_state=last, stream=stream, workspace=ws)

    ts = []
    with ClockSampler(dev.index) as clocks:
        for _ in range(warmup):
            flush.zero_()
            launch()
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            launch()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
    ms = sum(ts) / len(ts)
    nbytes = algorithmic_bytes(w)
    shape = selscan.ss_fwd_heuristic(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype,
                                     workspace_bytes=ws.numel() if ws is not None else 0)
    clk = clocks.summary()
    out = {"ms": ms, "ms_min": min(ts), "ms_max": max(ts), "steps": steps, "warmup": warmup,
           "updates_per_s": w.updates / (ms * 1e-3),
           "sfu_frac": w.updates / sfu_peak / (ms * 1e-3),
           "hbm_gbs": nbytes / (ms * 1e-3) / 1e9, "hbm_frac": nbytes / (ms * 1e-3) / 1e9 / hbm_peak,
           "algorithmic_bytes": nbytes, "launch": shape,
           "gpu_launches_per_step": 3 if shape["segments"] > 1 else 1, "clocks": clk}
    if clk.get("sm_mhz"):
        out["ms_x_median_sm_mhz"] = ms * clk["sm_mhz"]
    del d, y, last, ws
    torch.cuda.empty_cache()
    return out


def bench_dtproj(w: W.Workload, dev, stream, flush, steps: int, warmup: int, sfu_peak: float, unfused_ms: float):
    """Device time of the forward with delta produced inside the scan from its
    low-rank input (ss_fwd_dtproj: delta = W_dt delta_r on the tensor cores,
    dt_rank = ceil(d_model / 16) with d_model = dim / 2), beside the unfused
    forward's time on the same layer."""
    R = W.dt_rank_auto(w.dim // 2)
    host = W.make_dtproj_inputs(w, R)
    names_in = ("u", "delta_r", "W_dt", "A", "B", "C", "D", "z", "delta_bias")
    d = {k: (host[k].to(dev) if host[k] is not None else None) for k in names_in}
    y = torch.empty(d["u"].shape, dtype=w.dtype, device=dev)

    # x_proj's output as one tensor: feature rows delta_r, B, C (ss_fwd_xdbl reads them in place)
    x_dbl = torch.cat([d["delta_r"], d["B"], d["C"]], dim=1).contiguous()

    def launch():
        selscan.ss_fwd_dtproj(d["u"], d["delta_r"], d["W_dt"], d["A"], d["B"], d["C"], y, D=d["D"], z=d["z"],
                              delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus, stream=stream)

    def launch_xdbl():
        selscan.ss_fwd_xdbl(d["u"], x_dbl, d["W_dt"], d["A"], y, D=d["D"], z=d["z"], delta_bias=d["delta_bias"],
                            delta_softplus=w.delta_softplus, stream=stream)

    def timed(fn):
        for _ in range(warmup):
            flush.zero_()
            fn()
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        return statistics.median(ts)

    ms = timed(launch)
    xdbl_ms = timed(launch_xdbl)
    status = selscan.ss_device_status()
    del d, y, x_dbl
    return {"ms": ms, "dt_rank": R, "updates_per_s": w.updates / (ms * 1e-3),
            "sfu_frac": w.updates / sfu_peak / (ms * 1e-3), "unfused_ms": unfused_ms,
            "vs_unfused": unfused_ms / ms, "xdbl_ms": xdbl_ms, "steps": steps, "device_status": status,
            "note": "delta = W_dt delta_r (tcgen05 bf16 MMA into tensor memory, one 64-step stage ahead of "
                    "the scan) instead of reading delta; delta_r (B, dt_rank, L) and W_dt (D, dt_rank) bf16; "
                    "xdbl_ms: the same with delta_r, B and C read in place from one (B, dt_rank + 2 N, L) "
                    "x_proj output (ss_fwd_xdbl)"}


def bench_decode(w, d, out_dtype, stream, world, calls=200):
    """Latency of one recurrent decoding step (ss_step: the whole (batch, dim)
    layer advanced one token, state updated in place), averaged over
    back-to-back calls timed by CUDA events; bytes = state read + written plus
    the step's inputs and y."""
    dev = d["u"].device
    col = lambda x: None if x is None else x[..., 0].contiguous()  # noqa: E731
    u, delta, Bm, Cm, z = (col(d[k]) for k in ("u", "delta", "B", "C", "z"))
    state = torch.zeros((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev)
    y = torch.empty((w.batch, w.dim), dtype=out_dtype, device=dev)

    def step():
        selscan.ss_step(u, delta, d["A"], Bm, Cm, state, y, D=d["D"], z=z, delta_bias=d["delta_bias"],
                        delta_softplus=w.delta_softplus, stream=stream)

    for _ in range(10):
        step()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(calls):
        step()
    e1.record(stream)
    e1.synchronize()
    us_host = max_over_ranks(e0.elapsed_time(e1) * 1e3 / calls, world)
    # The same steps captured in a CUDA graph and replayed: the device time of
    # a step without the per-call host overhead of the Python binding.
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    per_graph = 50
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            for _ in range(per_graph):
                selscan.ss_step(u, delta, d["A"], Bm, Cm, state, y, D=d["D"], z=z,
                                delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus, stream=side)
    stream.wait_stream(side)
    graph.replay()
    torch.cuda.synchronize(dev)
    reps = max(1, calls // per_graph)
    e0.record(stream)
    for _ in range(reps):
        graph.replay()
    e1.record(stream)
    e1.synchronize()
    us = max_over_ranks(e0.elapsed_time(e1) * 1e3 / (reps * per_graph), world)
    del graph
    nbytes = (2 * state.numel() * 4 + y.numel() * y.element_size() +
              sum(t.numel() * t.element_size() for t in (u, delta, Bm, Cm, z) if t is not None))
    return {"us_per_step": us, "tokens_per_s": w.batch * world / (us * 1e-6), "bytes_per_step": nbytes,
            "hbm_gbs": nbytes / (us * 1e-6) / 1e9, "us_per_step_python_calls": us_host,
            "steps_timed": reps * per_graph, "gpu_launches_per_step": 1,
            "note": "ss_step replayed from a CUDA graph of 50 steps (device time per step); "
                    "us_per_step_python_calls: the same steps called one by one from Python"}


def _time_backward(w, d, dy, out_dtype, flush, stream, steps, warmup):
    """Device time (median ms) of ss_bwd (all gradients) on resident inputs,
    L2 flushed before each step; the workspace size and the launch plan."""
    dev = d["u"].device
    grads = {"du": torch.empty_like(d["u"]), "ddelta": torch.empty_like(d["u"]),
             "dA": torch.empty((w.dim, w.dstate), dtype=torch.float32, device=dev),
             "dB": torch.empty((w.batch, w.dstate, w.seqlen), dtype=torch.float32, device=dev),
             "dC": torch.empty((w.batch, w.dstate, w.seqlen), dtype=torch.float32, device=dev),
             "dD": torch.empty(w.dim, dtype=torch.float32, device=dev) if d["D"] is not None else None,
             "dz": torch.empty_like(d["u"]) if d["z"] is not None else None,
             "ddelta_bias": (torch.empty(w.dim, dtype=torch.float32, device=dev)
                             if d["delta_bias"] is not None else None)}
    nws = selscan.ss_bwd_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype)
    ws = torch.empty(nws, dtype=torch.uint8, device=dev)

    def launch():
        selscan.ss_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], dy, grads, D=d["D"], z=d["z"],
                       delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus, workspace=ws,
                       stream=stream)

    for _ in range(warmup):
        flush.zero_()
        launch()
    ts = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        launch()
        e1.record(stream)
        e1.synchronize()
        ts.append(e0.elapsed_time(e1))
    del ws, grads
    plan = selscan.ss_bwd_heuristic(w.batch, w.dim, w.seqlen, w.dstate, w.dtype, out_dtype)
    return statistics.median(ts), nws, plan


def _time_train_step(w, d, dy, out_dtype, flush, stream, steps, warmup):
    """A training step's device time (median ms over ``steps``, L2 flushed
    before each) two ways: the forward (ss_fwd, with the workspace that
    enables sequence segments) then ss_bwd, which runs its own forward pass
    for its checkpoints; and ss_fwd_ckpt, which writes them, then ss_bwd_ckpt,
    which reads them.  Each half is timed alone too."""
    dev = d["u"].device
    B, D, L, N = w.batch, w.dim, w.seqlen, w.dstate
    f32 = torch.float32
    y = torch.empty((B, D, L), dtype=out_dtype, device=dev)
    ck = torch.empty(selscan.ckpt_shape(B, D, L, N), dtype=f32, device=dev)
    wsf = selscan.workspace_for(B, D, L, N, w.dtype, out_dtype, device=dev)
    grads = {"du": torch.empty_like(d["u"]), "ddelta": torch.empty_like(d["u"]),
             "dA": torch.empty((D, N), dtype=f32, device=dev), "dB": torch.empty((B, N, L), dtype=f32, device=dev),
             "dC": torch.empty((B, N, L), dtype=f32, device=dev),
             "dD": torch.empty(D, dtype=f32, device=dev) if d["D"] is not None else None,
             "dz": torch.empty_like(d["u"]) if d["z"] is not None else None,
             "ddelta_bias": torch.empty(D, dtype=f32, device=dev) if d["delta_bias"] is not None else None}
    wsb = torch.empty(selscan.ss_bwd_workspace_bytes(B, D, L, N, w.dtype, out_dtype), dtype=torch.uint8, device=dev)
    kw = dict(D=d["D"], z=d["z"], delta_bias=d["delta_bias"], delta_softplus=w.delta_softplus, stream=stream)
    legs = {
        "fwd": lambda: selscan.ss_fwd(d["u"], d["delta"], d["A"], d["B"], d["C"], y, workspace=wsf, **kw),
        "bwd": lambda: selscan.ss_bwd(d["u"], d["delta"], d["A"], d["B"], d["C"], dy, grads, workspace=wsb, **kw),
        "fwd_ckpt": lambda: selscan.ss_fwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], y, ck, workspace=wsf,
                                                **kw),
        "bwd_ckpt": lambda: selscan.ss_bwd_ckpt(d["u"], d["delta"], d["A"], d["B"], d["C"], dy, ck, grads,
                                                workspace=wsb, **kw),
    }
    runs = {"step": ("fwd", "bwd"), "step_ckpt": ("fwd_ckpt", "bwd_ckpt"), "fwd": ("fwd",), "bwd": ("bwd",),
            "fwd_ckpt": ("fwd_ckpt",), "bwd_ckpt": ("bwd_ckpt",)}
    out = {}
    for name, parts in runs.items():
        for _ in range(warmup):
            flush.zero_()
            for leg in parts:
                legs[leg]()
        ts = []
        for _ in range(steps):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for leg in parts:
                legs[leg]()
            e1.record(stream)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        out[name + "_ms"] = statistics.median(ts)
    del y, ck, wsf, wsb, grads
    out["step_speedup"] = out["step_ms"] / out["step_ckpt_ms"]
    out["steps"] = steps
    out["note"] = ("training step = forward + backward: ss_fwd + ss_bwd (the backward's own checkpointing pass) "
                   "against ss_fwd_ckpt + ss_bwd_ckpt (checkpoints written by the forward); L2 flushed per step")
    return out


def _bwd_launches(w, plan):
    """Kernel launches of one ss_bwd call: per batch group the adjoint kernel
    and the dB/dC sum (plus, with sequence segments, the forward summary,
    its carry fold, the adjoint summary and its fold), then the row sums."""
    groups = -(-w.batch // plan["batch_group"])
    return groups * (2 + (4 if plan["segments"] > 1 else 0)) + 1


def bench_backward(args, w, d, host, out_dtype, flush, stream, sfu_peak, world):
    """Device time of ss_bwd (all gradients of sum(dy * y)) on the same inputs:
    a forward-state pass plus the adjoint pass recomputing the states, about
    two exps per state update (a seeded synthetic dy)."""
    dev = d["u"].device
    dy = gen.fill(tuple(host["u"].shape), out_dtype, w.seed, 9).to(dev)
    steps = max(3, min(args.steps, 30))
    ms, nws, plan = _time_backward(w, d, dy, out_dtype, flush, stream, steps, max(3, args.warmup))
    ms = max_over_ranks(ms, world)
    return {"ms_per_step": ms, "value": w.updates * world / (ms * 1e-3), "unit": "updates/s",
            "steps": steps, "workspace_bytes": nws, "plan": plan, "gpu_launches_per_step": _bwd_launches(w, plan),
            "ex2_per_update": 2, "sfu_frac": 2 * w.updates / sfu_peak / (ms * 1e-3),
            "note": "forward-state checkpoint pass + adjoint pass (recomputing the states) + "
                    "fixed-order reductions; L2 flushed before each step"}


def bench_backward_config(w: W.Workload, dev, stream, flush, steps: int, warmup: int, sfu_peak: float):
    """ss_bwd of workload ``w`` at full size (its own inputs and a seeded dy),
    as bench_backward; with sequence segments the two summary passes add
    about two exps per update to the two of the segmented adjoint kernel."""
    host = W.make_inputs(w)
    out_dtype = w.out_dtype or w.dtype
    names_in = ("u", "delta", "A", "B", "C", "D", "z", "delta_bias")
    d = {k: (host[k].to(dev) if host[k] is not None else None) for k in names_in}
    dy = gen.fill(tuple(host["u"].shape), out_dtype, w.seed, 9).to(dev)
    del host
    ms, nws, plan = _time_backward(w, d, dy, out_dtype, flush, stream, steps, warmup)
    train = _time_train_step(w, d, dy, out_dtype, flush, stream, steps, warmup)
    del d, dy
    torch.cuda.empty_cache()
    return {"ms": ms, "steps": steps, "warmup": warmup, "updates_per_s": w.updates / (ms * 1e-3),
            "sfu_frac": 2 * w.updates / sfu_peak / (ms * 1e-3), "ex2_per_update_counted": 2,
            "workspace_bytes": nws, "plan": plan, "gpu_launches_per_step": _bwd_launches(w, plan),
            "train_step": train}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(W.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-bwd", action="store_true", help="skip the backward measurement")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the forward of the other configurations")
    ap.add_argument("--traffic-bytes", type=float, default=None,
                    help="DRAM bytes per launch of the scan kernel from an ncu capture")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    w = W.WORKLOADS[args.workload]
    if args.impl == "reference":
        # The oracle runs on rank 0's host cores only; other ranks do no work.
        if int(os.environ.get("RANK", "0")) != 0:
            return
        line = bench_reference(args, w, 1, 0)
        print(json.dumps(line), flush=True)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py --impl ours needs a CUDA device")
    world, rank, local = dist_setup(args)
    try:
        line = bench_ours(args, w, world, rank, local)
        if line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
