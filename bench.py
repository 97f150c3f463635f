"""Throughput benchmark of the fused Hyena forward (B*D*L elements/s).

python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]

One step = one hyena_forward over the whole batch of the workload (all N
orders, every row), inputs resident in HBM. The default (headline) workload is
the order-3 bf16 B=1 D=768 L=65536 case, the longest single-GPU configuration
of the operator (padded transform M = 131072). The same line carries a
``workloads`` object with the other bench configurations (order-2 bf16 L=2048;
order-2 bf16 L=8192 with implicit filters; the 2D order-1 256x256 grid, plain
and through the HyenaND gate sandwich; the L=65536 case with channels-last
[B, L, D] activations), each
measured the same way: ms per step, throughput, roofline fraction, DRAM
traffic record, e2e, and the step with filter generation where the filters
are implicit. With N>1 (torchrun) every rank runs the
same workload on its own GPU with its own seed, with no collective on the data
path (weak scaling); the reported value is all ranks' elements divided by the
slowest rank's time.

Prints one JSON line on rank 0. The roofline object divides the operator's
flop convention (5 M log2 M per transform, two transforms per row and order)
by the kernel time, against the FP32 peak of 148 SMs x 128 lanes x 2 x the
maximum SM clock; it also reports the HBM fraction against the measured copy
bandwidth. e2e is the same metric through hyena_forward_host (page-locked host
buffers, copies inside the timed region).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

DEFAULT_WORKLOAD = "order3_bf16_b1_d768_l65536"
SIDE_WORKLOADS = ("order2_bf16_b8_d768_l2048", "order2_bf16_b4_d1024_l8192_implicit",
                  "order1_bf16_2d_b2_c256_256x256", "gated_order1_bf16_2d_b2_c256_256x256",
                  "order3_bf16_b1_d768_l65536_bld")
FP32_LANES_PER_SM = 128          # FP32 FMA lanes per SM (4 sub-partitions x 32)
SM_MAX_MHZ_FALLBACK = 1965.0
HBM_NOMINAL_GBS = 8000.0         # the operator's roofline convention (8 TB/s)
L2_FLUSH_BYTES = 512 << 20       # > 126 MB L2, written between timed steps


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU time of the oracle sample")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="reference arm: oracle time of the W + K steps together")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--channels", type=int, default=None,
                    help="override the workload's channel count (small cases for profiling)")
    ap.add_argument("--batch", type=int, default=None, help="override the workload's batch")
    ap.add_argument("--no-workloads", action="store_true",
                    help="measure the selected workload only (no side workloads in the line)")
    return ap.parse_args()


# ----------------------------------------------------------------- cost model
def cost_model(w):
    """Algorithmic flops and bytes of one step (whole batch), per the operator's
    roofline convention: 5 M log2 M flops per transform, two transforms per row
    per order; bytes = v (q and k for the gate sandwich), N gates and y once each, plus
    every spectrum row once."""
    io = 4 if w.dtype == "f32" else 2
    N = w.order
    if w.ndim == 1:
        L = w.shape[0]
        M = 1 << max(5, (2 * L - 1).bit_length())
        transforms = 2 * N * w.B * w.D
        flops = transforms * 5.0 * M * math.log2(M)
        spec_bytes = N * w.D * (M // 2 + 1) * 8
    else:
        H, W = w.shape
        M = (2 * H) * (2 * W)
        transforms = 2 * N * w.B * w.D
        flops = transforms * 5.0 * M * math.log2(M)
        spec_bytes = N * w.D * (2 * H) * (W + 1) * 8
    act_bytes = (N + 2 + (1 if w.gated else 0)) * w.elements * io   # the gate sandwich also reads k
    return {"flops": flops, "bytes": act_bytes + spec_bytes + N * w.D * 4, "M": M}


def device_fp32_peak_tflops(sm_mhz):
    import torch
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    return sms * FP32_LANES_PER_SM * 2 * sm_mhz * 1e6 / 1e12, sms


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": SM_MAX_MHZ_FALLBACK}, "fallback"


# ------------------------------------------------------------- clock sampler
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.samples = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) == 6:
                self.samples.append(parts)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        sm, smax = [], []
        for s in self.samples:
            try:
                sm.append(float(s[0]))
                smax.append(float(s[1]))
            except ValueError:
                continue
            for n, flag in zip(names, s[2:]):
                if flag.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------- multi-rank
def max_over_ranks(values, dist, device):
    """Element-wise max of per-rank timings (the slowest rank sets the job time)."""
    if dist is None:
        return list(values)
    import torch
    t = torch.tensor([float(x) for x in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


def job_throughput(elements_per_rank, world, ms):
    """Weak scaling: every rank processes its own full workload; the job's
    throughput is all ranks' elements over the slowest rank's time."""
    return elements_per_rank * world / (ms * 1e-3)


# ------------------------------------------------------------------ our arm
def run_ours(args, w, rank, world, dist):
    import torch
    from long_convolution_sequence_hyena_b200 import capi
    from long_convolution_sequence_hyena_b200.api import Plan
    from long_convolution_sequence_hyena_b200.workloads import make_inputs

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    inp = make_inputs(w, seed=w.seed + 1000 * rank)
    adt = inp["v"].dtype
    v = inp["v"].to(dev)
    gates = [g.to(dev) for g in inp["gates"]]
    dskip = inp["dskip"].to(dev)
    plan = Plan(w.shape, w.D, w.order, adt, layout=w.layout)
    if "h" in inp:
        H = plan.filter_spectrum(h=inp["h"].to(dev))
    else:
        imp = {k: (x.to(dev) if torch.is_tensor(x) else x) for k, x in inp["implicit"].items()}
        H = plan.filter_spectrum(implicit=imp)
    y = torch.empty_like(v)
    ws_bytes = plan.workspace_bytes(w.B)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()
    sptr = stream.cuda_stream
    gptrs = [g.data_ptr() for g in gates]

    # the C call with its arguments marshalled once, so that each timed step
    # enqueues its kernels with as little host work as possible
    import ctypes
    garr = (ctypes.c_void_p * len(gptrs))(*gptrs)
    if w.gated:
        # the gate sandwich: v is q, and the key k forms the inner gate q SiLU(k)
        kdev = inp["k"].to(dev)
        fwd_fn, fwd_name = capi.lib.hyena_forward_gated, "hyena_forward_gated"
        fwd_args = (plan.handle, w.B, v.data_ptr(), kdev.data_ptr(), garr, H.data_ptr(), dskip.data_ptr(),
                    y.data_ptr(), ws.data_ptr() if ws_bytes else None, ws_bytes, sptr)
    else:
        fwd_fn, fwd_name = capi.lib.hyena_forward, "hyena_forward"
        fwd_args = (plan.handle, w.B, v.data_ptr(), garr, H.data_ptr(), dskip.data_ptr(), y.data_ptr(),
                    ws.data_ptr() if ws_bytes else None, ws_bytes, sptr)

    def step():
        st = fwd_fn(*fwd_args)
        if st != capi.HYENA_OK:
            raise RuntimeError(fwd_name + ": " + capi.hyena_status_string(st))

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()

    clocks = ClockSampler(dev.index)
    clocks.start()
    time.sleep(0.3)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    n0 = capi.hyena_launch_count()
    for i in range(args.steps):
        flush.zero_()                      # L2 flush, outside the timed events
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    # the library's own count of the kernels it enqueued in the timed steps
    launches = (capi.hyena_launch_count() - n0) // args.steps
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    ms = sum(step_ms) / len(step_ms)

    # end to end through the C ABI with HOST buffers: hyena_forward_host copies the
    # page-locked inputs in and the output back, pipelined over the batch (the plain
    # operator only: the gate sandwich has no host-buffer entry point)
    if w.gated:
        return finish_gated(args, w, dist, dev, plan, ms, step_ms, clk, launches, imp if "implicit" in inp else None,
                            H, stream, step, flush)
    hv = inp["v"].pin_memory()
    hg = [g.pin_memory() for g in inp["gates"]]
    hy = torch.empty_like(hv).pin_memory()
    hws_bytes = capi.hyena_forward_host_workspace_bytes(plan.handle, w.B)
    hws = torch.empty(max(hws_bytes, 1), dtype=torch.uint8, device=dev)
    hgarr = (ctypes.c_void_p * len(hg))(*[g.data_ptr() for g in hg])
    host_args = (plan.handle, w.B, hv.data_ptr(), hgarr, H.data_ptr(), dskip.data_ptr(), hy.data_ptr(),
                 hws.data_ptr(), hws_bytes, sptr)

    def e2e_step():
        st = capi.lib.hyena_forward_host(*host_args)
        if st != capi.HYENA_OK:
            raise RuntimeError("hyena_forward_host: " + capi.hyena_status_string(st))

    for _ in range(max(1, args.warmup)):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps = max(3, min(args.steps, 20))
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps

    # the copy-bound figure of this box: the same input bytes copied host to
    # device from page-locked memory, one cudaMemcpyAsync per tensor on one stream
    dv = torch.empty_like(hv, device=dev)
    dg = [torch.empty_like(g, device=dev) for g in hg]

    def copy_in():
        dv.copy_(hv, non_blocking=True)
        for a, b in zip(dg, hg):
            a.copy_(b, non_blocking=True)
    copy_in()
    torch.cuda.synchronize()
    c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    c0.record(stream)
    for _ in range(3):
        copy_in()
    c1.record(stream)
    torch.cuda.synchronize()
    h2d_ms = c0.elapsed_time(c1) / 3
    del dv, dg

    # implicit filters: also time the filter network and its spectrum with the
    # forward, per step (filters regenerated every step, as in training)
    filt_ms = 0.0
    if "implicit" in inp:
        def filt_step():
            plan.filter_spectrum(implicit=imp, out=H, stream=stream)
            step()
        for _ in range(args.warmup):
            flush.zero_()
            filt_step()
        torch.cuda.synchronize()
        fs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            fs[i].record(stream)
            filt_step()
            fe[i].record(stream)
        torch.cuda.synchronize()
        filt_ms = sum(a.elapsed_time(b) for a, b in zip(fs, fe)) / args.steps

    ms, e2e_ms, filt_ms, h2d_ms = max_over_ranks([ms, e2e_ms, filt_ms, h2d_ms], dist, dev)
    io = 4 if w.dtype == "f32" else 2
    h2d = (w.order + 1) * w.elements * io
    d2h = w.elements * io
    plan.close()
    del v, gates, y, ws, flush, hws
    torch.cuda.empty_cache()
    return {"ms": ms, "step_ms": step_ms, "e2e_ms": e2e_ms, "h2d": h2d, "d2h": d2h, "clk": clk,
            "launches": launches, "filt_ms": filt_ms, "h2d_ms": h2d_ms}


def finish_gated(args, w, dist, dev, plan, ms, step_ms, clk, launches, imp, H, stream, step, flush):
    """The rest of run_ours for the gate sandwich: the step with filter generation (implicit
    kernels), no host-buffer leg."""
    import torch
    filt_ms = 0.0
    if imp is not None:
        def filt_step():
            plan.filter_spectrum(implicit=imp, out=H, stream=stream)
            step()
        for _ in range(args.warmup):
            flush.zero_()
            filt_step()
        torch.cuda.synchronize()
        fs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        fe = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
        for i in range(args.steps):
            flush.zero_()
            fs[i].record(stream)
            filt_step()
            fe[i].record(stream)
        torch.cuda.synchronize()
        filt_ms = sum(a.elapsed_time(b) for a, b in zip(fs, fe)) / args.steps
    ms, filt_ms = max_over_ranks([ms, filt_ms], dist, dev)
    plan.close()
    return {"ms": ms, "step_ms": step_ms, "e2e_ms": None, "h2d": 0, "d2h": 0, "clk": clk,
            "launches": launches, "filt_ms": filt_ms, "h2d_ms": None}


# ------------------------------------------------------------ oracle (CPU)
def oracle_runner(w):
    """Prepare the fp64 oracle on rows (planes) of the workload's recipe.
    Returns (run(rows) -> None, elements per row, threads, distinct rows); run(rows)
    evaluates `rows` rows, cycling over the distinct rows drawn."""
    import numpy as np

    import oracle
    from long_convolution_sequence_hyena_b200.workloads import make_inputs

    small = w.scaled(B=1, D=min(w.D, 64), name=w.name + "_sample")
    inp = make_inputs(small)
    threads = oracle.num_threads()
    N = w.order
    names = ("W1", "b1", "W2", "b2", "W3", "b3")
    if w.ndim == 1:
        L = w.shape[0]
        if "h" in inp:
            h64 = inp["h"].double().numpy()
        else:
            p = inp["implicit"]
            h64 = oracle.implicit_filter_1d(L, N, small.D, *(p[k].double().numpy() for k in names),
                                            p["alpha"].double().numpy(), p["num_freqs"], p["omega0"], p["omega_hidden"])
        v = inp["v"].double().reshape(small.D, L).numpy()
        g = inp["gates"].double().reshape(N, small.D, L).numpy()
        d = inp["dskip"].double().numpy()

        def run(rows):
            idx = np.arange(rows) % small.D
            oracle.hyena_1d(v[idx], g[:, idx], h64, d, fidx=idx)
        unit = L
    else:
        H, W = w.shape
        if "h" in inp:
            k64 = inp["h"].double().numpy()
        else:
            p = inp["implicit"]
            k64 = oracle.implicit_filter_2d(H, W, N, small.D, *(p[k].double().numpy() for k in names),
                                            p["sigma"].double().numpy(), p["omega0"], p["omega_hidden"])
        v = inp["v"].double().reshape(small.D, H, W).numpy()
        g = inp["gates"].double().reshape(N, small.D, H, W).numpy()
        d = inp["dskip"].double().numpy()

        def run(rows):
            idx = np.arange(rows) % small.D
            oracle.hyena_2d(v[idx], g[:, idx], k64, d, fidx=idx)
        unit = H * W
    return run, unit, threads, small.D


def calibrate_rows(run, threads, seconds):
    """Rows (a multiple of the thread count) whose oracle run takes about `seconds`."""
    rows = threads
    t0 = time.perf_counter()
    run(rows)
    dt = time.perf_counter() - t0
    while dt < seconds / 4 and rows < 4096 * threads:
        rows *= 2
        t0 = time.perf_counter()
        run(rows)
        dt = time.perf_counter() - t0
    return max(threads, int(rows * seconds / max(dt, 1e-9)) // threads * threads)


def oracle_sample(w, seconds):
    """Time the fp64 oracle on a bounded sample of the workload's rows (planes).
    Returns (elements/s, sample description, threads, seconds)."""
    run, unit, threads, distinct = oracle_runner(w)
    rows = calibrate_rows(run, threads, seconds)
    t0 = time.perf_counter()
    run(rows)
    dt = time.perf_counter() - t0
    what = "%d row evaluations (cycling over %d rows drawn with the workload's recipe; %d elements each), " \
           "direct fp64 sum" % (rows, distinct, unit)
    return rows * unit / dt, what, threads, dt


def run_reference(args, w):
    """The reference arm: the oracle as it stands, W warm-up and K timed steps,
    each step a bounded sample of the workload's rows (sized so the whole run
    takes about --ref-seconds, two minutes by default)."""
    run, unit, threads, distinct = oracle_runner(w)
    per_step = max(0.25, args.ref_seconds / (args.steps + args.warmup))
    rows = calibrate_rows(run, threads, per_step)
    for _ in range(args.warmup):
        run(rows)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        run(rows)
        times.append(time.perf_counter() - t0)
    value = rows * unit * len(times) / sum(times)
    sample = "%d row evaluations per step (cycling over %d rows drawn with the workload's recipe; " \
             "%d elements each), direct fp64 sum" % (rows, distinct, unit)
    return value, sample, threads


def traffic_record(w):
    """DRAM bytes per launch of the workload's dominant kernel from the committed ncu
    record, or None when there is none or the kernels changed since it was taken."""
    prof = os.path.join(ROOT, "profiles", "traffic_%s.json" % w.name)
    try:
        with open(prof) as f:
            pj = json.load(f)
        from long_convolution_sequence_hyena_b200.build import source_hash
        if pj.get("source_hash") == source_hash():
            return pj.get("dram_bytes_per_launch")
    except Exception:
        pass
    return None


def summarize(w, r, world):
    """The per-workload numbers of one measurement (see run_ours)."""
    cost = cost_model(w)
    peaks, peak_src = measured_peaks()
    sm_max = peaks.get("sm_max_mhz", SM_MAX_MHZ_FALLBACK)
    fp32_peak, sms = device_fp32_peak_tflops(sm_max)
    sec = r["ms"] * 1e-3
    achieved_tflops = cost["flops"] / sec / 1e12
    achieved_gbs = cost["bytes"] / sec / 1e9
    t_roof = max(cost["bytes"] / (HBM_NOMINAL_GBS * 1e9), cost["flops"] / (fp32_peak * 1e12))
    roof = {"bound": "alu", "achieved": achieved_tflops, "peak": fp32_peak, "unit": "TFLOP/s",
            "frac": achieved_tflops / fp32_peak, "traffic": traffic_record(w),
            "peak_source": "FP32 FMA lanes x2 x max SM clock (%d SMs, %.0f MHz)" % (sms, sm_max),
            "flops_convention": "5 M log2 M per transform, 2 transforms per row per order (M=%d)" % cost["M"],
            "algorithmic_bytes": cost["bytes"],
            "hbm_achieved_gbs": achieved_gbs, "hbm_peak_gbs": peaks.get("hbm_gbs"),
            "hbm_frac": achieved_gbs / peaks.get("hbm_gbs", 6650.0), "hbm_peak_source": peak_src,
            "operator_roofline_frac": t_roof / sec}
    e2e = None
    if r["e2e_ms"] is not None:
        e2e = {"value": w.elements * world / (r["e2e_ms"] * 1e-3), "unit": "elems/s", "ms_per_step": r["e2e_ms"],
               "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
               # copy-bound context: the step's input bytes over this box's measured pinned H2D
               # rate (the floor), and its input and output bytes at that rate (the time if the
               # two directions did not overlap at all)
               "h2d_gbs_measured": r["h2d"] / (r["h2d_ms"] * 1e-3) / 1e9, "h2d_ms_measured": r["h2d_ms"],
               "copies_serial_ms": (r["h2d"] + r["d2h"]) / r["h2d"] * r["h2d_ms"]}
    out = {"ms_per_step": r["ms"], "value": job_throughput(w.elements, world, r["ms"]), "unit": "elems/s",
           "roofline": roof, "e2e": e2e, "gpu_launches_per_step": r["launches"]}
    if r["filt_ms"] > 0:
        # the same metric with the implicit filter network and the filter spectra
        # computed inside every step (the operator as used in training)
        out["with_filter_generation"] = {"value": job_throughput(w.elements, world, r["filt_ms"]),
                                         "unit": "elems/s", "ms_per_step": r["filt_ms"]}
    return out


def main():
    args = parse()
    from long_convolution_sequence_hyena_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    if args.channels is not None or args.batch is not None:
        w = w.scaled(B=args.batch, D=args.channels, name=w.name)
    metric = "Hyena op throughput (B·D·L elems/s)"
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    cfg = {"workload": w.name, "batch": w.B, "global_batch": w.B * world, "seq_len": w.L, "channels": w.D, "order": w.order,
           "shape": list(w.shape), "parallelism": "independent replicas x%d (no data-path collective)" % world,
           "l2": "flushed between timed steps (512 MiB write)", "filters": w.filt}

    if args.impl == "reference":
        if rank != 0:
            return
        value, sample, threads = run_reference(args, w)
        line = {"metric": metric, "value": value, "unit": "elems/s", "n_gpus": args.gpus, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": w.elements * world / value * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
                "impl": "reference",
                "cpu_baseline": {"value": value, "unit": "elems/s", "cores": threads, "kind": "oracle", "sample": sample},
                "e2e": {"value": value, "unit": "elems/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist_mod
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = dist_mod
    r = run_ours(args, w, rank, world, dist)
    side = {}
    if not args.no_workloads and args.channels is None and args.batch is None:
        for name in SIDE_WORKLOADS:
            if name != w.name:
                side[name] = run_ours(args, WORKLOADS[name], rank, world, dist)
    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    head = summarize(w, r, world)
    line = {
        "metric": metric, "value": head["value"], "unit": "elems/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["ms"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.dtype == "bf16" else "f32", "data": "synthetic", "config": cfg,
        "roofline": head["roofline"], "e2e": head["e2e"],
        "gpu_launches": args.steps * r["launches"],
        "clocks": r["clk"],
        "step_ms_min": min(r["step_ms"]), "step_ms_max": max(r["step_ms"]),
    }
    if "with_filter_generation" in head:
        line["with_filter_generation"] = head["with_filter_generation"]
    if side:
        line["workloads"] = {}
        for name, rs in side.items():
            sw = WORKLOADS[name]
            line["workloads"][name] = dict(summarize(sw, rs, world), clocks=rs["clk"],
                                           config={"batch": sw.B, "channels": sw.D, "shape": list(sw.shape),
                                                   "order": sw.order, "dtype": sw.dtype, "filters": sw.filt})
    if world == 1 and not args.no_cpu_baseline:
        cv, sample, threads, _ = oracle_sample(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": cv, "unit": "elems/s", "cores": threads, "kind": "oracle", "sample": sample}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
