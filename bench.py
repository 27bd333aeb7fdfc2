#!/usr/bin/env python
"""Benchmark of exact attention forward + backward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the whole hot path, forward (fa_fwd) then backward
(fa_bwd), over the GPT-style causal workload B=2, H=32, N=4096, d=128 in bf16
(synthetic seeded inputs).  Throughput counts 4*B*H*N^2*d FLOPs for the
forward, halved when causal, and 2.5x that for the backward.

Timing follows "第17讲 Tensor Core、HBM、SRAM 与 FlashAttention" §10.1-10.2:
warm-up first, CUDA events on the launching stream with a synchronize on both
sides, fixed shapes and dtypes, and a check of the outputs before timing.  The
timed steps run as one CUDA graph (captured from the same library calls, which
never allocate or synchronise), so the step time holds no host launch gaps.  The
inputs and outputs of one step (about 0.6 GB) exceed the 126 MB L2, so no
flush is needed between steps.

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(heads are independent: weak scaling, no collective on the data path); the
step time is the maximum over ranks and the value is all ranks' FLOPs divided
by it.  Rank 0 prints one JSON line.

--impl reference times the fp64 CPU oracle (the reference arm) on a bounded
sample of the same workload, on the host cores.

--fp8 times fa_fwd_fp8 (E4M3 Q, K, V, per-head descale factors) on the same
shape, forward only, against twice the measured bf16 peak.

--gemm-sweep times fa_gemm on square sizes N = 256 i + {0, 1, 2, 8, 16}
(the lecture's divisibility classes) up to 8192 and prints the curve in the
same JSON line, with cuBLAS beside it; value = TFLOP/s at N = 8192.

--decode WORKLOAD times fa_decode instead (a decode step of Nq new queries per
head against a resident KV cache, same page §9.2-9.3) and prints its own line:
bytes of cache read per second, against the measured HBM copy bandwidth.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from tiled_attention_20_b200 import inputs, perf, ranks  # noqa: E402

WORKLOAD = inputs.GPT_CAUSAL
ATTN_WORKLOADS = {w.name: w for w in (inputs.SMALL_FWD, inputs.MID_NC, inputs.MID_C,
                                      inputs.GPT_CAUSAL, inputs.LONG_CONTEXT)}
DECODE_WORKLOADS = {w.name: w for w in (inputs.DECODE_B8, inputs.DECODE_B8_RAGGED,
                                        inputs.DECODE_SPEC, inputs.DECODE_LONG)}
METRIC = "attention fwd+bwd TFLOP/s (bf16, causal, N=4096 d=128) and % of dense BF16 peak"
# NVIDIA's B200 datasheet figure for dense BF16 tensor throughput (its 2:4
# sparse figure is twice this); context beside the measured peaks.
DATASHEET_BF16_DENSE_TFLOPS = 2250.0
UNIT = "TFLOP/s"
# The source file that defines each profiled kernel: a committed DRAM-traffic
# figure stays valid while that file is unchanged.
KERNEL_SOURCES = {"fa_fwd_kernel": "fwd_kernel.cuh", "fa_bwd_kernel": "bwd_kernel.cuh",
                  "fa_dq_kernel": "dq_kernel.cuh", "fa_decode_kernel": "decode_kernel.cuh",
                  "fa_gemm_kernel": "gemm_kernel.cuh"}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip the CPU oracle leg (used for profiler runs)")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer leg (profiler runs)")
    ap.add_argument("--deterministic", action="store_true",
                    help="time fa_bwd_deterministic (bit-reproducible dQ) instead of fa_bwd")
    ap.add_argument("--gemm-sweep", action="store_true",
                    help="time fa_gemm on square sizes of every divisibility class instead")
    ap.add_argument("--gemm-sizes", default=None,
                    help="comma-separated square sizes for --gemm-sweep (default: the full "
                         "sweep); the value is taken at the largest")
    ap.add_argument("--fp8", action="store_true",
                    help="time fa_fwd_fp8 (E4M3 operands) on the benchmark shape instead")
    ap.add_argument("--decode", default=None, metavar="WORKLOAD",
                    choices=sorted(DECODE_WORKLOADS),
                    help="time fa_decode on one decode workload instead of fwd+bwd")
    ap.add_argument("--workload", default=WORKLOAD.name, choices=sorted(ATTN_WORKLOADS),
                    help="attention workload of the fwd+bwd step (default: the benchmark's)")
    ap.add_argument("--quick", action="store_true",
                    help="headline pass only (no distribution or trace pass): for profiler runs")
    ap.add_argument("--sweep", action="store_true",
                    help="time forward and backward of the 48-case boundary/wave sweep instead")
    ap.add_argument("--cpu-table", action="store_true",
                    help="time the fp64 oracle on the small, mid and GPT-style workloads "
                         "(fwd and fwd+bwd; the small one also on one thread) instead")
    return ap.parse_args()


def workload_config(w=WORKLOAD, extra=None):
    in_bytes = 4 * w.B * w.H * w.N * w.d * 2  # Q, K, V, dO
    cfg = {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "causal": w.causal,
           "passes": "fwd+bwd" if w.backward else "fwd", "dist": w.dist, "seed": w.seed,
           "l2": ("inputs_exceed_l2 (no flush)" if in_bytes > 126e6 else
                  "inputs_fit_l2 (no flush: compute-bound)")}
    if extra:
        cfg.update(extra)
    return cfg


def workload_metric(w) -> str:
    """The headline metric for the benchmark workload; the same measure,
    named by its shape, for the others."""
    if w == WORKLOAD:
        return METRIC
    mask = "causal" if w.causal else "non-causal"
    return (f"attention {'fwd+bwd' if w.backward else 'fwd'} TFLOP/s (bf16, {mask}, "
            f"B={w.B} H={w.H} N={w.N} d={w.d}) and % of dense BF16 peak")


def step_flops(w=WORKLOAD) -> float:
    f = perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, False)
    if w.backward:
        f += perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, True)
    return f


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    with open(os.path.join(ROOT, "tiled_attention_20_b200", "csrc", KERNEL_SOURCES[kernel]), "rb") as f:
        h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary
    (profiles/dram_traffic.txt), if it was captured from the current kernel
    sources; else None."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        with open(path) as f:
            lines = [l.split() for l in f if l.strip() and not l.startswith("#")]
    except OSError:
        return None
    for name, src_hash, nbytes in (l[:3] for l in lines if len(l) >= 3):
        base = kernel.split(":")[0].replace("_nodq", "")
        if name == kernel and base in KERNEL_SOURCES and src_hash == kernel_source_hash(base):
            return int(nbytes)
    return None


# ---------------------------------------------------------------- end to end
def pipelined_e2e(dev, host_in, dev_in, dev_out, host_out, run, steps, dist=None):
    """Per-step milliseconds of host -> device -> host steps through the
    public API.  Two device buffer sets alternate: step i uploads its inputs
    (pinned host memory) into set i % 2 on one copy stream, its kernels run on
    the compute stream once that upload is done, and its results go back to
    pinned host memory on a second copy stream, so the upload of step i+1 and
    the download of step i-1 overlap the kernels of step i (the two copy
    directions use separate copy engines).  Events keep each set's reuse in
    order.  Every step moves its full inputs in and its full results out.
      host_in / host_out: lists of pinned host tensors;
      dev_in / dev_out:   two lists (one per set) of matching device tensors;
      run(k):             enqueues the step's library calls on set k."""
    comp = torch.cuda.Stream(dev)
    up = torch.cuda.Stream(dev)
    down = torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event(enable_timing=False)
    up_done = [ev(), ev()]
    comp_done = [ev(), ev()]
    down_done = [ev(), ev()]
    used = [False, False]

    def one(i):
        k = i % 2
        with torch.cuda.stream(up):
            if used[k]:
                up.wait_event(comp_done[k])  # set k's previous kernels have read their inputs
            for h, d in zip(host_in, dev_in[k]):
                d.copy_(h, non_blocking=True)
            up_done[k].record(up)
        with torch.cuda.stream(comp):
            comp.wait_event(up_done[k])
            if used[k]:
                comp.wait_event(down_done[k])  # set k's previous results are on the host
            run(k)
            comp_done[k].record(comp)
        with torch.cuda.stream(down):
            down.wait_event(comp_done[k])
            for d, h in zip(dev_out[k], host_out):
                h.copy_(d, non_blocking=True)
            down_done[k].record(down)
        used[k] = True

    one(0)
    one(1)
    torch.cuda.synchronize(dev)
    if dist is not None and dist.is_initialized():
        dist.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(up)
    for i in range(steps):
        one(i)
    t1.record(down)
    torch.cuda.synchronize(dev)
    return t0.elapsed_time(t1) / steps


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons every 200 ms."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        # keep samples taken under load (clock above idle) when there are any
        busy = [s for s in sm if s > 600] or sm
        return {"sm_mhz": statistics.median(busy) if busy else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


# ---------------------------------------------------------------- timing
def graph_of(step, steps):
    """One CUDA graph holding `steps` consecutive steps (every launch `step`
    enqueues, captured on a side stream), replayed once untimed so that a
    timed replay runs an instantiated, uploaded graph.  The library never
    allocates or synchronises inside a call, so its launches capture as they
    are; the graph removes the host launch gaps between the step's kernels."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, capture_error_mode="relaxed"):
        for _ in range(steps):
            step()
    g.replay()
    return g


def timed_passes(step, steps, stream, dev, dist, world, quick=False, dominant=None):
    """Timed passes of `step`, each bracketed by a barrier and a synchronize.
    Each pass captures its steps into one CUDA graph and times one replay of
    it on `stream` (the warm-up steps ran as plain launches):
      1. the headline: `steps` steps between two CUDA events, with the
         launches of the `dominant` kernel (and only those, so the step gets
         as few extra nodes as possible) bracketed by external event nodes:
         its duration for the roofline comes from the timed replay itself;
         returns the mean step time, max over ranks;
      2. the per-kernel table: `steps` steps with every library launch
         bracketed;
      3. the distribution: max(100, steps) steps with an event node after
         each, for the median, 10th and 90th percentile of the step time.
    Passes 2 and 3 run after the headline, when the power cap may have
    lowered the clock.  With quick (profiler runs) only pass 1 runs, as plain
    launches without events.  Returns (mean ms, stats, dominant kernel's
    trace, all kernels)."""
    import tiled_attention_20_b200.fa as fa

    def sync():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)

    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if quick:
        sync()
        e0.record(stream)
        for _ in range(steps):
            step()
        e1.record(stream)
        sync()
        return ranks.max_over_ranks(e0.elapsed_time(e1) / steps, dist, dev), {}, {}, {}

    fa.trace_start([dominant])
    g = graph_of(step, steps)
    sync()
    e0.record(stream)
    g.replay()
    e1.record(stream)
    sync()
    dom = fa.trace_stop()
    ms = ranks.max_over_ranks(e0.elapsed_time(e1) / steps, dist, dev)
    del g

    fa.trace_start()
    g = graph_of(step, steps)
    sync()
    g.replay()
    sync()
    traced = fa.trace_stop()
    del g

    n = max(100, steps)
    ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(n + 1)]

    def marked():
        ev[0].record()
        for i in range(n):
            step()
            ev[i + 1].record()

    g = graph_of(marked, 1)
    sync()
    g.replay()
    sync()
    per = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(n))
    del g
    pick = lambda f: per[min(n - 1, int(round(f * (n - 1))))]
    stats = {"n": n, "median_ms": statistics.median(per), "p10_ms": pick(0.1),
             "p90_ms": pick(0.9), "min_ms": per[0], "max_ms": per[-1],
             "after": "the headline and trace passes (the clock may be lower: power cap)"}
    return ms, stats, dom, traced


# ---------------------------------------------------------------- CPU oracle
def cpu_oracle_rate(q, k, v, dO, w, seconds: float, backward=None):
    """The oracle (fp64, as it stands) on whole heads of the workload until
    `seconds` of wall time have passed (forward, and backward when the
    workload has one); returns (TFLOP/s, heads, cores, s)."""
    import oracle  # the benchmark's CPU-baseline leg is one of the oracle's permitted users
    backward = w.backward if backward is None else backward
    t0 = time.time()
    heads = 0
    total = w.B * w.H
    while heads < total:
        b, h = divmod(heads, w.H)
        sl = lambda t: t[b:b + 1, h:h + 1]
        oracle.fwd(sl(q), sl(k), sl(v), causal=w.causal)
        if backward:
            oracle.bwd(sl(q), sl(k), sl(v), sl(dO), causal=w.causal)
        heads += 1
        if time.time() - t0 >= seconds:
            break
    el = time.time() - t0
    fl = perf.attention_flops(1, 1, w.N, w.d, w.causal, False)
    if backward:
        fl += perf.attention_flops(1, 1, w.N, w.d, w.causal, True)
    return fl * heads / el / 1e12, heads, oracle.num_threads(), el


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_cpu_table(args):
    """The fp64 oracle, as it stands, on the host cores: forward and
    forward+backward wall time of whole workloads (small, both mid masks,
    GPT-style), the small one also on one thread.  One JSON line."""
    import oracle
    rows = []
    for w in (inputs.SMALL_FWD, inputs.MID_NC, inputs.MID_C, inputs.GPT_CAUSAL):
        q, k, v, dO = inputs.for_workload(w)
        for backward in ((False,) if not w.backward else (False, True)):
            for threads in ((0, 1) if w is inputs.SMALL_FWD else (0,)):
                all_cores = oracle.num_threads()
                if threads:
                    oracle.set_num_threads(threads)
                rate, heads, cores, el = cpu_oracle_rate(q, k, v, dO, w, float("inf"), backward)
                oracle.set_num_threads(all_cores)
                rows.append({"workload": w.name, "passes": "fwd+bwd" if backward else "fwd",
                             "threads": cores, "heads": heads, "seconds": el,
                             "gflops": rate * 1e3})
    print(json.dumps({"metric": "fp64 CPU oracle wall time (whole workloads)",
                      "cpu_model": cpu_model(), "nproc": os.cpu_count(), "rows": rows}),
          flush=True)


SWEEP_METRIC = "attention TFLOP/s vs N, boundary/wave sweep (bf16, H=16)"


def run_sweep(args, rank, world, local_rank, dist):
    """Forward and backward of each of the 48 sweep workloads, timed with
    CUDA events (mean of `reps` calls each after warm-up, replayed as one
    CUDA graph like the main leg's timed passes), with the work units and
    waves of 148 SMs beside the rate.  Rank 0 prints one JSON line
    whose value is the median fwd+bwd rate over the cases."""
    import tiled_attention_20_b200.fa as fa
    from tiled_attention_20_b200 import build as fa_build
    if rank == 0 or world == 1:
        fa_build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = torch.cuda.current_stream(dev)
    peaks, peaks_src = measured_peaks()
    reps = max(5, min(args.steps, 50))
    sampler = ClockSampler(dev.index if world == 1 else local_rank)
    sampler.start()
    time.sleep(0.4)
    rows = []
    launches = 0
    for w in inputs.sweep_workloads():
        q, k, v, dO = (t.to(dev) for t in inputs.for_workload(w))
        o = torch.empty_like(q)
        lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
        grads = [torch.empty_like(q) for _ in range(3)]
        ws = torch.empty(fa.workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)

        def timed(fn):
            for _ in range(3):
                fn()
            g = graph_of(fn, reps)
            torch.cuda.synchronize(dev)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            g.replay()
            e1.record(stream)
            e1.synchronize()
            return e0.elapsed_time(e1) / reps

        fwd = lambda: fa.fwd(q, k, v, causal=w.causal, out=o, lse=lse)
        bwd = lambda: fa.bwd(q, k, v, o, dO, lse, causal=w.causal, workspace=ws, dq=grads[0],
                             dk=grads[1], dv=grads[2])
        ms_f = timed(fwd)
        ms_b = timed(bwd)
        launches += (3 + 2 * reps) * 4  # forward + preprocess, main, conversion
        f_f = perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, False)
        f_b = perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, True)
        ctas_f, units_f = fa.launch_shape(0, w.B, w.H, w.N, w.d, w.causal)
        ctas_b, units_b = fa.launch_shape(1, w.B, w.H, w.N, w.d, w.causal)
        rows.append({"workload": w.name, "N": w.N, "d": w.d, "B": w.B, "causal": w.causal,
                     "fwd_ms": ms_f, "bwd_ms": ms_b, "fwd_tflops": f_f / ms_f / 1e9,
                     "bwd_tflops": f_b / ms_b / 1e9,
                     "fwdbwd_tflops": (f_f + f_b) / (ms_f + ms_b) / 1e9,
                     "fwd_units": units_f, "bwd_units": units_b,
                     "fwd_waves": units_f / sms, "bwd_waves": units_b / sms})
        del q, k, v, dO, o, lse, grads, ws
    clocks = sampler.stop()
    fa.check_device_errors(dev)
    if rank == 0:
        rates = sorted(r["fwdbwd_tflops"] for r in rows)
        value = statistics.median(rates)
        print(json.dumps({
            "metric": SWEEP_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": reps, "warmup": 3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": "boundary_wave_sweep_48", "value": "median fwd+bwd over cases",
                       "l2": "no flush (compute-bound)", "sms": sms,
                       "launch": "cuda_graph (each pass: its calls captured back to back, one "
                                 "replay timed after an untimed one)"},
            "pct_of_peak": value / peaks["bf16_tflops"], "peak_source": peaks_src,
            "gpu_launches": launches, "clocks": clocks, "sweep": rows}), flush=True)


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle on the host cores, each step a bounded
    sample (one head, truncated to N' query/key rows so that all K + W steps
    end within about two minutes) of the benchmark workload."""
    if rank != 0:
        return
    import oracle
    w = WORKLOAD
    q, k, v, dO = inputs.for_workload(w)
    budget = 120.0 / max(1, args.steps + args.warmup)

    def sample_step(n):
        sl = lambda t: t[0:1, 0:1, :n].contiguous()
        t0 = time.time()
        oracle.fwd(sl(q), sl(k), sl(v), causal=w.causal)
        oracle.bwd(sl(q), sl(k), sl(v), sl(dO), causal=w.causal)
        return time.time() - t0

    t_cal = sample_step(512)
    n = int(512 * math.sqrt(max(budget, 1e-3) / max(t_cal, 1e-6)))
    n = max(128, min(w.N, n // 64 * 64))
    for _ in range(args.warmup):
        sample_step(n)
    t0 = time.time()
    for _ in range(args.steps):
        sample_step(n)
    el = time.time() - t0
    fl = (perf.attention_flops(1, 1, n, w.d, w.causal, False) +
          perf.attention_flops(1, 1, n, w.d, w.causal, True))
    value = fl * args.steps / el / 1e12
    sample = f"one head (b=0,h=0) truncated to N'={n} rows, fwd+bwd per step, fp64"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": workload_config(w, {"sample_N": n}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.num_threads(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank, dist):
    import tiled_attention_20_b200.fa as fa
    from tiled_attention_20_b200 import build as fa_build

    if rank == 0 or world == 1:
        fa_build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = ATTN_WORKLOADS[args.workload]
    q_h, k_h, v_h, dO_h = inputs.qkv_do(w.B, w.H, w.N, w.d, seed=ranks.rank_seed(w.seed, rank),
                                        dist=w.dist)
    q, k, v, dO = (t.to(dev) for t in (q_h, k_h, v_h, dO_h))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(fa.workspace_size(w.B, w.H, w.N, w.d), dtype=torch.uint8, device=dev)

    def step():
        fa.fwd(q, k, v, causal=w.causal, out=o, lse=lse)
        if w.backward:
            fa.bwd(q, k, v, o, dO, lse, causal=w.causal, workspace=ws, dq=dq, dk=dk, dv=dv,
                   deterministic=args.deterministic)

    # Output check before timing (no oracle here): finite results, and row 0
    # of a causal head sees only key 0, so O_0 must equal V_0 bit for bit.
    step()
    fa.check_device_errors(dev)
    for t in (o, lse, dq, dk, dv) if w.backward else (o, lse):
        if not torch.isfinite(t).all():
            raise RuntimeError("non-finite output")
    if w.causal and not torch.equal(o[:, :, 0], v[:, :, 0]):
        raise RuntimeError("causal row 0 does not equal V_0")

    for _ in range(max(0, args.warmup - 1)):
        step()
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(dev.index if world == 1 else local_rank)
    sampler.start()
    time.sleep(0.4)  # let the sampler come up
    # keep the GPU busy while the sampler starts, outside the timed region
    for _ in range(max(3, args.warmup)):
        step()
    dominant = "fa_bwd_kernel" if w.backward else "fa_fwd_kernel"
    ms, stats, dom_trace, traced = timed_passes(step, args.steps, stream, dev, dist, world,
                                                args.quick, dominant)
    clocks = sampler.stop()
    fa.check_device_errors(dev)
    flops = step_flops(w)
    value = ranks.weak_scaling_rate(flops, world, ms) / 1e12
    if args.quick:  # a profiler run: the headline pass alone
        if rank == 0:
            print(json.dumps({"metric": workload_metric(w), "value": value, "unit": UNIT,
                              "ms_per_step": ms, "config": workload_config(w), "quick": True}),
                  flush=True)
        return
    stats["tflops_at_median"] = flops / (stats["median_ms"] * 1e-3) / 1e12

    # dominant kernel (by the per-kernel pass), timed inside the headline pass
    top = max(traced.items(), key=lambda kv: kv[1][1])[0]
    if top != dominant:
        print(f"note: {top} took longer than {dominant} in the per-kernel pass",
              file=sys.stderr)
    dom_name = dominant
    dom_launches, dom_ms = dom_trace[dominant]
    per_launch_ms = dom_ms / dom_launches
    fwd_f = perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, False)
    kernel_flops = {
        "fa_fwd_kernel": fwd_f,
        "fa_bwd_kernel": perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, True),
    }
    if args.deterministic:
        # dK/dV kernel: S, dP, dV, dK (four GEMMs); dQ kernel: S, dP, dQ (three)
        kernel_flops["fa_bwd_kernel"] = 2.0 * fwd_f
        kernel_flops["fa_dq_kernel"] = 1.5 * fwd_f
    peaks, peaks_src = measured_peaks()
    if dom_name in kernel_flops:
        achieved = kernel_flops[dom_name] / (per_launch_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": profiled_traffic(dom_name + ("_nodq" if args.deterministic
                                                             and dom_name == "fa_bwd_kernel" else "")),
                "kernel": dom_name,
                "peak_source": f"{peaks_src} bf16_tflops (burst)",
                "frac_of_sustained": achieved / peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"]),
                "frac_of_datasheet_dense": achieved / DATASHEET_BF16_DENSE_TFLOPS,
                "launch_ms": per_launch_ms,
                "timed": "inside the headline pass, only this kernel's launches bracketed"}
    else:  # a memory-bound helper dominating would be a regression worth seeing
        roof = {"bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": None, "traffic": None, "kernel": dom_name}
    kernels = {name: {"launches": n, "avg_ms": t / n} for name, (n, t) in traced.items()}
    kernels["pass"] = "every launch bracketed, right after the headline pass"
    gpu_launches = sum(n for n, _ in traced.values())

    # end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        ins = (q_h, k_h, v_h, dO_h) if w.backward else (q_h, k_h, v_h)
        outs = (o, lse, dq, dk, dv) if w.backward else (o, lse)
        host_in = [t.pin_memory() for t in ins]
        host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs]
        dev_in = [[t.to(dev) for t in ins], [torch.empty(t.shape, dtype=t.dtype, device=dev)
                                             for t in ins]]
        dev_out = [list(outs), [torch.empty_like(t) for t in outs]]

        def run(kset):
            qq, kk, vv = dev_in[kset][:3]
            oo, ll = dev_out[kset][:2]
            fa.fwd(qq, kk, vv, causal=w.causal, out=oo, lse=ll)
            if w.backward:
                gq, gk, gv = dev_out[kset][2:]
                fa.bwd(qq, kk, vv, oo, dev_in[kset][3], ll, causal=w.causal, workspace=ws,
                       dq=gq, dk=gk, dv=gv, deterministic=args.deterministic)

        n_e2e = max(1, args.e2e_steps)
        ms_e2e = ranks.max_over_ranks(
            pipelined_e2e(dev, host_in, dev_in, dev_out, host_out, run, n_e2e, dist), dist, dev)
        fa.check_device_errors(dev)
        nb = lambda ts: sum(t.numel() * t.element_size() for t in ts)
        e2e = {"value": ranks.weak_scaling_rate(flops, world, ms_e2e) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": nb(host_in), "d2h_bytes_per_step": nb(host_out),
               "steps": n_e2e, "ms_per_step": ms_e2e,
               "pipeline": "two buffer sets; uploads and downloads overlap the kernels",
               "api": "tiled_attention_20_b200.fa.fwd/bwd (C ABI)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, heads, cores, el = cpu_oracle_rate(q_h, k_h, v_h, dO_h, w, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{heads} of {w.B * w.H} heads of the workload, fwd+bwd in fp64, "
                         f"{el:.1f} s wall"}

    if rank == 0:
        line = {
            "metric": workload_metric(w), "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": workload_config(w, {"parallelism": f"heads replicated per GPU x{world}",
                                          "bwd": "deterministic" if args.deterministic else "atomic_dq",
                                          "launch": "cuda_graph (each timed pass: its steps "
                                                    "captured back to back, one replay timed)"}),
            "pct_of_peak": value / world / peaks["bf16_tflops"],
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": gpu_launches,
            "kernels": kernels, "clocks": clocks, "step_stats": stats,
        }
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- decode leg
DECODE_METRIC = "decode attention cache-read bandwidth (bf16, KV cache in HBM)"
DECODE_UNIT = "GB/s"


def decode_bytes(w, lens) -> float:
    """Algorithmic bytes of one decode call: every valid K and V row once,
    q read, O (bf16) and lse (fp32) written."""
    rows = float(sum(int(n) for n in lens)) * w.H
    return rows * w.d * 2 * 2 + w.B * w.H * w.Nq * (w.d * 2 * 2 + 4)


def cpu_oracle_decode_rate(q, k, v, lens, w, seconds: float):
    """The oracle's decode (fp64, as it stands) on whole heads until `seconds`
    of wall time have passed; returns (GB/s of algorithmic bytes, heads, cores, s)."""
    import oracle  # CPU-baseline leg: one of the oracle's permitted users
    t0 = time.time()
    heads, done_bytes = 0, 0.0
    while heads < w.B * w.H:
        b, h = divmod(heads, w.H)
        sl = lambda t: t[b:b + 1, h:h + 1]
        oracle.decode(sl(q), sl(k), sl(v), causal=w.causal, lens=lens[b:b + 1].numpy())
        done_bytes += int(lens[b]) * w.d * 2 * 2 + w.Nq * (w.d * 2 * 2 + 4)
        heads += 1
        if time.time() - t0 >= seconds:
            break
    el = time.time() - t0
    return done_bytes / el / 1e9, heads, oracle.num_threads(), el


# ---------------------------------------------------------------- GEMM sweep
GEMM_METRIC = "bf16 GEMM TFLOP/s, square N x N x N (256x128 tiles, persistent over the SMs)"


def gemm_div_class(n: int) -> int:
    """Largest of 32, 16, 8, 2, 1 that divides n (the lecture's colour classes)."""
    for c in (32, 16, 8, 2):
        if n % c == 0:
            return c
    return 1


def run_gemm_sweep(args, rank, world, local_rank, dist):
    """Throughput of fa_gemm against the square size N, for N = 256 i + delta
    (i = 1..32, delta in 0, 1, 2, 8, 16: divisibility classes 32+, 1, 2, 8,
    16), each point the mean of `reps` launches with L2 flushed before each;
    torch.matmul (cuBLAS) is timed beside it for context."""
    import tiled_attention_20_b200.fa as fa
    from tiled_attention_20_b200 import build as fa_build
    if rank == 0 or world == 1:
        fa_build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)  # > 126 MB of L2
    g = torch.Generator(device=dev).manual_seed(ranks.rank_seed(0, rank))
    peaks, peaks_src = measured_peaks()
    reps = max(3, min(args.steps, 10))
    ws = torch.empty(320 << 20, dtype=torch.uint8, device=dev)  # aligned copies up to N = 8208
    n_warm = max(2, min(args.warmup, 3))

    def timed(fn):
        for _ in range(n_warm):
            fn()
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            e1.synchronize()
            tot += e0.elapsed_time(e1)
        return tot / reps

    sampler = ClockSampler(dev.index if world == 1 else local_rank)
    sampler.start()
    time.sleep(0.4)
    sweep = []
    sizes = ([int(x) for x in args.gemm_sizes.split(",")] if args.gemm_sizes else
             [256 * i + dlt for i in range(1, 33) for dlt in (0, 1, 2, 8, 16)])
    launches = 0
    for n in sizes:
        a = torch.randn((n, n), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        b = torch.randn((n, n), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
        c = torch.empty((n, n), dtype=torch.bfloat16, device=dev)
        ms = timed(lambda: fa.gemm(a, b, out=c, workspace=ws))
        ms_cublas = timed(lambda: torch.matmul(a, b, out=c))
        bn, tm, tn = fa.gemm_tiles(n, n, sms)
        launches += (n_warm + reps) * (1 if n % 8 == 0 else 3)  # GEMM (+ two aligned copies)
        fl = 2.0 * n * n * n
        sweep.append({"N": n, "div": gemm_div_class(n), "tile": f"256x{bn}", "tiles": tm * tn,
                      "rounds": -(-(tm * tn) // sms), "ms": ms, "tflops": fl / ms / 1e9,
                      "cublas_tflops": fl / ms_cublas / 1e9})
    clocks = sampler.stop()
    fa.check_device_errors(dev)
    top = next((r for r in sweep if r["N"] == 8192), max(sweep, key=lambda r: r["N"]))
    # whole-job rate: every rank ran the same point; the slowest rank sets the time
    top_ms = ranks.max_over_ranks(top["ms"], dist, dev)
    value = 2.0 * top["N"] ** 3 * world / top_ms / 1e9
    roof = {"bound": "tensor", "achieved": top["tflops"], "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": top["tflops"] / peaks["bf16_tflops"],
            "traffic": profiled_traffic(f"fa_gemm_kernel:{top['N']}"),
            "kernel": "fa_gemm_kernel", "peak_source": f"{peaks_src} bf16_tflops (burst)",
            "launch_ms": top["ms"], "at": f"N={top['N']}"}

    e2e = None
    if not args.no_e2e:
        n = top["N"]
        ha = torch.randn((n, n), generator=torch.Generator().manual_seed(1)).to(torch.bfloat16).pin_memory()
        hb = torch.randn((n, n), generator=torch.Generator().manual_seed(2)).to(torch.bfloat16).pin_memory()
        hc = torch.empty((n, n), dtype=torch.bfloat16).pin_memory()
        dev_in = [[torch.empty_like(ha, device=dev), torch.empty_like(hb, device=dev)]
                  for _ in range(2)]
        dev_out = [[torch.empty((n, n), dtype=torch.bfloat16, device=dev)] for _ in range(2)]

        def run(kset):
            fa.gemm(dev_in[kset][0], dev_in[kset][1], out=dev_out[kset][0], workspace=ws)

        k = max(1, args.e2e_steps)
        ms_e2e = ranks.max_over_ranks(
            pipelined_e2e(dev, [ha, hb], dev_in, dev_out, [hc], run, k, dist), dist, dev)
        e2e = {"value": 2.0 * n ** 3 / ms_e2e / 1e9 * world, "unit": UNIT,
               "h2d_bytes_per_step": 2 * n * n * 2, "d2h_bytes_per_step": n * n * 2,
               "steps": k, "ms_per_step": ms_e2e,
               "pipeline": "two buffer sets; uploads and downloads overlap the kernels",
               "api": "tiled_attention_20_b200.fa.gemm (C ABI)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle  # CPU-baseline leg: the fp64 oracle's plain product
        n = 1024
        a = torch.randn((n, n), generator=torch.Generator().manual_seed(3)).to(torch.bfloat16)
        t0 = time.time()
        done = 0
        while time.time() - t0 < args.cpu_seconds:
            oracle.gemm(a, a)
            done += 1
        el = time.time() - t0
        cpu = {"value": 2.0 * n ** 3 * done / el / 1e12, "unit": UNIT,
               "cores": oracle.num_threads(), "kind": "oracle",
               "sample": f"{done} products of {n} x {n} x {n} in fp64, {el:.1f} s wall"}

    if rank == 0:
        line = {
            "metric": GEMM_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": reps, "warmup": args.warmup, "ms_per_step": top["ms"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": ("gemm_square_sweep_N256_to_8208" if not args.gemm_sizes
                                    else "gemm_square_" + args.gemm_sizes.replace(",", "_")),
                       "value_at": f"N={top['N']}",
                       "tile": "256x256 when that fills the SMs, else 256x128", "sms": sms,
                       "l2": "flushed before every timed launch",
                       "parallelism": f"replicated per GPU x{world}"},
            "pct_of_peak": top["tflops"] / peaks["bf16_tflops"],
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": launches, "clocks": clocks, "sweep": sweep,
        }
        print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- FP8 leg
FP8_METRIC = "attention fwd TFLOP/s (fp8 e4m3 operands, causal, N=4096 d=128)"


def run_fp8(args, rank, world, local_rank, dist):
    """fa_fwd_fp8 on the benchmark workload's shape: E4M3 Q, K, V with
    per-head descale factors (inputs.fp8_qkv), bf16 O, fp32 lse."""
    import tiled_attention_20_b200.fa as fa
    from tiled_attention_20_b200 import build as fa_build
    if rank == 0 or world == 1:
        fa_build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = WORKLOAD
    host = inputs.fp8_qkv(w.B, w.H, w.N, w.d, seed=ranks.rank_seed(w.seed, rank), dist=w.dist)
    q8, k8, v8, fq, fk, fv = (t.to(dev) for t in host)
    o = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)

    def step():
        fa.fwd_fp8(q8, k8, v8, fq, fk, fv, causal=w.causal, out=o, lse=lse)

    step()
    fa.check_device_errors(dev)
    if not torch.isfinite(o).all():
        raise RuntimeError("non-finite FP8 output")
    for _ in range(max(0, args.warmup - 1)):
        step()
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(dev.index if world == 1 else local_rank)
    sampler.start()
    time.sleep(0.4)
    for _ in range(max(3, args.warmup)):
        step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    fa.trace_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    traced = fa.trace_stop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    fa.check_device_errors(dev)
    ms = ranks.max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, dev)
    flops = perf.attention_flops(w.B, w.H, w.N, w.d, w.causal, False)
    value = ranks.weak_scaling_rate(flops, world, ms) / 1e12
    n_l, t_l = traced["fa_fwd_kernel"]
    launch_ms = t_l / n_l
    peaks, peaks_src = measured_peaks()
    peak8 = 2.0 * peaks["bf16_tflops"]  # nominal dense fp8 / bf16 ratio: 4.5 / 2.25
    achieved = flops / (launch_ms * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak8, "unit": "TFLOP/s",
            "frac": achieved / peak8, "traffic": profiled_traffic("fa_fwd_kernel:fp8"),
            "kernel": "fa_fwd_kernel (fp8)",
            "peak_source": f"{peaks_src} bf16_tflops (burst) x 2, the nominal fp8/bf16 ratio",
            "launch_ms": launch_ms}
    kernels = {name: {"launches": n, "avg_ms": t / n} for name, (n, t) in traced.items()}

    e2e = None
    if not args.no_e2e:
        host_in = [t.pin_memory() for t in host[:3]]
        host_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (o, lse)]
        dev_in = [[q8, k8, v8], [torch.empty_like(t) for t in (q8, k8, v8)]]
        dev_out = [[o, lse], [torch.empty_like(t) for t in (o, lse)]]

        def run(kset):
            qq, kk, vv = dev_in[kset]
            fa.fwd_fp8(qq, kk, vv, fq, fk, fv, causal=w.causal, out=dev_out[kset][0],
                       lse=dev_out[kset][1])

        n_e2e = max(1, args.e2e_steps)
        ms_e2e = ranks.max_over_ranks(
            pipelined_e2e(dev, host_in, dev_in, dev_out, host_out, run, n_e2e, dist), dist, dev)
        fa.check_device_errors(dev)
        nb = lambda ts: sum(t.numel() * t.element_size() for t in ts)
        e2e = {"value": ranks.weak_scaling_rate(flops, world, ms_e2e) / 1e12, "unit": UNIT,
               "h2d_bytes_per_step": nb(host_in), "d2h_bytes_per_step": nb(host_out),
               "steps": n_e2e, "ms_per_step": ms_e2e,
               "pipeline": "two buffer sets; uploads and downloads overlap the kernels",
               "api": "tiled_attention_20_b200.fa.fwd_fp8 (C ABI)"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle  # CPU-baseline leg: the fp64 oracle on the dequantised inputs
        t0 = time.time()
        heads = 0
        while heads < w.B * w.H and time.time() - t0 < args.cpu_seconds:
            b, h = divmod(heads, w.H)
            deq = [host[i][b:b + 1, h:h + 1].to(torch.float64) * float(host[3 + i][b, h])
                   for i in range(3)]
            oracle.fwd(*deq, causal=w.causal)
            heads += 1
        el = time.time() - t0
        cpu = {"value": perf.attention_flops(1, 1, w.N, w.d, w.causal, False) * heads / el / 1e12,
               "unit": UNIT, "cores": oracle.num_threads(), "kind": "oracle",
               "sample": f"{heads} of {w.B * w.H} heads, forward in fp64 on the dequantised "
                         f"inputs, {el:.1f} s wall"}

    if rank == 0:
        line = {
            "metric": FP8_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "e4m3", "data": "synthetic",
            "config": workload_config(w, {"passes": "fwd", "operands": "e4m3, per-head descale",
                                          "parallelism": f"heads replicated per GPU x{world}"}),
            "pct_of_peak": value / world / peak8,
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": sum(n for n, _ in traced.values()), "kernels": kernels,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def run_decode(args, rank, world, local_rank, dist):
    import tiled_attention_20_b200.fa as fa
    from tiled_attention_20_b200 import build as fa_build
    if rank == 0 or world == 1:
        fa_build.build()
    if world > 1:
        dist.barrier()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = DECODE_WORKLOADS[args.decode]
    q_h, k_h, v_h, lens_h = inputs.decode_qkv(w.B, w.H, w.Nq, w.L, w.d,
                                              seed=ranks.rank_seed(w.seed, rank), ragged=w.ragged)
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    lens = lens_h.to(dev) if w.ragged else None
    o = torch.empty((w.B, w.H, w.Nq, w.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.H, w.Nq), dtype=torch.float32, device=dev)
    ws = torch.zeros(max(fa.decode_workspace_size(w.B, w.H, w.Nq, w.L, w.d), 16),
                     dtype=torch.uint8, device=dev)
    splits, chunk = fa.decode_plan(w.B * w.H, w.Nq, w.L, w.d,
                                   sms=torch.cuda.get_device_properties(dev).multi_processor_count)

    def step():
        fa.decode(q, k, v, cache_lens=lens, causal=w.causal, out=o, lse=lse, workspace=ws)

    step()
    fa.check_device_errors(dev)
    if not torch.isfinite(o).all():
        raise RuntimeError("non-finite decode output")
    for _ in range(max(0, args.warmup - 1)):
        step()
    stream = torch.cuda.current_stream(dev)
    sampler = ClockSampler(dev.index if world == 1 else local_rank)
    sampler.start()
    time.sleep(0.4)
    for _ in range(max(3, args.warmup)):
        step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    fa.trace_start()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    traced = fa.trace_stop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    fa.check_device_errors(dev)
    ms = ranks.max_over_ranks(e0.elapsed_time(e1) / args.steps, dist, dev)
    nbytes = decode_bytes(w, lens_h.tolist())
    value = nbytes * world / (ms * 1e-3) / 1e9
    n_l, t_l = traced["fa_decode_kernel"]
    launch_ms = t_l / n_l
    peaks, peaks_src = measured_peaks()
    achieved = nbytes / (launch_ms * 1e-3) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic(
                "fa_decode_kernel:" + w.name), "kernel": "fa_decode_kernel",
            "peak_source": f"{peaks_src} hbm_gbs (copy)", "launch_ms": launch_ms,
            "algorithmic_bytes": nbytes}
    kernels = {name: {"launches": n, "avg_ms": t / n} for name, (n, t) in traced.items()}

    e2e = None
    if not args.no_e2e:
        # The cache is resident state; a step's inputs are its new queries and
        # its results the attention output and lse.
        hq = q_h.pin_memory()
        ho = torch.empty(o.shape, dtype=torch.bfloat16).pin_memory()
        hlse = torch.empty(lse.shape, dtype=torch.float32).pin_memory()

        def e2e_step():
            q.copy_(hq, non_blocking=True)
            step()
            ho.copy_(o, non_blocking=True)
            hlse.copy_(lse, non_blocking=True)

        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        n_e2e = max(1, args.e2e_steps)
        e0.record(stream)
        for _ in range(n_e2e):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ms_e2e = ranks.max_over_ranks(e0.elapsed_time(e1) / n_e2e, dist, dev)
        nb = lambda *ts: sum(t.numel() * t.element_size() for t in ts)
        e2e = {"value": nbytes * world / (ms_e2e * 1e-3) / 1e9, "unit": DECODE_UNIT,
               "h2d_bytes_per_step": nb(hq), "d2h_bytes_per_step": nb(ho, hlse),
               "steps": n_e2e, "ms_per_step": ms_e2e,
               "api": "tiled_attention_20_b200.fa.decode (C ABI), cache resident"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, heads, cores, el = cpu_oracle_decode_rate(q_h, k_h, v_h, lens_h, w, args.cpu_seconds)
        cpu = {"value": rate, "unit": DECODE_UNIT, "cores": cores, "kind": "oracle",
               "sample": f"{heads} of {w.B * w.H} heads of the workload in fp64, {el:.1f} s wall"}

    if rank == 0:
        cfg = {"workload": w.name, "B": w.B, "H": w.H, "Nq": w.Nq, "L": w.L, "d": w.d,
               "causal": w.causal, "ragged": w.ragged, "seed": w.seed, "splits": splits,
               "chunk_keys": chunk, "l2": "inputs_exceed_l2 (no flush)" if nbytes > 126e6
               else "inputs_fit_l2",
               "parallelism": f"heads replicated per GPU x{world}"}
        line = {
            "metric": DECODE_METRIC, "value": value, "unit": DECODE_UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic", "config": cfg,
            "pct_of_peak": value / world / peaks["hbm_gbs"],
            "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": sum(n for n, _ in traced.values()), "kernels": kernels,
            "clocks": clocks,
        }
        print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    info = ranks.rank_info()
    world, rank, local_rank = info.world, info.rank, info.local_rank
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if args.cpu_table:
        if rank == 0:
            run_cpu_table(args)
        return
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        if args.decode:
            run_decode(args, rank, world, local_rank, dist)
        elif args.fp8:
            run_fp8(args, rank, world, local_rank, dist)
        elif args.gemm_sweep:
            run_gemm_sweep(args, rank, world, local_rank, dist)
        elif args.sweep:
            run_sweep(args, rank, world, local_rank, dist)
        else:
            run_ours(args, rank, world, local_rank, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
