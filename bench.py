#!/usr/bin/env python
"""Benchmark of the block-quantized projection path on B200.

One step = the paired Q8_0 decode projection workload: 64 back-to-back calls,
each quantizing a fresh fp32 activation (1 x 4096) to Q8 and running the
paired GEMV of two Q8_0 weights (8192 x 4096 each) against it, both in one
launch (dsq_gemv_paired_f32); the same calls as two launches each
(dsq_quantize_act_q8, then dsq_gemv_paired) are timed beside it.  Weights are
rotated over enough copies that L2 (126 MB) cannot serve them.  The headline
value is HBM GB/s of algorithmic bytes; the same JSON line also carries
us/call, the roofline of the dominant kernel, an end-to-end figure through
the public API with host buffers, the other decode workloads and the prefill
dequant-GEMM TFLOP/s sweep, the CPU oracle baseline and clock samples.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import platform
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_PAIR, K_PAIR, CALLS = 8192, 4096, 64
L2_BYTES = 126 * 1024 * 1024
METRIC = "decode GEMV HBM GB/s (% peak) and µs/call; prefill dequant-GEMM TFLOP/s"
WORKLOAD = "paired Q8_0 decode projection: 2 x (8192 x 4096) weights, shared 1 x 4096 activation, 64 calls"


def paired_bytes_per_call() -> dict:
    """Algorithmic bytes of one call.  fused: the one-launch form (weights,
    the fp32 activation, the outputs); two_call: the quantize step (x in,
    codes, scales and sums out) plus the paired GEMV on the codes (gemv)."""
    rb = K_PAIR // 32 * 34
    weights, out = 2 * N_PAIR * rb, 2 * N_PAIR * 4
    gemv = weights + K_PAIR + (K_PAIR // 32) * 4 + out
    quant = K_PAIR * 4 + K_PAIR + 2 * (K_PAIR // 32) * 4
    return {"fused": weights + K_PAIR * 4 + out, "gemv": gemv, "quant": quant, "two_call": gemv + quant}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def traffic_record(kernel: str, workload: str):
    """dram read+write bytes per launch from the committed ncu summary, or
    None when the kernel source changed since the counters were taken."""
    src = os.path.join(ROOT, "block_quantized_dsq_b200", "csrc", "gemv.cu")
    sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    for line in open(path):
        parts = line.split()
        if len(parts) == 4 and parts[0] == kernel and parts[1] == workload:
            return int(parts[3]) if parts[2] == sha else None
    return None


# ------------------------------------------------------------------ clocks --
class ClockSampler(threading.Thread):
    """Polls SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, torch_device: int, period: float = 0.01):
        super().__init__(daemon=True)
        self.period = period
        self.samples = []
        self.error = None
        self._halt = threading.Event()
        self.handle = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            pr = torch.cuda.get_device_properties(torch_device)
            bus = f"{pr.pci_domain_id:08X}:{pr.pci_bus_id:02X}:{pr.pci_device_id:02X}.0"
            self.nv = pynvml
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report, do not fail the bench
            self.error = f"{type(e).__name__}: {e}"

    def _reasons(self):
        nv = self.nv
        fn = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            getattr(nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
        return fn(self.handle)

    def sample(self):
        self.samples.append((self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM), self._reasons()))

    def run(self):
        if self.handle is None:
            return
        while not self._halt.is_set():
            try:
                self.sample()
            except Exception as e:
                self.error = str(e)
                return
            time.sleep(self.period)

    def stop(self):
        self._halt.set()
        if self.is_alive():
            self.join()
        if self.handle is not None and not self.samples:
            try:
                self.sample()
            except Exception:
                pass

    def summary(self):
        if self.handle is None:
            return {"error": self.error}
        busy = [s for s in self.samples if not (s[1] & 0x1)] or self.samples
        reasons = set()
        for _, r in busy:
            for bit, name in self.REASONS.items():
                if r & bit and bit != 0x1:
                    reasons.add(name)
        return {"sm_mhz": statistics.median([s[0] for s in busy]) if busy else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(reasons), "samples": len(self.samples)}


# -------------------------------------------------------------- helpers ----
def dist_setup():
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(local)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(world, v: float) -> float:
    """The largest of the ranks' values (device times: the slowest rank sets
    the job's time).  NCCL reduces a device tensor, gloo a host one."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def quantized_weights(dsq, qtype, seed, N, K):
    """Seeded N(0, 0.02^2) fp32 weights, quantized on the device by libdsq."""
    import torch

    from block_quantized_dsq_b200 import synth
    w32 = torch.from_numpy(synth.weights(seed, N, K)).cuda()
    w = torch.empty((N, dsq.dsq_row_bytes(qtype, K)), dtype=torch.uint8, device="cuda")
    dsq.dsq_quantize_weights(qtype, w32, N, K, w)
    del w32
    return w


def copies_for(nbytes: int, lo: int = 2) -> int:
    """Enough copies that the others exceed 3x L2 between two uses of one."""
    return max(lo, -(-3 * L2_BYTES // max(nbytes, 1)) + 1)


def paired_copies() -> int:
    """Weight copies the headline rotates over: past 3x L2, and the last call
    of a step and the first of the next never read the same copy."""
    R = copies_for(paired_bytes_per_call()["gemv"])
    while (CALLS - 1) % R == 0:
        R += 1
    return R


def bench_config(world: int) -> dict:
    """The workload description both arms print."""
    R = paired_copies()
    return {"workload": WORKLOAD, "weights": "N(0,0.02^2) fp32 quantized to Q8_0, seeds 1/2",
            "activations": "N(0,1) fp32, seeds 1000..1063, quantized to Q8 per call inside the GEMV launch",
            "l2": f"weights rotated over {R} copies ({R * paired_bytes_per_call()['gemv'] / 1e6:.0f} MB > 3x L2)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU"}


PROFILE = False   # --profile: run each selected workload a few times, untimed


def profile_calls(fn, n: int = 3):
    """Profile mode: n eager calls, no timing (for ncu captures)."""
    import torch
    st = torch.cuda.current_stream().cuda_stream
    for i in range(n):
        fn(i, st)
    torch.cuda.synchronize()
    return float("nan")


def time_calls(fn, n_calls: int, warmup: int = 5):
    """Device time per call (CUDA events around a batch of eager calls)."""
    import torch
    if PROFILE:
        return profile_calls(fn)
    st = torch.cuda.current_stream().cuda_stream
    for i in range(warmup):
        fn(i, st)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(n_calls):
        fn(i, st)
    e1.record()
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / 1e3 / n_calls


def time_graph(fn, calls_per_graph: int, replays: int = 21):
    """Device time per call with the calls captured in a CUDA graph, so host
    launch cost cannot hide in the figure.  Each replay is bracketed by its
    own CUDA events on the replay stream; returns the median per-call time
    and sets LAST_STATS to {median, min, max, replays} in microseconds."""
    import torch
    global LAST_STATS
    if PROFILE:
        return profile_calls(fn)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for i in range(3):
            fn(i, side.cuda_stream)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = torch.cuda.current_stream().cuda_stream
        for i in range(calls_per_graph):
            fn(i, st)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(replays + 1)]
    ev[0].record()
    for r in range(replays):
        g.replay()
        ev[r + 1].record()
    torch.cuda.synchronize()
    per_call = sorted(ev[r].elapsed_time(ev[r + 1]) / 1e3 / calls_per_graph for r in range(replays))
    del g
    LAST_STATS = {"median_us": round(statistics.median(per_call) * 1e6, 3), "min_us": round(per_call[0] * 1e6, 3),
                  "max_us": round(per_call[-1] * 1e6, 3), "replays": replays, "calls_per_replay": calls_per_graph}
    return statistics.median(per_call)


LAST_STATS: dict = {}


# ------------------------------------------------------------- the bench ---
def run_dsq(args, world, rank):
    import torch

    import block_quantized_dsq_b200 as dsq
    from block_quantized_dsq_b200 import synth
    from block_quantized_dsq_b200.build import build
    build()
    stream = torch.cuda.current_stream().cuda_stream
    L = dsq.lib()
    hbm_peak, bf16_peak, bf16_sust, peak_src = measured_peaks()

    # ---- paired workload: weights (rotated copies), 64 fresh activations
    seeds = synth.SEEDS["paired_q8_0_2x8192x4096"]
    W0 = quantized_weights(dsq, dsq.DSQ_Q8_0, seeds["w0"], N_PAIR, K_PAIR)
    W1 = quantized_weights(dsq, dsq.DSQ_Q8_0, seeds["w1"], N_PAIR, K_PAIR)
    bpc = paired_bytes_per_call()
    R = paired_copies()
    pairs = [(W0, W1)] + [(W0.clone(), W1.clone()) for _ in range(R - 1)]
    X_host = __import__("numpy").concatenate(
        [synth.activations(seeds["x_base"] + i, 1, K_PAIR) for i in range(CALLS)])
    X = torch.from_numpy(X_host).cuda()
    xq = torch.empty((CALLS, K_PAIR), dtype=torch.int8, device="cuda")
    xd = torch.empty((CALLS, K_PAIR // 32), dtype=torch.float32, device="cuda")
    xs = torch.empty((CALLS, K_PAIR // 32), dtype=torch.int32, device="cuda")
    Y = torch.empty((CALLS, 2, N_PAIR), dtype=torch.float32, device="cuda")
    p_x = [X[i].data_ptr() for i in range(CALLS)]
    p_xq = [xq[i].data_ptr() for i in range(CALLS)]
    p_xd = [xd[i].data_ptr() for i in range(CALLS)]
    p_xs = [xs[i].data_ptr() for i in range(CALLS)]
    p_y0 = [Y[i, 0].data_ptr() for i in range(CALLS)]
    p_y1 = [Y[i, 1].data_ptr() for i in range(CALLS)]
    p_w = [(a.data_ptr(), b.data_ptr()) for a, b in pairs]
    quant, paired, fused = L.dsq_quantize_act_q8, L.dsq_gemv_paired, L.dsq_gemv_paired_f32

    def one_call(c, st, form):
        """form: "fused" (the step: one launch quantizes x and runs the paired
        GEMV), "two_call" (quantize, then the GEMV on the codes) or "gemv"
        (the GEMV alone on codes already made)."""
        w0, w1 = p_w[c % R]
        if form == "fused":
            rc = fused(8, w0, N_PAIR, w1, N_PAIR, K_PAIR, p_x[c], p_y0[c], p_y1[c], st)
        else:
            rc = quant(p_x[c], 1, K_PAIR, p_xq[c], p_xd[c], p_xs[c], st) if form == "two_call" else 0
            rc |= paired(8, w0, N_PAIR, w1, N_PAIR, K_PAIR, p_xq[c], p_xd[c], p_xs[c], p_y0[c], p_y1[c], st)
        if rc:
            raise RuntimeError(dsq.dsq_last_error())

    def capture(form):
        """One step (64 calls) as a CUDA graph: the decode loop's launch
        pattern without host launch overhead between the kernels."""
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for c in range(CALLS):
                one_call(c, side.cuda_stream, form)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        n0 = dsq.dsq_launch_count()
        with torch.cuda.graph(g):
            st = torch.cuda.current_stream().cuda_stream
            for c in range(CALLS):
                one_call(c, st, form)
        return g, dsq.dsq_launch_count() - n0

    def replay_avg(graph, reps):
        """Average time of one replay over `reps` back-to-back replays."""
        graph.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            graph.replay()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 1e3 / reps

    step_graph, launches_per_step = capture("fused")
    for _ in range(args.warmup):
        step_graph.replay()
    torch.cuda.synchronize()
    assert dsq.dsq_device_status() == 0

    sampler = ClockSampler(torch.cuda.current_device())
    barrier(world)
    torch.cuda.synchronize()
    sampler.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record()
    for _ in range(args.steps):
        step_graph.replay()
    t1.record()
    torch.cuda.synchronize()
    barrier(world)
    sampler.stop()
    elapsed = max_over_ranks(world, t0.elapsed_time(t1) / 1e3)
    launches = launches_per_step * args.steps
    assert dsq.dsq_device_status() == 0, "a device wait timed out during the bench"
    ms_per_step = elapsed / args.steps * 1e3
    value = world * args.steps * CALLS * bpc["fused"] / elapsed / 1e9
    # the step is one kernel launch per call: the dominant kernel's average
    # launch duration is the timed region over its launches
    kern_avg = elapsed / launches

    # ---- the same step as two launches per call (quantize, then the GEMV on
    # the codes), and the GEMV alone, for comparison
    reps = max(3, args.steps // 4)
    two_graph, _ = capture("two_call")
    two_avg = replay_avg(two_graph, reps) / CALLS
    gemv_graph, _ = capture("gemv")
    gemv_avg = replay_avg(gemv_graph, reps) / CALLS
    del gemv_graph, two_graph, step_graph

    # ---- end to end through the public API with host buffers
    X_pin = torch.from_numpy(X_host).pin_memory()
    Y_pin = torch.empty((CALLS, 2, N_PAIR), dtype=torch.float32).pin_memory()
    e2e_steps = max(1, min(args.steps, 100))

    def e2e_step(s):
        X.copy_(X_pin, non_blocking=True)
        for c in range(CALLS):
            w0, w1 = p_w[c % R]
            dsq.dsq_gemv_paired_f32(8, w0, N_PAIR, w1, N_PAIR, K_PAIR, p_x[c], p_y0[c], p_y1[c], stream)
        Y_pin.copy_(Y, non_blocking=True)

    e2e_t = time_calls(lambda s_, st_: e2e_step(s_), e2e_steps, warmup=2)
    e2e_t = max_over_ranks(world, e2e_t)
    e2e_value = world * CALLS * bpc["fused"] / e2e_t / 1e9

    # ---- the other rows of the path (each its own short timed loop)
    rows, rows_clocks = {}, None
    if not args.skip_rows:
        rs = ClockSampler(torch.cuda.current_device(), period=0.05)
        rs.start()
        rows = measure_rows(dsq, L, stream, hbm_peak, bf16_peak,
                            only=set(args.rows.split(",")) if args.rows else None)
        rs.stop()
        rows_clocks = rs.summary()

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": bench_config(world),
        "us_per_call": round(ms_per_step * 1e3 / CALLS, 3),
        "hbm_frac": round(value / world / hbm_peak, 4),
        "timing": "CUDA graph of one step (64 calls of dsq_gemv_paired_f32: each quantizes its fp32 "
                  "activation and runs the paired GEMV in one launch, programmatic launch) replayed "
                  f"{args.steps} times; CUDA events on the replay stream",
        "roofline": {"bound": "hbm", "kernel": "gemv_kernel (paired Q8_0, activation quantized in the kernel)",
                     "achieved": round(bpc["fused"] / kern_avg / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(bpc["fused"] / kern_avg / 1e9 / hbm_peak, 4),
                     "traffic": traffic_record("gemv_kernel", "paired_f32_q8_0_2x8192x4096"),
                     "algorithmic_bytes": bpc["fused"], "avg_launch_us": round(kern_avg * 1e6, 3),
                     "measured": "the timed region over its launches (one per call)",
                     "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured"
                     else "fallback"},
        "two_call": {"us_per_call": round(two_avg * 1e6, 3), "GB/s": round(bpc["two_call"] / two_avg / 1e9, 1),
                     "gemv_us_per_call": round(gemv_avg * 1e6, 3),
                     "gemv_GB/s": round(bpc["gemv"] / gemv_avg / 1e9, 1),
                     "measured": f"{reps} replays of a graph of the 64 calls as dsq_quantize_act_q8 + "
                                 "dsq_gemv_paired, and of the 64 paired GEMVs alone"},
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": CALLS * K_PAIR * 4,
                "d2h_bytes_per_step": CALLS * 2 * N_PAIR * 4, "us_per_call": round(e2e_t / CALLS * 1e6, 3)},
        "gpu_launches": int(launches),
        "clocks": sampler.summary(),
        "rows": rows,
        "rows_clocks": rows_clocks,
        "rows_timing": "each row: a CUDA graph of calls rotating over weight copies past 3x L2, replayed 21 "
                       "times with CUDA events around every replay; median per call with min/max",
    }
    if rank == 0 and world == 1 and not args.skip_cpu:
        result["cpu_baseline"] = cpu_baseline(pairs[0], X_host, args.cpu_seconds)
        result["cpu_oracle_rows"] = cpu_oracle_rows()
    return result


PREFILL_SWEEP_M = (1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 1024, 2048)
NSWEEP_N = (1024, 2048, 4096, 8192, 16384, 32768, 65536)


def measure_rows(dsq, L, stream, hbm_peak, bf16_peak, only=None):
    """µs/call and GB/s (or TFLOP/s) for every other step of the path;
    `only` restricts the run to the named rows (a row family such as
    `prefill_sweep` or `gemv_nsweep` selects all of its points)."""
    import torch

    from block_quantized_dsq_b200 import synth
    rows = {}

    def want(name):
        return only is None or name in only or any(name.startswith(o + "_") for o in only)

    def act(seed, M, K):
        x = torch.from_numpy(synth.activations(seed, M, K)).cuda()
        xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
        xd = torch.empty((M, K // 32), dtype=torch.float32, device="cuda")
        xs = torch.empty((M, K // 32), dtype=torch.int32, device="cuda")
        dsq.dsq_quantize_act_q8(x, M, K, xq, xd, xs)
        return x, xq, xd, xs

    def stats_row(t, alg_bytes=None, flops=None):
        """One row: median µs/call (with min/max over the replays) and the
        rate of algorithmic bytes and/or flops against the measured peaks."""
        r = {"us_per_call": round(t * 1e6, 3), **{k: v for k, v in LAST_STATS.items()}}
        if alg_bytes is not None:
            gbs = alg_bytes / t / 1e9
            r.update({"GB/s": round(gbs, 1), "hbm_frac": round(gbs / hbm_peak, 4), "algorithmic_bytes": alg_bytes})
        if flops is not None:
            tf = flops / t / 1e12
            r.update({"TFLOP/s": round(tf, 1), "bf16_peak_frac": round(tf / bf16_peak, 4)})
        return r

    # activation prequantization, one decode row of K = 4096
    if want("quantize_act_q8_1x4096"):
        x, xq, xd, xs = act(101, 1, 4096)
        px, pq, pd, ps = x.data_ptr(), xq.data_ptr(), xd.data_ptr(), xs.data_ptr()
        t = time_graph(lambda i, st: L.dsq_quantize_act_q8(px, 1, 4096, pq, pd, ps, st), 500)
        rows["quantize_act_q8_1x4096"] = stats_row(t, 4096 * 4 + 4096 + 1024)

    def gemv_row(name, qtype, N, K, seed, xseed, G=1, fused=False):
        """fused: the *_f32 entry point (fp32 activation quantized in the
        kernel) instead of the two-call path's GEMV alone."""
        if not want(name):
            return
        w = quantized_weights(dsq, qtype, seed, G * N, K)
        nbytes = w.numel()
        R = copies_for(nbytes)
        ws = [w] + [w.clone() for _ in range(R - 1)]
        ptrs = [c.data_ptr() for c in ws]
        x, xq, xd, xs = act(xseed, G, K)
        y = torch.empty((G, N), dtype=torch.float32, device="cuda")
        pq, pd, ps, py = xq.data_ptr(), xd.data_ptr(), xs.data_ptr(), y.data_ptr()
        px = x.data_ptr()
        if fused and G > 1:
            fn = lambda i, st: L.dsq_gemv_grouped_f32(qtype, ptrs[i % R], G, N, K, px, py, st)  # noqa: E731
        elif fused:
            fn = lambda i, st: L.dsq_gemv_f32(qtype, ptrs[i % R], N, K, px, py, st)  # noqa: E731
        elif G > 1:
            fn = lambda i, st: L.dsq_gemv_grouped(qtype, ptrs[i % R], G, N, K, pq, pd, ps, py, st)  # noqa: E731
        elif qtype == dsq.DSQ_Q8_0:
            fn = lambda i, st: L.dsq_gemv_q8_0(ptrs[i % R], N, K, pq, pd, py, st)  # noqa: E731
        else:
            fn = lambda i, st: L.dsq_gemv_q4_k(ptrs[i % R], N, K, pq, pd, ps, py, st)  # noqa: E731
        t = time_graph(fn, R * max(1, 200 // R))
        if fused:
            alg = nbytes + G * K * 4 + G * N * 4
        else:
            alg = nbytes + G * (K + K // 32 * 4 * (2 if qtype == dsq.DSQ_Q4_K else 1)) + G * N * 4
        rows[name] = {**stats_row(t, alg), "weight_copies": R}
        del ws

    seeds = synth.SEEDS
    gemv_row("gemv_q8_0_1024x1024", dsq.DSQ_Q8_0, 1024, 1024, seeds["gemv_q8_0_1024"]["w"],
             seeds["gemv_q8_0_1024"]["x"])
    gemv_row("gemv_q4_k_4096x4096", dsq.DSQ_Q4_K, 4096, 4096, seeds["gemv_q4_k_4096"]["w"],
             seeds["gemv_q4_k_4096"]["x"])
    gemv_row("grouped_q8_0_8x1024x4096", dsq.DSQ_Q8_0, 1024, 4096, seeds["grouped_q8_0_8x1024x4096"]["w_base"],
             seeds["grouped_q8_0_8x1024x4096"]["x_base"], G=8)
    # the same decode GEMVs through the fused entry points (activation fp32
    # in, quantized inside the GEMV: one launch per call)
    gemv_row("f32_gemv_q8_0_1024x1024", dsq.DSQ_Q8_0, 1024, 1024, seeds["gemv_q8_0_1024"]["w"],
             seeds["gemv_q8_0_1024"]["x"], fused=True)
    gemv_row("f32_gemv_q4_k_4096x4096", dsq.DSQ_Q4_K, 4096, 4096, seeds["gemv_q4_k_4096"]["w"],
             seeds["gemv_q4_k_4096"]["x"], fused=True)
    gemv_row("f32_grouped_q8_0_8x1024x4096", dsq.DSQ_Q8_0, 1024, 4096,
             seeds["grouped_q8_0_8x1024x4096"]["w_base"], seeds["grouped_q8_0_8x1024x4096"]["x_base"], G=8,
             fused=True)
    if want("f32_paired_q8_0_2x8192x4096"):
        sp = seeds["paired_q8_0_2x8192x4096"]
        W0 = quantized_weights(dsq, dsq.DSQ_Q8_0, sp["w0"], N_PAIR, K_PAIR)
        W1 = quantized_weights(dsq, dsq.DSQ_Q8_0, sp["w1"], N_PAIR, K_PAIR)
        nb2 = W0.numel() + W1.numel()
        R = copies_for(nb2)
        pw = [(W0.data_ptr(), W1.data_ptr())]
        keep = []
        for _ in range(R - 1):
            c0, c1 = W0.clone(), W1.clone()
            keep += [c0, c1]
            pw.append((c0.data_ptr(), c1.data_ptr()))
        xs_ = torch.from_numpy(synth.activations(sp["x_base"], 1, K_PAIR)).cuda()
        y2 = torch.empty((2, N_PAIR), dtype=torch.float32, device="cuda")
        px, py0, py1 = xs_.data_ptr(), y2[0].data_ptr(), y2[1].data_ptr()
        fn = lambda i, st: L.dsq_gemv_paired_f32(dsq.DSQ_Q8_0, pw[i % R][0], N_PAIR, pw[i % R][1], N_PAIR,  # noqa: E731
                                                 K_PAIR, px, py0, py1, st)
        t = time_graph(fn, R * max(1, 128 // R))
        rows["f32_paired_q8_0_2x8192x4096"] = {**stats_row(t, nb2 + K_PAIR * 4 + 2 * N_PAIR * 4),
                                               "weight_copies": R}
        del keep, W0, W1

    # multi-token decode GEMV (dsq_gemv_tokens): M = 1..8 tokens per weight
    # read, next to M single-token GEMV calls on the same weights
    for qtype, tag, N, N1 in ((dsq.DSQ_Q4_K, "q4_k_4096x4096", 4096, 0),
                              (dsq.DSQ_Q8_0, "paired_q8_0_2x8192x4096", N_PAIR, N_PAIR)):
        Ms = [M for M in (1, 2, 4, 8) if want(f"tokens_{tag}_m{M}")]
        if not Ms:
            continue
        K = 4096
        w = quantized_weights(dsq, qtype, 620 + qtype, N + N1, K)
        R = copies_for(w.numel())
        ws = [w] + [w.clone() for _ in range(R - 1)]
        rbw = dsq.dsq_row_bytes(qtype, K)
        p0 = [c.data_ptr() for c in ws]
        x, xq, xd, xs = act(621, 8, K)
        pq, pd, ps = xq.data_ptr(), xd.data_ptr(), xs.data_ptr()
        y = torch.empty((8, N + N1), dtype=torch.float32, device="cuda")
        py = y.data_ptr()
        for M in Ms:
            fn = lambda i, st, M=M: L.dsq_gemv_tokens(  # noqa: E731
                qtype, p0[i % R], N, p0[i % R] + N * rbw if N1 else None, N1, K, M, pq, pd, ps, py,
                py + M * N * 4 if N1 else None, st)
            t = time_graph(fn, R * max(1, 64 // R))
            alg = w.numel() + M * (K + K // 32 * 4 * (2 if qtype == dsq.DSQ_Q4_K else 1)) + M * (N + N1) * 4
            row = {**stats_row(t, alg), "weight_copies": R, "tokens": M}
            # the same M tokens as M single-token calls, each reading its weights from HBM
            if N1:
                fn1 = lambda i, st, M=M: [L.dsq_gemv_paired(  # noqa: E731
                    qtype, p0[(i * M + m) % R], N, p0[(i * M + m) % R] + N * rbw, N1, K, pq + m * K,
                    pd + m * K // 8, ps + m * K // 8, py, py + N * 4, st) for m in range(M)]
            elif qtype == dsq.DSQ_Q8_0:
                fn1 = lambda i, st, M=M: [L.dsq_gemv_q8_0(p0[(i * M + m) % R], N, K, pq + m * K,  # noqa: E731
                                                          pd + m * K // 8, py, st) for m in range(M)]
            else:
                fn1 = lambda i, st, M=M: [L.dsq_gemv_q4_k(p0[(i * M + m) % R], N, K, pq + m * K,  # noqa: E731
                                                          pd + m * K // 8, ps + m * K // 8, py, st)
                                          for m in range(M)]
            t1 = time_graph(fn1, max(1, 64 // M))
            row["m_single_calls_us"] = round(t1 * 1e6, 3)
            rows[f"tokens_{tag}_m{M}"] = row
        del ws, w

    # decode GEMV N-sweep at K = 4096: the asymptotic HBM fraction once the
    # launch and first-byte latency are amortised over more rows.  The rows
    # of a 4096-row seeded matrix are repeated on the device (distinct
    # addresses; the weight stream does not depend on the values).
    K = 4096
    for qtype, tag in ((dsq.DSQ_Q8_0, "q8_0"), (dsq.DSQ_Q4_K, "q4_k")):
        Ns = [N for N in NSWEEP_N if want(f"gemv_nsweep_{tag}_n{N}")]
        if not Ns:
            continue
        base = quantized_weights(dsq, qtype, 600 + qtype, 4096, K)
        x, xq, xd, xs = act(601, 1, K)
        pq, pd, ps = xq.data_ptr(), xd.data_ptr(), xs.data_ptr()
        for N in Ns:
            w = base.repeat((N + 4095) // 4096, 1)[:N].contiguous()
            R = copies_for(w.numel())
            ws = [w] + [w.clone() for _ in range(R - 1)]
            ptrs = [c.data_ptr() for c in ws]
            y = torch.empty(N, dtype=torch.float32, device="cuda")
            py = y.data_ptr()
            if qtype == dsq.DSQ_Q8_0:
                fn = lambda i, st, ptrs=ptrs, R=R, N=N, py=py: L.dsq_gemv_q8_0(  # noqa: E731
                    ptrs[i % R], N, K, pq, pd, py, st)
            else:
                fn = lambda i, st, ptrs=ptrs, R=R, N=N, py=py: L.dsq_gemv_q4_k(  # noqa: E731
                    ptrs[i % R], N, K, pq, pd, ps, py, st)
            t = time_graph(fn, R * max(1, 64 // R))
            alg = w.numel() + K + K // 32 * 4 * (2 if qtype == dsq.DSQ_Q4_K else 1) + N * 4
            rows[f"gemv_nsweep_{tag}_n{N}"] = {**stats_row(t, alg), "weight_copies": R}
            del ws, w, y
        del base

    # prefill dequant-GEMM M sweep (1 .. 2048) for both weight types; for
    # M <= 64 the same M tokens as M separate decode calls (quantize the M
    # rows once, then one GEMV per token, each reading its weights from HBM)
    for qtype, N, tag in ((dsq.DSQ_Q4_K, 4096, "q4_k_n4096"), (dsq.DSQ_Q8_0, 8192, "q8_0_n8192")):
        Ms = [M for M in PREFILL_SWEEP_M if want(f"prefill_{tag}_m{M}")]
        if not Ms:
            continue
        w = quantized_weights(dsq, qtype, seeds["prefill"]["w_q4_k" if qtype == dsq.DSQ_Q4_K else "w_q8_0"], N, K)
        wbytes = w.numel()
        R = copies_for(wbytes)
        ws = [w] + [w.clone() for _ in range(R - 1)]
        pw = [c.data_ptr() for c in ws]
        for M in Ms:
            x = torch.from_numpy(synth.activations(seeds["prefill"]["x_base"] + M, M, K)).cuda()
            y = torch.empty((M, N), dtype=torch.float32, device="cuda")
            nb = dsq.dsq_prefill_workspace_bytes(qtype, N, K, M)
            wsp = torch.empty(nb, dtype=torch.uint8, device="cuda")
            px, py, pws = x.data_ptr(), y.data_ptr(), wsp.data_ptr()
            t = time_graph(lambda i, st: L.dsq_gemm_prefill(qtype, pw[i % R], N, K, px, M, py, pws, nb, st),
                           R * max(1, 24 // R))
            flops = 2.0 * M * N * K
            alg = wbytes + 4 * M * K + 4 * M * N
            bound_t = max(flops / (bf16_peak * 1e12), alg / (hbm_peak * 1e9))
            row = {**stats_row(t, alg, flops), "weight_copies": R,
                   "bound": "tensor" if flops / (bf16_peak * 1e12) >= alg / (hbm_peak * 1e9) else "hbm",
                   "roofline_frac": round(bound_t / t, 4)}
            if M <= 64:
                xq = torch.empty((M, K), dtype=torch.int8, device="cuda")
                xd = torch.empty((M, K // 32), dtype=torch.float32, device="cuda")
                xs = torch.empty((M, K // 32), dtype=torch.int32, device="cuda")
                pq, pd, ps = xq.data_ptr(), xd.data_ptr(), xs.data_ptr()
                rbq = K  # xq row stride (int8)
                rbd = K // 32 * 4

                def per_token(i, st, M=M, pq=pq, pd=pd, ps=ps, px=px, py=py):
                    L.dsq_quantize_act_q8(px, M, K, pq, pd, ps, st)
                    for m in range(M):
                        wp = pw[(i * M + m) % R]
                        if qtype == dsq.DSQ_Q8_0:
                            L.dsq_gemv_q8_0(wp, N, K, pq + m * rbq, pd + m * rbd, py + m * N * 4, st)
                        else:
                            L.dsq_gemv_q4_k(wp, N, K, pq + m * rbq, pd + m * rbd, ps + m * rbd, py + m * N * 4,
                                            st)
                t2 = time_graph(per_token, max(1, 48 // M))
                row["m_decode_calls_us"] = round(t2 * 1e6, 3)
                row["m_decode_calls_stats"] = dict(LAST_STATS)
                if M <= 8:
                    # the same tokens through the multi-token GEMV: one
                    # quantize of the M rows, one weight read for all of them
                    def tokens(i, st, M=M, pq=pq, pd=pd, ps=ps, px=px, py=py):
                        L.dsq_quantize_act_q8(px, M, K, pq, pd, ps, st)
                        L.dsq_gemv_tokens(qtype, pw[i % R], N, None, 0, K, M, pq, pd, ps, py, None, st)
                    t3 = time_graph(tokens, R * max(1, 24 // R))
                    row["tokens_call_us"] = round(t3 * 1e6, 3)
                    row["tokens_call_stats"] = dict(LAST_STATS)
                del xq, xd, xs
            rows[f"prefill_{tag}_m{M}"] = row
            del x, y, wsp
        del ws, w
    # grouped attention-A prefill: two Q4_K weights (4096 and 1024 rows) that
    # read the same X, one launch against two back-to-back single calls
    for M in (512, 2048):
        name = f"prefill_grouped_q4_k_4096+1024_m{M}"
        if not want(name):
            continue
        Ns = [4096, 1024]
        wl = [quantized_weights(dsq, dsq.DSQ_Q4_K, 630 + g, n, K) for g, n in enumerate(Ns)]
        wbytes = sum(w.numel() for w in wl)
        R = copies_for(wbytes)
        copies = [wl] + [[w.clone() for w in wl] for _ in range(R - 1)]
        x = torch.from_numpy(synth.activations(631 + M, M, K)).cuda()
        ys = [torch.empty((M, n), dtype=torch.float32, device="cuda") for n in Ns]
        nbg = dsq.dsq_prefill_grouped_workspace_bytes(dsq.DSQ_Q4_K, Ns, K, M)
        wsg = torch.empty(nbg, dtype=torch.uint8, device="cuda")
        nbs = [dsq.dsq_prefill_workspace_bytes(dsq.DSQ_Q4_K, n, K, M) for n in Ns]
        wss = [torch.empty(b, dtype=torch.uint8, device="cuda") for b in nbs]
        pw = [[w.data_ptr() for w in c] for c in copies]
        arr_n = (ctypes.c_int64 * 2)(*Ns)
        arr_y = (ctypes.c_void_p * 2)(*[y.data_ptr() for y in ys])
        arr_w = [(ctypes.c_void_p * 2)(*p) for p in pw]
        px = x.data_ptr()

        def grouped(i, st):
            L.dsq_gemm_prefill_grouped(dsq.DSQ_Q4_K, 2, arr_w[i % R], arr_n, K, px, M, arr_y, wsg.data_ptr(), nbg, st)

        def singles(i, st):
            for g in range(2):
                L.dsq_gemm_prefill(dsq.DSQ_Q4_K, pw[i % R][g], Ns[g], K, px, M, ys[g].data_ptr(), wss[g].data_ptr(),
                                   nbs[g], st)
        t = time_graph(grouped, R * max(1, 24 // R))
        flops = 2.0 * M * sum(Ns) * K
        row = {**stats_row(t, wbytes + 4 * M * K + 4 * M * sum(Ns), flops), "weight_copies": R}
        t2 = time_graph(singles, R * max(1, 24 // R))
        row["single_calls_us"] = round(t2 * 1e6, 3)
        rows[name] = row
        del copies, wl, wsg, wss
    assert dsq.dsq_device_status() == 0
    return rows


def run_profile(args):
    """Untimed runs of selected workloads for ncu (committed so that every
    profile summary names a command over committed files only)."""
    global PROFILE
    PROFILE = True
    import torch

    import block_quantized_dsq_b200 as dsq
    from block_quantized_dsq_b200.build import build
    build()
    L = dsq.lib()
    stream = torch.cuda.current_stream().cuda_stream
    if not args.skip_headline:
        from block_quantized_dsq_b200 import synth
        seeds = synth.SEEDS["paired_q8_0_2x8192x4096"]
        W0 = quantized_weights(dsq, dsq.DSQ_Q8_0, seeds["w0"], N_PAIR, K_PAIR)
        W1 = quantized_weights(dsq, dsq.DSQ_Q8_0, seeds["w1"], N_PAIR, K_PAIR)
        x = torch.from_numpy(synth.activations(seeds["x_base"], 1, K_PAIR)).cuda()
        xq = torch.empty(K_PAIR, dtype=torch.int8, device="cuda")
        xd = torch.empty(K_PAIR // 32, dtype=torch.float32, device="cuda")
        xs = torch.empty(K_PAIR // 32, dtype=torch.int32, device="cuda")
        y = torch.empty((2, N_PAIR), dtype=torch.float32, device="cuda")
        for _ in range(3):
            dsq.dsq_gemv_paired_f32(8, W0, N_PAIR, W1, N_PAIR, K_PAIR, x, y[0], y[1], stream)
        for _ in range(3):
            dsq.dsq_quantize_act_q8(x, 1, K_PAIR, xq, xd, xs, stream)
            dsq.dsq_gemv_paired(8, W0, N_PAIR, W1, N_PAIR, K_PAIR, xq, xd, xs, y[0], y[1], stream)
        torch.cuda.synchronize()
    hbm_peak, bf16_peak, _, _ = measured_peaks()
    if args.rows:
        measure_rows(dsq, L, stream, hbm_peak, bf16_peak, only=set(args.rows.split(",")))
    assert dsq.dsq_device_status() == 0


def cpu_baseline(pair, X_host, budget_s: float):
    """The CPU oracle (single-threaded C) on a bounded sample of the workload:
    as many of the 64 paired calls as fit in the time budget."""
    import numpy as np

    import oracle as ref
    w0, w1 = pair[0].cpu().numpy(), pair[1].cpu().numpy()
    bpc = paired_bytes_per_call()
    t0 = time.perf_counter()
    n = 0
    while n < CALLS:
        xq, xd, xs = ref.quantize_act_q8(X_host[n:n + 1])
        ref.gemv(8, w0, K_PAIR, xq, xd, xs)
        ref.gemv(8, w1, K_PAIR, xq, xd, xs)
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": round(n * bpc["fused"] / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} of the 64 paired calls (oracle act-quantize + two integer-form GEMVs), {dt:.1f} s",
            "cpu": platform.processor() or platform.machine(), "host_cores": os.cpu_count()}


def cpu_oracle_rows(budget_s: float = 1.5) -> dict:
    """The CPU oracle (single-threaded C, 1 core) per workload, each timed for
    about budget_s seconds: activation quantize, the integer-form GEMV of the
    three other decode workloads, and the fp64 prefill reference on a bounded
    sample (256 weight rows x 128 tokens of the Q4_K N = 4096 workload)."""
    import numpy as np

    import oracle as ref
    from block_quantized_dsq_b200 import synth
    seeds = synth.SEEDS
    out = {}

    def timed(fn):
        n, t0 = 0, time.perf_counter()
        while True:
            fn()
            n += 1
            dt = time.perf_counter() - t0
            if dt > budget_s:
                return dt / n

    x1 = synth.activations(seeds["gemv_q4_k_4096"]["x"], 1, 4096)
    t = timed(lambda: ref.quantize_act_q8(x1))
    out["quantize_act_q8_1x4096"] = {"us_per_call": round(t * 1e6, 2),
                                     "GB/s": round((4096 * 4 + 4096 + 1024) / t / 1e9, 4)}
    for name, qtype, N, K, sw, sx, G in (
            ("gemv_q8_0_1024x1024", 8, 1024, 1024, seeds["gemv_q8_0_1024"]["w"], seeds["gemv_q8_0_1024"]["x"], 1),
            ("gemv_q4_k_4096x4096", 12, 4096, 4096, seeds["gemv_q4_k_4096"]["w"], seeds["gemv_q4_k_4096"]["x"], 1),
            ("grouped_q8_0_8x1024x4096", 8, 1024, 4096, seeds["grouped_q8_0_8x1024x4096"]["w_base"],
             seeds["grouped_q8_0_8x1024x4096"]["x_base"], 8)):
        w = np.concatenate([ref.quantize(qtype, synth.weights(sw + g, N, K)) for g in range(G)])
        xq, xd, xs = ref.quantize_act_q8(np.concatenate([synth.activations(sx + g, 1, K) for g in range(G)]))

        def run(w=w, xq=xq, xd=xd, xs=xs, qtype=qtype, N=N, K=K, G=G):
            for g in range(G):
                ref.gemv(qtype, w[g * N:(g + 1) * N], K, xq[g], xd[g], xs[g])
        t = timed(run)
        alg = w.nbytes + G * (K + K // 32 * 4 * (2 if qtype == 12 else 1)) + G * N * 4
        out[name] = {"us_per_call": round(t * 1e6, 1), "GB/s": round(alg / t / 1e9, 4)}
    K, N, M, rows = 4096, 4096, 128, 256
    w = ref.quantize(12, synth.weights(seeds["prefill"]["w_q4_k"], rows, K))
    x = synth.activations(seeds["prefill"]["x_base"] + M, M, K)
    t = timed(lambda: ref.prefill_f64(12, w, K, x))
    out["prefill_q4_k_n4096_m128"] = {"sample": f"{rows} of {N} weight rows x {M} tokens, fp64",
                                      "GFLOP/s": round(2.0 * M * rows * K / t / 1e9, 4),
                                      "us_per_full_call": round(t * N / rows * 1e6, 1)}
    out["cores"] = 1
    out["kind"] = "oracle"
    return out


def run_reference(args, world, rank):
    """The oracle as the reference arm: same metric and workload, a bounded
    sample per step, host cores only (rank 0)."""
    import numpy as np

    import oracle as ref
    from block_quantized_dsq_b200 import synth
    seeds = synth.SEEDS["paired_q8_0_2x8192x4096"]
    w0 = ref.quantize(8, synth.weights(seeds["w0"], N_PAIR, K_PAIR))
    w1 = ref.quantize(8, synth.weights(seeds["w1"], N_PAIR, K_PAIR))
    X = np.concatenate([synth.activations(seeds["x_base"] + i, 1, K_PAIR) for i in range(CALLS)])
    per_step = 2      # calls per step: bounded so the whole run ends within minutes
    bpc = paired_bytes_per_call()

    def step(s):
        for j in range(per_step):
            c = (s * per_step + j) % CALLS
            xq, xd, xs = ref.quantize_act_q8(X[c:c + 1])
            ref.gemv(8, w0, K_PAIR, xq, xd, xs)
            ref.gemv(8, w1, K_PAIR, xq, xd, xs)

    for s in range(args.warmup):
        step(s)
    t0 = time.perf_counter()
    for s in range(args.steps):
        step(s)
    dt = time.perf_counter() - t0
    value = args.steps * per_step * bpc["fused"] / dt / 1e9
    sample = f"{per_step} of the 64 paired calls per step (oracle act-quantize + two integer-form GEMVs)"
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
            "data": "synthetic", "config": bench_config(world),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=None)
    ap.add_argument("--impl", choices=["dsq", "reference"], default="dsq")
    ap.add_argument("--skip-rows", action="store_true", help="only the headline workload")
    ap.add_argument("--skip-cpu", action="store_true", help="no CPU oracle baseline")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--rows", default=None,
                    help="comma-separated row names to run (e.g. prefill_q8_0_n8192_m2048)")
    ap.add_argument("--profile", action="store_true",
                    help="for ncu: run the selected rows (and, unless --skip-headline, one headline "
                         "step) a few times untimed and print nothing")
    ap.add_argument("--skip-headline", action="store_true")
    args = ap.parse_args()
    if args.impl == "reference":
        args.steps = 5 if args.steps is None else args.steps
        args.warmup = 1 if args.warmup is None else args.warmup
        if int(os.environ.get("RANK", "0")) != 0:
            return 0
        print(json.dumps(run_reference(args, int(os.environ.get("WORLD_SIZE", "1")), 0)))
        return 0
    args.steps = 500 if args.steps is None else args.steps
    args.warmup = 5 if args.warmup is None else args.warmup
    if args.warmup < 3:
        args.warmup = 3
    world, rank, _ = dist_setup()
    try:
        if args.profile:
            run_profile(args)
            return 0
        res = run_dsq(args, world, rank)
        if rank == 0:
            print(json.dumps(res))
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
