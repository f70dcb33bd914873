#!/usr/bin/env python
"""Benchmark of the H-BitLinear forward (BitNet v2) on B200.

Headline workload (one step): the prefill down_proj H-BitLinear, M=4096 tokens,
K=16384, N=4096, W1.58A4 with the Hadamard on -- the largest single-GPU
configuration. A step is one forward of that batch: the Hadamard + INT4
quantiser kernel, then the tcgen05 GEMM with its dequant epilogue. Two input
sets (bf16 X 128 MiB and packed weights 16 MiB each) alternate between steps,
so no step finds its inputs in the 126 MB L2. value = tokens/s over the whole
job; the roofline is the GEMM's int8 tensor rate from CUDA events recorded
around each launch inside the timed region.

Also reported: the same metric end to end through the C ABI with the
host<->device copies in the timed region, SM clocks during the run, the CPU
oracle on a bounded sample of the batch, the decode o_proj (M=16, K=N=4096)
with its HBM roofline, other decode shapes, the seven projections of a
7B-shaped block at M in {1, 64, 512, 4096}, an M x K x N sweep with the
decode-to-prefill crossover, and the rows beyond the forward.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                  [--sweep default|full|none] [--no-extras] [--no-cpu]

Under torchrun each rank runs the same step on its own GPU (token-sharded
replicas, weak scaling, no collective in the data path); rank 0 prints one
JSON line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "H-BitLinear fwd TOPS & tokens/s (W1.58A4) + % of HBM/tensor roofline"
LAYERS = 64                    # decode weight sets per graph
HEAD = dict(M=4096, K=16384, N=4096, act_bits=4, use_hadamard=1)
DECODE = dict(M=16, K=4096, N=4096, act_bits=4, use_hadamard=1)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def csrc_hash() -> str:
    h = hashlib.sha256()
    for f in sorted(glob.glob(os.path.join(ROOT, "hadamard_bit_quant_b200", "csrc", "*"))):
        with open(f, "rb") as fh:
            h.update(os.path.basename(f).encode())
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current kernels."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{workload}/{kernel}")
    if not e or e.get("csrc_sha") != csrc_hash():
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi clock/throttle samples every 200 ms while running."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.idx), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                     hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
                except ValueError:
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        reasons = set()
        for r in rows:
            for k, nm in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                          ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(r["sm"] for r in rows), "sm_max_mhz": max(r["smax"] for r in rows),
                "reasons": sorted(reasons), "samples": len(rows),
                "power_w_max": max(r["power"] for r in rows)}


class ClockPoller:
    """SM clock and clock-event (throttle) reasons read through NVML from a background
    thread, back to back, while running: read-only queries, as fine-grained as NVML allows
    for a timed region of a few milliseconds (nvidia-smi samples every 200 ms at best)."""
    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, torch, local, period_s=0.0):
        self.torch, self.local, self.period = torch, local, period_s
        self.samples, self.thread, self.h, self.nv = [], None, None, None
        self.stop_flag = False

    def _handle(self):
        import pynvml as nv
        nv.nvmlInit()
        self.nv = nv
        try:
            uuid = str(self.torch.cuda.get_device_properties(self.local).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(gpu_index(self.torch, self.local))

    def _reasons(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return f(self.h)

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM), self._reasons()))
            except Exception:
                pass
            if self.period > 0:
                time.sleep(self.period)

    def start(self):
        import threading
        try:
            self.h = self._handle()
            self.smax = self.nv.nvmlDeviceGetMaxClockInfo(self.h, self.nv.NVML_CLOCK_SM)
        except Exception:
            self.h = None
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join(2)
        if not self.samples:
            return None
        reasons = set()
        for _, r in self.samples:
            for bit, nm in self.REASONS.items():
                if r & bit:
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(c for c, _ in self.samples), "sm_max_mhz": float(self.smax),
                "reasons": sorted(reasons), "samples": len(self.samples),
                "sm_mhz_min": min(c for c, _ in self.samples),
                "source": "NVML clock and clock-event reasons polled back to back during the timed region"}


# ----------------------------------------------------------------------------- workloads
def headline_workload_name():
    return (f"prefill_down M={HEAD['M']} K={HEAD['K']} N={HEAD['N']} W1.58A{HEAD['act_bits']} "
            f"H{'on' if HEAD['use_hadamard'] else 'off'}")


def headline_config(world):
    """The config dict both arms print (identical keys and values)."""
    return {"workload": headline_workload_name(), "M": HEAD["M"], "K": HEAD["K"], "N": HEAD["N"],
            "act_bits": HEAD["act_bits"], "use_hadamard": HEAD["use_hadamard"],
            "tokens_per_step_per_gpu": HEAD["M"],
            "l2": "inputs larger than L2: two input sets (bf16 X 128 MiB + packed weights 16 MiB each) "
                  "alternate between steps",
            "parallelism": f"dp{world} (token-sharded replicas, no collective)"}


def headline_cases(inputs):
    """Two input sets of the prefill down_proj workload (the second drawn the same way, seed + 100)."""
    import dataclasses
    c0 = inputs.prefill_down_case()
    return [c0, dataclasses.replace(c0, seed=c0.seed + 100, x_stream=c0.x_stream + 1)]


def oracle_threads():
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        return len(os.sched_getaffinity(0))


def oracle_sampled_rows(X64, T, alpha, rows_per_call, budget_s=None, calls=None, seed=0):
    """The oracle forward on sampled token rows of the headline batch (tokens are independent,
    so each sampled row is an exact part of the forward). Runs for budget_s seconds or `calls`
    calls; returns (tokens, seconds)."""
    import numpy as np
    import oracle
    rng = np.random.default_rng(seed)
    M = X64.shape[0]
    oracle.forward_rows(X64, T, alpha, HEAD["act_bits"], HEAD["use_hadamard"], [0])   # builds H once
    t0 = time.perf_counter()
    n = 0
    while True:
        rows = rng.choice(M, rows_per_call, replace=False)
        oracle.forward_rows(X64, T, alpha, HEAD["act_bits"], HEAD["use_hadamard"], rows)
        n += 1
        dt = time.perf_counter() - t0
        if (calls is not None and n >= calls) or (budget_s is not None and dt > budget_s):
            break
    return n * rows_per_call, dt


def cpu_oracle_baseline(case, budget_s=12.0, rows_per_call=8):
    """The oracle, as it stands, on a bounded sample of the headline batch (rank 0, N=1)."""
    import oracle
    X64 = case.make_x().double().numpy()
    a, T = oracle.weight_quant(case.make_w().numpy())       # offline weight packing: not timed
    tokens, dt = oracle_sampled_rows(X64, T, a, rows_per_call, budget_s=budget_s)
    return {"value": tokens / dt, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
            "sample": f"{tokens} sampled token rows of the M={case.M} headline batch, {rows_per_call} per "
                      f"oracle call (explicit O(K^2) fp64 Hadamard, fp64 quantiser, exact GEMM against all "
                      f"N={case.N} outputs) in {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    """The oracle as the reference arm: each step is the oracle forward of 8 sampled token rows
    of the headline batch (rank 0 only; other ranks exit without work)."""
    if rank != 0:
        return 0
    import oracle
    from hadamard_bit_quant_b200 import inputs
    case = headline_cases(inputs)[0]
    X64 = case.make_x().double().numpy()
    a, T = oracle.weight_quant(case.make_w().numpy())
    rows = 8
    oracle_sampled_rows(X64, T, a, rows, calls=args.warmup, seed=1)
    tokens, dt = oracle_sampled_rows(X64, T, a, rows, calls=args.steps, seed=2)
    val = tokens / dt
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": headline_config(world), "impl": "reference",
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": oracle_threads(), "kind": "oracle",
                             "sample": f"each step: the oracle forward of {rows} sampled token rows of the "
                                       f"M={case.M} headline batch ({args.steps} steps in {dt:.1f} s)"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- timing helpers
def capture_step(torch, hbl, X, Wpks, wsc, Y, ws, case):
    """A CUDA graph of one forward per packed weight set (decode shapes: launch-bound)."""
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        for Wpk in Wpks:
            hbl.hbl_forward_ws(X, case["M"], case["K"], case["N"], Wpk, wsc, case["act_bits"],
                               case["use_hadamard"], Y, ws, ws.numel())
    return g


def timed_replays(torch, dist, g, warmup, steps, world):
    for _ in range(warmup):
        g.replay()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        g.replay()
    e1.record()
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    if world > 1:
        from hadamard_bit_quant_b200.shard import max_over_ranks
        ms = max_over_ranks(ms, device="cuda")
        dist.barrier()
    return ms


KERNEL_BYTES = {
    # algorithmic bytes per launch (what the step must move), per kernel kind
    # fused forward: packed weights + bf16 X + bf16 Y + alpha
    "fused_decode": lambda M, K, N: N * K / 4 + 2 * M * K + 2 * M * N + 4,
    "gemm_decode": lambda M, K, N: N * K / 4 + M * K + 2 * M * N + 8 * M + 4,
    "gemm_mma": lambda M, K, N: N * K / 4 + M * K + 2 * M * N + 4 * M + 4,
    "fwht_quant": lambda M, K, N: M * (2 * K + K + 8),
    "quant_rows": lambda M, K, N: M * (2 * K + K + 8),
    "dequant_store": lambda M, K, N: 4 * M * N + 2 * M * N + 8 * M,
}
TENSOR_KERNELS = ("gemm_tc",)


def int8_peak(peaks, peak_kind):
    """Dense int8 tensor-core peak: the measured bf16 burst figure times the nominal dense
    int8:bf16 ratio of 2 (no int8 GEMM peak is measured on this machine)."""
    return 2.0 * peaks["bf16_tflops"], f"2 x {peak_kind} bf16_tflops (burst; nominal dense int8:bf16 = 2)"


def kernel_table(prof, case, peaks, peak_kind):
    """Per-kernel average launch time and its roofline fraction (bytes for HBM-bound kernels,
    2MNK int8 ops for the tensor-core GEMM)."""
    out = {}
    M, K, N = case["M"], case["K"], case["N"]
    for k, v in prof.items():
        e = dict(v)
        t = v["ms_per_launch"] * 1e-3
        if k in KERNEL_BYTES and t > 0:
            gbs = KERNEL_BYTES[k](M, K, N) / t / 1e9
            e.update(bound="hbm", GBps=gbs, frac=gbs / peaks["hbm_gbs"])
        elif k in TENSOR_KERNELS and t > 0:
            tops = 2.0 * M * N * K / t / 1e12
            e.update(bound="tensor", TOPS=tops, frac=tops / int8_peak(peaks, peak_kind)[0])
        out[k] = e
    return out


def prof_dict(hbl):
    return {k: {"launches": n, "ms_per_launch": ms / max(n, 1)} for k, (n, ms) in hbl.profile_table().items()}


def profile_kernels(torch, hbl, X, Wpks, wsc, Y, ws, case, reps):
    """Per-kernel CUDA-event durations of the forward, weights cold (L2 flushed before each)."""
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    hbl.hbl_profile_enable(1)
    for r in range(reps):
        flush.zero_()
        hbl.hbl_forward_ws(X, case["M"], case["K"], case["N"], Wpks[r % len(Wpks)], wsc, case["act_bits"],
                           case["use_hadamard"], Y, ws, ws.numel())
    torch.cuda.synchronize()
    prof = prof_dict(hbl)
    hbl.hbl_profile_enable(0)
    del flush
    return prof


# ----------------------------------------------------------------------------- headline: prefill
def prefill_headline(torch, dist, hbl, layer, inputs, args, world, local, peaks, peak_kind):
    """K steps of the prefill forward, eager (a forward is ~0.3 ms, launch cost is hidden), with
    the library's per-launch CUDA events on (recorded on the launching stream, inside the timed
    region): value from the region's two events, the roofline from the per-kernel events."""
    M, K, N = HEAD["M"], HEAD["K"], HEAD["N"]
    a, h = HEAD["act_bits"], HEAD["use_hadamard"]
    cases = headline_cases(inputs)
    Xc = [c.make_x() for c in cases]
    X = [x.cuda() for x in Xc]
    W = [layer.pack_weights(c.make_w().cuda()) for c in cases]
    Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(M, K, N, "cuda")

    def fwd(i, y=Y, x=None):
        Wpk, wsc = W[i % 2]
        hbl.hbl_forward_ws(X[i % 2] if x is None else x, M, K, N, Wpk, wsc, a, h, y, ws, ws.numel())

    fwd(0)
    torch.cuda.synchronize()
    smi = ClockSampler(gpu_index(torch, local))
    smi.start()
    for i in range(args.warmup):
        fwd(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    hbl.hbl_profile_enable(1)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    poll = ClockPoller(torch, local)
    poll.start()
    e0.record()
    for i in range(args.steps):
        fwd(i)
    e1.record()
    torch.cuda.synchronize()
    clk = poll.stop()
    ms = e0.elapsed_time(e1)
    prof = prof_dict(hbl)
    hbl.hbl_profile_enable(0)
    clk_smi = smi.stop()
    if clk is None:
        clk = clk_smi
    if world > 1:
        from hadamard_bit_quant_b200.shard import max_over_ranks
        ms = max_over_ranks(ms, device="cuda")
        dist.barrier()
    tokens = world * args.steps * M
    ops = 2.0 * M * N * K
    c = dict(HEAD)
    kt = kernel_table(prof, c, peaks, peak_kind)
    g = prof["gemm_tc"]
    t_gemm = g["ms_per_launch"] * 1e-3
    peak, peak_src = int8_peak(peaks, peak_kind)
    ach = ops / t_gemm / 1e12
    roof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
            "traffic": traffic_for("gemm_tc", "prefill_down"), "kernel": "gemm_tc",
            "ops_per_launch": ops, "ops": "int8 multiply-adds, 2 ops each (2*M*N*K)",
            "launch_us": t_gemm * 1e6,
            "duration_source": "CUDA events around each launch on its launching stream, inside the timed region",
            "peak_source": peak_src,
            "forward_frac": ops * world * args.steps / (ms * 1e-3) / 1e12 / peak}

    # e2e: the same steps through the C ABI from pinned host memory: each step copies its X in
    # (128 MiB) and its Y out (32 MiB) on copy streams beside the compute stream (two device
    # buffers each, so step i+1's input copy overlaps step i's forward)
    Xh = [x.pin_memory() for x in Xc]
    Xd = [torch.empty(M, K, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    Yd = [torch.empty(M, N, dtype=torch.bfloat16, device="cuda") for _ in range(2)]
    Yh = [torch.empty(M, N, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    s = torch.cuda.current_stream()
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def e2e_steps(n):
        ev_in = [torch.cuda.Event() for _ in range(n)]
        ev_fw = [torch.cuda.Event() for _ in range(n)]
        ev_out = [torch.cuda.Event() for _ in range(n)]
        s_in.wait_stream(s)
        s_out.wait_stream(s)
        for i in range(n):
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_fw[i - 2])       # forward i-2 has read Xd[i % 2]
                Xd[i % 2].copy_(Xh[i % 2], non_blocking=True)
                ev_in[i].record(s_in)
            s.wait_event(ev_in[i])
            if i >= 2:
                s.wait_event(ev_out[i - 2])             # Yd[i % 2] has been copied out
            fwd(i, y=Yd[i % 2], x=Xd[i % 2])
            ev_fw[i].record(s)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_fw[i])
                Yh[i % 2].copy_(Yd[i % 2], non_blocking=True)
                ev_out[i].record(s_out)
        s.wait_stream(s_in)
        s.wait_stream(s_out)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    e2e_steps(args.steps)
    e1.record()
    torch.cuda.synchronize()
    ms_e2e = e0.elapsed_time(e1)
    if world > 1:
        ms_e2e = max_over_ranks(ms_e2e, device="cuda")
    # the copied-back output of the last step is the forward's output
    last = args.steps - 1
    fwd(last, y=Y)
    torch.cuda.synchronize()
    if not torch.equal(Yh[last % 2].cuda(), Y):
        raise RuntimeError("e2e: copied-back output differs from the device-side forward")
    e2e = {"value": tokens / (ms_e2e * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": M * K * 2,
           "d2h_bytes_per_step": M * N * 2, "ms_per_step": ms_e2e / args.steps,
           "copies": "per step, pinned host <-> device on two copy streams beside the compute stream"}
    gpu_launches = sum(v["launches"] for k, v in prof.items() if k != "memset_acc")
    out = {"value": tokens / (ms * 1e-3), "ms": ms, "tops": ops * world * args.steps / (ms * 1e-3) / 1e12,
           "roofline": roof, "kernels": kt, "e2e": e2e, "gpu_launches": gpu_launches, "clocks": clk,
           "clocks_smi": clk_smi}
    del X, W, Y, ws, Xd, Yd
    torch.cuda.empty_cache()
    return out


# ----------------------------------------------------------------------------- decode roofline
def decode_roofline(torch, hbl, layer, inputs, peaks, peak_kind, steps=20):
    """The decode o_proj (M=16, K=N=4096, A4, H on): a graph of 64 forwards over 64 weight copies
    (256 MiB, larger than L2), replayed; one kernel per forward, so its average launch duration
    is the timed region / launches."""
    case = [c for c in inputs.decode_oproj_cases((DECODE["M"],), (DECODE["act_bits"],))][0]
    c = dict(DECODE)
    X = case.make_x().cuda()
    Wpk, wsc = layer.pack_weights(case.make_w().cuda())
    Wpks = [Wpk] + [Wpk.clone() for _ in range(LAYERS - 1)]
    Y = torch.empty(c["M"], c["N"], dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(c["M"], c["K"], c["N"], "cuda")
    hbl.hbl_forward_ws(X, c["M"], c["K"], c["N"], Wpk, wsc, c["act_bits"], c["use_hadamard"], Y, ws, ws.numel())
    torch.cuda.synchronize()
    g = capture_step(torch, hbl, X, Wpks, wsc, Y, ws, c)
    ms = timed_replays(torch, None, g, 3, steps, 1)
    us = ms / (steps * LAYERS) * 1e3
    prof = profile_kernels(torch, hbl, X, Wpks, wsc, Y, ws, c, 64)
    ours = {k: v for k, v in prof.items() if k in KERNEL_BYTES}
    dom = max(ours, key=lambda k: ours[k]["ms_per_launch"] * ours[k]["launches"])
    b = KERNEL_BYTES[dom](c["M"], c["K"], c["N"])
    single = len(prof) == 1
    t = us * 1e-6 if single else ours[dom]["ms_per_launch"] * 1e-3
    ach = b / t / 1e9
    wbytes = c["N"] * c["K"] / 4
    del g, Wpks
    floor = launch_floors(torch, int(b), LAYERS)
    floor["forward_over_floor"] = us / floor["copy_us"]
    return {"workload": f"decode_oproj M={c['M']} K={c['K']} N={c['N']} W1.58A4 Hon, {LAYERS} weight sets per graph",
            "us_per_forward": us, "tokens_per_s": c["M"] / (us * 1e-6),
            "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": ach / peaks["hbm_gbs"], "traffic": traffic_for(dom, "decode_oproj_m16"),
                         "kernel": dom, "bytes_per_launch": b, "launch_us": t * 1e6,
                         "duration_source": ("timed region / launches (CUDA events on the launching stream)"
                                             if single else "CUDA events around each launch, L2 flushed"),
                         "peak_source": f"{peak_kind} hbm_gbs",
                         "weights_frac": wbytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"],
                         "single_launch_floor": floor},
            "kernels_cold": prof}


def launch_floors(torch, nbytes, sets, reps=20):
    """What one launch that moves `nbytes` costs on this GPU, measured like the decode forwards
    (a graph of `sets` launches over `sets` distinct buffers, larger than L2 together, replayed):
    a device-to-device copy of half of the bytes (the same bytes in total, half read and half
    written). A library copy, timed only as a floor for the decode rooflines; it is not on the
    product path."""
    n32 = nbytes // 4
    srcs = [torch.randint(-1000, 1000, (n32 // 2,), dtype=torch.int32, device="cuda") for _ in range(sets)]
    dsts = [torch.empty(n32 // 2, dtype=torch.int32, device="cuda") for _ in range(sets)]

    def graph_us(fn):
        fn(0)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=st):
            for i in range(sets):
                fn(i)
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) * 1e3 / (reps * sets)

    copy_us = graph_us(lambda i: dsts[i].copy_(srcs[i]))
    del srcs, dsts
    torch.cuda.empty_cache()
    return {"bytes": nbytes, "copy_us": copy_us,
            "kind": f"graph of {sets} launches over distinct buffers: device copy of half the bytes "
                    "(read + written = the bytes)"}


def secondary(torch, hbl, layer, inputs):
    """Other decode shapes (graph of 64 forwards, 20 replays) and a large decode shape."""
    out = {}
    for case in inputs.decode_oproj_cases():
        if case.M == DECODE["M"] and case.act_bits == DECODE["act_bits"]:
            continue
        c = dict(M=case.M, K=case.K, N=case.N, act_bits=case.act_bits, use_hadamard=case.use_hadamard)
        X = case.make_x().cuda()
        Wpk, wsc = layer.pack_weights(case.make_w().cuda())
        Wpks = [Wpk] + [Wpk.clone() for _ in range(LAYERS - 1)]
        Y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device="cuda")
        ws = layer.workspace(case.M, case.K, case.N, "cuda")
        hbl.hbl_forward_ws(X, case.M, case.K, case.N, Wpk, wsc, case.act_bits, case.use_hadamard, Y, ws, ws.numel())
        g = capture_step(torch, hbl, X, Wpks, wsc, Y, ws, c)
        ms = timed_replays(torch, None, g, 3, 20, 1) / (20 * LAYERS)
        out[f"decode M={case.M} a{case.act_bits}"] = {
            "us_per_forward": ms * 1e3, "tokens_per_s": case.M / (ms * 1e-3),
            "weight_GBps": case.N * case.K / 4 / (ms * 1e-3) / 1e9}
        del g, Wpks
    # a large decode shape: 64 MiB of packed weights per forward (16 weight sets, 1 GiB per step)
    big = inputs.sweep_case(16, 16384, 16384, 4, 1)
    c = dict(M=big.M, K=big.K, N=big.N, act_bits=big.act_bits, use_hadamard=big.use_hadamard)
    X = big.make_x().cuda()
    Wpk, wsc = layer.pack_weights(big.make_w().cuda())
    Wpks = [Wpk] + [Wpk.clone() for _ in range(15)]
    Y = torch.empty(big.M, big.N, dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(big.M, big.K, big.N, "cuda")
    hbl.hbl_forward_ws(X, big.M, big.K, big.N, Wpk, wsc, 4, 1, Y, ws, ws.numel())
    g = capture_step(torch, hbl, X, Wpks, wsc, Y, ws, c)
    ms = timed_replays(torch, None, g, 3, 10, 1) / (10 * len(Wpks))
    prof = profile_kernels(torch, hbl, X, Wpks, wsc, Y, ws, c, 16)
    del g, Wpks
    floor = launch_floors(torch, big.N * big.K // 4, 16, reps=10)
    floor["forward_over_floor"] = ms * 1e3 / floor["copy_us"]
    out["decode M=16 K=16384 N=16384 a4"] = {
        "us_per_forward": ms * 1e3, "tokens_per_s": big.M / (ms * 1e-3),
        "weight_GBps": big.N * big.K / 4 / (ms * 1e-3) / 1e9, "kernels_cold": prof,
        "single_launch_floor": floor}
    torch.cuda.empty_cache()
    return out


def forward_model(M, K, N, peaks, peak_kind):
    """Roofline model of one forward: algorithmic bytes over HBM and 2MNK ops over the int8 peak."""
    b = N * K / 4 + 2 * M * K + 2 * M * N + 4 * M + 4
    ops = 2.0 * M * N * K
    return b, ops, b / (peaks["hbm_gbs"] * 1e9), ops / (int8_peak(peaks, peak_kind)[0] * 1e12)


def graph_time_us(torch, hbl, X, Wpks, wsc, Y, ws, c, reps):
    hbl.hbl_forward_ws(X, c["M"], c["K"], c["N"], Wpks[0], wsc, c["act_bits"], c["use_hadamard"], Y, ws, ws.numel())
    torch.cuda.synchronize()
    g = capture_step(torch, hbl, X, Wpks, wsc, Y, ws, c)
    ms = timed_replays(torch, None, g, 2, reps, 1)
    del g
    return ms / (reps * len(Wpks)) * 1e3


def block7b(torch, hbl, layer, inputs, peaks, peak_kind):
    """All seven projections of one synthetic 7B-shaped block (q/k/v/up/gate plain BitLinear INT8,
    o/down H-BitLinear INT4) at M in {1, 64, 512, 4096}: per-block tokens/s = M / sum of the seven
    forwards. Each graph runs the block over enough weight copies (67 MB of packed weights each)
    that the weights never sit in L2 between uses."""
    out = {}
    for M in (1, 64, 512, 4096):
        cases = inputs.block7b_cases(M)
        copies = 3 if M <= 64 else 2
        Xs = [c.make_x().cuda() for c in cases]
        Ws = [[layer.pack_weights(c.make_w().cuda())] for c in cases]
        for wl in Ws:
            wl += [(wl[0][0].clone(), wl[0][1]) for _ in range(copies - 1)]
        Ys = [torch.empty(M, c.N, dtype=torch.bfloat16, device="cuda") for c in cases]
        wsz = max(hbl.hbl_workspace_bytes(M, c.K, c.N) for c in cases)
        ws = torch.empty(wsz, dtype=torch.uint8, device="cuda")
        for c, x, wl, y in zip(cases, Xs, Ws, Ys):
            hbl.hbl_forward_ws(x, M, c.K, c.N, wl[0][0], wl[0][1], c.act_bits, c.use_hadamard, y, ws, ws.numel())
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        st = torch.cuda.Stream()
        with torch.cuda.graph(g, stream=st):
            for r in range(copies):
                for c, x, wl, y in zip(cases, Xs, Ws, Ys):
                    hbl.hbl_forward_ws(x, M, c.K, c.N, wl[r][0], wl[r][1], c.act_bits, c.use_hadamard, y, ws,
                                       ws.numel())
        reps = 20 if M <= 64 else 5
        ms = timed_replays(torch, None, g, 2, reps, 1) / (reps * copies)
        del g
        b = sum(forward_model(M, c.K, c.N, peaks, peak_kind)[0] for c in cases)
        ops = sum(2.0 * M * c.N * c.K for c in cases)
        t_mem, t_ten = b / (peaks["hbm_gbs"] * 1e9), ops / (int8_peak(peaks, peak_kind)[0] * 1e12)
        t = ms * 1e-3
        gbs, tops = b / t / 1e9, ops / t / 1e12
        bound = "hbm" if t_mem >= t_ten else "tensor"
        out[f"M={M}"] = {"us_per_block": ms * 1e3, "tokens_per_s": M / t, "TOPS": tops, "GBps": gbs,
                         "bound": bound,
                         "frac": (gbs / peaks["hbm_gbs"]) if bound == "hbm" else (tops / int8_peak(peaks, peak_kind)[0]),
                         "algorithmic_bytes": b, "ops": ops}
        del Xs, Ws, Ys, ws
        torch.cuda.empty_cache()
    return out


def sweep(torch, hbl, layer, inputs, peaks, peak_kind, full=False):
    """M x K x N sweep (Student-t(3) inputs): every M in 2^0..2^14 at K=N in {4096, 16384} (all
    16 K,N pairs with full=True), act 4/8, Hadamard on/off. Per point: forward time (graph over
    enough packed weight copies that at least 256 MiB of weights stream per replay), TOPS and
    GB/s of algorithmic bytes. Per series: the model ridge M* (where the HBM time of the
    algorithmic bytes equals the int8 tensor time of 2MNK) and the measured crossover (the
    smallest M whose forward takes twice the M=1 forward: time no longer set by the weights)."""
    kn = [(k, n) for k in inputs.SWEEP_KN for n in inputs.SWEEP_KN] if full else [(4096, 4096), (16384, 16384)]
    Mmax = max(inputs.SWEEP_MS)
    kmax = max(k for k, _ in kn)
    nmax = max(n for _, n in kn)
    Y = torch.empty(Mmax * nmax, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(hbl.hbl_workspace_bytes(Mmax, kmax, nmax), dtype=torch.uint8, device="cuda")
    series = {}
    xcache = {}
    for (K, N) in kn:
        if K not in xcache:
            xcache.clear()
            torch.cuda.empty_cache()
            xcache[K] = inputs.student_t(Mmax, K, 4 + K).cuda()
        Xall = xcache[K]
        Wpk, wsc = layer.pack_weights(inputs.gaussian_weights(N, K, 4 + N).cuda())
        copies = max(2, (256 << 20) // (N * K // 4))
        Wpks = [Wpk] + [Wpk.clone() for _ in range(copies - 1)]
        for a in (4, 8):
            for h in (1, 0):
                pts = []
                for M in inputs.SWEEP_MS:
                    c = dict(M=M, K=K, N=N, act_bits=a, use_hadamard=h)
                    X = Xall[:M]
                    Yv = Y[:M * N].view(M, N)
                    reps = 5 if M * K * N < (1 << 40) else 2
                    us = graph_time_us(torch, hbl, X, Wpks, wsc, Yv, ws, c, reps)
                    b, ops, _, _ = forward_model(M, K, N, peaks, peak_kind)
                    pts.append([M, round(us, 3), round(ops / (us * 1e-6) / 1e12, 2), round(b / (us * 1e-6) / 1e9, 1)])
                t1 = pts[0][1]
                meas = next((p[0] for p in pts if p[1] > 2.0 * t1), None)
                # model ridge: M with HBM time of the algorithmic bytes = int8 tensor time
                P, B = int8_peak(peaks, peak_kind)[0] * 1e12, peaks["hbm_gbs"] * 1e9
                denom = 2.0 * N * K / P - (2.0 * K + 2.0 * N + 4.0) / B
                ridge = (N * K / 4 / B) / denom if denom > 0 else None
                series[f"K={K} N={N} a{a} H{'on' if h else 'off'}"] = {
                    "points[M, us, TOPS, GBps]": pts, "M_star_model": ridge, "M_star_measured": meas,
                    "peak_TOPS": max(p[2] for p in pts), "peak_GBps": max(p[3] for p in pts)}
        del Wpks
        torch.cuda.empty_cache()
    del Y, ws, xcache
    torch.cuda.empty_cache()
    return series


def _event_ms(torch, fn, reps=5, flush=None):
    """Median CUDA-event time (ms) of fn(), L2 flushed before each run."""
    times = []
    for _ in range(reps):
        if flush is not None:
            flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def next_rows(torch, hbl, layer, inputs, peak_gbs):
    """The next rows beyond the forward: RMSNorm prologue (f1), rotated-weight packing (f2),
    Hadamard backward (f3), post-RoPE QKV quantiser (f4). Bytes per call are algorithmic
    (what the kernel must read and write); all are bound by HBM."""
    out = {}
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    g = torch.Generator().manual_seed(7)

    def rec(name, ms, nbytes, **extra):
        gbs = nbytes / (ms * 1e-3) / 1e9
        out[name] = {"us": ms * 1e3, "bytes": nbytes, "GBps": gbs, "frac_of_hbm": gbs / peak_gbs, **extra}

    # f1: RMSNorm + Hadamard + INT4 quantiser, prefill-sized
    M, K = 4096, 16384
    X = (torch.randn(M, K, generator=g)).to(torch.bfloat16).cuda()
    gain = (0.5 + torch.rand(K, generator=g)).cuda()
    codes = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sc = torch.empty(M, device="cuda")
    cs = torch.empty(M, dtype=torch.int32, device="cuda")
    ms = _event_ms(torch, lambda: hbl.hbl_quantize_ln(X, M, K, gain, 4, 1, codes, sc, cs), flush=flush)
    rec("f1 quantize_ln M=4096 K=16384 A4 H on", ms, M * (2 * K + K + 8) + 4 * K)
    ms = _event_ms(torch, lambda: hbl.hbl_quantize(X, M, K, 4, 1, codes, sc, cs), flush=flush)
    rec("a1+a2 quantize (no LN) M=4096 K=16384 A4 H on", ms, M * (2 * K + K + 8))
    # f1: the whole forward with the prologue, decode o_proj shape (fused kernel), 64 weight sets
    case = [c for c in inputs.decode_oproj_cases((DECODE["M"],), (DECODE["act_bits"],))][0]
    Xd = case.make_x().cuda()
    gd = (0.5 + torch.rand(case.K, generator=g)).cuda()
    Wpk, wsc = layer.pack_weights(case.make_w().cuda())
    Wpks = [Wpk] + [Wpk.clone() for _ in range(LAYERS - 1)]
    Y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(case.M, case.K, case.N, "cuda")
    hbl.hbl_forward_ln_ws(Xd, case.M, case.K, case.N, gd, Wpk, wsc, case.act_bits, 1, Y, ws, ws.numel())
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    with torch.cuda.graph(graph, stream=st):
        for w in Wpks:
            hbl.hbl_forward_ln_ws(Xd, case.M, case.K, case.N, gd, w, wsc, case.act_bits, 1, Y, ws, ws.numel(),
                                  torch.cuda.current_stream().cuda_stream)
    ms = timed_replays(torch, None, graph, 3, 20, 1) / (20 * LAYERS)
    rec(f"f1 forward_ln decode M={case.M} K={case.K} N={case.N} A{case.act_bits}", ms,
        case.N * case.K // 4 + 2 * case.M * case.K + 2 * case.M * case.N + 4 * case.K + 4,
        tokens_per_s=case.M / (ms * 1e-3))
    del graph, Wpks
    # f2: rotated-weight packing (offline), 4096 x 4096
    N2 = K2 = 4096
    W = (0.02 * torch.randn(N2, K2, generator=g)).cuda()
    Wpk2 = torch.empty(hbl.hbl_packed_bytes(N2, K2), dtype=torch.uint8, device="cuda")
    a2 = torch.empty(1, device="cuda")
    Wrot = torch.empty(N2, K2, device="cuda")
    ms = _event_ms(torch, lambda: hbl.hbl_pack_weights_rotated(W, N2, K2, Wpk2, a2, Wrot), flush=flush)
    rec("f2 pack_weights_rotated N=K=4096", ms, 4 * N2 * K2 + 4 * N2 * K2 + N2 * K2 // 4)
    # f3: Hadamard backward, fp32 gradients, prefill-sized
    dXr = torch.randn(M, K, generator=g).cuda()
    dX = torch.empty_like(dXr)
    ms = _event_ms(torch, lambda: hbl.hbl_hadamard_backward_f32(dXr, M, K, dX), flush=flush)
    rec("f3 hadamard_backward_f32 M=4096 K=16384", ms, 8 * M * K)
    del dXr, dX
    # f4: post-RoPE QKV quantiser, 4 bits, BOS at 8 bits
    T, H, d = 4096, 32, 128
    Xq = torch.randn(T, H, d, generator=g).to(torch.bfloat16).cuda()
    cq = torch.empty(T, H, d, dtype=torch.uint8, device="cuda")
    gq = torch.empty(T, H, device="cuda")
    ms = _event_ms(torch, lambda: hbl.hbl_quantize_qkv(Xq, T, H, d, 4, 0, cq, gq), flush=flush)
    rec("f4 quantize_qkv T=4096 H=32 d=128 4-bit", ms, 2 * T * H * d + T * H * d + 4 * T * H)
    return out


def gpu_index(torch, local):
    if "CUDA_VISIBLE_DEVICES" in os.environ:
        return int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local])
    return torch.cuda.current_device()


def run_ours(args, rank, world, local):
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from hadamard_bit_quant_b200 import build, hbl, inputs, layer
    if not os.path.exists(os.path.join(ROOT, "hadamard_bit_quant_b200", "libhbl.so")):
        build.build()
    hbl.lib()
    peaks, peak_kind = load_peaks()
    head = prefill_headline(torch, dist, hbl, layer, inputs, args, world, local, peaks, peak_kind)
    line = {
        "metric": METRIC, "value": head["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": headline_config(world),
        "tops": head["tops"],
        "roofline": head["roofline"],
        "kernels": head["kernels"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "clocks_smi_whole_warmup_and_timed": head["clocks_smi"],
    }
    if rank == 0 and world == 1 and not args.no_extras:
        for key, fn in (("decode", lambda: decode_roofline(torch, hbl, layer, inputs, peaks, peak_kind)),
                        ("secondary", lambda: secondary(torch, hbl, layer, inputs)),
                        ("block7b", lambda: block7b(torch, hbl, layer, inputs, peaks, peak_kind)),
                        ("sweep", lambda: sweep(torch, hbl, layer, inputs, peaks, peak_kind,
                                                full=args.sweep == "full") if args.sweep != "none" else None),
                        ("next_rows", lambda: next_rows(torch, hbl, layer, inputs, peaks["hbm_gbs"]))):
            try:
                v = fn()
                if v is not None:
                    line[key] = v
            except Exception as ex:  # extra sections are context; the headline stands without them
                line[key] = {"error": repr(ex)}
            torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_oracle_baseline(headline_cases(inputs)[0])
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def profile_next(torch, hbl):
    """The next rows' kernels, each called twice, at the sizes bench.py times them."""
    g = torch.Generator().manual_seed(7)
    M, K = 4096, 16384
    X = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    gain = (0.5 + torch.rand(K, generator=g)).cuda()
    codes = torch.empty(M, K, dtype=torch.int8, device="cuda")
    sc = torch.empty(M, device="cuda")
    cs = torch.empty(M, dtype=torch.int32, device="cuda")
    dXr = torch.randn(M, K, generator=g).cuda()
    dX = torch.empty_like(dXr)
    T, H, d = 4096, 32, 128
    Xq = torch.randn(T, H, d, generator=g).to(torch.bfloat16).cuda()
    cq = torch.empty(T, H, d, dtype=torch.uint8, device="cuda")
    gq = torch.empty(T, H, device="cuda")
    for _ in range(2):
        hbl.hbl_quantize_ln(X, M, K, gain, 4, 1, codes, sc, cs)      # f1
        hbl.hbl_hadamard_backward_f32(dXr, M, K, dX)                 # f3
        hbl.hbl_quantize_qkv(Xq, T, H, d, 4, 0, cq, gq)              # f4
    torch.cuda.synchronize()
    assert hbl.hbl_get_device_error() == 0
    print("profile case next: f1, f3, f4 kernels twice each ok")
    return 0


def profile_case(which: str):
    """A short, fixed run for ncu captures: pack once, then two forwards of one config."""
    import torch
    from hadamard_bit_quant_b200 import hbl, inputs, layer
    torch.cuda.set_device(0)
    hbl.lib()
    if which == "prefill":
        case = inputs.prefill_down_case()
    elif which == "decode":
        case = [c for c in inputs.decode_oproj_cases((DECODE["M"],), (DECODE["act_bits"],))][0]
    elif which == "decode_big":
        case = inputs.sweep_case(16, 16384, 16384, 4, 1)
    elif which == "next":
        return profile_next(torch, hbl)
    else:
        raise SystemExit(f"unknown profile case {which}")
    X = case.make_x().cuda()
    Wpk, wsc = layer.pack_weights(case.make_w().cuda())
    ws = layer.workspace(case.M, case.K, case.N, "cuda")
    for _ in range(2):
        Y = layer.forward(X, Wpk, wsc, case.N, case.act_bits, case.use_hadamard, ws=ws)
    torch.cuda.synchronize()
    assert hbl.hbl_get_device_error() == 0
    print(f"profile case {which}: {case.label} ok, |Y|max={Y.float().abs().max().item():.3f}")
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--sweep", choices=["default", "full", "none"], default="default",
                    help="M x K x N sweep: K=N in {4096, 16384} (default), all 16 K,N pairs (full), or none")
    ap.add_argument("--profile-case", choices=["prefill", "decode", "decode_big", "next"], default=None,
                    help="run one short fixed case (for ncu captures) and exit")
    args = ap.parse_args()
    if args.profile_case:
        return profile_case(args.profile_case)
    if args.warmup < 3:
        args.warmup = 3
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
