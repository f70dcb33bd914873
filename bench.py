#!/usr/bin/env python
"""Benchmark of the H-BitLinear forward (BitNet v2) on B200.

Workload (one step): the decode-shaped o_proj H-BitLinear, M=16 tokens,
K=N=4096, W1.58A4 with the Hadamard on, run once for each of 64 distinct
packed weight sets (64 x 4 MiB = 256 MiB, larger than the 126 MB L2, so every
forward streams its weights from HBM). The 64 forwards of a step are captured
in one CUDA graph. value = tokens/s over the whole job (tokens = M per forward).

Also reported: the dominant kernel's roofline fraction (CUDA-event duration
of that kernel, algorithmic bytes), the same metric end to end through the C
ABI with the host<->device copies in the timed region, SM clocks during the
run, the CPU oracle on a bounded sample, and secondary configurations.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

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
LAYERS = 64
HEAD = dict(M=16, K=4096, N=4096, act_bits=4, use_hadamard=1)
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


def headline_workload_name():
    return (f"decode_oproj M={HEAD['M']} K={HEAD['K']} N={HEAD['N']} W1.58A{HEAD['act_bits']} "
            f"H{'on' if HEAD['use_hadamard'] else 'off'}, {LAYERS} weight sets per step")


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


def cpu_oracle_baseline(X, W, case, budget_s=12.0):
    """The oracle, as it stands, on a bounded sample of the headline batch (rank 0, N=1)."""
    import numpy as np
    import oracle
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = len(os.sched_getaffinity(0))
    Xn = X.double().numpy()
    a, T = oracle.weight_quant(W.numpy())          # offline weight packing: not timed
    oracle.forward(Xn[:1], T, a, case["act_bits"], case["use_hadamard"])   # builds H once
    t0 = time.perf_counter()
    n = 0
    while True:
        oracle.forward(Xn, T, a, case["act_bits"], case["use_hadamard"])
        n += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    return {"value": n * case["M"] / dt, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} full oracle forwards of the M={case['M']} headline batch "
                      f"(explicit O(K^2) fp64 Hadamard, fp64 quantiser, exact GEMM) in {dt:.1f} s"}


# ----------------------------------------------------------------------------- reference arm
def run_reference(args, rank, world):
    if rank != 0:
        return 0
    import numpy as np
    import torch
    import oracle
    from hadamard_bit_quant_b200 import inputs
    case = [c for c in inputs.decode_oproj_cases((HEAD["M"],), (HEAD["act_bits"],))][0]
    X = case.make_x().double().numpy()
    a, T = oracle.weight_quant(case.make_w().numpy())
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:
        threads = len(os.sched_getaffinity(0))
    # one step = the oracle forward of the whole headline batch (M tokens), as cpu_baseline times it
    def step(i):
        oracle.forward(X, T, a, case.act_bits, case.use_hadamard)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    dt = time.perf_counter() - t0
    val = args.steps * case.M / dt
    cfg = {"workload": headline_workload_name(), "M": case.M, "K": case.K, "N": case.N,
           "act_bits": case.act_bits, "use_hadamard": case.use_hadamard}
    line = {"metric": METRIC, "value": val, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "impl": "reference",
            "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                             "sample": f"the M={case.M} headline batch per step through the oracle forward "
                                       f"({args.steps} steps in {dt:.1f} s)"},
            "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- our arm
def capture_step(torch, hbl, X, Wpks, wsc, Y, ws, case, Xh=None, Yh=None):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        for Wpk in Wpks:
            if Xh is not None:
                X.copy_(Xh, non_blocking=True)
            hbl.hbl_forward_ws(X, case["M"], case["K"], case["N"], Wpk, wsc, case["act_bits"],
                               case["use_hadamard"], Y, ws, ws.numel())
            if Yh is not None:
                Yh.copy_(Y, non_blocking=True)
    return g


def capture_step_e2e(torch, hbl, Xh, Wpks, wsc, ws, case):
    """The step end to end: every forward's input is copied from pinned host memory and its
    output back, on two copy streams that run beside the compute stream (per-forward device
    buffers; each forward waits for its input copy, each output copy for its forward). Both
    copy streams rejoin the compute stream before the step ends, so every copy is inside it."""
    M, K, N = case["M"], case["K"], case["N"]
    L = len(Wpks)
    Xs = torch.empty(L, M, K, dtype=torch.bfloat16, device="cuda")
    Ys = torch.empty(L, M, N, dtype=torch.bfloat16, device="cuda")
    Yh = torch.empty(L, M, N, dtype=torch.bfloat16).pin_memory()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.graph(g, stream=s):
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        s_in.wait_stream(s)
        s_out.wait_stream(s)
        ev_in = [torch.cuda.Event() for _ in range(L)]
        ev_fw = [torch.cuda.Event() for _ in range(L)]
        with torch.cuda.stream(s_in):
            for i in range(L):
                Xs[i].copy_(Xh, non_blocking=True)
                ev_in[i].record(s_in)
        for i, Wpk in enumerate(Wpks):
            s.wait_event(ev_in[i])
            hbl.hbl_forward_ws(Xs[i], M, K, N, Wpk, wsc, case["act_bits"], case["use_hadamard"], Ys[i], ws,
                               ws.numel(), s.cuda_stream)
            ev_fw[i].record(s)
        with torch.cuda.stream(s_out):
            for i in range(L):
                s_out.wait_event(ev_fw[i])
                Yh[i].copy_(Ys[i], non_blocking=True)
        s.wait_stream(s_in)
        s.wait_stream(s_out)
    return g, Yh


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


def profile_kernels(torch, hbl, X, Wpks, wsc, Y, ws, case, reps):
    """Per-kernel CUDA-event durations of the forward, weights cold (L2 flushed before each)."""
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    hbl.hbl_profile_enable(1)
    for r in range(reps):
        flush.zero_()
        hbl.hbl_forward_ws(X, case["M"], case["K"], case["N"], Wpks[r % len(Wpks)], wsc, case["act_bits"],
                           case["use_hadamard"], Y, ws, ws.numel())
    torch.cuda.synchronize()
    tab = hbl.profile_table()
    hbl.hbl_profile_enable(0)
    del flush
    return {k: {"launches": n, "ms_per_launch": ms / max(n, 1)} for k, (n, ms) in tab.items()}


def roofline_of(prof, case, peaks, peak_kind, workload, timed_us_per_forward=None):
    """Roofline of the dominant kernel. When the forward is ONE kernel, its
    average launch duration is the timed region divided by the launches in it
    (measured live, programmatic-launch overlap included); otherwise the
    per-kernel CUDA-event durations of the profiling loop are used."""
    ours = {k: v for k, v in prof.items() if k in KERNEL_BYTES}
    dom = max(ours, key=lambda k: ours[k]["ms_per_launch"] * ours[k]["launches"])
    b = KERNEL_BYTES[dom](case["M"], case["K"], case["N"])
    single = len(prof) == 1 and timed_us_per_forward is not None
    if single:
        t = timed_us_per_forward * 1e-6
        src = "timed region / launches (CUDA events on the launching stream)"
    else:
        t = ours[dom]["ms_per_launch"] * 1e-3
        src = "CUDA events around each launch, L2 flushed before each forward"
    ach = b / t / 1e9
    peak = peaks["hbm_gbs"]
    return {"bound": "hbm", "achieved": ach, "peak": peak, "unit": "GB/s", "frac": ach / peak,
            "traffic": traffic_for(dom, workload), "kernel": dom, "bytes_per_launch": b,
            "launch_us": t * 1e6, "duration_source": src, "peak_source": f"{peak_kind} hbm_gbs"}


def secondary(torch, hbl, layer, inputs):
    """Other decode shapes (graph of 64 forwards, 20 replays) and the prefill config."""
    out = {}
    for case in inputs.decode_oproj_cases():
        if case.M == HEAD["M"] and case.act_bits == HEAD["act_bits"]:
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
    out["decode M=16 K=16384 N=16384 a4"] = {
        "us_per_forward": ms * 1e3, "tokens_per_s": big.M / (ms * 1e-3),
        "weight_GBps": big.N * big.K / 4 / (ms * 1e-3) / 1e9}
    del g, Wpks
    torch.cuda.empty_cache()
    case = inputs.prefill_down_case()
    X = case.make_x().cuda()
    Wpk, wsc = layer.pack_weights(case.make_w().cuda())
    Y = torch.empty(case.M, case.N, dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(case.M, case.K, case.N, "cuda")
    c = dict(M=case.M, K=case.K, N=case.N, act_bits=case.act_bits, use_hadamard=case.use_hadamard)
    hbl.hbl_forward_ws(X, case.M, case.K, case.N, Wpk, wsc, case.act_bits, case.use_hadamard, Y, ws, ws.numel())
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    times = []
    for _ in range(5):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        hbl.hbl_forward_ws(X, case.M, case.K, case.N, Wpk, wsc, case.act_bits, case.use_hadamard, Y, ws, ws.numel())
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    prof = profile_kernels(torch, hbl, X, [Wpk], wsc, Y, ws, c, 3)
    ms = statistics.median(times)
    ops = 2.0 * case.M * case.N * case.K
    gemm_ms = (prof.get("gemm_tc") or prof.get("gemm_mma") or {}).get("ms_per_launch")
    out["prefill M=4096 K=16384 N=4096 a4"] = {
        "ms_forward": ms, "tokens_per_s": case.M / (ms * 1e-3), "TOPS": ops / (ms * 1e-3) / 1e12,
        "gemm_ms": gemm_ms, "gemm_TOPS": (ops / (gemm_ms * 1e-3) / 1e12) if gemm_ms else None,
        "kernels": prof}
    return out


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
    # f1: the whole forward with the prologue, decode o_proj shape (fused kernel), 64 weight sets
    case = [c for c in inputs.decode_oproj_cases((HEAD["M"],), (HEAD["act_bits"],))][0]
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
    case = [c for c in inputs.decode_oproj_cases((HEAD["M"],), (HEAD["act_bits"],))][0]
    c = dict(HEAD)
    Xc, Wc = case.make_x(), case.make_w()
    X = Xc.cuda()
    Wpk, wsc = layer.pack_weights(Wc.cuda())
    Wpks = [Wpk] + [Wpk.clone() for _ in range(LAYERS - 1)]
    Y = torch.empty(c["M"], c["N"], dtype=torch.bfloat16, device="cuda")
    ws = layer.workspace(c["M"], c["K"], c["N"], "cuda")
    # eager call first: library init (device probe, kernel attributes) happens outside capture
    hbl.hbl_forward_ws(X, c["M"], c["K"], c["N"], Wpk, wsc, c["act_bits"], c["use_hadamard"], Y, ws, ws.numel())
    torch.cuda.synchronize()
    g = capture_step(torch, hbl, X, Wpks, wsc, Y, ws, c)

    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else int(os.environ["CUDA_VISIBLE_DEVICES"].split(",")[local]))
    clocks.start()
    ms = timed_replays(torch, dist, g, args.warmup, args.steps, world)
    clk = clocks.stop()
    tokens = world * args.steps * LAYERS * c["M"]
    value = tokens / (ms * 1e-3)
    ops_per_step = 2.0 * LAYERS * c["M"] * c["N"] * c["K"]

    # e2e: same step with the H2D copy of each forward's input and the D2H copy of its output,
    # the copies pipelined against the forwards on their own streams
    Xh = Xc.pin_memory()
    g2, Yh = capture_step_e2e(torch, hbl, Xh, Wpks, wsc, ws, c)
    ms_e2e = timed_replays(torch, dist, g2, args.warmup, args.steps, world)
    e2e = {"value": tokens / (ms_e2e * 1e-3), "unit": "tokens/s",
           "h2d_bytes_per_step": LAYERS * Xh.numel() * 2, "d2h_bytes_per_step": Yh.numel() * 2,
           "copies": "per forward, on two copy streams beside the compute stream"}
    # the copied-back outputs are the forwards' outputs
    if not torch.equal(Yh[-1].cuda(), Y):
        raise RuntimeError("e2e step: copied-back output differs from the device-side forward")

    prof = profile_kernels(torch, hbl, X, Wpks, wsc, Y, ws, c, 64)
    launches_per_forward = sum(v["launches"] for k, v in prof.items() if k != "memset_acc") / 64
    roof = roofline_of(prof, c, peaks, peak_kind, "decode_oproj_m16",
                       timed_us_per_forward=ms / (args.steps * LAYERS) * 1e3)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "i8", "data": "synthetic",
        "config": {"workload": headline_workload_name(), "M": c["M"], "K": c["K"], "N": c["N"],
                   "act_bits": c["act_bits"], "use_hadamard": c["use_hadamard"], "layers_per_step": LAYERS,
                   "tokens_per_step_per_gpu": LAYERS * c["M"],
                   "l2": "inputs larger than L2: 64 packed weight sets (256 MiB) rotate within each step",
                   "parallelism": f"dp{world} (token-sharded replicas, no collective)", "graph": True},
        "tops": ops_per_step * args.steps * world / (ms * 1e-3) / 1e12,
        "roofline": roof,
        "kernels": prof,
        "e2e": e2e,
        "gpu_launches": int(round(launches_per_forward * LAYERS * args.steps)),
        "clocks": clk,
    }
    if rank == 0 and world == 1 and not args.no_extras:
        try:
            line["secondary"] = secondary(torch, hbl, layer, inputs)
        except Exception as ex:  # secondary numbers are optional context
            line["secondary"] = {"error": repr(ex)}
        try:
            line["next_rows"] = next_rows(torch, hbl, layer, inputs, peaks["hbm_gbs"])
        except Exception as ex:
            line["next_rows"] = {"error": repr(ex)}
    if rank == 0 and world == 1 and not args.no_cpu:
        line["cpu_baseline"] = cpu_oracle_baseline(Xc, Wc, c)
    if rank == 0:
        print(json.dumps(line), flush=True)
    del g, g2
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
        case = [c for c in inputs.decode_oproj_cases((HEAD["M"],), (HEAD["act_bits"],))][0]
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
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
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
