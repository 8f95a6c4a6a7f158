#!/usr/bin/env python
"""Benchmark: one HALO-2 linear layer, forward + both backward GEMMs, on B200.

A step is the whole hot path over one batch: the six Hadamard-rotate + quantize passes
(X along K and M, W along K and N, dY along N and M) and the three tcgen05 GEMMs with the
dequantizing epilogue (Y = X W^T, dX = dY W, dW = dY^T X).  Workload: Llama-style MLP
up-projection, 4096 tokens (batch 4 x seq 1024), d_in 4096 -> d_out 11008, bf16 inputs,
INT8 codes, k = 256, synthetic seeded inputs (N(0,1) activations with 1% outlier channels
x U[30,100], N(0,0.02) weights, Student-t(3) x 1e-3 output gradients).

Prints one JSON line (rank 0).  `value` = 6*M*N*K / device time per step (TOPS), inputs
resident in HBM; `e2e` = the same metric through the public API with the inputs copied
from pinned host memory and the three outputs copied back inside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun every rank runs its own replica (weak scaling, no collective on the data
path); times are the max over ranks.  `--impl reference` times the CPU oracle (the plain
reference implementation of the method) on a token sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from hadamard_rotated_precision_b200 import synthetic  # noqa: E402

WORKLOAD_ID = 2
METRIC = "HALO-2 linear fwd+bwd TOPS, % of INT8/FP8 tensor peak; FWHT+quant HBM GB/s"
UNIT = "TOPS"
INT8_OVER_BF16 = 2.0  # nominal dense INT8 / bf16 tensor throughput ratio on B200 (4.5 / 2.25)
GEMM_SRC = os.path.join(ROOT, "hadamard_rotated_precision_b200", "csrc", "gemm_tcgen05.cuh")
QUANT_SRC = os.path.join(ROOT, "hadamard_rotated_precision_b200", "csrc", "fwht_quant.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CPU_SAMPLE_TOKENS = 512
REF_STEP_TOKENS = 256


# ----------------------------------------------------------------------------- distributed

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=120))
    return dist


def reduce_max(value: float, world: int, device=None) -> float:
    """Max of a per-rank float over all ranks (identity at world size 1)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ----------------------------------------------------------------------------- helpers

def file_digest(path: str) -> str:
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def recorded_traffic(kind: str):
    """Per-launch DRAM bytes of a kernel from the committed ncu summary, if that summary was
    taken on the current source of the kernel (else None)."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(kind)
    if not e:
        return None
    src = GEMM_SRC if kind.startswith("gemm") else QUANT_SRC
    if e.get("source_sha") != file_digest(src):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms during the timed region."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def __enter__(self):
        import tempfile
        fd, self.path = tempfile.mkstemp(prefix="hq_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (FileNotFoundError, OSError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return None
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
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
        load = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["smax"] for r in rows), "samples": len(rows),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- CPU (oracle)

def oracle_layer_seconds(d, k: int, fmt: int) -> float:
    import oracle
    t0 = time.perf_counter()
    oracle.linear_fwd(d["X"], d["W"], k, fmt)
    oracle.linear_bwd_dx(d["dY"], d["W"], k, fmt)
    oracle.linear_bwd_dw(d["dY"], d["X"], k, fmt)
    return time.perf_counter() - t0


def cpu_baseline(w, tokens: int):
    """The oracle, untuned, on a token-prefix sample of the workload (full K, N, k, format)."""
    import oracle
    L = w.layers[0]
    d = synthetic.draw(w, 0, M=tokens)
    fmt = 0 if w.fmt == "int8" else 1
    secs = oracle_layer_seconds(d, w.k, fmt)
    ops = 6.0 * tokens * L.K * L.N
    return {"value": ops / secs / 1e12, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"{L.name} layer fwd+dX+dW at {tokens} of {L.M} tokens (K={L.K}, N={L.N}, "
                      f"k={w.k}, {w.fmt}), {secs:.2f} s"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = synthetic.WORKLOADS[WORKLOAD_ID]
    L = w.layers[0]
    d = synthetic.draw(w, 0, M=REF_STEP_TOKENS)
    fmt = 0 if w.fmt == "int8" else 1
    for _ in range(args.warmup):
        oracle_layer_seconds(d, w.k, fmt)
    total = 0.0
    for _ in range(args.steps):
        total += oracle_layer_seconds(d, w.k, fmt)
    ops = 6.0 * REF_STEP_TOKENS * L.K * L.N
    value = ops * args.steps / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: M={L.M} K={L.K} N={L.N} k={w.k} {w.fmt} bf16 inputs",
                   "step_sample_tokens": REF_STEP_TOKENS, "parallelism": "rank 0 only (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"each step: fwd+dX+dW at {REF_STEP_TOKENS} of {L.M} tokens"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU

def run_gpu(args):
    import torch
    import hadamard_rotated_precision_b200 as hq
    from hadamard_rotated_precision_b200 import build

    world, rank, local = dist_env()
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    build.build()
    hq.lib()

    w = synthetic.WORKLOADS[WORKLOAD_ID]
    L = w.layers[0]
    M, K, N, k = L.M, L.K, L.N, w.k
    fmt = hq.HQ_INT8 if w.fmt == "int8" else hq.HQ_FP8_E4M3
    d = synthetic.draw(w, 0)
    def dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)
    X, W, dY = dev(d["X"]), dev(d["W"]), dev(d["dY"])
    Y = torch.empty(M, N, dtype=torch.bfloat16, device=device)
    dX = torch.empty(M, K, dtype=torch.bfloat16, device=device)
    dW = torch.empty(N, K, dtype=torch.bfloat16, device=device)
    qX_K = torch.empty(M, K, dtype=torch.uint8, device=device)
    qX_M = torch.empty(K, M, dtype=torch.uint8, device=device)
    qW_K = torch.empty(N, K, dtype=torch.uint8, device=device)
    qW_N = torch.empty(K, N, dtype=torch.uint8, device=device)
    qdY_N = torch.empty(M, N, dtype=torch.uint8, device=device)
    qdY_M = torch.empty(N, M, dtype=torch.uint8, device=device)
    scales = torch.empty(8, dtype=torch.float32, device=device)
    lws = torch.empty(hq.hq_linear_fwd_bwd_workspace_bytes(M, K, N), dtype=torch.uint8, device=device)
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731

    # The step, as pre-marshalled C-ABI calls in the schedule hq_linear_fwd_bwd uses: X and W
    # quantized in both rotations and the forward GEMM on the main stream, dY in both
    # rotations on a side stream alongside them, joined by an event before the backward
    # GEMMs.  CUDA events on each stream time every group of launches.
    L_ = hq.lib()
    side = torch.cuda.Stream(device)
    sh, sh2 = stream.cuda_stream, side.cuda_stream
    sp = lambda i: scales[i:i + 1].data_ptr()  # noqa: E731
    pw = hq.hq_quantize_dual_workspace_bytes()
    part = torch.empty(2 * pw, dtype=torch.uint8, device=device)
    ws_main, ws_side = part.data_ptr(), part.data_ptr() + pw

    def dual(src, codes_c, si_c, codes_r, si_r, ws, st):
        return (src.data_ptr(), hq.HQ_BF16, src.shape[0], src.shape[1], k, fmt, codes_c.data_ptr(), sp(si_c),
                codes_r.data_ptr(), sp(si_r), ws, pw, st)

    # the GEMMs run one after another on the main stream and share one split scratch
    gws_len = max(hq.hq_gemm_workspace_bytes(M, N, K), hq.hq_gemm_workspace_bytes(M, K, N),
                  hq.hq_gemm_workspace_bytes(N, K, M))
    gws = torch.empty(max(gws_len, 16), dtype=torch.uint8, device=device)

    def gemm(a, ai, b, bi, out):
        return (a.data_ptr(), sp(ai), b.data_ptr(), sp(bi), a.shape[0], b.shape[0], a.shape[1], fmt,
                hq.HQ_OUT_BF16, out.data_ptr(), gws.data_ptr(), gws_len, sh)

    pq = hq.hq_quantize_workspace_bytes()

    def single(src, dim, codes, si, ws, st):
        return (src.data_ptr(), hq.HQ_BF16, src.shape[0], src.shape[1], dim, k, fmt, codes.data_ptr(), sp(si),
                ws, pq, st)

    q_main = [single(X, 1, qX_K, 0, ws_main, sh), single(W, 1, qW_K, 2, ws_main, sh)]
    q_side_dual = [dual(dY, qdY_N, 4, qdY_M, 5, ws_side, sh2)]
    q_side_wn = [single(W, 0, qW_N, 3, ws_side, sh2)]
    q_side_xm = [single(X, 0, qX_M, 1, ws_side, sh2)]
    g_fwd, g_dx, g_dw = gemm(qX_K, 0, qW_K, 2, Y), gemm(qdY_N, 4, qW_N, 3, dX), gemm(qdY_M, 5, qX_M, 1, dW)

    def run(calls, fn, what):
        for c in calls:
            st = fn(*c)
            if st:
                raise hq.HQError(st, what)

    def step(ev_main=None, ev_side=None):
        rec = (lambda lst, i, s_: lst[i].record(s_)) if ev_main is not None else (lambda *a: None)
        fork = torch.cuda.Event()
        fork.record(stream)
        side.wait_event(fork)
        rec(ev_side, 0, side)
        run(q_side_dual, L_.hq_quantize_dual, "hq_quantize_dual")
        rec(ev_side, 1, side)
        run(q_side_wn, L_.hq_quantize, "hq_quantize")
        join_dx = torch.cuda.Event()
        join_dx.record(side)
        run(q_side_xm, L_.hq_quantize, "hq_quantize")
        rec(ev_side, 2, side)
        join = torch.cuda.Event()
        join.record(side)
        rec(ev_main, 0, stream)
        run(q_main, L_.hq_quantize, "hq_quantize")
        rec(ev_main, 1, stream)
        run([g_fwd], L_.hq_gemm_ws, "hq_gemm_ws")
        rec(ev_main, 2, stream)
        stream.wait_event(join_dx)
        rec(ev_main, 3, stream)
        run([g_dx], L_.hq_gemm_ws, "hq_gemm_ws")
        stream.wait_event(join)  # X along M, the weight gradient's operand
        rec(ev_main, 4, stream)
        run([g_dw], L_.hq_gemm_ws, "hq_gemm_ws")
        rec(ev_main, 5, stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    if hq.hq_get_error(stream) != 0:
        raise SystemExit("device status error during warm-up")

    # ---------------------------------------------------------------- timed region (device)
    ev_main = [[ev() for _ in range(6)] for _ in range(args.steps)]
    ev_side = [[ev() for _ in range(3)] for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()  # L2 flush (256 MiB > 126 MB L2), outside the step's events
            step(ev_main[i], ev_side[i])
        torch.cuda.synchronize(device)
    barrier(world, device)
    torch.cuda.synchronize(device)
    status = hq.hq_get_error(stream)
    step_ms_local = sum(e[0].elapsed_time(e[5]) for e in ev_main) / args.steps
    gemm_ms = sum(e[1].elapsed_time(e[2]) + e[3].elapsed_time(e[5]) for e in ev_main)
    quant_ms = sum(e[0].elapsed_time(e[1]) for e in ev_main) + sum(e[0].elapsed_time(e[2]) for e in ev_side)
    def mean_ms(pairs):
        return sum(a.elapsed_time(b) for a, b in pairs) / args.steps
    phases = {
        "main_quant_fwd_operands": mean_ms((e[0], e[1]) for e in ev_main),
        "gemm_fwd": mean_ms((e[1], e[2]) for e in ev_main),
        "wait_side_dy": mean_ms((e[2], e[3]) for e in ev_main),
        "gemm_dx": mean_ms((e[3], e[4]) for e in ev_main),
        "gemm_dw": mean_ms((e[4], e[5]) for e in ev_main),
        "side_quant_dy_both_rotations": mean_ms((e[0], e[1]) for e in ev_side),
        "side_quant_w_n_x_m": mean_ms((e[1], e[2]) for e in ev_side),
    }
    step_ms = reduce_max(step_ms_local, world, device)
    gemm_ms_launch = reduce_max(gemm_ms / (3 * args.steps), world, device)
    quant_ms_step = reduce_max(quant_ms / args.steps, world, device)
    launches = 13 * args.steps  # per step: 5 quantization calls x 2 kernels + 3 GEMMs

    # ---------------------------------------------------------------- quantizer alone
    # The three two-rotation quantizations one after another on one stream (nothing
    # overlapping), L2 flushed before each, to report the quantization kernels' own throughput;
    # and, for comparison, the six rotations as single-rotation calls (two reads each).
    def alone(calls, fn, what):
        tot = 0.0
        for c in calls:
            flush.zero_()
            a, b = ev(), ev()
            a.record(stream)
            st = fn(*c)
            if st:
                raise hq.HQError(st, what)
            b.record(stream)
            torch.cuda.synchronize(device)
            tot += a.elapsed_time(b)
        return tot

    reps = max(3, min(args.steps, 10))
    single = [(src.data_ptr(), hq.HQ_BF16, src.shape[0], src.shape[1], dim, k, fmt, codes.data_ptr(), sp(si),
               ws_main, pq, sh)
              for src, dim, codes, si in ((X, 1, qX_K, 0), (X, 0, qX_M, 1), (W, 1, qW_K, 2), (W, 0, qW_N, 3),
                                          (dY, 1, qdY_N, 4), (dY, 0, qdY_M, 5))]
    dual_calls = [dual(X, qX_K, 0, qX_M, 1, ws_main, sh), dual(W, qW_K, 2, qW_N, 3, ws_main, sh),
                  dual(dY, qdY_N, 4, qdY_M, 5, ws_main, sh)]
    alone_ms = sum(alone(dual_calls, L_.hq_quantize_dual, "hq_quantize_dual") for _ in range(reps))
    alone_ms_step = reduce_max(alone_ms / reps, world, device)
    single_ms = sum(alone(single, L_.hq_quantize, "hq_quantize") for _ in range(reps))
    single_ms_step = reduce_max(single_ms / reps, world, device)

    # ---------------------------------------------------------------- end to end (host buffers)
    # Every step copies X, W, dY from pinned host memory, runs hq_linear_fwd_bwd and copies Y,
    # dX, dW back.  Steps are pipelined over two device buffer sets and three streams: the
    # host->device copy of step i+1 and the device->host copy of step i-1 overlap step i's
    # kernels (PCIe is full duplex).  Timed from the first copy in to the last copy out.
    hX = torch.empty(M, K, dtype=torch.bfloat16, pin_memory=True).copy_(X)
    hW = torch.empty(N, K, dtype=torch.bfloat16, pin_memory=True).copy_(W)
    hdY = torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True).copy_(dY)
    hY = torch.empty(M, N, dtype=torch.bfloat16, pin_memory=True)
    hdX = torch.empty(M, K, dtype=torch.bfloat16, pin_memory=True)
    hdW = torch.empty(N, K, dtype=torch.bfloat16, pin_memory=True)
    e2e_steps = max(2, min(args.steps, 10))
    bufs = [(X, W, dY, Y, dX, dW)]
    bufs.append(tuple(torch.empty_like(t) for t in bufs[0]))
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_cmp = stream

    def e2e_run(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_cmp = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = ev(), ev()
        t0.record(s_in)
        for i in range(nsteps):
            bX, bW, bdY, bY, bdX, bdW = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])  # step i-2 finished reading these inputs
                bX.copy_(hX, non_blocking=True)
                bW.copy_(hW, non_blocking=True)
                bdY.copy_(hdY, non_blocking=True)
                ev_in[i].record(s_in)
            s_cmp.wait_event(ev_in[i])
            if i >= 2:
                s_cmp.wait_event(ev_out[i - 2])  # step i-2's outputs are on the host
            hq.hq_linear_fwd_bwd(bX, bW, bdY, k, fmt, Y=bY, dX=bdX, dW=bdW, workspace=lws, stream=s_cmp)
            ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                hY.copy_(bY, non_blocking=True)
                hdX.copy_(bdX, non_blocking=True)
                hdW.copy_(bdW, non_blocking=True)
                ev_out[i].record(s_out)
        s_cmp.wait_event(ev_out[nsteps - 1])
        s_cmp.wait_event(ev_in[nsteps - 1])
        t1.record(s_cmp)
        torch.cuda.synchronize(device)
        return t0.elapsed_time(t1) / nsteps

    e2e_run(2)
    barrier(world, device)
    e2e_ms = reduce_max(e2e_run(e2e_steps), world, device)
    status |= hq.hq_get_error(stream)

    # ---------------------------------------------------------------- report
    ops = 6.0 * M * N * K
    value = world * ops / (step_ms * 1e-3) / 1e12
    peaks = load_peaks()
    int8_peak = peaks["bf16"] * INT8_OVER_BF16
    gemm_ops = 2.0 * M * N * K
    gemm_tops = gemm_ops / (gemm_ms_launch * 1e-3) / 1e12
    elem = 2  # bf16 source bytes
    # each rotation: its bf16 source read once + its 1-byte codes written
    quant_bytes = (elem + 1) * 2 * (M * K + N * K + M * N)
    quant_gbs = quant_bytes / (quant_ms_step * 1e-3) / 1e9
    traffic = recorded_traffic("gemm_pair_int8_llama_up_proj")
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": f"{w.name}: M={M} K={K} N={N} k={k} {w.fmt} codes, bf16 inputs",
                   "l2": "flushed between steps (256 MiB write, outside the step timing)",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "tensor", "kernel": "gemm_pair_kernel<int8,bf16 out> (tcgen05.mma.cta_group::2 kind::i8)",
                     "achieved": gemm_tops, "peak": int8_peak, "unit": "TFLOP/s",
                     "frac": gemm_tops / int8_peak, "traffic": traffic,
                     "peak_note": f"{peaks['src']} burst bf16 {peaks['bf16']} x {INT8_OVER_BF16} (nominal INT8/bf16 ratio; the timed region lasts tens of ms, clocks stay at max); ops = 2*M*N*K per launch"},
        "fwht_quant": {"achieved_gbs": quant_bytes / (alone_ms_step * 1e-3) / 1e9, "peak_gbs": peaks["hbm"],
                       "frac": quant_bytes / (alone_ms_step * 1e-3) / 1e9 / peaks["hbm"],
                       "bytes_per_step": quant_bytes, "ms_per_step": alone_ms_step,
                       "in_step_gbs": quant_gbs, "in_step_ms": quant_ms_step,
                       "kernel": "fwhtq_dual_kernel (both rotations of X, W, dY from one read per pass)",
                       "single_rotation_gbs": quant_bytes / (single_ms_step * 1e-3) / 1e9,
                       "single_rotation_ms": single_ms_step,
                       "note": "algorithmic bytes of the six rotations (bf16 source + 1-byte codes each); achieved: the three two-rotation quantizations timed alone with CUDA events, L2 flushed before each; in_step: summed event time of the same launches inside the overlapped step (sharing the GPU with the GEMMs); single_rotation: the six rotations as one-rotation calls"},
        "phases_ms": phases,
        "gemm_ms_per_step": gemm_ms_launch * 3,
        "schedule": "X and W along K + forward GEMM on the main stream; dY in both rotations (one read per pass), W along N and X along M on a side stream overlapping them; the dX GEMM waits for W along N, the dW GEMM for X along M",
        "frac_of_int8_peak_end_to_end": value / world / int8_peak,
        "e2e": {"value": world * ops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": elem * (M * K + N * K + M * N),
                "d2h_bytes_per_step": elem * (M * N + M * K + N * K),
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "note": "copies of step i+1 (in) and i-1 (out) overlap step i's kernels"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "device_status": int(status),
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, CPU_SAMPLE_TOKENS)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0 if status == 0 else 1


def run_sweep(args):
    """Every workload's layer (and the Llama-2-7B block over INT8/FP8 x k): the whole step
    through hq_linear_fwd_bwd, each GEMM alone and each rotation alone, CUDA events, L2
    flushed before every timed launch group.  One JSON line per point."""
    import torch
    import hadamard_rotated_precision_b200 as hq
    from hadamard_rotated_precision_b200 import build
    build.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    int8_peak = peaks["bf16"] * INT8_OVER_BF16
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    L_ = hq.lib()
    reps = max(3, args.steps)

    def timed(fn):
        for _ in range(2):
            flush.zero_()
            fn()
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            tot += a.elapsed_time(b)
        return tot / reps

    out_lines = []
    wids = [WORKLOAD_ID] if args.formats else sorted(synthetic.WORKLOADS)
    for wid in wids:
        w = synthetic.WORKLOADS[wid]
        points = list(w.sweep) if w.sweep else [(w.fmt, w.k)]
        if args.formats:  # the bench workload's layer in every code format at its k
            points = [(f, w.k) for f in ("int8", "fp8", "fp6_e3m2", "fp6_e2m3", "fp4_e2m1")]
        for li, Lr in enumerate(w.layers):
            d = synthetic.draw(w, li)
            def dev_t(a):
                if a.dtype == np.uint16:
                    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
                return torch.from_numpy(a).to(dev)
            X, W, dY = dev_t(d["X"]), dev_t(d["W"]), dev_t(d["dY"])
            M, K, N = Lr.M, Lr.K, Lr.N
            ws = torch.empty(hq.hq_linear_fwd_bwd_workspace_bytes(M, K, N), dtype=torch.uint8, device=dev)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
            dW = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
            for fmt_name, k in points:
                fmt = hq._fmt(fmt_name)
                step_ms = timed(lambda: hq.hq_linear_fwd_bwd(X, W, dY, k, fmt, Y=Y, dX=dX, dW=dW, workspace=ws))
                codes = {}
                quant_ms = 0.0
                for (nc, nr), src in ((("XK", "XM"), X), (("WK", "WN"), W), (("DN", "DM"), dY)):
                    cc = torch.empty(src.shape[0], src.shape[1], dtype=torch.uint8, device=dev)
                    cr = torch.empty(src.shape[1], src.shape[0], dtype=torch.uint8, device=dev)
                    sc, sr = (torch.empty(1, dtype=torch.float32, device=dev) for _ in range(2))
                    quant_ms += timed(lambda: hq.hq_quantize_dual(src, k, fmt, codes_c=cc, scale_c=sc,
                                                                  codes_r=cr, scale_r=sr))
                    codes[nc], codes[nr] = (cc, sc), (cr, sr)
                gemm_ms = 0.0
                for a, b, o in (("XK", "WK", Y), ("DN", "WN", dX), ("DM", "XM", dW)):
                    (ca, sa), (cb, sb) = codes[a], codes[b]
                    gws = torch.empty(max(16, hq.hq_gemm_workspace_bytes(ca.shape[0], cb.shape[0], ca.shape[1])),
                                      dtype=torch.uint8, device=dev)
                    gemm_ms += timed(lambda: hq.hq_gemm(ca, sa, cb, sb, fmt, out=o, workspace=gws))
                elem = X.element_size()
                qbytes = (elem + 1) * 2 * (M * K + N * K + M * N)
                ops = 6.0 * M * N * K
                line = {"workload": w.name, "layer": Lr.name, "M": M, "K": K, "N": N, "fmt": fmt_name, "k": k,
                        "dtype": "bf16" if elem == 2 else "f32",
                        "step_ms": step_ms, "step_tops": ops / (step_ms * 1e-3) / 1e12,
                        "gemm_ms": gemm_ms, "gemm_tops": ops / (gemm_ms * 1e-3) / 1e12,
                        "gemm_frac_of_peak": ops / (gemm_ms * 1e-3) / 1e12 / int8_peak,
                        "quant_ms": quant_ms, "quant_gbs": qbytes / (quant_ms * 1e-3) / 1e9,
                        "quant_frac_of_hbm": qbytes / (quant_ms * 1e-3) / 1e9 / peaks["hbm"],
                        "status": hq.hq_get_error()}
                out_lines.append(line)
                print(json.dumps(line), flush=True)
            del X, W, dY, ws, Y, dX, dW
            torch.cuda.empty_cache()
    return 0 if all(l["status"] == 0 for l in out_lines) else 1


def run_reuse(args):
    """The backward placement that reuses the forward's codes against the HALO-2 saved-codes
    flow, per workload and layer (INT8 / FP8 at the workload's k): hq_linear_fwd_keep +
    hq_linear_bwd_reuse (four rotations, the contraction-outermost dX GEMM, the output's
    de-rotation) against hq_linear_fwd_save + hq_linear_bwd (six rotations), each timed whole
    with CUDA events, L2 flushed before each; the reuse dX alone (GEMM + de-rotation) beside
    the HALO-2 dX GEMM alone.  One JSON line per point."""
    import torch
    import hadamard_rotated_precision_b200 as hq
    from hadamard_rotated_precision_b200 import build
    build.build()
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    peaks = load_peaks()
    int8_peak = peaks["bf16"] * INT8_OVER_BF16
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=dev)
    reps = max(3, args.steps)

    def timed(fn):
        for _ in range(2):
            flush.zero_()
            fn()
        tot = 0.0
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            tot += a.elapsed_time(b)
        return tot / reps

    def dev_t(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(a).to(dev)

    out_lines = []
    for wid in (2, 3, 4, 5):
        w = synthetic.WORKLOADS[wid]
        for li, Lr in enumerate(w.layers):
            d = synthetic.draw(w, li)
            X, W, dY = dev_t(d["X"]), dev_t(d["W"]), dev_t(d["dY"])
            M, K, N = Lr.M, Lr.K, Lr.N
            fmt, k = hq._fmt(w.fmt), w.k
            Y = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
            dX = torch.empty(M, K, dtype=torch.bfloat16, device=dev)
            dW = torch.empty(N, K, dtype=torch.bfloat16, device=dev)
            xqt = torch.empty(K, M, dtype=torch.uint8, device=dev)
            wq = torch.empty(N, K, dtype=torch.uint8, device=dev)
            sx, sw = (torch.empty(1, dtype=torch.float32, device=dev) for _ in range(2))
            ws = torch.empty(max(hq.hq_linear_fwd_save_workspace_bytes(M, K, N), hq.hq_linear_bwd_workspace_bytes(M, K, N),
                                 hq.hq_linear_fwd_keep_workspace_bytes(M, K, N),
                                 hq.hq_linear_bwd_reuse_workspace_bytes(M, K, N)), dtype=torch.uint8, device=dev)

            def halo2():
                hq.hq_linear_fwd_save(X, W, k, fmt, Y=Y, xqt=xqt, xqt_scale=sx, workspace=ws)
                hq.hq_linear_bwd(dY, W, xqt, sx, k, fmt, dX=dX, dW=dW, workspace=ws)

            def reuse():
                hq.hq_linear_fwd_keep(X, W, k, fmt, Y=Y, xqt=xqt, xqt_scale=sx, wq=wq, wq_scale=sw, workspace=ws)
                hq.hq_linear_bwd_reuse(dY, xqt, sx, wq, sw, k, fmt, dX=dX, dW=dW, workspace=ws)

            halo2_ms = timed(halo2)
            reuse_ms = timed(reuse)
            g, sg = hq.hq_quantize(dY, 0, k, fmt)
            dx_reuse_ms = timed(lambda: hq.hq_linear_bwd_dx_reuse(g, sg, wq, sw, k, fmt, dX=dX, workspace=ws))
            gn, sgn = hq.hq_quantize(dY, 1, k, fmt)
            wn, swn = hq.hq_quantize(W, 0, k, fmt)
            dx_gemm_ms = timed(lambda: hq.hq_gemm(gn, sgn, wn, swn, fmt, out=dX))
            ops = 6.0 * M * N * K
            line = {"workload": w.name, "layer": Lr.name, "M": M, "K": K, "N": N, "fmt": w.fmt, "k": k,
                    "halo2_step_ms": halo2_ms, "halo2_step_tops": ops / (halo2_ms * 1e-3) / 1e12,
                    "reuse_step_ms": reuse_ms, "reuse_step_tops": ops / (reuse_ms * 1e-3) / 1e12,
                    "reuse_frac_of_peak": ops / (reuse_ms * 1e-3) / 1e12 / int8_peak,
                    "dx_reuse_ms": dx_reuse_ms, "dx_halo2_gemm_ms": dx_gemm_ms,
                    "derotate_bytes": 14 * M * K,
                    "status": hq.hq_get_error()}
            out_lines.append(line)
            print(json.dumps(line), flush=True)
            del X, W, dY, Y, dX, dW, xqt, wq, ws
            torch.cuda.empty_cache()
    # the next layer's rotation in the epilogue, on the bench layer's forward GEMM: the GEMM
    # writing its output rotated along N in fp32 plus the quantization of that output as it is,
    # against the bf16 GEMM plus the rotating quantization of its output along N
    w = synthetic.WORKLOADS[WORKLOAD_ID]
    Lr = w.layers[0]
    M, K, N = Lr.M, Lr.K, Lr.N
    fmt, k = hq._fmt(w.fmt), w.k
    g = torch.Generator(device="cuda").manual_seed(1)
    qa = torch.randint(-127, 128, (M, K), generator=g, device=dev, dtype=torch.int32).to(torch.int8).view(torch.uint8)
    qb = torch.randint(-127, 128, (N, K), generator=g, device=dev, dtype=torch.int32).to(torch.int8).view(torch.uint8)
    s1 = torch.full((1,), 1e-3, device=dev)
    yr = torch.empty(M, N, dtype=torch.float32, device=dev)
    yb = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
    codes = torch.empty(M, N, dtype=torch.uint8, device=dev)
    sc = torch.empty(1, dtype=torch.float32, device=dev)
    ws = torch.empty(hq.hq_quantize_workspace_bytes(), dtype=torch.uint8, device=dev)
    rot_gemm_ms = timed(lambda: hq.hq_gemm_rotout(qa, s1, qb, s1, k, fmt, out=yr))
    prerot_ms = timed(lambda: hq.hq_quantize_prerotated(yr, fmt, codes=codes, scale=sc, workspace=ws))
    plain_gemm_ms = timed(lambda: hq.hq_gemm(qa, s1, qb, s1, fmt, out=yb))
    plain_quant_ms = timed(lambda: hq.hq_quantize(yb, 1, k, fmt, codes=codes, scale=sc, workspace=ws))
    line = {"case": "next_layer_rotation_in_epilogue", "workload": w.name, "M": M, "K": K, "N": N, "fmt": w.fmt,
            "k": k, "gemm_rotout_ms": rot_gemm_ms, "gemm_rotout_tops": 2.0 * M * N * K / (rot_gemm_ms * 1e-3) / 1e12,
            "quantize_prerotated_ms": prerot_ms,
            # two passes reading 4 B and one 1-byte code per element
            "quantize_prerotated_gbs": 9.0 * M * N / (prerot_ms * 1e-3) / 1e9,
            "gemm_bf16_ms": plain_gemm_ms, "quantize_rotating_ms": plain_quant_ms,
            "fused_ms": rot_gemm_ms + prerot_ms, "unfused_ms": plain_gemm_ms + plain_quant_ms,
            "status": hq.hq_get_error()}
    out_lines.append(line)
    print(json.dumps(line), flush=True)
    return 0 if all(l["status"] == 0 for l in out_lines) else 1


def run_kernel_case(args):
    """One small standalone invocation of a hot kernel, for profiler captures: a warm-up
    call, then the captured call(s).  Inputs exceed L2 (126 MB) but stay near 200 MB."""
    import torch
    import hadamard_rotated_precision_b200 as hq
    from hadamard_rotated_precision_b200 import build
    build.build()
    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(0)
    case = args.kernel_case
    if case.startswith("gemm"):
        fmt = "fp8" if case == "gemm_fp8" else "int8"
        # the Llama up-projection forward shape, or the ViT-B fc1 forward (contraction 768)
        M, N, K = (12608, 3072, 768) if case == "gemm_short_k" else (4096, 11008, 4096)
        A = torch.randint(-127, 128, (M, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        B = torch.randint(-127, 128, (N, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        if fmt == "fp8":
            A = A & 0x77  # finite e4m3 codes, magnitude <= 240
            B = B & 0x77
        s = torch.full((1,), 0.01, device="cuda")
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        for _ in range(2):
            hq.hq_gemm(A, s, B, s, fmt, out=out)
    elif case == "dx_reuse":
        # a dX of the reuse placement at 4096 tokens, K = 4096, contraction 8192 (codes 2 x 32 MB,
        # fp32 output 64 MB + bf16 32 MB: more than L2)
        M, K, N = 4096, 4096, 8192
        gq = torch.randint(-127, 128, (N, M), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        wq = torch.randint(-127, 128, (N, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        s = torch.full((1,), 0.01, device="cuda")
        for _ in range(2):
            hq.hq_linear_bwd_dx_reuse(gq, s, wq, s, 128, "int8")
    elif case == "quant_dual":
        x = torch.randn(11008, 4096, generator=g, device="cuda").to(torch.bfloat16)
        for _ in range(2):
            hq.hq_quantize_dual(x, 256, "int8")
    else:
        rows, cols, dim = (11008, 4096, 1) if case == "quant_rows" else (11008, 4096, 0)
        x = torch.randn(rows, cols, generator=g, device="cuda").to(torch.bfloat16)
        for _ in range(2):
            hq.hq_quantize(x, dim, 256, "int8")
    torch.cuda.synchronize()
    st = hq.hq_get_error()
    print(json.dumps({"kernel_case": case, "status": st}))
    return 0 if st == 0 else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("hq", "reference"), default="hq")
    ap.add_argument("--kernel-case", choices=("gemm", "gemm_fp8", "gemm_short_k", "quant_rows", "quant_cols", "quant_dual",
                                              "dx_reuse"),
                    help="run one small standalone kernel case (for profiler captures) and exit")
    ap.add_argument("--formats", action="store_true",
                    help="with --sweep: the bench workload's layer in every code format (INT8, FP8, FP6, FP4)")
    ap.add_argument("--reuse", action="store_true",
                    help="time the backward placement that reuses the forward's codes against HALO-2, every workload, and exit")
    ap.add_argument("--sweep", action="store_true",
                    help="time every workload (one JSON line per workload/layer/format/k) and exit")
    args = ap.parse_args(argv)
    if args.kernel_case:
        return run_kernel_case(args)
    if args.sweep:
        return run_sweep(args)
    if args.reuse:
        return run_reuse(args)
    args.warmup = max(args.warmup, 3)  # timing rule: at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
