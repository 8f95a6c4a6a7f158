#!/usr/bin/env python
"""Benchmark: the HALO-2 linear layers of a Llama-2-7B-shaped decoder block, forward + both
backward GEMMs, on B200.

A step is the whole hot path over one batch for every linear layer of the block (qkv 4096 ->
12288, o 4096 -> 4096, gate and up 4096 -> 11008, down 11008 -> 4096; 8192 tokens): per
layer the six Hadamard-rotate + quantize passes (X along K and M, W along K and N, dY along N
and M) and the three tcgen05 GEMMs with the dequantizing epilogue (Y = X W^T, dX = dY W,
dW = dY^T X), each layer through the library's own entry point hq_linear_fwd_bwd.  INT8
codes, k = 256, bf16 inputs drawn seeded (N(0,1) activations with 1% outlier channels x
U[30,100], N(0,0.02) weights, Student-t(3) x 1e-3 output gradients).

Prints one JSON line (rank 0).  `value` = sum over layers of 6*M*N*K / device time per step
(TOPS), inputs resident in HBM; `e2e` = the same metric through the same entry point with the
inputs copied from pinned host memory and the three outputs of every layer copied back inside
the timed region.  The dense INT8 / FP8 tensor peaks are measured in the same run
(hq_mma_peak: MMA-only, operands in shared memory).

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

WORKLOAD_ID = 5        # the Llama-2-7B block at 8192 tokens (INT8, k = 256 for the headline step)
LAYER_WORKLOAD_ID = 2  # the Llama up-projection layer at 4096 tokens (an extra key of the line)
METRIC = "HALO-2 linear fwd+bwd TOPS, % of INT8/FP8 tensor peak; FWHT+quant HBM GB/s"
UNIT = "TOPS"
NOMINAL_INT8_TOPS = 4500.0  # B200 dense INT8 / FP8, nominal (context only)
GEMM_SRC = os.path.join(ROOT, "hadamard_rotated_precision_b200", "csrc", "gemm_tcgen05.cuh")
QUANT_SRC = os.path.join(ROOT, "hadamard_rotated_precision_b200", "csrc", "fwht_dual.cuh")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
CPU_SAMPLE_TOKENS = 256   # cpu_baseline: every layer of the block at this many tokens
REF_STEP_TOKENS = 256     # --impl reference: one layer of the block per step (in turn), this many tokens
# (token samples are multiples of k: the weight gradient's operands are rotated along the tokens)
MMA_OPS = 2 * 256 * 256 * 32  # operations of one CTA-pair MMA instruction of the peak probe
# the roofline kernel: the block's largest GEMM launch, the qkv weight gradient
ROOFLINE_GEMM = ("qkv", "dW")
ROOFLINE_GEMM_KEY = "gemm_pair_int8_12288x4096x8192"


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


def draw_block(w, tokens=None):
    """Every layer's inputs (seeded, numpy), drawn in parallel worker processes started with
    spawn before any CUDA call of this process."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    n = len(w.layers)
    with ProcessPoolExecutor(max_workers=max(1, min(n, os.cpu_count() or 1)),
                             mp_context=mp.get_context("spawn")) as ex:
        futs = [ex.submit(synthetic.draw, w, li, tokens) for li in range(n)]
        return [f.result() for f in futs]


def block_ops(w, tokens=None) -> float:
    return sum(6.0 * (L.M if tokens is None else tokens) * L.N * L.K for L in w.layers)


def measure_mma_peaks(hq, torch, sustained: bool = True):
    """Dense tensor-core peaks of this GPU, measured with the MMA-only probe (operands in
    shared memory, accumulator in TMEM, no global traffic): burst = best of ten ~1 ms runs,
    sustained = one run of about a quarter second (under the power cap)."""
    def run(fmt, n_blocks, reps):
        best, pairs = 0.0, 0
        for _ in range(reps):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            pairs = hq.hq_mma_peak(fmt, n_blocks)
            b.record()
            torch.cuda.synchronize()
            best = max(best, pairs * n_blocks * 4 * MMA_OPS / (a.elapsed_time(b) * 1e-3) / 1e12)
        return best
    out = {}
    for name in ("int8", "fp8"):
        run(name, 256, 2)
        out[name] = run(name, 4096, 10)
        if sustained and name == "int8":
            out["int8_sustained"] = run(name, 1000000, 1)
    if hq.hq_get_error() != 0:
        raise SystemExit("tensor-core peak probe reported a device error")
    return out


# ----------------------------------------------------------------------------- CPU (oracle)

def oracle_block_seconds(ds, w, fmt: int) -> float:
    import oracle
    t0 = time.perf_counter()
    for d in ds:
        oracle.linear_fwd(d["X"], d["W"], w.k, fmt)
        oracle.linear_bwd_dx(d["dY"], d["W"], w.k, fmt)
        oracle.linear_bwd_dw(d["dY"], d["X"], w.k, fmt)
    return time.perf_counter() - t0


def cpu_baseline(w, ds_sample, tokens: int):
    """The oracle, untuned, on a token-prefix sample of every layer of the block (full K, N,
    k, format)."""
    import oracle
    fmt = 0 if w.fmt == "int8" else 1
    secs = oracle_block_seconds(ds_sample, w, fmt)
    ops = block_ops(w, tokens)
    return {"value": ops / secs / 1e12, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
            "sample": f"all {len(w.layers)} layers of {w.name} (fwd+dX+dW) at {tokens} of {w.layers[0].M} tokens "
                      f"(full K, N, k={w.k}, {w.fmt}), {secs:.2f} s"}


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = synthetic.WORKLOADS[WORKLOAD_ID]
    ds = draw_block(w, REF_STEP_TOKENS)
    fmt = 0 if w.fmt == "int8" else 1
    n = len(w.layers)

    def layer_step(i):
        d, L = ds[i % n], w.layers[i % n]
        t0 = time.perf_counter()
        oracle.linear_fwd(d["X"], d["W"], w.k, fmt)
        oracle.linear_bwd_dx(d["dY"], d["W"], w.k, fmt)
        oracle.linear_bwd_dw(d["dY"], d["X"], w.k, fmt)
        return time.perf_counter() - t0, 6.0 * REF_STEP_TOKENS * L.N * L.K

    for i in range(args.warmup):
        layer_step(i)
    total, ops = 0.0, 0.0
    for i in range(args.steps):
        t, o = layer_step(i)
        total += t
        ops += o
    value = ops / total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: Llama-2-7B block linears (qkv, o, gate, up, down) at "
                               f"{w.layers[0].M} tokens, k={w.k} {w.fmt}, bf16 inputs",
                   "step_sample_tokens": REF_STEP_TOKENS, "parallelism": "rank 0 only (CPU)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": oracle.threads(), "kind": "oracle",
                         "sample": f"step i: layer i mod {n} of the block, fwd+dX+dW at {REF_STEP_TOKENS} of "
                                   f"{w.layers[0].M} tokens (full K, N)"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU

def run_gpu(args):
    world, rank, local = dist_env()
    w = synthetic.WORKLOADS[WORKLOAD_ID]
    # host-side draws first: the worker pool starts (spawn) before this process touches CUDA
    inputs = draw_block(w)
    cpu_sample = draw_block(w, CPU_SAMPLE_TOKENS) if (rank == 0 and world == 1) else None

    import torch
    import hadamard_rotated_precision_b200 as hq
    from hadamard_rotated_precision_b200 import build

    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 must be launched with torchrun (one process per GPU)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    init_dist(world, "nccl")
    build.build()
    hq.lib()
    k = w.k
    fmt = hq.HQ_INT8 if w.fmt == "int8" else hq.HQ_FP8_E4M3

    def dev(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(device)

    layers = []
    for L, d in zip(w.layers, inputs):
        M, K, N = L.M, L.K, L.N
        layers.append(dict(
            L=L, X=dev(d["X"]), W=dev(d["W"]), dY=dev(d["dY"]),
            Y=torch.empty(M, N, dtype=torch.bfloat16, device=device),
            dX=torch.empty(M, K, dtype=torch.bfloat16, device=device),
            dW=torch.empty(N, K, dtype=torch.bfloat16, device=device),
            ws=torch.empty(hq.hq_linear_fwd_bwd_workspace_bytes(M, K, N), dtype=torch.uint8, device=device)))
    del inputs
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    peaks_file = load_peaks()
    mma = measure_mma_peaks(hq, torch)
    int8_peak = mma["int8"]

    # The step: every layer through the public entry point, one after another on one stream.
    def step(evs=None):
        for i, l in enumerate(layers):
            if evs is not None:
                evs[i].record(stream)
            hq.hq_linear_fwd_bwd(l["X"], l["W"], l["dY"], k, fmt, Y=l["Y"], dX=l["dX"], dW=l["dW"],
                                 workspace=l["ws"], stream=stream)
        if evs is not None:
            evs[-1].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize(device)
    if hq.hq_get_error(stream) != 0:
        raise SystemExit("device status error during warm-up")
    # outputs of an untimed call, compared bit for bit with the timed steps' afterwards
    ref_out = [tuple(l[n].clone() for n in ("Y", "dX", "dW")) for l in layers]

    # ---------------------------------------------------------------- timed region (device)
    evs = [[ev() for _ in range(len(layers) + 1)] for _ in range(args.steps)]
    barrier(world, device)
    torch.cuda.synchronize(device)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.zero_()  # L2 flush (256 MiB > 126 MB L2), outside the step's events
            step(evs[i])
        torch.cuda.synchronize(device)
    barrier(world, device)
    torch.cuda.synchronize(device)
    status = hq.hq_get_error(stream)
    outputs_match = all(torch.equal(l[n].view(torch.int16), r.view(torch.int16))
                        for l, rr in zip(layers, ref_out) for n, r in zip(("Y", "dX", "dW"), rr))
    del ref_out
    step_ms_local = sum(e[0].elapsed_time(e[-1]) for e in evs) / args.steps
    layer_ms = {l["L"].name: sum(e[i].elapsed_time(e[i + 1]) for e in evs) / args.steps
                for i, l in enumerate(layers)}
    step_ms = reduce_max(step_ms_local, world, device)
    # our kernels per layer call: X and W in both rotations and dY in both (2 launches per
    # rotation pass pair: 5 quantizations x 2) plus the three GEMMs
    launches = 13 * len(layers) * args.steps

    # ---------------------------------------------------------------- kernels alone
    # Every layer's X, W and dY quantized in both rotations by the fused two-rotation kernel
    # (hq_quantize_dual), each call timed alone with L2 flushed before it; then the three GEMMs
    # of every layer on those codes (hq_gemm_ws, the same kernels and split rule as the step),
    # each launch timed alone.
    reps = max(3, min(args.steps, 5))

    quant = []
    gemm = []
    for l in layers:
        L = l["L"]
        codes = {}
        for (nc, nr), src in ((("XK", "XM"), l["X"]), (("WK", "WN"), l["W"]), (("DN", "DM"), l["dY"])):
            cc = torch.empty(src.shape[0], src.shape[1], dtype=torch.uint8, device=device)
            cr = torch.empty(src.shape[1], src.shape[0], dtype=torch.uint8, device=device)
            sc, sr = (torch.empty(1, dtype=torch.float32, device=device) for _ in range(2))
            qws = torch.empty(hq.hq_quantize_dual_workspace_bytes(), dtype=torch.uint8, device=device)
            fn = lambda: hq.hq_quantize_dual(src, k, fmt, codes_c=cc, scale_c=sc, codes_r=cr, scale_r=sr,  # noqa: E731
                                             workspace=qws, stream=stream)
            fn()
            torch.cuda.synchronize(device)
            ms = []
            for _ in range(reps):
                flush.zero_()
                a, b = ev(), ev()
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize(device)
                ms.append(a.elapsed_time(b))
            t = statistics.median(ms)
            nbytes = 2 * (2 + 1) * src.numel()  # two rotations: bf16 source + 1-byte codes each
            quant.append({"layer": L.name, "tensor": nc[0] if nc[0] != "D" else "dY",
                          "shape": list(src.shape), "us": 1e3 * t, "gbs": nbytes / (t * 1e-3) / 1e9})
            codes[nc], codes[nr] = (cc, sc), (cr, sr)
        for name, (a_, b_, o) in (("fwd", ("XK", "WK", l["Y"])), ("dX", ("DN", "WN", l["dX"])),
                                  ("dW", ("DM", "XM", l["dW"]))):
            (ca, sa), (cb, sb) = codes[a_], codes[b_]
            Mg, Ng, Kg = ca.shape[0], cb.shape[0], ca.shape[1]
            gws = torch.empty(max(16, hq.hq_gemm_workspace_bytes(Mg, Ng, Kg)), dtype=torch.uint8, device=device)
            fn = lambda: hq.hq_gemm(ca, sa, cb, sb, fmt, out=o, workspace=gws, stream=stream)  # noqa: E731
            fn()
            ms = []
            for _ in range(reps):
                flush.zero_()
                a, b = ev(), ev()
                a.record(stream)
                fn()
                b.record(stream)
                torch.cuda.synchronize(device)
                ms.append(a.elapsed_time(b))
            t = statistics.median(ms)
            gemm.append({"layer": L.name, "gemm": name, "M": Mg, "N": Ng, "K": Kg, "us": 1e3 * t,
                         "tops": 2.0 * Mg * Ng * Kg / (t * 1e-3) / 1e12})
        del codes
    status |= hq.hq_get_error(stream)
    gemm_ops = sum(2.0 * g["M"] * g["N"] * g["K"] for g in gemm)
    gemm_ms = sum(g["us"] for g in gemm) * 1e-3
    all_gemm_tops = reduce_max(gemm_ops / (gemm_ms * 1e-3) / 1e12, world, device)
    rg = next(g for g in gemm if (g["layer"], g["gemm"]) == ROOFLINE_GEMM)
    gemm_tops = reduce_max(rg["tops"], world, device)
    quant_bytes = sum(2 * 3 * l[n].numel() for l in layers for n in ("X", "W", "dY"))
    quant_ms = sum(q["us"] for q in quant) * 1e-3
    quant_gbs = quant_bytes / (quant_ms * 1e-3) / 1e9

    # pinned host copies of the inputs for the end-to-end leg below
    hosts = []
    for l in layers:
        L = l["L"]
        hosts.append(dict(X=l["X"].cpu().pin_memory(), W=l["W"].cpu().pin_memory(), dY=l["dY"].cpu().pin_memory(),
                          Y=torch.empty(L.M, L.N, dtype=torch.bfloat16, pin_memory=True),
                          dX=torch.empty(L.M, L.K, dtype=torch.bfloat16, pin_memory=True),
                          dW=torch.empty(L.N, L.K, dtype=torch.bfloat16, pin_memory=True)))

    # ---------------------------------------------------------------- one layer (extra key)
    wl = synthetic.WORKLOADS[LAYER_WORKLOAD_ID]
    Ll = wl.layers[0]
    del layers
    torch.cuda.empty_cache()
    dl = synthetic.draw(wl, 0)
    lX, lW, ldY = dev(dl["X"]), dev(dl["W"]), dev(dl["dY"])
    lws = torch.empty(hq.hq_linear_fwd_bwd_workspace_bytes(Ll.M, Ll.K, Ll.N), dtype=torch.uint8, device=device)
    lY = torch.empty(Ll.M, Ll.N, dtype=torch.bfloat16, device=device)
    ldX = torch.empty(Ll.M, Ll.K, dtype=torch.bfloat16, device=device)
    ldW = torch.empty(Ll.N, Ll.K, dtype=torch.bfloat16, device=device)
    lfn = lambda: hq.hq_linear_fwd_bwd(lX, lW, ldY, wl.k, fmt, Y=lY, dX=ldX, dW=ldW, workspace=lws,  # noqa: E731
                                       stream=stream)
    lfn()
    lms = []
    for _ in range(reps):
        flush.zero_()
        a, b = ev(), ev()
        a.record(stream)
        lfn()
        b.record(stream)
        torch.cuda.synchronize(device)
        lms.append(a.elapsed_time(b))
    layer_step_ms = statistics.median(lms)
    del lX, lW, ldY, lws, lY, ldX, ldW, dl
    torch.cuda.empty_cache()

    # ---------------------------------------------------------------- end to end (host buffers)
    # Every step copies every layer's X, W, dY from pinned host memory, runs hq_linear_fwd_bwd
    # for each layer and copies every Y, dX, dW back.  Steps are pipelined over two device
    # buffer sets and three streams: the host->device copies of step i+1 and the device->host
    # copies of step i-1 overlap step i's kernels (PCIe is full duplex).  Timed from the first
    # copy in to the last copy out.
    e2e_steps = max(2, min(args.steps, 5))
    bufs = [[], []]
    for L in w.layers:
        M, K, N = L.M, L.K, L.N
        for b in bufs:
            b.append(dict(X=torch.empty(M, K, dtype=torch.bfloat16, device=device),
                          W=torch.empty(N, K, dtype=torch.bfloat16, device=device),
                          dY=torch.empty(M, N, dtype=torch.bfloat16, device=device),
                          Y=torch.empty(M, N, dtype=torch.bfloat16, device=device),
                          dX=torch.empty(M, K, dtype=torch.bfloat16, device=device),
                          dW=torch.empty(N, K, dtype=torch.bfloat16, device=device),
                          ws=torch.empty(hq.hq_linear_fwd_bwd_workspace_bytes(M, K, N), dtype=torch.uint8,
                                         device=device)))
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    s_cmp = stream
    h2d = sum(2 * (L.M * L.K + L.N * L.K + L.M * L.N) for L in w.layers)

    def e2e_run(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_cmp = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = ev(), ev()
        t0.record(s_in)
        for i in range(nsteps):
            bset = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_cmp[i - 2])  # step i-2 finished reading these inputs
                for h, b in zip(hosts, bset):
                    for n in ("X", "W", "dY"):
                        b[n].copy_(h[n], non_blocking=True)
                ev_in[i].record(s_in)
            s_cmp.wait_event(ev_in[i])
            if i >= 2:
                s_cmp.wait_event(ev_out[i - 2])  # step i-2's outputs are on the host
            for b in bset:
                hq.hq_linear_fwd_bwd(b["X"], b["W"], b["dY"], k, fmt, Y=b["Y"], dX=b["dX"], dW=b["dW"],
                                     workspace=b["ws"], stream=s_cmp)
            ev_cmp[i].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[i])
                for h, b in zip(hosts, bset):
                    for n in ("Y", "dX", "dW"):
                        h[n].copy_(b[n], non_blocking=True)
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
    ops = block_ops(w)
    value = world * ops / (step_ms * 1e-3) / 1e12
    traffic = recorded_traffic(ROOFLINE_GEMM_KEY)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8", "data": "synthetic",
        "config": {"workload": f"{w.name}: Llama-2-7B block linears qkv 4096->12288, o 4096->4096, "
                               f"gate/up 4096->11008, down 11008->4096 at {w.layers[0].M} tokens; "
                               f"k={k} {w.fmt} codes, bf16 inputs",
                   "l2": "flushed between steps (256 MiB write, outside the step timing); inputs exceed L2",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "roofline": {"bound": "tensor", "kernel": "gemm_pair_kernel<int8,bf16 out> (tcgen05.mma.cta_group::2 kind::i8): "
                                                  "the block's largest launch, the qkv weight gradient 12288 x 4096 x 8192, "
                                                  "timed alone (median of the repetitions)",
                     "achieved": gemm_tops, "peak": int8_peak, "unit": "TFLOP/s",
                     "frac": gemm_tops / int8_peak, "traffic": traffic,
                     "algorithmic_bytes": float(rg["M"] * rg["K"] + rg["N"] * rg["K"] + 2 * rg["M"] * rg["N"]),
                     "frac_of_nominal": gemm_tops / NOMINAL_INT8_TOPS,
                     "all_gemms_tops": all_gemm_tops, "all_gemms_frac": all_gemm_tops / int8_peak,
                     "peak_note": "measured in this run: hq_mma_peak INT8, tcgen05 kind::i8 CTA-pair MMAs with "
                                  "operands in shared memory, best of ten ~1 ms runs (burst); ops = 2*M*N*K per "
                                  f"launch; nominal {NOMINAL_INT8_TOPS:.0f} for context; traffic = ncu DRAM read + "
                                  "write of one launch of that shape (profiles/traffic.json, null when the kernel "
                                  "source changed since)"},
        "mma_peak_tops": {"int8_burst": mma["int8"], "int8_sustained": mma.get("int8_sustained"),
                          "fp8_burst": mma["fp8"], "bf16_burst_measured_file": peaks_file["bf16"],
                          "source": "hq_mma_peak in this run"},
        "fwht_quant": {"achieved_gbs": quant_gbs, "peak_gbs": peaks_file["hbm"], "frac": quant_gbs / peaks_file["hbm"],
                       "bytes_per_step": quant_bytes, "ms_per_step": quant_ms,
                       "kernel": "fwhtq_dual_kernel (both rotations of one tensor from one read per pass)",
                       "per_shape": quant,
                       "note": "algorithmic bytes of the 30 rotations (bf16 source + 1-byte codes each) over the "
                               "15 two-rotation calls' CUDA-event times, each call alone with L2 flushed before "
                               f"it; HBM peak: {peaks_file['src']} copy bandwidth"},
        "gemms": gemm,
        "phases_ms": layer_ms,
        "gemm_ms_per_step": gemm_ms,
        "frac_of_int8_peak_end_to_end": value / world / int8_peak,
        "frac_of_nominal_end_to_end": value / world / NOMINAL_INT8_TOPS,
        "outputs_match_untimed_call": bool(outputs_match),
        "llama_up_proj_layer": {"workload": f"{wl.name}: M={Ll.M} K={Ll.K} N={Ll.N} k={wl.k} {wl.fmt}",
                                "ms": layer_step_ms,
                                "tops": 6.0 * Ll.M * Ll.N * Ll.K / (layer_step_ms * 1e-3) / 1e12},
        "e2e": {"value": world * ops / (e2e_ms * 1e-3) / 1e12, "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": h2d,
                "ms_per_step": e2e_ms, "steps": e2e_steps,
                "note": "hq_linear_fwd_bwd per layer with host buffers; copies of step i+1 (in) and i-1 (out) "
                        "overlap step i's kernels"},
        "gpu_launches": launches,
        "clocks": clocks.summary(),
        "device_status": int(status),
    }
    if rank == 0 and world == 1:
        line["cpu_baseline"] = cpu_baseline(w, cpu_sample, CPU_SAMPLE_TOKENS)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0 if (status == 0 and outputs_match) else 1


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
    mma = measure_mma_peaks(hq, torch, sustained=False)
    # INT8 GEMMs against the measured INT8 peak, the kind::f8f6f4 formats against the FP8 one
    peak_of = lambda f: mma["int8"] if f == "int8" else mma["fp8"]  # noqa: E731
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
                        "gemm_frac_of_peak": ops / (gemm_ms * 1e-3) / 1e12 / peak_of(fmt_name),
                        "peak_tops": peak_of(fmt_name),
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
    mma = measure_mma_peaks(hq, torch, sustained=False)
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
                    "reuse_frac_of_peak": ops / (reuse_ms * 1e-3) / 1e12 / (mma["int8"] if fmt == hq.HQ_INT8 else mma["fp8"]),
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
    if case == "block_step":
        # two steps of the bench's headline workload (every layer of the Llama-2-7B block through
        # hq_linear_fwd_bwd), for the launch list of the step
        w = synthetic.WORKLOADS[WORKLOAD_ID]
        ls = []
        for li, L in enumerate(w.layers):
            d = synthetic.draw(w, li)
            t = {n: torch.from_numpy(d[n].view(np.int16)).view(torch.bfloat16).cuda() for n in ("X", "W", "dY")}
            t["ws"] = torch.empty(hq.hq_linear_fwd_bwd_workspace_bytes(L.M, L.K, L.N), dtype=torch.uint8, device="cuda")
            ls.append(t)
        for _ in range(2):
            for t in ls:
                hq.hq_linear_fwd_bwd(t["X"], t["W"], t["dY"], w.k, w.fmt, workspace=t["ws"])
        torch.cuda.synchronize()
        st = hq.hq_get_error()
        print(json.dumps({"kernel_case": case, "status": st}))
        return 0 if st == 0 else 1
    if case.startswith("gemm"):
        fmt = "fp8" if case == "gemm_fp8" else "int8"
        # the Llama up-projection forward shape, or the ViT-B fc1 forward (contraction 768), or its
        # dX (contraction 11008: 3.46 waves of tiles, the last wave split along the contraction
        # through the workspace), or --shape M,N,K
        M, N, K = {"gemm_short_k": (12608, 3072, 768), "gemm_split": (4096, 4096, 11008)}.get(case, (4096, 11008, 4096))
        if args.shape:
            M, N, K = (int(v) for v in args.shape.split(","))
        A = torch.randint(-127, 128, (M, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        B = torch.randint(-127, 128, (N, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        if fmt == "fp8":
            A = A & 0x77  # finite e4m3 codes, magnitude <= 240
            B = B & 0x77
        s = torch.full((1,), 0.01, device="cuda")
        out = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        ws = None
        if case == "gemm_split":
            ws = torch.empty(max(16, hq.hq_gemm_workspace_bytes(M, N, K)), dtype=torch.uint8, device="cuda")
        for _ in range(2):
            hq.hq_gemm(A, s, B, s, fmt, out=out, workspace=ws)
    elif case == "rotout":
        # the next layer's rotation in the epilogue: 4096 x 4096 x 4096 INT8, fp32 output rotated
        # along its columns in blocks of 256 (64 MB)
        M = N = K = 4096
        A = torch.randint(-127, 128, (M, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        B = torch.randint(-127, 128, (N, K), generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
        s = torch.full((1,), 0.01, device="cuda")
        for _ in range(2):
            hq.hq_gemm_rotout(A, s, B, s, 256, "int8")
    elif case == "prerot":
        # codes of already-rotated fp32 values, 4096 x 11008 (180 MB)
        y = torch.randn(4096, 11008, generator=g, device="cuda")
        for _ in range(2):
            hq.hq_quantize_prerotated(y, "int8")
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
    ap.add_argument("--kernel-case", choices=("gemm", "gemm_fp8", "gemm_short_k", "gemm_split", "rotout", "prerot",
                                              "quant_rows", "quant_cols", "quant_dual",
                                              "dx_reuse", "block_step"),
                    help="run one small standalone kernel case (for profiler captures) and exit")
    ap.add_argument("--shape", help="with --kernel-case gemm / gemm_fp8: M,N,K of the GEMM")
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
