"""Seeded synthetic inputs shaped like the pages' linear-layer workloads.

This module only draws random numbers; it holds none of the method's arithmetic and is the
one piece of code shared by the CUDA path's tests/benchmark and the CPU oracle.

Distributions stand in for what the pages describe about real tensors: activations with a
few feature-wise outlier channels ("Training Transformers with 4-bit Integers", section 3.2
"Activation Outliers"), small Gaussian weights, and heavy-tailed, mostly-small output
gradients (same page, section 4.1 "Structural Sparsity of Gradients").  No dataset, trained
weight or checkpoint is used.

Seeding: numpy ``default_rng(SeedSequence([workload_seed, layer_index, tensor_id]))`` with
tensor ids X=0, W=1, dY=2, outlier-channel choice=3.  Values are drawn in fp64, cast to fp32,
and for bf16 workloads rounded to bf16 (round-to-nearest-even) and returned as uint16 bit
patterns.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

X_ID, W_ID, DY_ID, OUTLIER_ID = 0, 1, 2, 3


@dataclass(frozen=True)
class Layer:
    name: str
    M: int  # tokens
    K: int  # d_in
    N: int  # d_out


@dataclass(frozen=True)
class Workload:
    name: str
    seed: int
    dtype: str                       # "f32" | "bf16"
    fmt: str                         # "int8" | "fp8"
    k: int
    layers: Tuple[Layer, ...]
    x_outlier_frac: float            # fraction of X channels that are outliers
    x_outlier_count: Optional[int]   # exact count if the workload states one
    x_outlier_scale: Tuple[float, float]  # uniform range of the outlier multiplier
    dy_dist: str                     # "student_t3" | "laplace"
    sweep: Tuple[Tuple[str, int], ...] = field(default_factory=tuple)


def _llama(seed, name, fmt, k, layers, sweep=()):
    return Workload(name, seed, "bf16", fmt, k, layers, 0.01, None, (30.0, 100.0), "student_t3",
                    tuple(sweep))


WORKLOADS = {
    # Tiny single layer, INT8 k=16, fp32, 4 outlier columns x50.
    1: Workload("tiny_int8_k16", 0, "f32", "int8", 16, (Layer("tiny", 64, 256, 128),),
                0.0, 4, (50.0, 50.0), "student_t3"),
    # Llama-style MLP up-projection: 4096 tokens (4 x 1024), 4096 -> 11008, INT8 k=256.
    2: _llama(1, "llama_up_proj_int8_k256", "int8", 256, (Layer("up_proj", 4096, 4096, 11008),)),
    # Attention output projection: 8192 tokens, 4096 -> 4096, FP8 e4m3 k=128.
    3: _llama(2, "attn_out_proj_fp8_k128", "fp8", 128, (Layer("o_proj", 8192, 4096, 4096),)),
    # ViT-B MLP: 12608 tokens (64 x 197), fc1 768 -> 3072 and fc2 3072 -> 768, INT8 k=64.
    4: Workload("vitb_mlp_int8_k64", 3, "bf16", "int8", 64,
                (Layer("fc1", 12608, 768, 3072), Layer("fc2", 12608, 3072, 768)),
                0.005, None, (50.0, 50.0), "laplace"),
    # Llama-2-7B decoder block linears at 8192 tokens, INT8/FP8 x k in {16..256}.
    5: _llama(4, "llama2_7b_block_sweep", "int8", 256,
              (Layer("qkv", 8192, 4096, 12288), Layer("o", 8192, 4096, 4096),
               Layer("gate", 8192, 4096, 11008), Layer("up", 8192, 4096, 11008),
               Layer("down", 8192, 11008, 4096)),
              sweep=[(f, k) for f in ("int8", "fp8") for k in (16, 32, 64, 128, 256)]),
}


def _rng(seed: int, layer: int, tensor: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([seed, layer, tensor]))


def outlier_count(w: Workload, K: int) -> int:
    if w.x_outlier_count is not None:
        return w.x_outlier_count
    return max(1, int(round(w.x_outlier_frac * K)))


def draw_fp32(w: Workload, layer_index: int = 0, M: Optional[int] = None):
    """Return dict X[M][K], W[N][K], dY[M][N] as fp32 numpy arrays.

    Passing a smaller M draws a token-prefix sample of the same workload: numpy fills each
    array in row-major order from its own stream, so X and dY are the first M rows of the
    full-size draw and W is unchanged."""
    L = w.layers[layer_index]
    M = L.M if M is None else M
    K, N = L.K, L.N
    rx = _rng(w.seed, layer_index, X_ID)
    X = rx.standard_normal((M, K))
    ro = _rng(w.seed, layer_index, OUTLIER_ID)
    n_out = outlier_count(w, K)
    cols = np.sort(ro.choice(K, size=n_out, replace=False))
    lo, hi = w.x_outlier_scale
    mult = ro.uniform(lo, hi, size=n_out) if hi > lo else np.full(n_out, lo)
    X[:, cols] *= mult
    rw = _rng(w.seed, layer_index, W_ID)
    W = rw.normal(0.0, 0.02, size=(N, K))
    rd = _rng(w.seed, layer_index, DY_ID)
    if w.dy_dist == "student_t3":
        dY = rd.standard_t(3, size=(M, N)) * 1e-3
    elif w.dy_dist == "laplace":
        dY = rd.laplace(0.0, 1e-3, size=(M, N))
    else:
        raise ValueError(w.dy_dist)
    return dict(X=X.astype(np.float32), W=W.astype(np.float32), dY=dY.astype(np.float32),
                outlier_cols=cols)


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the bit patterns as uint16."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def draw(w: Workload, layer_index: int = 0, M: Optional[int] = None):
    """Inputs in the workload's storage dtype: fp32 arrays, or bf16 bits as uint16."""
    d = draw_fp32(w, layer_index, M)
    if w.dtype == "bf16":
        for key in ("X", "W", "dY"):
            d[key] = to_bf16_bits(d[key])
    return d


def tiny_random(shape, seed: int, dist: str = "normal", scale: float = 1.0) -> np.ndarray:
    """Small seeded fp32 arrays for edge-case tests."""
    r = np.random.default_rng(np.random.SeedSequence([1000 + seed]))
    if dist == "normal":
        v = r.standard_normal(shape) * scale
    elif dist == "int":
        v = r.integers(-8, 9, size=shape).astype(np.float64) * scale
    else:
        raise ValueError(dist)
    return v.astype(np.float32)


def sign_flags(n: int, seed: int) -> np.ndarray:
    """Seeded random sign flags for the randomized Hadamard variant: n bytes, each 0 or 1 with
    probability 1/2 (a Rademacher diagonal D = diag(1 - 2 * flags))."""
    r = np.random.default_rng(np.random.SeedSequence([seed, 1 << 20, n]))
    return r.integers(0, 2, size=n).astype(np.uint8)


def layer_list(w: Workload) -> List[Layer]:
    return list(w.layers)
