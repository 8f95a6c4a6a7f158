"""Shared test plumbing: moving seeded inputs to the device and comparing results."""
import numpy as np


def to_device(x: np.ndarray):
    """fp32 numpy -> float32 CUDA tensor; bf16 bit patterns (uint16) -> bfloat16 CUDA tensor."""
    import torch
    if x.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(x)).cuda()
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    raise TypeError(x.dtype)


def bf16_bits(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def sample_rows(n: int, tile: int = 128, extra: int = 16, seed: int = 0) -> np.ndarray:
    """Rows at tile boundaries, the ragged tail, and a seeded random handful."""
    r = np.random.default_rng(seed)
    fixed = [0, 1, tile - 1, tile, tile + 1, n // 2, n - tile - 1, n - tile, n - 2, n - 1,
             (n // tile) * tile - 1, (n // tile) * tile]
    rand = r.integers(0, n, size=extra).tolist()
    return np.array(sorted({v for v in fixed + rand if 0 <= v < n}), dtype=np.int64)


def bf16_ulp_diff(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 ulps between two arrays of bf16 bit patterns (same sign assumed or zero)."""
    def key(b):
        b = b.astype(np.int64)
        return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)
    return np.abs(key(a_bits) - key(b_bits))


def rel_fro(got: np.ndarray, want: np.ndarray) -> float:
    got = got.astype(np.float64)
    want = want.astype(np.float64)
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / den) if den > 0 else float(np.linalg.norm(got))
