"""Plain CPU oracle for the Hadamard-rotated, tensor-wise quantized linear layer.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  It shares no code with the CUDA
library and never imports it.

The arithmetic lives in ``hq_oracle.c`` (plain C, fp32 FWHT without FMA contraction, RNE
quantizers, int32 / fp64 GEMMs); this module only marshals numpy arrays into it and composes
the three GEMMs of one linear layer the way the pages describe them:

* "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs", "Approach": right-hand
  Hadamard on X and W in the forward pass, left-hand Hadamard on the output gradient in the
  backward pass (HALO-2), tensor-wise quantization.
* "Training Transformers with 4-bit Integers", section 3.3: a block-diagonal transform of
  H_k blocks applied to both operands of a product cancels in the product; section 3.1:
  the integer product is dequantized by the two scales.

Every rotation runs along the contraction dimension of its GEMM:

    forward   Y  = X  W^T   contraction over K (d_in):  X along K, W along K
    backward  dX = dY W     contraction over N (d_out): dY along N, W along N
    backward  dW = dY^T X   contraction over M (tokens): dY along M, X along M  (left-hand)

A second placement reuses the forward's codes (``linear_bwd_reuse``): dY is rotated along M
only, dX multiplies its codes with the forward's K-rotated weight codes and undoes both
rotations on the GEMM output.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libhq_oracle.so")

INT8, FP8_E4M3 = 0, 1
FP6_E3M2, FP6_E2M3, FP4_E2M1 = 2, 3, 4  # minifloats below FP8 (one code per byte, low bits)
MINIFLOATS = (FP6_E3M2, FP6_E2M3, FP4_E2M1)
F32, BF16 = 0, 1

OK, ERR_ARG, ERR_SHAPE, ERR_NONFINITE = 0, 1, 2, 5

GCC_FLAGS = ["-O3", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile hq_oracle.c into libhq_oracle.so next to it (plain gcc, no CUDA)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        L.hq_oracle_rotate.argtypes = [p, i32, i64, i64, i32, i32, p]
        L.hq_oracle_rotate.restype = i32
        L.hq_oracle_quantize.argtypes = [p, i32, i64, i64, i32, i32, i32, p, p]
        L.hq_oracle_quantize.restype = i32
        L.hq_oracle_rotate_signed.argtypes = [p, i32, i64, i64, i32, i32, p, p]
        L.hq_oracle_rotate_signed.restype = i32
        L.hq_oracle_quantize_signed.argtypes = [p, i32, i64, i64, i32, i32, p, i32, p, p]
        L.hq_oracle_quantize_signed.restype = i32
        L.hq_oracle_quantize_rotated.argtypes = [p, i64, i32, p, p]
        L.hq_oracle_quantize_rotated.restype = i32
        L.hq_oracle_quantize_rotated_given.argtypes = [p, i64, i32, ctypes.c_float, p, p]
        L.hq_oracle_quantize_rotated_given.restype = i32
        L.hq_oracle_absmax.argtypes = [p, i64]
        L.hq_oracle_absmax.restype = ctypes.c_float
        L.hq_oracle_fwht_block.argtypes = [p, i32]
        L.hq_oracle_fwht_block.restype = None
        L.hq_oracle_norm_const.argtypes = [i32]
        L.hq_oracle_norm_const.restype = ctypes.c_float
        L.hq_oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.hq_oracle_e4m3_decode.restype = ctypes.c_double
        L.hq_oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.hq_oracle_e4m3_encode.restype = ctypes.c_uint8
        L.hq_oracle_bf16_from_f64.argtypes = [ctypes.c_double]
        L.hq_oracle_bf16_from_f64.restype = ctypes.c_uint16
        L.hq_oracle_bf16_from_f32.argtypes = [ctypes.c_float]
        L.hq_oracle_bf16_from_f32.restype = ctypes.c_uint16
        L.hq_oracle_gemm_i8.argtypes = [p, p, i64, i64, i64, p, i64, p]
        L.hq_oracle_gemm_i8.restype = None
        L.hq_oracle_gemm_f8.argtypes = [p, p, i64, i64, i64, p, i64, p]
        L.hq_oracle_gemm_f8.restype = None
        L.hq_oracle_gemm_fp.argtypes = [i32, p, p, i64, i64, i64, p, i64, p]
        L.hq_oracle_gemm_fp.restype = None
        L.hq_oracle_minifloat_max.argtypes = [i32]
        L.hq_oracle_minifloat_max.restype = ctypes.c_double
        L.hq_oracle_minifloat_decode.argtypes = [i32, ctypes.c_uint8]
        L.hq_oracle_minifloat_decode.restype = ctypes.c_double
        L.hq_oracle_minifloat_encode.argtypes = [i32, ctypes.c_float]
        L.hq_oracle_minifloat_encode.restype = ctypes.c_uint8
        L.hq_oracle_epilogue.argtypes = [p, i32, i64, ctypes.c_float, ctypes.c_float, p, p]
        L.hq_oracle_epilogue.restype = None
        L.hq_oracle_dequant_f32.argtypes = [p, i32, i64, ctypes.c_float, ctypes.c_float, p]
        L.hq_oracle_dequant_f32.restype = None
        L.hq_oracle_f32_to_bf16.argtypes = [p, i64, p]
        L.hq_oracle_f32_to_bf16.restype = None
        L.hq_oracle_threads.argtypes = []
        L.hq_oracle_threads.restype = i32
        _lib = L
    return _lib


class OracleError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: oracle status {status}")
        self.status = status


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _src(x: np.ndarray):
    """Accept fp32 arrays or bf16 bit patterns stored as uint16."""
    x = np.ascontiguousarray(x)
    if x.dtype == np.float32:
        return x, F32
    if x.dtype == np.uint16:
        return x, BF16
    raise TypeError(f"oracle source must be float32 or bf16 bits (uint16), got {x.dtype}")


# ------------------------------------------------------------------------------- primitives

def fwht_block(x: np.ndarray) -> np.ndarray:
    """Unnormalised fp32 Sylvester FWHT of one block (length k), stage h = 1, 2, ..., k/2."""
    buf = np.array(x, dtype=np.float32, copy=True)
    lib().hq_oracle_fwht_block(_ptr(buf), buf.size)
    return buf


def norm_const(k: int) -> np.float32:
    return np.float32(lib().hq_oracle_norm_const(k))


def _neg_flags(neg, length: int):
    if neg is None:
        return None
    f = np.ascontiguousarray(np.asarray(neg).astype(np.uint8) != 0, dtype=np.uint8)
    if f.shape != (length,):
        raise ValueError(f"sign flags must have one entry per position of the rotated dim ({length})")
    return f


def rotate(x: np.ndarray, dim: int, k: int, neg=None) -> np.ndarray:
    """y = blockdiag(H_k / sqrt(k)) applied along `dim` of x[rows][cols], in fp32.

    dim=1: along columns, result [rows][cols].  dim=0: along rows, result [cols][rows]
    (rotated dimension innermost, i.e. K-major for the GEMM that contracts it).
    neg: optional flags, one per position of the rotated dim; a set flag negates that
    position before the Hadamard blocks (randomized Hadamard: H_k D x)."""
    x, dt = _src(x)
    rows, cols = x.shape
    f = _neg_flags(neg, cols if dim == 1 else rows)
    y = np.empty((rows, cols) if dim == 1 else (cols, rows), dtype=np.float32)
    st = lib().hq_oracle_rotate_signed(_ptr(x), dt, rows, cols, dim, k, None if f is None else _ptr(f), _ptr(y))
    if st != OK:
        raise OracleError(st, "rotate")
    return y


def absmax(y: np.ndarray) -> np.float32:
    """max |y| of rotated values (+inf if any is not finite)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    return np.float32(lib().hq_oracle_absmax(_ptr(y), y.size))


def quantize_rotated(y: np.ndarray, fmt: int, absmax_of_whole=None):
    """Tensor-wise quantization of rotated values; absmax_of_whole: the absmax of the tensor
    y is a slice of (sharded quantization), else y's own."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    codes = np.empty(y.shape, dtype=np.uint8)
    scale = np.zeros(1, dtype=np.float32)
    if absmax_of_whole is not None:
        st = lib().hq_oracle_quantize_rotated_given(_ptr(y), y.size, fmt, float(absmax_of_whole), _ptr(codes),
                                                    _ptr(scale))
        if st != OK:
            raise OracleError(st, "quantize")
        return codes, np.float32(scale[0])
    st = lib().hq_oracle_quantize_rotated(_ptr(y), y.size, fmt, _ptr(codes), _ptr(scale))
    if st != OK:
        raise OracleError(st, "quantize")
    return codes, np.float32(scale[0])


def quantize(x: np.ndarray, dim: int, k: int, fmt: int, neg=None):
    """hq_quantize's definition: rotate along `dim`, tensor-wise absmax, RNE codes.
    neg: optional sign flags of the randomized variant (see rotate).

    Returns (codes uint8 with the rotated dim innermost, fp32 scale)."""
    x, dt = _src(x)
    rows, cols = x.shape
    f = _neg_flags(neg, cols if dim == 1 else rows)
    codes = np.empty((rows, cols) if dim == 1 else (cols, rows), dtype=np.uint8)
    scale = np.zeros(1, dtype=np.float32)
    st = lib().hq_oracle_quantize_signed(_ptr(x), dt, rows, cols, dim, k, None if f is None else _ptr(f), fmt,
                                         _ptr(codes), _ptr(scale))
    if st != OK:
        raise OracleError(st, "quantize")
    return codes, np.float32(scale[0])


def minifloat_max(fmt: int) -> float:
    return lib().hq_oracle_minifloat_max(fmt)


def minifloat_decode(fmt: int, code: int) -> float:
    return lib().hq_oracle_minifloat_decode(fmt, code)


def minifloat_encode(fmt: int, x: float) -> int:
    return lib().hq_oracle_minifloat_encode(fmt, float(x))


def minifloat_bits(fmt: int) -> int:
    """Bits of a code of the format (sign included): 6 for FP6, 4 for FP4."""
    return 4 if fmt == FP4_E2M1 else 6


def device_codes(codes: np.ndarray, fmt: int) -> np.ndarray:
    """The library's storage layout of a code tensor (rotated dimension innermost): INT8 and
    FP8 one code per byte as they are; FP6 / FP4 in the tensor cores' operand form, each group
    of 16 consecutive codes along the last axis packed LSB-first (code i at bits b*i .. b*i+b-1,
    b = 6 or 4, of the little-endian chunk) into the leading 12 or 8 bytes of one 16-byte
    chunk, the rest zero.  Plain integer bit packing, no arithmetic of the method."""
    if fmt not in MINIFLOATS:
        return codes
    b = minifloat_bits(fmt)
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, n = c.reshape(-1, c.shape[-1]).shape
    if n % 16:
        raise ValueError("the packed layout needs the rotated dimension to be a multiple of 16")
    g = c.reshape(rows, n // 16, 16).astype(np.uint64)
    lo = np.zeros((rows, n // 16), dtype=np.uint64)  # bits 0..63 of each chunk
    hi = np.zeros((rows, n // 16), dtype=np.uint64)  # bits 64..127
    for i in range(16):
        sh = b * i
        v = g[:, :, i] & np.uint64((1 << b) - 1)
        if sh + b <= 64:
            lo |= v << np.uint64(sh)
        elif sh >= 64:
            hi |= v << np.uint64(sh - 64)
        else:  # straddles bit 64
            lo |= (v << np.uint64(sh)) & np.uint64(0xFFFFFFFFFFFFFFFF)
            hi |= v >> np.uint64(64 - sh)
    out = np.concatenate([lo[..., None], hi[..., None]], axis=-1).view(np.uint8)
    return out.reshape(c.shape)


def e4m3_decode(code: int) -> float:
    return lib().hq_oracle_e4m3_decode(code)


def e4m3_encode(x: float) -> int:
    return lib().hq_oracle_e4m3_encode(x)


E4M3_TABLE = None


def e4m3_table() -> np.ndarray:
    """Decoded value of each of the 256 e4m3 codes (NaN for 0x7F / 0xFF)."""
    global E4M3_TABLE
    if E4M3_TABLE is None:
        E4M3_TABLE = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
    return E4M3_TABLE


def bf16_from_f64(v: float) -> int:
    return lib().hq_oracle_bf16_from_f64(v)


def bf16_from_f32(v: float) -> int:
    return lib().hq_oracle_bf16_from_f32(v)


def gemm(A: np.ndarray, B: np.ndarray, fmt: int, rows=None) -> np.ndarray:
    """C[i][j] = sum_l A[i][l] B[j][l] over codes (both operands contraction-innermost).

    INT8: int32 accumulators.  FP8 / FP6 / FP4: exact fp64 accumulators.  `rows` selects
    rows of A."""
    A = np.ascontiguousarray(A)
    B = np.ascontiguousarray(B)
    M, K = A.shape
    N, K2 = B.shape
    if K != K2:
        raise ValueError("contraction lengths differ")
    if rows is not None:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        R, rp = rows.size, _ptr(rows)
    else:
        R, rp = M, None
    if fmt == INT8:
        C = np.empty((R, N), dtype=np.int32)
        lib().hq_oracle_gemm_i8(_ptr(A.view(np.int8)), _ptr(B.view(np.int8)), M, N, K, rp,
                                R, _ptr(C))
    else:
        C = np.empty((R, N), dtype=np.float64)
        lib().hq_oracle_gemm_fp(int(fmt), _ptr(A.view(np.uint8)), _ptr(B.view(np.uint8)), M, N, K, rp,
                                R, _ptr(C))
    return C


def epilogue(acc: np.ndarray, sa: float, sb: float):
    """Dequantize accumulators to bf16 bit patterns.

    Returns (ref, fast): ref = bf16(fp64(acc)*sa*sb); fast = bf16(fp32(acc)*fp32(sa*sb))."""
    acc = np.ascontiguousarray(acc)
    kind = 0 if acc.dtype == np.int32 else 1
    if kind == 1:
        acc = acc.astype(np.float64, copy=False)
    ref = np.empty(acc.shape, dtype=np.uint16)
    fast = np.empty(acc.shape, dtype=np.uint16)
    lib().hq_oracle_epilogue(_ptr(acc), kind, acc.size, float(sa), float(sb), _ptr(ref),
                             _ptr(fast))
    return ref, fast


def threads() -> int:
    """OpenMP threads the oracle's parallel loops use."""
    return int(lib().hq_oracle_threads())


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ------------------------------------------------------------------------------- the layer

def _gemm_layer(a_src, a_dim, b_src, b_dim, k, fmt, rows=None, neg=None):
    # neg: optional sign flags of the randomized variant over the contraction dimension, the
    # same D for both operands (D^2 = I cancels in the product like H)
    qa, sa = quantize(a_src, a_dim, k, fmt, neg=neg)
    qb, sb = quantize(b_src, b_dim, k, fmt, neg=neg)
    acc = gemm(qa, qb, fmt, rows)
    ref, fast = epilogue(acc, sa, sb)
    return dict(qa=qa, sa=sa, qb=qb, sb=sb, acc=acc, ref=ref, fast=fast)


def linear_fwd(X, W, k, fmt, rows=None, neg=None):
    """Y[M][N] = (X H)(W H)^T, both operands rotated along K (HALO right-hand rotation).
    neg: optional sign flags over K (randomized variant, (X D H)(W D H)^T)."""
    return _gemm_layer(X, 1, W, 1, k, fmt, rows, neg)


def linear_bwd_dx(dY, W, k, fmt, rows=None, neg=None):
    """dX[M][K] = dY W: dY rotated along N (its columns), W rotated along N (its rows).
    neg: optional sign flags over N."""
    return _gemm_layer(dY, 1, W, 0, k, fmt, rows, neg)


def linear_bwd_dw(dY, X, k, fmt, rows=None, neg=None):
    """dW[N][K] = dY^T X: both rotated along the token dimension M (HALO-2 left-hand).
    neg: optional sign flags over M."""
    return _gemm_layer(dY, 0, X, 0, k, fmt, rows, neg)


# ------------------------------------------------- rotated-output placement (forward codes reused)
#
# "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs", Approach: the quantized
# rotated tensors of the forward pass are reused, and the backward pass puts a left-hand
# Hadamard on the output gradient; "Training Transformers with 4-bit Integers", section 4: the
# backward GEMMs quantize only the output gradient and reuse the forward's quantized activations
# and weights.  With Wq = Q(W H) kept from the forward (rotated along K, [N][K]) and dY rotated
# along the tokens M once (G = Q(H dY), stored [N][M] as for dW):
#
#     dX = dY W = H (H dY) (W H) H      (H symmetric and orthonormal: H H = I)
#        ~ H [ s_g s_w * G^T Wq ] H     GEMM contraction over N, then both rotations undone on
#                                       the output: along its columns (K), then its rows (M).
#
# Reading: the de-rotation runs on the fp32 dequantized accumulators (the epilogue's
# fp32(acc) * fp32(s_g * s_w)), as two rotations like `rotate` (butterflies bit 0 first, then
# x fp32(1/sqrt(k))), columns first; the result is rounded to bf16 once at the end.


def dequant_f32(acc: np.ndarray, sa: float, sb: float) -> np.ndarray:
    """fp32(acc) * fp32(sa * sb) elementwise, fp32 (the epilogue before its bf16 rounding)."""
    acc = np.ascontiguousarray(acc)
    kind = 0 if acc.dtype == np.int32 else 1
    if kind == 1:
        acc = acc.astype(np.float64, copy=False)
    z = np.empty(acc.shape, dtype=np.float32)
    lib().hq_oracle_dequant_f32(_ptr(acc), kind, acc.size, float(sa), float(sb), _ptr(z))
    return z


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of fp32 values, round to nearest even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().hq_oracle_f32_to_bf16(_ptr(x), x.size, _ptr(out))
    return out


def derotate_output(Z: np.ndarray, k: int) -> np.ndarray:
    """blockdiag(H_k/sqrt k) applied to Z[rows][cols] on both sides, in fp32: along the columns
    (each row's k-blocks) first, then along the rows.  Both dims must be multiples of k."""
    Z1 = rotate(np.ascontiguousarray(Z, dtype=np.float32), 1, k)  # [rows][cols]
    return np.ascontiguousarray(rotate(Z1, 0, k).T)                # rotate gives [cols][rows]


def linear_bwd_dx_reuse(g_codes, s_g, wq_codes, s_w, k, fmt, rows=None):
    """dX[M][K] from dY's token-rotated codes g_codes[N][M] (scale s_g) and the forward's
    weight codes wq_codes[N][K] (rotated along K, scale s_w):
    bf16( H [fp32(G^T Wq) scaled] H ).

    rows: optional first row of each k-row block to evaluate (sampling whole blocks, since the
    rows of a block mix); returns the rows of those blocks in order.

    Returns dict(acc, z, out): accumulators, fp32 de-rotated values, bf16 bits."""
    A = np.ascontiguousarray(np.asarray(g_codes).T)   # [M][N]
    B = np.ascontiguousarray(np.asarray(wq_codes).T)  # [K][N]
    sel = None
    if rows is not None:
        sel = np.concatenate([np.arange(r, r + k) for r in np.asarray(rows, dtype=np.int64)])
    acc = gemm(A, B, fmt, sel)
    z = derotate_output(dequant_f32(acc, s_g, s_w), k)
    return dict(acc=acc, z=z, out=f32_to_bf16(z))


def linear_bwd_reuse(dY, xqt_codes, s_x, wq_codes, s_w, k, fmt):
    """Backward of the reuse placement: dY is quantized once, rotated along M ([N][M]); dW uses
    it with the saved token-rotated X codes (as linear_bwd_dw), dX with the forward's weight
    codes (linear_bwd_dx_reuse).  Returns dict(g, s_g, dw, dx) with bf16 bits."""
    g, s_g = quantize(dY, 0, k, fmt)
    dw_acc = gemm(g, np.asarray(xqt_codes), fmt)
    _, dw = epilogue(dw_acc, s_g, s_x)
    dx = linear_bwd_dx_reuse(g, s_g, wq_codes, s_w, k, fmt)
    return dict(g=g, s_g=s_g, dw=dw, dx=dx["out"], dx_z=dx["z"])


# ------------------------------------------------- next layer's rotation in the GEMM's epilogue
#
# "Training Transformers with 4-bit Integers", section 3.3 (the Hadamard blocks are applied to
# an operand before it is quantized): when a GEMM's output is the next GEMM's operand along its
# columns, the producing GEMM can apply that rotation to its fp32 dequantized output, and the
# next operand is then only quantized (quantize_rotated).  Reading: the rotation acts on the
# fp32 values fp32(acc) * fp32(s_a * s_b), as `rotate` does (butterflies, then x c_k).


def gemm_rotout(A, B, sa, sb, fmt: int, k: int, rows=None) -> np.ndarray:
    """fp32 [M][N]: blockdiag(H_k/sqrt k) along the columns of the dequantized A B^T."""
    return rotate(dequant_f32(gemm(A, B, fmt, rows), sa, sb), 1, k)
