"""Python binding of libhq.so: Hadamard-rotated, tensor-wise quantized linear layer (INT8, FP8
e4m3, FP6 e3m2 / e2m3 and FP4 e2m1 codes) for B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the library's CUDA
kernels; PyTorch provides device memory and streams.  The functions carry the names of the
C entry points declared in include/hq.h.  There is no CPU fallback: CPU tensors, a missing
library or a non-sm_100 device raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")

HQ_OK = 0
HQ_INT8, HQ_FP8_E4M3 = 0, 1
HQ_FP6_E3M2, HQ_FP6_E2M3, HQ_FP4_E2M1 = 2, 3, 4
HQ_F32, HQ_BF16 = 0, 1
HQ_OUT_BF16, HQ_OUT_ACC = 0, 1
HQ_MAX_K_INT8 = 133143

STATUS_NAMES = {0: "HQ_OK", 1: "HQ_ERR_ARG", 2: "HQ_ERR_SHAPE", 3: "HQ_ERR_DTYPE",
                4: "HQ_ERR_ALIGN", 5: "HQ_ERR_NONFINITE", 6: "HQ_ERR_TIMEOUT", 7: "HQ_ERR_CUDA",
                8: "HQ_ERR_WORKSPACE", 9: "HQ_ERR_UNSUPPORTED"}

EXPORTS = ("hq_quantize_workspace_bytes", "hq_quantize", "hq_quantize_noalloc",
           "hq_quantize_dual_workspace_bytes", "hq_quantize_dual", "hq_gemm",
           "hq_linear_workspace_bytes", "hq_linear_fwd", "hq_linear_bwd_dx", "hq_linear_bwd_dw",
           "hq_linear_fwd_bwd_workspace_bytes", "hq_linear_fwd_bwd",
           "hq_linear_fwd_save_workspace_bytes", "hq_linear_fwd_save",
           "hq_linear_bwd_workspace_bytes", "hq_linear_bwd", "hq_selftest_gemm_timeout",
           "hq_quantize_rht", "hq_quantize_dual_rht", "hq_linear_fwd_bwd_rht",
           "hq_quantize_absmax", "hq_quantize_codes",
           "hq_linear_fwd_keep_workspace_bytes", "hq_linear_fwd_keep",
           "hq_linear_bwd_dx_reuse_workspace_bytes", "hq_linear_bwd_dx_reuse",
           "hq_linear_bwd_reuse_workspace_bytes", "hq_linear_bwd_reuse",
           "hq_gemm_rotout", "hq_quantize_prerotated_workspace_bytes", "hq_quantize_prerotated",
           "hq_gemm_workspace_bytes", "hq_gemm_ws",
           "hq_workspace_bytes", "hq_mma_peak", "hq_get_error",
           "hq_last_cuda_error", "hq_status_string", "hq_version")


class HQError(RuntimeError):
    def __init__(self, status: int, where: str, cuda_error: int = 0):
        name = STATUS_NAMES.get(status, str(status))
        msg = f"{where}: {name}"
        if status == 7:
            msg += f" (cudaError {cuda_error})"
        super().__init__(msg)
        self.status = status
        self.cuda_error = cuda_error


_lib = None


def lib() -> ctypes.CDLL:
    """Load libhq.so (built in-tree by ``build.build()``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libhq.so is not built ({LIB_PATH}); run "
                              "`python -m hadamard_rotated_precision_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        p, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
        L.hq_quantize_workspace_bytes.argtypes = []
        L.hq_quantize_workspace_bytes.restype = sz
        L.hq_quantize.argtypes = [p, i32, i64, i64, i32, i32, i32, p, p, p, sz, p]
        L.hq_quantize.restype = i32
        L.hq_quantize_noalloc.argtypes = [p, i32, i64, i64, i32, i32, i32, p, p, p]
        L.hq_quantize_noalloc.restype = i32
        L.hq_quantize_rht.argtypes = [p, i32, i64, i64, i32, i32, i32, p, p, p, p, sz, p]
        L.hq_quantize_rht.restype = i32
        L.hq_quantize_dual_rht.argtypes = [p, i32, i64, i64, i32, i32, p, p, p, p, p, p, p, sz, p]
        L.hq_quantize_dual_rht.restype = i32
        L.hq_linear_fwd_bwd_rht.argtypes = [p, p, p, i32, i64, i64, i64, i32, i32, p, p, p, p, p, p, p, sz, p]
        L.hq_linear_fwd_bwd_rht.restype = i32
        L.hq_quantize_absmax.argtypes = [p, i32, i64, i64, i32, i32, p, p, p, sz, p]
        L.hq_quantize_absmax.restype = i32
        L.hq_quantize_codes.argtypes = [p, i32, i64, i64, i32, i32, i32, p, p, p, p, p]
        L.hq_quantize_codes.restype = i32
        L.hq_quantize_dual_workspace_bytes.argtypes = []
        L.hq_quantize_dual_workspace_bytes.restype = sz
        L.hq_quantize_dual.argtypes = [p, i32, i64, i64, i32, i32, p, p, p, p, p, sz, p]
        L.hq_quantize_dual.restype = i32
        L.hq_linear_fwd_bwd_workspace_bytes.argtypes = [i64, i64, i64]
        L.hq_linear_fwd_bwd_workspace_bytes.restype = sz
        L.hq_linear_fwd_bwd.argtypes = [p, p, p, i32, i64, i64, i64, i32, i32, p, p, p, p, sz, p]
        L.hq_linear_fwd_bwd.restype = i32
        for name in ("hq_linear_fwd_save_workspace_bytes", "hq_linear_bwd_workspace_bytes"):
            getattr(L, name).argtypes = [i64, i64, i64]
            getattr(L, name).restype = sz
        L.hq_linear_fwd_save.argtypes = [p, p, i32, i64, i64, i64, i32, i32, p, p, p, p, sz, p]
        L.hq_linear_fwd_save.restype = i32
        L.hq_linear_bwd.argtypes = [p, p, p, p, i32, i64, i64, i64, i32, i32, p, p, p, sz, p]
        L.hq_linear_bwd.restype = i32
        for name in ("hq_linear_fwd_keep_workspace_bytes", "hq_linear_bwd_dx_reuse_workspace_bytes",
                     "hq_linear_bwd_reuse_workspace_bytes"):
            getattr(L, name).argtypes = [i64, i64, i64]
            getattr(L, name).restype = sz
        L.hq_linear_fwd_keep.argtypes = [p, p, i32, i64, i64, i64, i32, i32, p, p, p, p, p, p, sz, p]
        L.hq_linear_fwd_keep.restype = i32
        L.hq_linear_bwd_dx_reuse.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, p, sz, p]
        L.hq_linear_bwd_dx_reuse.restype = i32
        L.hq_linear_bwd_reuse.argtypes = [p, i32, p, p, p, p, i64, i64, i64, i32, i32, p, p, p, sz, p]
        L.hq_linear_bwd_reuse.restype = i32
        L.hq_gemm_workspace_bytes.argtypes = [i64, i64, i64]
        L.hq_gemm_workspace_bytes.restype = sz
        L.hq_gemm_ws.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, p, sz, p]
        L.hq_gemm_ws.restype = i32
        L.hq_gemm_rotout.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, p]
        L.hq_gemm_rotout.restype = i32
        L.hq_quantize_prerotated_workspace_bytes.argtypes = []
        L.hq_quantize_prerotated_workspace_bytes.restype = sz
        L.hq_quantize_prerotated.argtypes = [p, i64, i64, i32, p, p, p, sz, p]
        L.hq_quantize_prerotated.restype = i32
        L.hq_gemm.argtypes = [p, p, p, p, i64, i64, i64, i32, i32, p, p]
        L.hq_gemm.restype = i32
        L.hq_linear_workspace_bytes.argtypes = [i64, i64, i64]
        L.hq_linear_workspace_bytes.restype = sz
        for name in ("hq_linear_fwd", "hq_linear_bwd_dx", "hq_linear_bwd_dw"):
            f = getattr(L, name)
            f.argtypes = [p, p, i32, i64, i64, i64, i32, i32, p, p, sz, p]
            f.restype = i32
        L.hq_selftest_gemm_timeout.argtypes = [p, p, p, i64, i64, i64, p]
        L.hq_selftest_gemm_timeout.restype = i32
        L.hq_workspace_bytes.argtypes = [i64, i64, i64, i32]
        L.hq_workspace_bytes.restype = sz
        L.hq_mma_peak.argtypes = [i32, i64, p, p]
        L.hq_mma_peak.restype = i32
        L.hq_get_error.argtypes = [p]
        L.hq_get_error.restype = i32
        L.hq_last_cuda_error.argtypes = []
        L.hq_last_cuda_error.restype = i32
        L.hq_status_string.argtypes = [i32]
        L.hq_status_string.restype = ctypes.c_char_p
        L.hq_version.argtypes = []
        L.hq_version.restype = i32
        _lib = L
    return _lib


def _check(status: int, where: str):
    if status != HQ_OK:
        raise HQError(status, where, lib().hq_last_cuda_error() if status == 7 else 0)


def _torch():
    import torch
    return torch


def _stream_handle(stream) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _dev_tensor(t, name: str):
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _src_dtype(t, name: str) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return HQ_F32
    if t.dtype == torch.bfloat16:
        return HQ_BF16
    raise TypeError(f"{name} must be float32 or bfloat16, got {t.dtype}")


def _fmt(fmt) -> int:
    names = {"int8": HQ_INT8, "fp8": HQ_FP8_E4M3, "fp8_e4m3": HQ_FP8_E4M3, "fp6_e3m2": HQ_FP6_E3M2,
             "fp6_e2m3": HQ_FP6_E2M3, "fp4_e2m1": HQ_FP4_E2M1}
    if isinstance(fmt, str) and fmt in names:
        return names[fmt]
    if fmt in (HQ_INT8, HQ_FP8_E4M3, HQ_FP6_E3M2, HQ_FP6_E2M3, HQ_FP4_E2M1):
        return int(fmt)
    raise ValueError(f"unknown format {fmt!r}")


def hq_quantize_workspace_bytes() -> int:
    return int(lib().hq_quantize_workspace_bytes())


def hq_linear_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_workspace_bytes(M, K, N))


def _workspace(nbytes: int, device, workspace=None):
    torch = _torch()
    if workspace is None:
        return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)
    _dev_tensor(workspace, "workspace")
    if workspace.numel() * workspace.element_size() < nbytes:
        raise ValueError("workspace too small")
    return workspace


def hq_quantize(src, dim: int, k: int, fmt, codes=None, scale=None, workspace=None,
                stream=None) -> Tuple["torch.Tensor", "torch.Tensor"]:
    """Rotate `src` [rows][cols] along `dim` with blockdiag(H_k)/sqrt(k), quantize it
    tensor-wise.  Returns (codes uint8 with the rotated dim innermost, scale fp32[1])."""
    torch = _torch()
    _dev_tensor(src, "src")
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    dt = _src_dtype(src, "src")
    rows, cols = src.shape
    shape = (rows, cols) if dim == 1 else (cols, rows)
    if codes is None:
        codes = torch.empty(shape, dtype=torch.uint8, device=src.device)
    if scale is None:
        scale = torch.empty(1, dtype=torch.float32, device=src.device)
    _dev_tensor(codes, "codes")
    _dev_tensor(scale, "scale")
    ws = _workspace(hq_quantize_workspace_bytes(), src.device, workspace)
    st = lib().hq_quantize(src.data_ptr(), dt, rows, cols, dim, k, _fmt(fmt), codes.data_ptr(),
                           scale.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                           _stream_handle(stream))
    _check(st, "hq_quantize")
    return codes, scale


def _sign_flags(neg, length: int, name: str):
    """Device uint8 flags (bit 0 = negate), one per position of a rotated dimension; None = plain."""
    if neg is None:
        return None
    _dev_tensor(neg, name)
    torch = _torch()
    if neg.dtype != torch.uint8 or neg.dim() != 1 or neg.numel() != length or not neg.is_contiguous():
        raise ValueError(f"{name} must be a contiguous uint8 CUDA tensor of {length} flags")
    return neg


def _ptr_or_none(t):
    return None if t is None else t.data_ptr()


def hq_quantize_rht(src, dim: int, k: int, fmt, neg, codes=None, scale=None, workspace=None, stream=None):
    """hq_quantize with the randomized Hadamard's sign flags `neg` (uint8 CUDA tensor, one per
    position of the rotated dimension, bit 0 = negate before the blocks; None = plain)."""
    torch = _torch()
    _dev_tensor(src, "src")
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    dt = _src_dtype(src, "src")
    rows, cols = src.shape
    neg = _sign_flags(neg, cols if dim == 1 else rows, "neg")
    shape = (rows, cols) if dim == 1 else (cols, rows)
    codes = torch.empty(shape, dtype=torch.uint8, device=src.device) if codes is None else codes
    scale = torch.empty(1, dtype=torch.float32, device=src.device) if scale is None else scale
    _dev_tensor(codes, "codes")
    _dev_tensor(scale, "scale")
    ws = _workspace(hq_quantize_workspace_bytes(), src.device, workspace)
    st = lib().hq_quantize_rht(src.data_ptr(), dt, rows, cols, dim, k, _fmt(fmt), _ptr_or_none(neg),
                               codes.data_ptr(), scale.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                               _stream_handle(stream))
    _check(st, "hq_quantize_rht")
    return codes, scale


def hq_quantize_dual_rht(src, k: int, fmt, neg_c, neg_r, codes_c=None, scale_c=None, codes_r=None,
                         scale_r=None, workspace=None, stream=None):
    """hq_quantize_dual with sign flags neg_c over the columns and neg_r over the rows."""
    torch = _torch()
    _dev_tensor(src, "src")
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    dt = _src_dtype(src, "src")
    rows, cols = src.shape
    neg_c = _sign_flags(neg_c, cols, "neg_c")
    neg_r = _sign_flags(neg_r, rows, "neg_r")
    dev = src.device
    codes_c = torch.empty((rows, cols), dtype=torch.uint8, device=dev) if codes_c is None else codes_c
    codes_r = torch.empty((cols, rows), dtype=torch.uint8, device=dev) if codes_r is None else codes_r
    scale_c = torch.empty(1, dtype=torch.float32, device=dev) if scale_c is None else scale_c
    scale_r = torch.empty(1, dtype=torch.float32, device=dev) if scale_r is None else scale_r
    for t, n in ((codes_c, "codes_c"), (codes_r, "codes_r"), (scale_c, "scale_c"), (scale_r, "scale_r")):
        _dev_tensor(t, n)
    ws = _workspace(hq_quantize_dual_workspace_bytes(), dev, workspace)
    st = lib().hq_quantize_dual_rht(src.data_ptr(), dt, rows, cols, k, _fmt(fmt), _ptr_or_none(neg_c),
                                    _ptr_or_none(neg_r), codes_c.data_ptr(), scale_c.data_ptr(), codes_r.data_ptr(),
                                    scale_r.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                                    _stream_handle(stream))
    _check(st, "hq_quantize_dual_rht")
    return codes_c, scale_c, codes_r, scale_r


def hq_quantize_absmax(src, dim: int, k: int, neg=None, absmax=None, workspace=None, stream=None):
    """Pass 1 alone: max |y| of the rotation of `src` along `dim`, as a float32[1] CUDA tensor."""
    torch = _torch()
    _dev_tensor(src, "src")
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    dt = _src_dtype(src, "src")
    rows, cols = src.shape
    neg = _sign_flags(neg, cols if dim == 1 else rows, "neg")
    absmax = torch.empty(1, dtype=torch.float32, device=src.device) if absmax is None else absmax
    _dev_tensor(absmax, "absmax")
    ws = _workspace(hq_quantize_workspace_bytes(), src.device, workspace)
    st = lib().hq_quantize_absmax(src.data_ptr(), dt, rows, cols, dim, k, _ptr_or_none(neg), absmax.data_ptr(),
                                  ws.data_ptr(), ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_quantize_absmax")
    return absmax


def hq_quantize_codes(src, dim: int, k: int, fmt, absmax, neg=None, codes=None, scale=None, stream=None):
    """Pass 2 from a given absmax (float32[1] CUDA tensor): codes and scale of `src` as the
    slice of a tensor whose absmax that is."""
    torch = _torch()
    _dev_tensor(src, "src")
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    _dev_tensor(absmax, "absmax")
    dt = _src_dtype(src, "src")
    rows, cols = src.shape
    neg = _sign_flags(neg, cols if dim == 1 else rows, "neg")
    shape = (rows, cols) if dim == 1 else (cols, rows)
    codes = torch.empty(shape, dtype=torch.uint8, device=src.device) if codes is None else codes
    scale = torch.empty(1, dtype=torch.float32, device=src.device) if scale is None else scale
    _dev_tensor(codes, "codes")
    _dev_tensor(scale, "scale")
    st = lib().hq_quantize_codes(src.data_ptr(), dt, rows, cols, dim, k, _fmt(fmt), _ptr_or_none(neg),
                                 absmax.data_ptr(), codes.data_ptr(), scale.data_ptr(), _stream_handle(stream))
    _check(st, "hq_quantize_codes")
    return codes, scale


def sharded_quantize_flow(absmax_pass, reduce_max, codes_pass):
    """The sharded quantization of quantized FSDP communication: this rank's absmax, the maximum
    over ranks, then this rank's codes scaled by the whole tensor's absmax.  The passes and the
    collective are arguments so the same flow runs on the library's kernels with NCCL and, in the
    CPU tests, on other implementations with gloo."""
    a = absmax_pass()
    a = reduce_max(a)
    return codes_pass(a)


def hq_quantize_sharded(shard, dim: int, k: int, fmt, group=None, neg=None, stream=None):
    """This rank's slice `shard` of a tensor distributed over the ranks of `group`, quantized
    with the whole tensor's tensor-wise scale (slices along the non-rotated dimension, or along
    the rotated one in multiples of k).  Returns (codes of the slice, scale)."""
    import torch.distributed as dist

    def reduce_max(a):
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(a, op=dist.ReduceOp.MAX, group=group)
        return a

    return sharded_quantize_flow(lambda: hq_quantize_absmax(shard, dim, k, neg=neg, stream=stream), reduce_max,
                                 lambda a: hq_quantize_codes(shard, dim, k, fmt, a, neg=neg, stream=stream))


def hq_fsdp_all_gather(w_shard, k: int, fmt, group=None, neg=None):
    """Quantized weight all-gather: this rank holds rows [r*n, (r+1)*n) of W [N][K]; every rank
    gets the codes of the whole W rotated along K (1 byte per element on the wire instead of 2)
    and its scale, equal to hq_quantize(W, dim=1) bit for bit."""
    import torch.distributed as dist
    torch = _torch()
    codes, scale = hq_quantize_sharded(w_shard, 1, k, fmt, group=group, neg=neg)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    if world == 1:
        return codes, scale
    full = torch.empty((world * codes.shape[0], codes.shape[1]), dtype=torch.uint8, device=codes.device)
    dist.all_gather_into_tensor(full, codes, group=group)
    return full, scale


def fsdp_prefetch_schedule(n_layers: int, start_gather, wait_gather, compute):
    """Order of a forward pass over a stack of linear layers whose weights are sharded over the
    ranks and all-gathered as quantized codes (the quantized FSDP communication of HALO): the
    gather of layer i + 1 is started before layer i computes, so the communication of the next
    weight overlaps the current layer's GEMMs, and layer i computes only once its own gather
    has completed.  start_gather(i) issues layer i's gather without waiting for it;
    wait_gather(i) blocks (or orders the compute stream) until it is done and returns the
    gathered weight; compute(i, gathered) runs the layer.  Returns the computes' results in
    layer order.  The callbacks are arguments so the same order runs on CUDA streams with NCCL
    (hq_fsdp_forward) and, in the CPU tests, with gloo."""
    out = []
    if n_layers <= 0:
        return out
    start_gather(0)
    for i in range(n_layers):
        g = wait_gather(i)
        if i + 1 < n_layers:
            start_gather(i + 1)
        out.append(compute(i, g))
    return out


def hq_fsdp_forward(w_shards, xs, k: int, fmt, group=None, comm_stream=None):
    """Forward GEMMs Y_i = Q(X_i H) Q(W_i H)^T of a stack of layers with quantized FSDP weights.
    Rank r holds rows [r n_i, (r + 1) n_i) of every W_i [N_i][K_i] (w_shards[i]); xs[i] is
    the layer's full input X_i [M][K_i] on this rank.  Each layer's weight is quantized shard by
    shard with the whole tensor's scale and its 1-byte codes all-gathered (hq_fsdp_all_gather)
    on `comm_stream` (a new CUDA stream by default), the gather of layer i + 1 overlapping the
    quantization of X_i and the GEMM of layer i on the current stream (fsdp_prefetch_schedule).
    Returns the bf16 outputs; each equals hq_linear_fwd(X_i, W_i) bit for bit."""
    torch = _torch()
    compute = torch.cuda.current_stream()
    comm = comm_stream if comm_stream is not None else torch.cuda.Stream()
    pending = {}

    def start(i):
        ready = torch.cuda.Event()
        ready.record(compute)  # the shard as the compute stream left it
        with torch.cuda.stream(comm):
            comm.wait_event(ready)
            codes, scale = hq_fsdp_all_gather(w_shards[i], k, fmt, group=group)
            done = torch.cuda.Event()
            done.record(comm)
        codes.record_stream(compute)
        scale.record_stream(compute)
        pending[i] = (codes, scale, done)

    def wait(i):
        codes, scale, done = pending.pop(i)
        compute.wait_event(done)
        return codes, scale

    def run(i, g):
        wq, sw = g
        xq, sx = hq_quantize(xs[i], 1, k, fmt)
        return hq_gemm(xq, sx, wq, sw, fmt)

    return fsdp_prefetch_schedule(len(w_shards), start, wait, run)


def hq_quantize_dual_workspace_bytes() -> int:
    return int(lib().hq_quantize_dual_workspace_bytes())


def hq_quantize_dual(src, k: int, fmt, codes_c=None, scale_c=None, codes_r=None, scale_r=None,
                     workspace=None, stream=None):
    """Both rotations of `src` [rows][cols] at once.  Returns (codes_c [rows][cols], scale_c,
    codes_r [cols][rows], scale_r): rotated along cols and along rows respectively."""
    torch = _torch()
    _dev_tensor(src, "src")
    if src.dim() != 2:
        raise ValueError("src must be 2-D")
    dt = _src_dtype(src, "src")
    rows, cols = src.shape
    dev = src.device
    codes_c = torch.empty((rows, cols), dtype=torch.uint8, device=dev) if codes_c is None else codes_c
    codes_r = torch.empty((cols, rows), dtype=torch.uint8, device=dev) if codes_r is None else codes_r
    scale_c = torch.empty(1, dtype=torch.float32, device=dev) if scale_c is None else scale_c
    scale_r = torch.empty(1, dtype=torch.float32, device=dev) if scale_r is None else scale_r
    for t, n in ((codes_c, "codes_c"), (codes_r, "codes_r"), (scale_c, "scale_c"), (scale_r, "scale_r")):
        _dev_tensor(t, n)
    ws = _workspace(hq_quantize_dual_workspace_bytes(), dev, workspace)
    st = lib().hq_quantize_dual(src.data_ptr(), dt, rows, cols, k, _fmt(fmt), codes_c.data_ptr(),
                                scale_c.data_ptr(), codes_r.data_ptr(), scale_r.data_ptr(),
                                ws.data_ptr(), ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_quantize_dual")
    return codes_c, scale_c, codes_r, scale_r


def hq_linear_fwd_bwd_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_fwd_bwd_workspace_bytes(M, K, N))


def hq_linear_fwd_bwd(X, W, dY, k: int, fmt, Y=None, dX=None, dW=None, workspace=None, stream=None):
    """The layer step: (Y, dX, dW) = (X W^T, dY W, dY^T X), every operand quantized once in both
    rotations."""
    torch = _torch()
    for t, n in ((X, "X"), (W, "W"), (dY, "dY")):
        _dev_tensor(t, n)
    dt = _src_dtype(X, "X")
    if _src_dtype(W, "W") != dt or _src_dtype(dY, "dY") != dt:
        raise TypeError("X, W and dY must have the same dtype")
    M, K = X.shape
    N = W.shape[0]
    dev = X.device
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if Y is None else Y
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if dX is None else dX
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if dW is None else dW
    for t, n in ((Y, "Y"), (dX, "dX"), (dW, "dW")):
        _dev_tensor(t, n)
    ws = _workspace(hq_linear_fwd_bwd_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_fwd_bwd(X.data_ptr(), W.data_ptr(), dY.data_ptr(), dt, M, K, N, k, _fmt(fmt),
                                 Y.data_ptr(), dX.data_ptr(), dW.data_ptr(), ws.data_ptr(),
                                 ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_linear_fwd_bwd")
    return Y, dX, dW


def hq_linear_fwd_bwd_rht(X, W, dY, k: int, fmt, neg_k, neg_n, neg_m, Y=None, dX=None, dW=None, workspace=None,
                          stream=None):
    """hq_linear_fwd_bwd with the randomized Hadamard's sign flags per contraction dimension:
    neg_k [K] (forward), neg_n [N] (dX), neg_m [M] (dW); None = plain for that dimension."""
    torch = _torch()
    for t, n in ((X, "X"), (W, "W"), (dY, "dY")):
        _dev_tensor(t, n)
    dt = _src_dtype(X, "X")
    if _src_dtype(W, "W") != dt or _src_dtype(dY, "dY") != dt:
        raise TypeError("X, W and dY must have the same dtype")
    M, K = X.shape
    N = W.shape[0]
    neg_k, neg_n, neg_m = _sign_flags(neg_k, K, "neg_k"), _sign_flags(neg_n, N, "neg_n"), _sign_flags(neg_m, M, "neg_m")
    dev = X.device
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if Y is None else Y
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if dX is None else dX
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if dW is None else dW
    for t, n in ((Y, "Y"), (dX, "dX"), (dW, "dW")):
        _dev_tensor(t, n)
    ws = _workspace(hq_linear_fwd_bwd_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_fwd_bwd_rht(X.data_ptr(), W.data_ptr(), dY.data_ptr(), dt, M, K, N, k, _fmt(fmt),
                                     _ptr_or_none(neg_k), _ptr_or_none(neg_n), _ptr_or_none(neg_m), Y.data_ptr(),
                                     dX.data_ptr(), dW.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                                     _stream_handle(stream))
    _check(st, "hq_linear_fwd_bwd_rht")
    return Y, dX, dW


def hq_linear_fwd_save_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_fwd_save_workspace_bytes(M, K, N))


def hq_linear_fwd_save(X, W, k: int, fmt, Y=None, xqt=None, xqt_scale=None, workspace=None, stream=None):
    """Y = X W^T, and X's codes rotated along the tokens (xqt [K][M] uint8 + device scale) kept
    for hq_linear_bwd.  Returns (Y, xqt, xqt_scale)."""
    torch = _torch()
    _dev_tensor(X, "X")
    _dev_tensor(W, "W")
    dt = _src_dtype(X, "X")
    if _src_dtype(W, "W") != dt:
        raise TypeError("X and W must have the same dtype")
    M, K = X.shape
    N = W.shape[0]
    dev = X.device
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if Y is None else Y
    xqt = torch.empty((K, M), dtype=torch.uint8, device=dev) if xqt is None else xqt
    xqt_scale = torch.empty((1,), dtype=torch.float32, device=dev) if xqt_scale is None else xqt_scale
    for t, n in ((Y, "Y"), (xqt, "xqt"), (xqt_scale, "xqt_scale")):
        _dev_tensor(t, n)
    ws = _workspace(hq_linear_fwd_save_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_fwd_save(X.data_ptr(), W.data_ptr(), dt, M, K, N, k, _fmt(fmt), Y.data_ptr(),
                                  xqt.data_ptr(), xqt_scale.data_ptr(), ws.data_ptr(),
                                  ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_linear_fwd_save")
    return Y, xqt, xqt_scale


def hq_linear_bwd_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_bwd_workspace_bytes(M, K, N))


def hq_linear_bwd(dY, W, xqt, xqt_scale, k: int, fmt, dX=None, dW=None, workspace=None, stream=None):
    """(dX, dW) = (dY W, dY^T X) with X given by the codes hq_linear_fwd_save kept."""
    torch = _torch()
    for t, n in ((dY, "dY"), (W, "W"), (xqt, "xqt"), (xqt_scale, "xqt_scale")):
        _dev_tensor(t, n)
    dt = _src_dtype(dY, "dY")
    if _src_dtype(W, "W") != dt:
        raise TypeError("dY and W must have the same dtype")
    M, N = dY.shape
    K = W.shape[1]
    if tuple(xqt.shape) != (K, M):
        raise ValueError(f"xqt must be [K][M] = [{K}][{M}]")
    dev = dY.device
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if dX is None else dX
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if dW is None else dW
    for t, n in ((dX, "dX"), (dW, "dW")):
        _dev_tensor(t, n)
    ws = _workspace(hq_linear_bwd_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_bwd(dY.data_ptr(), W.data_ptr(), xqt.data_ptr(), xqt_scale.data_ptr(), dt, M, K, N, k,
                             _fmt(fmt), dX.data_ptr(), dW.data_ptr(), ws.data_ptr(),
                             ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_linear_bwd")
    return dX, dW


def hq_linear_fwd_keep_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_fwd_keep_workspace_bytes(M, K, N))


def hq_linear_fwd_keep(X, W, k: int, fmt, Y=None, xqt=None, xqt_scale=None, wq=None, wq_scale=None,
                       workspace=None, stream=None):
    """hq_linear_fwd_save that also returns W's K-rotated codes (wq [N][K] uint8 + device scale)
    for hq_linear_bwd_reuse.  Returns (Y, xqt, xqt_scale, wq, wq_scale)."""
    torch = _torch()
    _dev_tensor(X, "X")
    _dev_tensor(W, "W")
    dt = _src_dtype(X, "X")
    if _src_dtype(W, "W") != dt:
        raise TypeError("X and W must have the same dtype")
    M, K = X.shape
    N = W.shape[0]
    dev = X.device
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev) if Y is None else Y
    xqt = torch.empty((K, M), dtype=torch.uint8, device=dev) if xqt is None else xqt
    xqt_scale = torch.empty((1,), dtype=torch.float32, device=dev) if xqt_scale is None else xqt_scale
    wq = torch.empty((N, K), dtype=torch.uint8, device=dev) if wq is None else wq
    wq_scale = torch.empty((1,), dtype=torch.float32, device=dev) if wq_scale is None else wq_scale
    for t, n in ((Y, "Y"), (xqt, "xqt"), (xqt_scale, "xqt_scale"), (wq, "wq"), (wq_scale, "wq_scale")):
        _dev_tensor(t, n)
    ws = _workspace(hq_linear_fwd_keep_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_fwd_keep(X.data_ptr(), W.data_ptr(), dt, M, K, N, k, _fmt(fmt), Y.data_ptr(),
                                  xqt.data_ptr(), xqt_scale.data_ptr(), wq.data_ptr(), wq_scale.data_ptr(),
                                  ws.data_ptr(), ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_linear_fwd_keep")
    return Y, xqt, xqt_scale, wq, wq_scale


def hq_linear_bwd_dx_reuse_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_bwd_dx_reuse_workspace_bytes(M, K, N))


def hq_linear_bwd_dx_reuse(g, g_scale, wq, wq_scale, k: int, fmt, dX=None, workspace=None, stream=None):
    """dX [M][K] bf16 = H [G^T-contraction with Wq, dequantized in fp32] H from dY's token-rotated
    codes g [N][M] and the forward's K-rotated weight codes wq [N][K]."""
    torch = _torch()
    for t, n in ((g, "g"), (g_scale, "g_scale"), (wq, "wq"), (wq_scale, "wq_scale")):
        _dev_tensor(t, n)
    N, M = g.shape
    if wq.shape[0] != N:
        raise ValueError("g and wq must share their first (contraction) dimension")
    K = wq.shape[1]
    dev = g.device
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if dX is None else dX
    _dev_tensor(dX, "dX")
    ws = _workspace(hq_linear_bwd_dx_reuse_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_bwd_dx_reuse(g.data_ptr(), g_scale.data_ptr(), wq.data_ptr(), wq_scale.data_ptr(), M, K, N,
                                      k, _fmt(fmt), dX.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                                      _stream_handle(stream))
    _check(st, "hq_linear_bwd_dx_reuse")
    return dX


def hq_linear_bwd_reuse_workspace_bytes(M: int, K: int, N: int) -> int:
    return int(lib().hq_linear_bwd_reuse_workspace_bytes(M, K, N))


def hq_linear_bwd_reuse(dY, xqt, xqt_scale, wq, wq_scale, k: int, fmt, dX=None, dW=None, workspace=None,
                        stream=None):
    """(dX, dW) of one layer from dY and the codes hq_linear_fwd_keep kept: dY quantized once
    along the tokens, dW from the saved X codes, dX from the weight codes with both rotations
    undone on the output."""
    torch = _torch()
    for t, n in ((dY, "dY"), (xqt, "xqt"), (xqt_scale, "xqt_scale"), (wq, "wq"), (wq_scale, "wq_scale")):
        _dev_tensor(t, n)
    dt = _src_dtype(dY, "dY")
    M, N = dY.shape
    K = wq.shape[1]
    if tuple(xqt.shape) != (K, M) or wq.shape[0] != N:
        raise ValueError(f"xqt must be [K][M] = [{K}][{M}] and wq [N][K] = [{N}][{K}]")
    dev = dY.device
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev) if dX is None else dX
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=dev) if dW is None else dW
    for t, n in ((dX, "dX"), (dW, "dW")):
        _dev_tensor(t, n)
    ws = _workspace(hq_linear_bwd_reuse_workspace_bytes(M, K, N), dev, workspace)
    st = lib().hq_linear_bwd_reuse(dY.data_ptr(), dt, xqt.data_ptr(), xqt_scale.data_ptr(), wq.data_ptr(),
                                   wq_scale.data_ptr(), M, K, N, k, _fmt(fmt), dX.data_ptr(), dW.data_ptr(),
                                   ws.data_ptr(), ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_linear_bwd_reuse")
    return dX, dW


def hq_gemm_rotout(A, scale_a, B, scale_b, k: int, fmt, out=None, stream=None):
    """out [M][N] fp32: the dequantized A B^T rotated along its columns in blocks of k (the next
    layer's rotation applied in the GEMM's epilogue)."""
    torch = _torch()
    for t, n in ((A, "A"), (scale_a, "scale_a"), (B, "B"), (scale_b, "scale_b")):
        _dev_tensor(t, n)
    M, K = A.shape
    N = B.shape[0]
    out = torch.empty((M, N), dtype=torch.float32, device=A.device) if out is None else out
    _dev_tensor(out, "out")
    st = lib().hq_gemm_rotout(A.data_ptr(), scale_a.data_ptr(), B.data_ptr(), scale_b.data_ptr(), M, N, K, k,
                              _fmt(fmt), out.data_ptr(), _stream_handle(stream))
    _check(st, "hq_gemm_rotout")
    return out


def hq_quantize_prerotated_workspace_bytes() -> int:
    return int(lib().hq_quantize_prerotated_workspace_bytes())


def hq_quantize_prerotated(y, fmt, codes=None, scale=None, workspace=None, stream=None):
    """Tensor-wise codes of already-rotated fp32 values y [rows][cols] (no transform).
    Returns (codes uint8 [rows][cols], scale)."""
    torch = _torch()
    _dev_tensor(y, "y")
    if y.dtype != torch.float32:
        raise TypeError("y must be float32")
    rows, cols = y.shape
    codes = torch.empty((rows, cols), dtype=torch.uint8, device=y.device) if codes is None else codes
    scale = torch.empty((1,), dtype=torch.float32, device=y.device) if scale is None else scale
    ws = _workspace(hq_quantize_prerotated_workspace_bytes(), y.device, workspace)
    st = lib().hq_quantize_prerotated(y.data_ptr(), rows, cols, _fmt(fmt), codes.data_ptr(), scale.data_ptr(),
                                      ws.data_ptr(), ws.numel() * ws.element_size(), _stream_handle(stream))
    _check(st, "hq_quantize_prerotated")
    return codes, scale


def hq_gemm_workspace_bytes(M: int, N: int, K: int) -> int:
    return int(lib().hq_gemm_workspace_bytes(M, N, K))


def hq_gemm(A, scale_a, B, scale_b, fmt, out_kind: int = HQ_OUT_BF16, out=None, stream=None, workspace=None):
    """out[M][N] = sum_l A[i][l] B[j][l] on codes (both contraction-innermost), dequantized
    to bf16 by scale_a*scale_b (HQ_OUT_BF16) or raw int32/fp32 accumulators (HQ_OUT_ACC).
    workspace: optional device scratch (hq_gemm_ws) that lets the last wave's tiles split."""
    torch = _torch()
    _dev_tensor(A, "A")
    _dev_tensor(B, "B")
    M, K = A.shape
    N, K2 = B.shape
    if K != K2:
        raise ValueError("contraction lengths differ")
    f = _fmt(fmt)
    if out is None:
        if out_kind == HQ_OUT_BF16:
            dtype = torch.bfloat16
        else:
            dtype = torch.int32 if f == HQ_INT8 else torch.float32
        out = torch.empty((M, N), dtype=dtype, device=A.device)
    _dev_tensor(out, "out")
    sa = scale_a.data_ptr() if scale_a is not None else None
    sb = scale_b.data_ptr() if scale_b is not None else None
    if workspace is None:
        st = lib().hq_gemm(A.data_ptr(), sa, B.data_ptr(), sb, M, N, K, f, out_kind, out.data_ptr(),
                           _stream_handle(stream))
    else:
        _dev_tensor(workspace, "workspace")
        st = lib().hq_gemm_ws(A.data_ptr(), sa, B.data_ptr(), sb, M, N, K, f, out_kind, out.data_ptr(),
                              workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                              _stream_handle(stream))
    _check(st, "hq_gemm")
    return out


def _linear(name, a, b, M, K, N, out_shape, k, fmt, out, workspace, stream):
    torch = _torch()
    _dev_tensor(a, "a")
    _dev_tensor(b, "b")
    dt = _src_dtype(a, "a")
    if _src_dtype(b, "b") != dt:
        raise TypeError("both operands must have the same dtype")
    if out is None:
        out = torch.empty(out_shape, dtype=torch.bfloat16, device=a.device)
    _dev_tensor(out, "out")
    ws = _workspace(hq_linear_workspace_bytes(M, K, N), a.device, workspace)
    st = getattr(lib(), name)(a.data_ptr(), b.data_ptr(), dt, M, K, N, k, _fmt(fmt),
                              out.data_ptr(), ws.data_ptr(), ws.numel() * ws.element_size(),
                              _stream_handle(stream))
    _check(st, name)
    return out


def hq_linear_fwd(X, W, k: int, fmt, out=None, workspace=None, stream=None):
    """Y[M][N] = (X H)(W H)^T, X [M][K], W [N][K]: HALO right-hand rotation along K."""
    M, K = X.shape
    N = W.shape[0]
    return _linear("hq_linear_fwd", X, W, M, K, N, (M, N), k, fmt, out, workspace, stream)


def hq_linear_bwd_dx(dY, W, k: int, fmt, out=None, workspace=None, stream=None):
    """dX[M][K] = dY W with dY and W rotated along N (d_out)."""
    M, N = dY.shape
    K = W.shape[1]
    return _linear("hq_linear_bwd_dx", dY, W, M, K, N, (M, K), k, fmt, out, workspace, stream)


def hq_linear_bwd_dw(dY, X, k: int, fmt, out=None, workspace=None, stream=None):
    """dW[N][K] = dY^T X with dY and X rotated along the tokens M (HALO-2 left-hand)."""
    M, N = dY.shape
    K = X.shape[1]
    return _linear("hq_linear_bwd_dw", dY, X, M, K, N, (N, K), k, fmt, out, workspace, stream)


def hq_workspace_bytes(M: int, K: int, N: int, fmt) -> int:
    """One workspace size for every layer-level call of the shape (any code format)."""
    return int(lib().hq_workspace_bytes(M, K, N, _fmt(fmt)))


def hq_mma_peak(fmt, n_blocks: int, stream=None) -> int:
    """Launch the dense tensor-core throughput probe (n_blocks x 4 CTA-pair MMAs of 256 x 256 x 32
    per pair, operands in shared memory) on `stream`; returns the number of CTA pairs.  The
    caller times it: operations = pairs * n_blocks * 4 * 2 * 256 * 256 * 32."""
    pairs = ctypes.c_int(0)
    _check(lib().hq_mma_peak(_fmt(fmt), int(n_blocks), ctypes.byref(pairs), _stream_handle(stream)), "hq_mma_peak")
    return int(pairs.value)


def hq_get_error(stream=None) -> int:
    """Synchronise the stream and return/clear the device status word (0 = HQ_OK)."""
    return int(lib().hq_get_error(_stream_handle(stream)))


def hq_status_string(status: int) -> str:
    return lib().hq_status_string(status).decode()


def hq_version() -> int:
    return int(lib().hq_version())
