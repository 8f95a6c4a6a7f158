"""GPU check of hq_quantize_noalloc, the quantizer entry point for callers that cannot
allocate device memory (for example plugin code that is handed only its input and output
buffers).  It must give exactly what hq_quantize gives with a caller-provided workspace:
codes and scale bit-exact, on two calls in a row through the C ABI (the second call reuses
the library's fixed scratch array left over from the first).

Kept in a file that pytest collects last so that a run stopping at the first failure has
already run every other test.  Needs no fixture from the other files: it passes alone in a
fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import build

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    build.build()
    return hq.lib()


def _cases():
    # (rows, cols, dim, k, fmt, dtype): both kernels (dim 1 and 0), both formats and dtypes,
    # one large enough for the absmax pass to use its full grid of partial maxima
    return [(4096, 4096, 1, 256, hq.HQ_INT8, torch.bfloat16),
            (4096, 2048, 0, 64, hq.HQ_FP8_E4M3, torch.bfloat16),
            (96, 512, 1, 16, hq.HQ_FP8_E4M3, torch.float32),
            (768, 208, 0, 128, hq.HQ_INT8, torch.float32)]


@pytest.mark.parametrize("case", _cases())
def test_noalloc_matches_workspace_version(L, case):
    rows, cols, dim, k, fmt, dtype = case
    g = torch.Generator(device="cuda").manual_seed(rows + cols + k)
    stream = torch.cuda.current_stream()
    sh = ctypes.c_void_p(stream.cuda_stream)
    dt = hq.HQ_BF16 if dtype == torch.bfloat16 else hq.HQ_F32
    out_shape = (rows, cols) if dim == 1 else (cols, rows)
    for call in range(2):
        x = torch.randn(rows, cols, generator=g, device="cuda")
        x[:, 5] *= 40.0 + call
        x = x.to(dtype)
        want_codes = torch.empty(out_shape, dtype=torch.uint8, device="cuda")
        want_scale = torch.empty(1, dtype=torch.float32, device="cuda")
        ws = torch.empty(hq.hq_quantize_workspace_bytes(), dtype=torch.uint8, device="cuda")
        st = L.hq_quantize(x.data_ptr(), dt, rows, cols, dim, k, fmt, want_codes.data_ptr(),
                           want_scale.data_ptr(), ws.data_ptr(), ws.numel(), sh)
        assert st == 0
        codes = torch.full(out_shape, 0xAB, dtype=torch.uint8, device="cuda")
        scale = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
        st = L.hq_quantize_noalloc(x.data_ptr(), dt, rows, cols, dim, k, fmt, codes.data_ptr(),
                                   scale.data_ptr(), sh)
        assert st == 0
        assert L.hq_get_error(sh) == 0
        assert torch.equal(codes, want_codes), f"call {call}: codes differ"
        assert np.array_equal(scale.cpu().numpy().view(np.uint32), want_scale.cpu().numpy().view(np.uint32))


def test_noalloc_argument_errors(L):
    x = torch.randn(64, 96, device="cuda")
    codes = torch.empty(64, 96, dtype=torch.uint8, device="cuda")
    scale = torch.empty(1, device="cuda")
    sh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.hq_quantize_noalloc(x.data_ptr(), hq.HQ_F32, 64, 96, 1, 64, hq.HQ_INT8, codes.data_ptr(),
                                 scale.data_ptr(), sh) == 2   # 96 is not a multiple of k
    assert L.hq_quantize_noalloc(x.data_ptr(), hq.HQ_F32, 64, 96, 1, 24, hq.HQ_INT8, codes.data_ptr(),
                                 scale.data_ptr(), sh) == 1   # k not supported
