"""Device-side failure path, exercised without faulting the GPU.

Every mbarrier wait inside the GEMM is bounded (about one second).  The test hook
hq_selftest_gemm_timeout leaves one pipeline stage un-armed so that such a wait expires: the
kernel must record HQ_ERR_TIMEOUT in the status word, stop every role, drain its copies and
MMAs, free tensor memory and return, leaving the CUDA context usable.
"""
import ctypes
import time

import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import build

pytestmark = pytest.mark.gpu


def _codes(shape, seed):
    r = np.random.default_rng(seed)
    return r.integers(-127, 128, size=shape).astype(np.int8).view(np.uint8)


def test_gemm_wait_timeout_reported_and_context_survives(oracle_lib):
    build.build()
    L = hq.lib()
    M, N, K = 200, 272, 640
    A, B = _codes((M, K), 1), _codes((N, K), 2)
    At, Bt = torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()
    out = torch.zeros(M, N, dtype=torch.int32, device="cuda")
    sh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert hq.hq_get_error() == 0
    t0 = time.time()
    assert L.hq_selftest_gemm_timeout(At.data_ptr(), Bt.data_ptr(), out.data_ptr(), M, N, K, sh) == 0
    assert L.hq_get_error(sh) == 6  # HQ_ERR_TIMEOUT
    assert time.time() - t0 < 60
    assert L.hq_get_error(sh) == 0  # cleared
    # the context still works: a normal GEMM matches the oracle exactly
    acc = hq.hq_gemm(At, None, Bt, None, "int8", hq.HQ_OUT_ACC)
    np.testing.assert_array_equal(acc.cpu().numpy(), oracle.gemm(A, B, oracle.INT8))
    assert hq.hq_get_error() == 0


def test_selftest_rejects_large_shapes():
    build.build()
    L = hq.lib()
    a = torch.zeros(16, 16, dtype=torch.uint8, device="cuda")
    sh = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert L.hq_selftest_gemm_timeout(a.data_ptr(), a.data_ptr(), a.data_ptr(), 8192, 16, 16, sh) == 2
