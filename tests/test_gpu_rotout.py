"""GPU parity of the next layer's rotation in the GEMM's epilogue: hq_gemm_rotout (the
dequantized product rotated along its columns by the epilogue) and hq_quantize_prerotated (the
tensor-wise codes of values that are already rotated), against the oracle.  INT8 bit-exact;
FP8 against the oracle's exact product with the relative Frobenius bound 2e-3."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import synthetic

pytestmark = pytest.mark.gpu

FP8_TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_lib):
    from hadamard_rotated_precision_b200 import build
    build.build()
    assert torch.cuda.is_available()
    hq.lib()
    yield
    assert hq.hq_get_error() == 0


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _scale(s):
    return torch.tensor([float(s)], dtype=torch.float32, device="cuda")


def _fmt_name(fmt):
    return "int8" if fmt == oracle.INT8 else "fp8"


# (M, N, K, k): ragged M, M below one CTA's rows, N tails against 256-wide tiles (N % k == 0),
# contraction tails against 128-deep k-blocks
SHAPES = [(256, 256, 256, 16), (300, 384, 208, 128), (64, 256, 96, 256), (1024, 768, 1024, 64),
          (512, 4096, 4096, 256), (200, 48, 64, 16)]


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3), ids=_fmt_name)
@pytest.mark.parametrize("M,N,K,k", SHAPES)
def test_gemm_rotout(fmt, M, N, K, k):
    x = synthetic.tiny_random((M, K), M + N)
    w = synthetic.tiny_random((N, K), K + k, scale=0.02)
    qa, sa = oracle.quantize(x, 1, 16, fmt)
    qb, sb = oracle.quantize(w, 1, 16, fmt)
    want = oracle.gemm_rotout(qa, qb, sa, sb, fmt, k)
    got = hq.hq_gemm_rotout(_dev(qa), _scale(sa), _dev(qb), _scale(sb), k, fmt).cpu().numpy()
    if fmt == oracle.INT8:
        bad = np.argwhere(got.view(np.uint32) != want.view(np.uint32))
        assert bad.size == 0, f"{len(bad)} mismatches, first at {bad[0].tolist()}"
    else:
        rel = np.linalg.norm(got.astype(np.float64) - want) / np.linalg.norm(want.astype(np.float64))
        assert rel <= FP8_TOL


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3), ids=_fmt_name)
@pytest.mark.parametrize("rows,cols", [(64, 256), (1000, 4096), (3, 16)])
def test_quantize_prerotated(fmt, rows, cols):
    y = synthetic.tiny_random((rows, cols), rows + cols)
    y[rows // 2, 5] = 37.0  # the absmax element
    codes, scale = hq.hq_quantize_prerotated(_dev(y), fmt)
    want, ws = oracle.quantize_rotated(y, fmt)
    assert np.array_equal(codes.cpu().numpy(), want)
    assert scale.item() == ws


def test_quantize_prerotated_zero_and_nonfinite():
    codes, scale = hq.hq_quantize_prerotated(torch.zeros(32, 64, device="cuda"), oracle.INT8)
    assert scale.item() == 1.0 and torch.count_nonzero(codes).item() == 0
    y = torch.ones(32, 64, device="cuda")
    y[3, 7] = float("nan")
    hq.hq_quantize_prerotated(y, oracle.INT8)
    assert hq.hq_get_error() == 5  # HQ_ERR_NONFINITE, read and cleared


def test_next_layer_flow():
    """Layer 1 with the next layer's rotation in its epilogue, its output quantized as it is,
    and layer 2's GEMM: every intermediate equals the oracle's (INT8)."""
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw_fp32(w)
    X, W1 = d["X"], d["W"]
    W2 = synthetic.tiny_random((96, 128), 4, scale=0.05)
    k, fmt = 16, oracle.INT8
    qx, sx = oracle.quantize(X, 1, k, fmt)
    qw1, sw1 = oracle.quantize(W1, 1, k, fmt)
    qw2, sw2 = oracle.quantize(W2, 1, k, fmt)
    y_rot = hq.hq_gemm_rotout(_dev(qx), _scale(sx), _dev(qw1), _scale(sw1), k, fmt)
    qy, sy = hq.hq_quantize_prerotated(y_rot, fmt)
    y2 = hq.hq_gemm(qy, sy, _dev(qw2), _scale(sw2), fmt)
    torch.cuda.synchronize()
    want_rot = oracle.gemm_rotout(qx, qw1, sx, sw1, fmt, k)
    want_qy, want_sy = oracle.quantize_rotated(want_rot, fmt)
    _, want_y2 = oracle.epilogue(oracle.gemm(want_qy, qw2, fmt), want_sy, sw2)
    assert np.array_equal(y_rot.cpu().numpy().view(np.uint32), want_rot.view(np.uint32))
    assert np.array_equal(qy.cpu().numpy(), want_qy) and sy.item() == want_sy
    assert np.array_equal(y2.contiguous().view(torch.int16).cpu().numpy().view(np.uint16), want_y2)
