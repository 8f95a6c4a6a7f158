"""GPU parity of the backward placement that reuses the forward's codes ("HALO: Hadamard-Assisted
Lower-Precision Optimization for LLMs", Approach): dY rotated along the tokens once, dX from
its codes and the forward's K-rotated weight codes through the GEMM that reads both operands
contraction-outermost, both rotations undone on the fp32 output.

INT8: every result bit-exact against the oracle (integer accumulators, the same fp32 rounding
steps).  FP8: the tensor cores accumulate in fp32, the oracle exactly, so the de-rotated output
is compared to the oracle's fp32 values with the relative Frobenius bound 2e-3."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import synthetic
from _helpers import to_device, bf16_bits, bits_to_f32

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


def _dev(a: np.ndarray):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _scale(s):
    return torch.tensor([float(s)], dtype=torch.float32, device="cuda")


def _fmt_name(fmt):
    return "int8" if fmt == oracle.INT8 else "fp8"


def _inputs(M, K, N, seed):
    dY = synthetic.tiny_random((M, N), seed) * 1e-3
    dY[seed % M, :] *= 40.0  # one outlier token
    W = synthetic.tiny_random((N, K), seed + 1, scale=0.02)
    X = synthetic.tiny_random((M, K), seed + 2)
    X[:, (3 * seed) % K] *= 50.0  # one outlier channel
    return X, W, dY


def _check_dx(got: torch.Tensor, want: dict, fmt, tag=""):
    g = bf16_bits(got)
    if fmt == oracle.INT8:
        bad = np.argwhere(g != want["out"])
        assert bad.size == 0, f"{tag}{len(bad)} mismatches, first at {bad[0].tolist()}"
    else:
        z = want["z"].astype(np.float64)
        rel = np.linalg.norm(bits_to_f32(g).astype(np.float64) - z) / np.linalg.norm(z)
        assert rel <= FP8_TOL, f"{tag}relative error {rel:.3g}"


# (M, K, N, k): several 256 x 256 tiles, M and K not multiples of 256, contraction N ragged
# against the 128-deep k-blocks, M below one CTA's 128 rows, N below one k-block
SHAPES = [(256, 256, 128, 16), (320, 384, 200, 64), (512, 512, 1000, 256), (64, 128, 48, 32),
          (1024, 768, 4096, 128), (768, 256, 16, 256)]


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3), ids=_fmt_name)
@pytest.mark.parametrize("M,K,N,k", SHAPES)
def test_dx_reuse_from_codes(fmt, M, K, N, k):
    _, W, dY = _inputs(M, K, N, M + K + N)
    g, sg = oracle.quantize(dY, 0, k, fmt)   # [N][M]
    wq, sw = oracle.quantize(W, 1, k, fmt)   # [N][K]
    want = oracle.linear_bwd_dx_reuse(g, sg, wq, sw, k, fmt)
    got = hq.hq_linear_bwd_dx_reuse(_dev(g), _scale(sg), _dev(wq), _scale(sw), k, fmt)
    torch.cuda.synchronize()
    _check_dx(got, want, fmt, f"{M}x{K}x{N} k={k}: ")


def test_dx_reuse_zero_and_one_hot():
    """All-zero codes give exact zeros; a single nonzero product gives the closed form
    s * c^2 * h_i h_j^T on one block pair (both rotations undone)."""
    M, K, N, k = 256, 256, 128, 64
    g = np.zeros((N, M), dtype=np.uint8)
    wq = np.zeros((N, K), dtype=np.uint8)
    got = hq.hq_linear_bwd_dx_reuse(_dev(g), _scale(1.0), _dev(wq), _scale(1.0), k, oracle.INT8)
    assert torch.count_nonzero(got.float()).item() == 0
    g[5, 70] = 3       # G[n=5][m=70]
    wq[5, 129] = 0xFE  # Wq[n=5][j=129] = -2
    want = oracle.linear_bwd_dx_reuse(g, np.float32(0.5), wq, np.float32(0.25), k, oracle.INT8)
    got = hq.hq_linear_bwd_dx_reuse(_dev(g), _scale(0.5), _dev(wq), _scale(0.25), k, oracle.INT8)
    _check_dx(got, want, oracle.INT8)
    nz = np.argwhere(want["out"] != 0)
    assert nz[:, 0].min() == 64 and nz[:, 0].max() == 127 and nz[:, 1].min() == 128 and nz[:, 1].max() == 191


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3), ids=_fmt_name)
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("M,K,N,k", [(256, 512, 384, 128), (192, 320, 448, 64), (512, 256, 256, 256)])
def test_keep_and_reuse_flow(fmt, dtype, M, K, N, k):
    """hq_linear_fwd_keep then hq_linear_bwd_reuse against the oracle: every code tensor and
    scale bit-exact, Y and dW as the HALO-2 calls give them, dX as the reuse placement."""
    X, W, dY = _inputs(M, K, N, 7 * M + k)
    if dtype == "bf16":
        X, W, dY = (synthetic.to_bf16_bits(a) for a in (X, W, dY))
    Xd, Wd, dYd = to_device(X), to_device(W), to_device(dY)
    Y, xqt, sx, wq, sw = hq.hq_linear_fwd_keep(Xd, Wd, k, fmt)
    Y2, xqt2, sx2 = hq.hq_linear_fwd_save(Xd, Wd, k, fmt)
    dX, dW = hq.hq_linear_bwd_reuse(dYd, xqt, sx, wq, sw, k, fmt)
    torch.cuda.synchronize()
    assert torch.equal(Y, Y2) and torch.equal(xqt, xqt2) and torch.equal(sx, sx2)
    want_wq, want_sw = oracle.quantize(W, 1, k, fmt)
    want_xq, want_sx = oracle.quantize(X, 0, k, fmt)
    assert np.array_equal(wq.cpu().numpy(), want_wq) and sw.item() == want_sw
    assert np.array_equal(xqt.cpu().numpy(), want_xq) and sx.item() == want_sx
    r = oracle.linear_bwd_reuse(dY, want_xq, want_sx, want_wq, want_sw, k, fmt)
    want_dx = oracle.linear_bwd_dx_reuse(r["g"], r["s_g"], want_wq, want_sw, k, fmt)
    _check_dx(dX, want_dx, fmt, "dX: ")
    if fmt == oracle.INT8:
        assert np.array_equal(bf16_bits(dW), r["dw"])
        assert np.array_equal(bf16_bits(Y), oracle.linear_fwd(X, W, k, fmt)["fast"])
    else:
        dw_ref = bits_to_f32(oracle.linear_bwd_dw(dY, X, k, fmt)["ref"]).astype(np.float64)
        rel = np.linalg.norm(bits_to_f32(bf16_bits(dW)) - dw_ref) / np.linalg.norm(dw_ref)
        assert rel <= FP8_TOL


@pytest.mark.parametrize("wid", (2, 3))
def test_reuse_flow_full_size(wid):
    """The Llama up-projection (INT8, k=256) and the attention output projection (FP8, k=128)
    at full size: the kept codes in full, dX on two whole k-row blocks (first and last), dW on
    sampled rows."""
    w = synthetic.WORKLOADS[wid]
    fmt = oracle.INT8 if w.fmt == "int8" else oracle.FP8_E4M3
    k = w.k
    d = synthetic.draw(w)
    X, W, dY = d["X"], d["W"], d["dY"]
    M, K = X.shape
    N = W.shape[0]
    Xd, Wd, dYd = to_device(X), to_device(W), to_device(dY)
    Y, xqt, sx, wq, sw = hq.hq_linear_fwd_keep(Xd, Wd, k, fmt)
    dX, dW = hq.hq_linear_bwd_reuse(dYd, xqt, sx, wq, sw, k, fmt)
    torch.cuda.synchronize()
    want_wq, want_sw = oracle.quantize(W, 1, k, fmt)
    assert np.array_equal(wq.cpu().numpy(), want_wq) and sw.item() == want_sw
    g, sg = oracle.quantize(dY, 0, k, fmt)
    blocks = [0, M - k]
    want = oracle.linear_bwd_dx_reuse(g, sg, want_wq, want_sw, k, fmt, rows=blocks)
    got = torch.cat([dX[r:r + k] for r in blocks])
    _check_dx(got, want, fmt, f"{w.name}: ")
    xq, sxo = oracle.quantize(X, 0, k, fmt)
    assert sx.item() == sxo
    rows = np.array([0, 1, 255, 256, N // 2, N - 1], dtype=np.int64)
    acc = oracle.gemm(g, xq, fmt, rows)
    ref, fast = oracle.epilogue(acc, sg, sxo)
    got_dw = bf16_bits(dW[torch.from_numpy(rows).cuda()])
    if fmt == oracle.INT8:
        assert np.array_equal(got_dw, fast)
    else:
        r = bits_to_f32(ref).astype(np.float64)
        assert np.linalg.norm(bits_to_f32(got_dw) - r) / np.linalg.norm(r) <= FP8_TOL
