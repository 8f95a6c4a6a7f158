"""GPU parity of the randomized Hadamard variant (a sign diagonal D before the blocks,
t = H_k D x) against the CPU oracle: codes and scales bit-exact, layer outputs as for the
plain rotation (INT8 bit-exact with the oracle's device-formula epilogue, FP8 within 2e-3
relative Frobenius error).  Sign flags are seeded random draws passed in as inputs."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import synthetic
from _helpers import to_device, bf16_bits, bits_to_f32, bf16_ulp_diff, rel_fro

pytestmark = pytest.mark.gpu

KS = (16, 32, 64, 128, 256)
FMTS = (oracle.INT8, oracle.FP8_E4M3)
FP8_TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_lib):
    from hadamard_rotated_precision_b200 import build
    build.build()
    assert torch.cuda.is_available()
    hq.lib()
    yield
    assert hq.hq_get_error() == 0


def _flags_dev(f):
    return torch.from_numpy(f).cuda()


def _outlier_input(rows, cols, seed, dtype):
    x = synthetic.tiny_random((rows, cols), seed)
    x[:, 3 % cols] *= 60.0
    x[:, (cols // 2) % cols] *= -35.0
    return synthetic.to_bf16_bits(x) if dtype == "bf16" else x


def _check_codes(codes, scale, x, dim, k, fmt, neg, tag=""):
    want_codes, want_scale = oracle.quantize(x, dim, k, fmt, neg=neg)
    got = codes.cpu().numpy()
    mism = np.count_nonzero(got != want_codes)
    assert mism == 0, f"{tag}: {mism} code mismatches of {got.size}"
    assert scale.cpu().numpy()[0].view(np.uint32) == np.float32(want_scale).view(np.uint32), tag


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_rht_both_dims(dtype, k, fmt):
    """Ragged shapes (rows and cols not multiples of the kernels' tiles; for k = 16 the
    contiguous kernel's 32-element thread chunks straddle rows)."""
    x = _outlier_input(512 + 2 * k, 3 * k, 90 + k, dtype)
    rows, cols = (512 + 2 * k, 3 * k)
    for dim in (0, 1):
        neg = synthetic.sign_flags(cols if dim == 1 else rows, 7 * k + dim)
        codes, scale = hq.hq_quantize_rht(to_device(x), dim, k, fmt, _flags_dev(neg))
        _check_codes(codes, scale, x, dim, k, fmt, neg, f"{dtype}/k{k}/dim{dim}")


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
def test_quantize_rht_many_steps(dtype):
    """Large enough that every CTA runs several grid-stride steps, in the forward (absmax) and
    reversed (codes) order, so the per-thread column tracking wraps many times."""
    x = _outlier_input(2048, 2 * 1536, 5, dtype)
    for dim, k in ((1, 256), (1, 16), (0, 64)):
        n = x.shape[1] if dim == 1 else x.shape[0]
        neg = synthetic.sign_flags(n, 100 + k + dim)
        for fmt in FMTS:
            codes, scale = hq.hq_quantize_rht(to_device(x), dim, k, fmt, _flags_dev(neg))
            _check_codes(codes, scale, x, dim, k, fmt, neg, f"{dtype}/k{k}/dim{dim}")


def test_quantize_rht_identities():
    """All flags clear = the plain rotation; all set = every INT8 code negated with the same
    scale (H is linear, the flip exact, rounding to nearest-even symmetric)."""
    x = _outlier_input(1024, 768, 3, "bf16")
    xd = to_device(x)
    for dim in (0, 1):
        n = 768 if dim == 1 else 1024
        c0, s0 = hq.hq_quantize(xd, dim, 64, "int8")
        cz, sz = hq.hq_quantize_rht(xd, dim, 64, "int8", torch.zeros(n, dtype=torch.uint8, device="cuda"))
        assert torch.equal(c0, cz) and torch.equal(s0, sz)
        co, so = hq.hq_quantize_rht(xd, dim, 64, "int8", torch.ones(n, dtype=torch.uint8, device="cuda"))
        assert torch.equal(s0, so)
        assert torch.equal(co.view(torch.int8), -c0.view(torch.int8))


@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_dual_rht(k, fmt):
    """Both rotations with their own flags: the fused kernel (bf16, multiples of 64, more tiles
    than SMs for k = 64) and the four-pass path (fp32 source)."""
    cases = [("bf16", (3200, 3200) if k < 256 else (3328, 3328)), ("f32", (512 + 2 * k, 3 * k))]
    if k <= 64:
        cases.append(("bf16", (1344, 1216)))
    for dtype, (rows, cols) in cases:
        x = _outlier_input(rows, cols, 11 * k + rows, dtype)
        nc, nr = synthetic.sign_flags(cols, k + 1), synthetic.sign_flags(rows, k + 2)
        cc, sc, cr, sr = hq.hq_quantize_dual_rht(to_device(x), k, fmt, _flags_dev(nc), _flags_dev(nr))
        _check_codes(cc, sc, x, 1, k, fmt, nc, f"{dtype}/{rows}x{cols}/cols")
        _check_codes(cr, sr, x, 0, k, fmt, nr, f"{dtype}/{rows}x{cols}/rows")
    # one vector given, the other NULL (plain for that rotation)
    x = _outlier_input(1024, 1024, 77, "bf16")
    nc = synthetic.sign_flags(1024, 5)
    cc, sc, cr, sr = hq.hq_quantize_dual_rht(to_device(x), k, fmt, _flags_dev(nc), None)
    _check_codes(cc, sc, x, 1, k, fmt, nc, "cols only")
    _check_codes(cr, sr, x, 0, k, fmt, None, "rows plain")


def _layer_rht_check(d, k, fmt, tag, rows=None):
    X, W, dY = d["X"], d["W"], d["dY"]
    M, K = X.shape
    N = W.shape[0]
    nk, nn, nm = synthetic.sign_flags(K, 1), synthetic.sign_flags(N, 2), synthetic.sign_flags(M, 3)
    Y, dX, dW = hq.hq_linear_fwd_bwd_rht(to_device(X), to_device(W), to_device(dY), k, fmt,
                                        _flags_dev(nk), _flags_dev(nn), _flags_dev(nm))
    want = {"Y": oracle.linear_fwd(X, W, k, fmt, rows, neg=nk),
            "dX": oracle.linear_bwd_dx(dY, W, k, fmt, rows, neg=nn),
            "dW": oracle.linear_bwd_dw(dY, X, k, fmt, rows, neg=nm)}
    for name, out in (("Y", Y), ("dX", dX), ("dW", dW)):
        got = bf16_bits(out)
        if rows is not None:
            got = got[rows]
        w = want[name]
        if fmt == oracle.INT8:
            np.testing.assert_array_equal(got, w["fast"], err_msg=f"{tag}{name}")
            assert bf16_ulp_diff(got, w["ref"]).max() <= 1, f"{tag}{name}"
        else:
            assert rel_fro(bits_to_f32(got), bits_to_f32(w["ref"])) <= FP8_TOL, f"{tag}{name}"
    assert hq.hq_get_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_layer_rht_tiny_workload(fmt):
    w = synthetic.WORKLOADS[1]
    _layer_rht_check(synthetic.draw(w), w.k, fmt, "tiny/")


@pytest.mark.parametrize("wid", (2, 3, 4))
def test_layer_rht_token_prefix(wid):
    """Each workload's layer at its full K and N and a 512-token prefix."""
    w = synthetic.WORKLOADS[wid]
    fmt = oracle.INT8 if w.fmt == "int8" else oracle.FP8_E4M3
    for li in range(len(w.layers)):
        _layer_rht_check(synthetic.draw(w, li, M=512), w.k, fmt, f"{w.name}/{li}/")


def test_layer_rht_zero_flags_equal_plain():
    w = synthetic.WORKLOADS[2]
    d = synthetic.draw(w, 0, M=512)
    X, W, dY = (to_device(d[n]) for n in ("X", "W", "dY"))
    M, K = X.shape
    N = W.shape[0]
    z = lambda n: torch.zeros(n, dtype=torch.uint8, device="cuda")  # noqa: E731
    a = hq.hq_linear_fwd_bwd_rht(X, W, dY, w.k, "int8", z(K), z(N), z(M))
    b = hq.hq_linear_fwd_bwd(X, W, dY, w.k, "int8")
    for u, v in zip(a, b):
        assert torch.equal(u.view(torch.int16), v.view(torch.int16))
