"""GPU parity of the CUDA path (called through the C ABI) against the CPU oracle.

Bar (stated for the method, see include/hq.h for the readings):
  * quantized codes and scales: bit-exact;
  * INT8 GEMM int32 accumulators: bit-exact;
  * bf16 outputs: within 1 bf16 ulp of the oracle's fp64-dequantized value (and, for INT8,
    bit-exact with the oracle's evaluation of the device epilogue formula);
  * FP8 path: relative Frobenius error of the output <= 2e-3 against the oracle's exact
    fp64 product of the same codes.
"""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import synthetic
from _helpers import to_device, bf16_bits, bits_to_f32, sample_rows, bf16_ulp_diff, rel_fro

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


def _quant_check(x_np, dim, k, fmt):
    codes, scale = hq.hq_quantize(to_device(x_np), dim, k, fmt)
    want_codes, want_scale = oracle.quantize(x_np, dim, k, fmt)
    want_codes = oracle.device_codes(want_codes, fmt)
    got = codes.cpu().numpy()
    assert got.shape == want_codes.shape
    mism = np.count_nonzero(got != want_codes)
    assert mism == 0, f"{mism} code mismatches of {got.size}"
    got_scale = scale.cpu().numpy()[0]
    assert got_scale.view(np.uint32) == np.float32(want_scale).view(np.uint32)
    return codes, scale


def _outlier_input(rows, cols, seed, dtype):
    x = synthetic.tiny_random((rows, cols), seed)
    x[:, 3 % cols] *= 60.0
    x[:, (cols // 2) % cols] *= -35.0
    return synthetic.to_bf16_bits(x) if dtype == "bf16" else x


# ------------------------------------------------------------------------------ quantize

@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_along_cols_ragged(dtype, k, fmt):
    # 37 rows x 5k cols: the element count is not a multiple of the 256-element warp chunk
    # nor of the per-step 1024 elements, so the tail paths run
    x = _outlier_input(37, 5 * k, 10 + k, dtype)
    _quant_check(x, 1, k, fmt)


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_along_rows_ragged(dtype, k, fmt):
    # rows = 3 tiles of 256 + 2k (ragged last row tile); cols = 208: ragged column tile
    x = _outlier_input(768 + 2 * k, 208, 20 + k, dtype)
    _quant_check(x, 0, k, fmt)


@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_large_grid(fmt):
    # big enough that every CTA runs several grid-stride steps in both passes
    x = _outlier_input(2048, 4096, 3, "bf16")
    _quant_check(x, 1, 256, fmt)
    _quant_check(x, 0, 64, fmt)


def test_quantize_zero_tensor():
    for dim in (0, 1):
        for fmt in FMTS:
            codes, scale = hq.hq_quantize(torch.zeros(64, 64, device="cuda"), dim, 16, fmt)
            assert scale.item() == 1.0 and int(codes.count_nonzero()) == 0


def test_quantize_single_outlier():
    x = np.zeros((32, 256), np.float32)
    x[5, 100] = 1000.0
    for dim in (0, 1):
        _quant_check(x, dim, 32, oracle.INT8)
        _quant_check(x, dim, 32, oracle.FP8_E4M3)


@pytest.mark.parametrize("bad", (float("nan"), float("inf")))
def test_quantize_nonfinite_sets_status(bad):
    x = torch.randn(64, 128, device="cuda")
    x[7, 9] = bad
    assert hq.hq_get_error() == 0
    hq.hq_quantize(x, 1, 64, "int8")
    assert hq.hq_get_error() == 5
    assert hq.hq_get_error() == 0  # cleared
    hq.hq_quantize(x, 0, 64, "fp8")
    assert hq.hq_get_error() == 5


def test_quantize_empty():
    codes, scale = hq.hq_quantize(torch.zeros(0, 64, device="cuda"), 1, 16, "int8")
    assert codes.numel() == 0 and scale.item() == 1.0


def test_argument_errors():
    x = torch.randn(64, 96, device="cuda")
    with pytest.raises(hq.HQError) as e:
        hq.hq_quantize(x, 1, 64, "int8")  # 96 % 64 != 0
    assert e.value.status == 2
    with pytest.raises(hq.HQError) as e:
        hq.hq_quantize(x, 1, 24, "int8")
    assert e.value.status == 1
    with pytest.raises(hq.HQError) as e:
        hq.hq_quantize(torch.randn(64, 24, device="cuda"), 0, 16, "int8")  # cols % 16
    assert e.value.status == 2
    buf = torch.randn(64 * 64 + 4, device="cuda")
    with pytest.raises(hq.HQError) as e:
        hq.hq_quantize(buf[1:1 + 64 * 64].view(64, 64), 1, 16, "int8")
    assert e.value.status == 4
    with pytest.raises(hq.HQError) as e:  # K = 40 is not a multiple of 16
        hq.hq_gemm(torch.zeros(128, 40, dtype=torch.uint8, device="cuda"), None,
                   torch.zeros(128, 40, dtype=torch.uint8, device="cuda"), None, "int8", hq.HQ_OUT_ACC)
    assert e.value.status == 2
    with pytest.raises(hq.HQError) as e:
        hq.hq_linear_fwd(torch.randn(64, 256, device="cuda"), torch.randn(100, 256, device="cuda"), 16, "int8")
    assert e.value.status == 2
    with pytest.raises(TypeError):
        hq.hq_quantize(torch.randn(16, 16), 1, 16, "int8")  # CPU tensor: no fallback


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_dual(dtype, k, fmt):
    """Both rotations from one call equal the oracle's two quantizations bit for bit."""
    x = _outlier_input(512 + 2 * k, 3 * k, 40 + k, dtype)
    cc, sc, cr, sr = hq.hq_quantize_dual(to_device(x), k, fmt)
    for codes, scale, dim in ((cc, sc, 1), (cr, sr, 0)):
        want_codes, want_scale = oracle.quantize(x, dim, k, fmt)
        assert np.array_equal(codes.cpu().numpy(), want_codes), f"dim {dim}"
        assert scale.cpu().numpy()[0].view(np.uint32) == np.float32(want_scale).view(np.uint32)


# Shapes for the fused two-rotation kernel (bf16, rows and cols multiples of 64, 256 x 256
# tiles): ragged last tiles in both directions where k allows it, and a case with more
# tiles than SMs so that CTAs run several tiles and the strip ring wraps.
def _fused_shapes(k):
    small = {16: (1344, 1216), 32: (1344, 1216), 64: (1344, 1216), 128: (1408, 1152), 256: (1536, 1280)}[k]
    many = (3328, 3328) if k == 256 else (3200, 3200)
    return (small, many)


@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_quantize_dual_fused_tiles(k, fmt):
    """The fused kernel's codes and scales equal the oracle's for both rotations."""
    for rows, cols in _fused_shapes(k):
        x = _outlier_input(rows, cols, 7 * k + rows, "bf16")
        cc, sc, cr, sr = hq.hq_quantize_dual(to_device(x), k, fmt)
        for codes, scale, dim in ((cc, sc, 1), (cr, sr, 0)):
            want_codes, want_scale = oracle.quantize(x, dim, k, fmt)
            got = codes.cpu().numpy()
            mism = np.count_nonzero(got != want_codes)
            assert mism == 0, f"{rows}x{cols} dim {dim}: {mism} code mismatches"
            assert scale.cpu().numpy()[0].view(np.uint32) == np.float32(want_scale).view(np.uint32)
    assert hq.hq_get_error() == 0


@pytest.mark.parametrize("k", (64, 256))
def test_quantize_dual_fused_matches_single(k):
    """At a full weight size (11008 x 4096, every CTA several tiles deep) the fused kernel
    writes the same bytes as the two single-rotation calls."""
    w = synthetic.WORKLOADS[2]
    W = to_device(synthetic.draw(w)["W"])
    for fmt in FMTS:
        cc, sc, cr, sr = hq.hq_quantize_dual(W, k, fmt)
        c1, s1 = hq.hq_quantize(W, 1, k, fmt)
        c0, s0 = hq.hq_quantize(W, 0, k, fmt)
        assert torch.equal(cc, c1) and torch.equal(sc, s1)
        assert torch.equal(cr, c0) and torch.equal(sr, s0)
    assert hq.hq_get_error() == 0


def test_quantize_dual_fused_special_values():
    """Zero tensor (scale 1, zero codes); a NaN (both rotations flagged); two near-maximal
    values in one row block, which overflow the rotation along the columns only: that
    rotation is flagged and the other is still written, equal to the oracle's."""
    z = torch.zeros(256, 512, dtype=torch.bfloat16, device="cuda")
    cc, sc, cr, sr = hq.hq_quantize_dual(z, 64, "int8")
    assert sc.item() == 1.0 and sr.item() == 1.0
    assert int(cc.count_nonzero()) == 0 and int(cr.count_nonzero()) == 0
    x = torch.randn(256, 512, device="cuda").to(torch.bfloat16)
    x[100, 300] = float("nan")
    assert hq.hq_get_error() == 0
    hq.hq_quantize_dual(x, 128, "fp8")
    assert hq.hq_get_error() == 5
    xb = _outlier_input(512, 512, 11, "bf16")
    big = np.uint16(0x7F7F)  # largest finite bf16, about 3.39e38
    xb[40, 0] = big
    xb[40, 1] = big
    cc, sc, cr, sr = hq.hq_quantize_dual(to_device(xb), 64, "int8")
    assert hq.hq_get_error() == 5
    assert not np.isfinite(sc.cpu().numpy()[0])
    want_codes, want_scale = oracle.quantize(xb, 0, 64, oracle.INT8)
    assert np.array_equal(cr.cpu().numpy(), want_codes)
    assert sr.cpu().numpy()[0].view(np.uint32) == np.float32(want_scale).view(np.uint32)


# ------------------------------------------------------------------------------ GEMM

def _rand_codes(shape, fmt, seed):
    r = np.random.default_rng(seed)
    if fmt == oracle.INT8:
        return r.integers(-127, 128, size=shape).astype(np.int8).view(np.uint8)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    return r.choice(finite, size=shape)


GEMM_SHAPES = [(128, 256, 128), (200, 272, 400), (384, 768, 1024), (64, 16, 16), (1, 32, 48),
               (300, 512, 12608 // 64 * 16)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int8_accumulators_exact(M, N, K):
    A = _rand_codes((M, K), oracle.INT8, M + K)
    B = _rand_codes((N, K), oracle.INT8, N + 7 * K)
    acc = hq.hq_gemm(torch.from_numpy(A).cuda(), None, torch.from_numpy(B).cuda(), None, "int8",
                     hq.HQ_OUT_ACC)
    want = oracle.gemm(A, B, oracle.INT8)
    np.testing.assert_array_equal(acc.cpu().numpy(), want)


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES[:4])
def test_gemm_int8_bf16_epilogue(M, N, K):
    A = _rand_codes((M, K), oracle.INT8, 3 * M + K)
    B = _rand_codes((N, K), oracle.INT8, 5 * N + K)
    sa = np.float32(0.0173)
    sb = np.float32(2.9e-4)
    out = hq.hq_gemm(torch.from_numpy(A).cuda(), torch.tensor([sa], device="cuda"),
                     torch.from_numpy(B).cuda(), torch.tensor([sb], device="cuda"), "int8")
    ref, fast = oracle.epilogue(oracle.gemm(A, B, oracle.INT8), sa, sb)
    got = bf16_bits(out)
    np.testing.assert_array_equal(got, fast)
    assert bf16_ulp_diff(got, ref).max() <= 1


# CTA-pair kernel (M >= 256) with ragged row and column edges: its bf16 epilogue stores 32 x 64
# boxes with TMA, clipped at the tensor's edge, and skips boxes wholly past it.
PAIR_EDGE_SHAPES = [(520, 400, 256), (300, 48, 512), (256, 16, 128), (777, 1040, 384), (1000, 1008, 768)]


@pytest.mark.parametrize("M,N,K", PAIR_EDGE_SHAPES)
@pytest.mark.parametrize("fmt", FMTS)
def test_gemm_pair_bf16_edges(M, N, K, fmt):
    A = _rand_codes((M, K), fmt, 17 * M + K)
    B = _rand_codes((N, K), fmt, 19 * N + K)
    sa, sb = np.float32(0.0123), np.float32(7.1e-4)
    out = torch.full((M, N), 3.0, dtype=torch.bfloat16, device="cuda")
    hq.hq_gemm(torch.from_numpy(A).cuda(), torch.tensor([sa], device="cuda"), torch.from_numpy(B).cuda(),
               torch.tensor([sb], device="cuda"), fmt, out=out)
    got = bf16_bits(out)
    ref, fast = oracle.epilogue(oracle.gemm(A, B, fmt), sa, sb)
    if fmt == oracle.INT8:
        np.testing.assert_array_equal(got, fast)
        assert bf16_ulp_diff(got, ref).max() <= 1
    else:
        assert rel_fro(bits_to_f32(got), bits_to_f32(ref)) <= FP8_TOL
    # nothing outside [M][N] exists to be written; every element inside was written
    assert not np.any(got == np.uint16(0x4040)) or np.count_nonzero(bits_to_f32(ref) == 3.0) > 0


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES[:5])
def test_gemm_fp8(M, N, K):
    A = _rand_codes((M, K), oracle.FP8_E4M3, 11 * M + K)
    B = _rand_codes((N, K), oracle.FP8_E4M3, 13 * N + K)
    At, Bt = torch.from_numpy(A).cuda(), torch.from_numpy(B).cuda()
    acc = hq.hq_gemm(At, None, Bt, None, "fp8", hq.HQ_OUT_ACC)
    want = oracle.gemm(A, B, oracle.FP8_E4M3)
    assert rel_fro(acc.cpu().numpy(), want) <= FP8_TOL
    sa, sb = np.float32(0.011), np.float32(0.0037)
    out = hq.hq_gemm(At, torch.tensor([sa], device="cuda"), Bt, torch.tensor([sb], device="cuda"), "fp8")
    ref, _ = oracle.epilogue(want, sa, sb)
    assert rel_fro(bits_to_f32(bf16_bits(out)), bits_to_f32(ref)) <= FP8_TOL


def test_gemm_k_zero_writes_zeros():
    a = torch.zeros(32, 0, dtype=torch.uint8, device="cuda")
    out = torch.full((32, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    b = torch.zeros(64, 0, dtype=torch.uint8, device="cuda")
    s = torch.ones(1, device="cuda")
    hq.hq_gemm(a, s, b, s, "int8", out=out)
    assert int(out.count_nonzero()) == 0


# ------------------------------------------------------------------------------ the layer

def _layer_check(d, k, fmt, rows_sample=None, tag="", step=False):
    """All three GEMMs of one layer: codes, scales, accumulators (via the split entry points)
    and the fused linear entry points' bf16 outputs.  step=True: the whole-layer entry point
    hq_linear_fwd_bwd's outputs are compared with the oracle on the same rows as well."""
    X, W, dY = d["X"], d["W"], d["dY"]
    Xd, Wd, dYd = to_device(X), to_device(W), to_device(dY)
    step_out = dict(zip(("fwd", "dx", "dw"), hq.hq_linear_fwd_bwd(Xd, Wd, dYd, k, fmt))) if step else {}
    cases = (
        ("fwd", hq.hq_linear_fwd, (Xd, Wd), oracle.linear_fwd, (X, W), (X, 1), (W, 1)),
        ("dx", hq.hq_linear_bwd_dx, (dYd, Wd), oracle.linear_bwd_dx, (dY, W), (dY, 1), (W, 0)),
        ("dw", hq.hq_linear_bwd_dw, (dYd, Xd), oracle.linear_bwd_dw, (dY, X), (dY, 0), (X, 0)),
    )
    for name, gfun, gargs, ofun, oargs, (a_src, a_dim), (b_src, b_dim) in cases:
        out = gfun(*gargs, k, fmt)
        n_out_rows = out.shape[0]
        rows = None if rows_sample is None else sample_rows(n_out_rows, seed=n_out_rows)
        want = ofun(*oargs, k, fmt, rows=rows)
        # codes and scales of both operands, bit-exact
        qa, sa = hq.hq_quantize(to_device(a_src), a_dim, k, fmt)
        qb, sb = hq.hq_quantize(to_device(b_src), b_dim, k, fmt)
        assert np.array_equal(qa.cpu().numpy(), oracle.device_codes(want["qa"], fmt)), f"{tag}{name}: A codes"
        assert np.array_equal(qb.cpu().numpy(), oracle.device_codes(want["qb"], fmt)), f"{tag}{name}: B codes"
        assert sa.cpu().numpy()[0] == want["sa"] and sb.cpu().numpy()[0] == want["sb"], f"{tag}{name}: scales"
        got = bf16_bits(out)
        if rows is not None:
            got = got[rows]
        if fmt == oracle.INT8:
            acc = hq.hq_gemm(qa, None, qb, None, fmt, hq.HQ_OUT_ACC).cpu().numpy()
            if rows is not None:
                acc = acc[rows]
            np.testing.assert_array_equal(acc, want["acc"], err_msg=f"{tag}{name}: int32")
            np.testing.assert_array_equal(got, want["fast"], err_msg=f"{tag}{name}: bf16 formula")
            assert bf16_ulp_diff(got, want["ref"]).max() <= 1, f"{tag}{name}: ulp"
        else:
            e = rel_fro(bits_to_f32(got), bits_to_f32(want["ref"]))
            assert e <= FP8_TOL, f"{tag}{name}: fp8 rel fro {e}"
        if step:
            gs = bf16_bits(step_out[name])
            if rows is not None:
                gs = gs[rows]
            if fmt == oracle.INT8:
                np.testing.assert_array_equal(gs, want["fast"], err_msg=f"{tag}{name}: step bf16 formula")
                assert bf16_ulp_diff(gs, want["ref"]).max() <= 1, f"{tag}{name}: step ulp"
            else:
                e = rel_fro(bits_to_f32(gs), bits_to_f32(want["ref"]))
                assert e <= FP8_TOL, f"{tag}{name}: step fp8 rel fro {e}"
    assert hq.hq_get_error() == 0


def _fwd_bwd_check(d, k, fmt, rows_sample=None, tag=""):
    """hq_linear_fwd_bwd (quantize once, both rotations) equals the three separate layer
    entry points bit for bit, and those are checked against the oracle by _layer_check."""
    Xd, Wd, dYd = to_device(d["X"]), to_device(d["W"]), to_device(d["dY"])
    Y, dX, dW = hq.hq_linear_fwd_bwd(Xd, Wd, dYd, k, fmt)
    sep = (hq.hq_linear_fwd(Xd, Wd, k, fmt), hq.hq_linear_bwd_dx(dYd, Wd, k, fmt),
           hq.hq_linear_bwd_dw(dYd, Xd, k, fmt))
    for name, a, b in zip(("Y", "dX", "dW"), (Y, dX, dW), sep):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"{tag}{name}"
    assert hq.hq_get_error() == 0


def _saved_codes_check(d, k, fmt, tag=""):
    """Training flow: hq_linear_fwd_save keeps X's token-rotated codes (equal to the oracle's
    quantization of X along M bit for bit), and hq_linear_bwd from those codes gives the same
    dX and dW as the separate entry points given X itself."""
    X = d["X"]
    Xd, Wd, dYd = to_device(X), to_device(d["W"]), to_device(d["dY"])
    Y, xqt, sx = hq.hq_linear_fwd_save(Xd, Wd, k, fmt)
    want_codes, want_scale = oracle.quantize(X, 0, k, fmt)
    assert np.array_equal(xqt.cpu().numpy(), oracle.device_codes(want_codes, fmt)), f"{tag}saved codes"
    assert sx.cpu().numpy()[0].view(np.uint32) == np.float32(want_scale).view(np.uint32), f"{tag}saved scale"
    dX, dW = hq.hq_linear_bwd(dYd, Wd, xqt, sx, k, fmt)
    sep = (hq.hq_linear_fwd(Xd, Wd, k, fmt), hq.hq_linear_bwd_dx(dYd, Wd, k, fmt),
           hq.hq_linear_bwd_dw(dYd, Xd, k, fmt))
    for name, a, b in zip(("Y", "dX", "dW"), (Y, dX, dW), sep):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), f"{tag}{name}"
    assert hq.hq_get_error() == 0


@pytest.mark.parametrize("fmt", FMTS)
def test_fwd_bwd_tiny_workload(fmt):
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw(w)
    _layer_check(d, w.k, fmt)
    _fwd_bwd_check(d, w.k, fmt)
    _saved_codes_check(d, w.k, fmt)


@pytest.mark.parametrize("wid", (2, 3, 4))
def test_fwd_bwd_full_size(wid):
    w = synthetic.WORKLOADS[wid]
    fmt = oracle.INT8 if w.fmt == "int8" else oracle.FP8_E4M3
    for li in range(len(w.layers)):
        d = synthetic.draw(w, li)
        _fwd_bwd_check(d, w.k, fmt, tag=f"{w.name}/{li}/")
        _saved_codes_check(d, w.k, fmt, tag=f"{w.name}/{li}/")


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("k", KS)
@pytest.mark.parametrize("fmt", FMTS)
def test_saved_codes_every_k(dtype, k, fmt):
    """The saved-codes flow at every k, both formats and both source dtypes, on a layer of
    3k tokens, 2k inputs and 5k outputs (several GEMM tiles only at the larger k)."""
    M, K, N = 3 * k, 2 * k, 5 * k
    X = _outlier_input(M, K, 70 + k, dtype)
    W = synthetic.tiny_random((N, K), 80 + k, scale=0.02)
    dY = synthetic.tiny_random((M, N), 90 + k, scale=1e-3)
    if dtype == "bf16":
        W, dY = synthetic.to_bf16_bits(W), synthetic.to_bf16_bits(dY)
    _saved_codes_check({"X": X, "W": W, "dY": dY}, k, fmt, tag=f"{dtype}/{k}/{fmt}/")


# Weight gradients with few output tiles and a long token contraction run as two halves of
# the contraction whose partial sums are combined in the GEMM (split contraction): ragged
# output edges, both formats, through the layer entry points and the layer step.
SPLIT_SHAPES = [(4096, 272, 400), (8192, 256, 256), (3072, 768, 512)]


@pytest.mark.parametrize("M,K,N", SPLIT_SHAPES)
@pytest.mark.parametrize("fmt", FMTS)
def test_split_contraction_dw(M, K, N, fmt):
    k = 16
    X = _outlier_input(M, K, 3 + K, "bf16")
    dY = synthetic.to_bf16_bits(synthetic.tiny_random((M, N), 5 + N, scale=1e-3))
    W = synthetic.to_bf16_bits(synthetic.tiny_random((N, K), 7 + K, scale=0.02))
    d = {"X": X, "W": W, "dY": dY}
    out = hq.hq_linear_bwd_dw(to_device(dY), to_device(X), k, fmt)
    want = oracle.linear_bwd_dw(dY, X, k, fmt)
    got = bf16_bits(out)
    if fmt == oracle.INT8:
        np.testing.assert_array_equal(got, want["fast"])
        assert bf16_ulp_diff(got, want["ref"]).max() <= 1
    else:
        assert rel_fro(bits_to_f32(got), bits_to_f32(want["ref"])) <= FP8_TOL
    _fwd_bwd_check(d, k, fmt, tag=f"split/{M}/{K}/{N}/")
    _saved_codes_check(d, k, fmt, tag=f"split/{M}/{K}/{N}/")


@pytest.mark.parametrize("fmt", FMTS)
def test_layer_tiny_workload(fmt):
    w = synthetic.WORKLOADS[1]
    _layer_check(synthetic.draw(w), w.k, fmt)


@pytest.mark.parametrize("wid", (2, 3, 4))
def test_layer_token_prefix(wid):
    """Each workload at its full K and N but a 512-token prefix (exact, full comparison)."""
    w = synthetic.WORKLOADS[wid]
    fmt = oracle.INT8 if w.fmt == "int8" else oracle.FP8_E4M3
    for li in range(len(w.layers)):
        _layer_check(synthetic.draw(w, li, M=512), w.k, fmt, tag=f"{w.name}/{li}/")


@pytest.mark.parametrize("wid", (1, 2, 3, 4))
def test_layer_full_size(wid):
    """Each workload at its full size, outputs of the separate entry points and of the
    whole-layer step hq_linear_fwd_bwd compared with the oracle on sampled rows; codes and
    scales compared in full."""
    w = synthetic.WORKLOADS[wid]
    fmt = oracle.INT8 if w.fmt == "int8" else oracle.FP8_E4M3
    for li in range(len(w.layers)):
        _layer_check(synthetic.draw(w, li), w.k, fmt, rows_sample=True, tag=f"{w.name}/{li}/", step=True)


@pytest.mark.parametrize("fmt_name,k", synthetic.WORKLOADS[5].sweep)
def test_llama_block_sweep_o_proj(fmt_name, k):
    """Llama-2-7B block sweep over formats and k on the 4096 -> 4096 projection (8192 tokens)."""
    w = synthetic.WORKLOADS[5]
    fmt = oracle.INT8 if fmt_name == "int8" else oracle.FP8_E4M3
    _layer_check(synthetic.draw(w, 1), k, fmt, rows_sample=True, tag=f"o/{fmt_name}/{k}/")


@pytest.mark.parametrize("li", (0, 1, 2, 3, 4))
def test_llama_block_step_vs_oracle(li):
    """The bench's headline step: every layer of the Llama-2-7B block (qkv, o, gate, up, down
    at 8192 tokens) through hq_linear_fwd_bwd at INT8 k = 256, outputs against the oracle on
    sampled rows, codes and scales in full."""
    w = synthetic.WORKLOADS[5]
    _layer_check(synthetic.draw(w, li), 256, oracle.INT8, rows_sample=True, tag=f"{w.layers[li].name}/", step=True)


@pytest.mark.parametrize("li", (0, 2, 3, 4))
def test_llama_block_sweep_other_layers(li):
    """The block's sweep over INT8 / FP8 x k = 16 .. 256 on qkv, gate, up and down (8192
    tokens; the o projection has its own test above): codes and scales in full, the separate
    entry points' and the whole-layer step's outputs on sampled rows."""
    w = synthetic.WORKLOADS[5]
    d = synthetic.draw(w, li)
    for fmt_name, k in w.sweep:
        fmt = oracle.INT8 if fmt_name == "int8" else oracle.FP8_E4M3
        _layer_check(d, k, fmt, rows_sample=True, tag=f"{w.layers[li].name}/{fmt_name}/{k}/", step=(k in (16, 256)))
