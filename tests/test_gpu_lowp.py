"""GPU parity of the FP6 (e3m2, e2m3) and FP4 (e2m1) code formats against the CPU oracle:
codes and scales bit-exact, GEMMs on tcgen05 kind::f8f6f4 within 2e-3 relative Frobenius error
of the oracle's exact fp64 product of the same codes (the FP8 bar), layer outputs likewise."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import synthetic
from _helpers import to_device, bf16_bits, bits_to_f32, rel_fro
from test_gpu_parity import (_quant_check, _outlier_input, _layer_check, _fwd_bwd_check, _fused_shapes,
                             _saved_codes_check)

pytestmark = pytest.mark.gpu

LOWP = (oracle.FP6_E3M2, oracle.FP6_E2M3, oracle.FP4_E2M1)
TOL = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_lib):
    from hadamard_rotated_precision_b200 import build
    build.build()
    assert torch.cuda.is_available()
    hq.lib()
    yield
    assert hq.hq_get_error() == 0


@pytest.mark.parametrize("fmt", LOWP)
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("k", (16, 64, 256))
def test_quantize_lowp(fmt, dtype, k):
    x = _outlier_input(512 + 2 * k, 3 * k, 50 + k + fmt, dtype)
    for dim in (0, 1):
        _quant_check(x, dim, k, fmt)


@pytest.mark.parametrize("fmt", LOWP)
@pytest.mark.parametrize("k", (32, 128, 256))
def test_quantize_dual_lowp(fmt, k):
    """The fused two-rotation kernel (bf16, multiples of 64, several tiles per CTA) and the
    four-pass path (fp32)."""
    cases = [("bf16", s) for s in _fused_shapes(k)] + [("f32", (512 + 2 * k, 3 * k))]
    for dtype, (rows, cols) in cases:
        x = _outlier_input(rows, cols, 3 * k + rows + fmt, dtype)
        cc, sc, cr, sr = hq.hq_quantize_dual(to_device(x), k, fmt)
        for codes, scale, dim in ((cc, sc, 1), (cr, sr, 0)):
            want_codes, want_scale = oracle.quantize(x, dim, k, fmt)
            mism = np.count_nonzero(codes.cpu().numpy() != oracle.device_codes(want_codes, fmt))
            assert mism == 0, f"{dtype}/{rows}x{cols}/dim{dim}: {mism} mismatches"
            assert scale.cpu().numpy()[0].view(np.uint32) == np.float32(want_scale).view(np.uint32)


def _rand_lowp_codes(shape, fmt, seed):
    return np.random.default_rng(seed).integers(0, 1 << oracle.minifloat_bits(fmt), size=shape).astype(np.uint8)


@pytest.mark.parametrize("fmt", LOWP)
@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (200, 272, 400), (384, 768, 1024), (64, 16, 32),
                                   (512, 512, 3072)])
def test_gemm_lowp(fmt, M, N, K):
    """Single-CTA (M < 256) and CTA-pair kernels, ragged tiles, short and long contractions."""
    A = _rand_lowp_codes((M, K), fmt, 7 * M + K + fmt)
    B = _rand_lowp_codes((N, K), fmt, 5 * N + K + fmt)
    # the library's operand layout: 16-code groups packed into 16-byte chunks
    At = torch.from_numpy(oracle.device_codes(A, fmt)).cuda()
    Bt = torch.from_numpy(oracle.device_codes(B, fmt)).cuda()
    acc = hq.hq_gemm(At, None, Bt, None, fmt, hq.HQ_OUT_ACC)
    want = oracle.gemm(A, B, fmt)
    assert rel_fro(acc.cpu().numpy(), want) <= 1e-6  # products of these codes sum exactly here
    sa, sb = np.float32(0.013), np.float32(0.0041)
    out = hq.hq_gemm(At, torch.tensor([sa], device="cuda"), Bt, torch.tensor([sb], device="cuda"), fmt)
    ref, _ = oracle.epilogue(want, sa, sb)
    assert rel_fro(bits_to_f32(bf16_bits(out)), bits_to_f32(ref)) <= TOL


@pytest.mark.parametrize("fmt", LOWP)
def test_layer_lowp_tiny(fmt):
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw(w)
    _layer_check(d, w.k, fmt, tag=f"tiny/{fmt}/")
    _fwd_bwd_check(d, w.k, fmt, tag=f"tiny/{fmt}/")


@pytest.mark.parametrize("fmt", LOWP)
def test_layer_lowp_token_prefix(fmt):
    """The Llama up-projection at full K and N, 512 tokens (HALO-1 with FP6 / FP4 codes)."""
    w = synthetic.WORKLOADS[2]
    d = synthetic.draw(w, 0, M=512)
    _layer_check(d, w.k, fmt, tag=f"llama512/{fmt}/")
    _fwd_bwd_check(d, w.k, fmt, tag=f"llama512/{fmt}/")


@pytest.mark.parametrize("fmt", LOWP)
def test_layer_lowp_saved_codes(fmt):
    """Training flow with saved codes in FP6 / FP4: the kept token-rotated codes equal the
    oracle's (packed layout) and the backward from them equals the separate entry points."""
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw(w)
    _saved_codes_check(d, w.k, fmt, tag=f"tiny/{fmt}/")
    d = synthetic.draw(synthetic.WORKLOADS[4], 0, M=512)
    _saved_codes_check(d, 64, fmt, tag=f"vit512/{fmt}/")


@pytest.mark.parametrize("fmt", LOWP)
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
def test_quantize_rht_lowp(fmt, dtype):
    """The randomized variant's sign flags with minifloat codes: single rotations in both
    directions and both rotations at once (fused kernel for the bf16 source)."""
    k = 64
    rows, cols = (1344, 1216) if dtype == "bf16" else (512 + 2 * k, 3 * k)
    x = _outlier_input(rows, cols, 21 + fmt, dtype)
    nc, nr = synthetic.sign_flags(cols, 30 + fmt), synthetic.sign_flags(rows, 40 + fmt)
    f = lambda a: torch.from_numpy(a).cuda()  # noqa: E731
    for dim, neg in ((1, nc), (0, nr)):
        codes, scale = hq.hq_quantize_rht(to_device(x), dim, k, fmt, f(neg))
        want, ws = oracle.quantize(x, dim, k, fmt, neg=neg)
        assert np.array_equal(codes.cpu().numpy(), oracle.device_codes(want, fmt)), f"dim {dim}"
        assert scale.cpu().numpy()[0].view(np.uint32) == np.float32(ws).view(np.uint32)
    cc, sc, cr, sr = hq.hq_quantize_dual_rht(to_device(x), k, fmt, f(nc), f(nr))
    for codes, scale, dim, neg in ((cc, sc, 1, nc), (cr, sr, 0, nr)):
        want, ws = oracle.quantize(x, dim, k, fmt, neg=neg)
        assert np.array_equal(codes.cpu().numpy(), oracle.device_codes(want, fmt)), f"dual dim {dim}"
        assert scale.cpu().numpy()[0].view(np.uint32) == np.float32(ws).view(np.uint32)
