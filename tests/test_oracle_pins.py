"""Pins of the CPU oracle to facts that do not come from the oracle itself.

Each test checks one oracle function against a closed form, a textbook or library routine,
a hand-derived fixture, an exact rational computation, or brute force on tiny inputs, so
that a dropped term, a wrong sign or index, or a transposed operand fails at least one test.
Sources: "Training Transformers with 4-bit Integers" section 3.3 (block-diagonal H_k,
cancellation in the product) and section 3.1 (symmetric integer range, INT32 product
dequantized); "HALO: Hadamard-Assisted Lower-Precision Optimization for LLMs" Approach
(right-hand rotation of X and W, left-hand rotation of the output gradient, tensor-wise
scale) and Limitations (round-to-nearest, FP8).
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from hadamard_rotated_precision_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
KS = (16, 32, 64, 128, 256)


def _ints(shape, seed, lo=-8, hi=8):
    r = np.random.default_rng(seed)
    return r.integers(lo, hi + 1, size=shape).astype(np.float32)


# ------------------------------------------------------------------------- Hadamard transform

@pytest.mark.parametrize("k", KS)
def test_fwht_equals_dense_sylvester_matrix(oracle_lib, k):
    """Integer inputs keep every fp32 partial sum exact, so the butterfly must equal the
    dense product with scipy's Sylvester-construction Hadamard matrix bit for bit."""
    H = scipy.linalg.hadamard(k).astype(np.int64)
    for seed in range(4):
        x = _ints(k, seed)
        got = oracle.fwht_block(x)
        want = (x.astype(np.int64) @ H).astype(np.float32)
        np.testing.assert_array_equal(got, want)


def test_fwht_hand_fixture(oracle_lib):
    lines = [l for l in open(os.path.join(GOLDEN, "fwht_ramp_k16.txt")) if not l.startswith("#")]
    x = np.array(lines[0].split(":")[1].split(), dtype=np.float32)
    want = np.array(lines[1].split(":")[1].split(), dtype=np.float32)
    np.testing.assert_array_equal(oracle.fwht_block(x), want)


@pytest.mark.parametrize("k", KS)
def test_one_hot_maps_to_signed_constant(oracle_lib, k):
    """e_i -> (+-1/sqrt(k)) with sign (-1)^popcount(i&j): row i of Sylvester's H, normalised."""
    c = oracle.norm_const(k)
    for i in (0, 1, k // 2 - 1, k - 1, 5 % k):
        x = np.zeros((1, k), dtype=np.float32)
        x[0, i] = 1.0
        y = oracle.rotate(x, 1, k)[0]
        signs = np.array([(-1) ** bin(i & j).count("1") for j in range(k)], dtype=np.float32)
        np.testing.assert_array_equal(y, signs * c)


@pytest.mark.parametrize("k", KS)
def test_orthogonality_exact(oracle_lib, k):
    """Rows of the unnormalised transform of the identity give H; H H^T = k I exactly."""
    H = np.stack([oracle.fwht_block(np.eye(k, dtype=np.float32)[i]) for i in range(k)])
    np.testing.assert_array_equal(H @ H.T, k * np.eye(k, dtype=np.float32))
    # the normalised rotation is orthonormal to fp32 rounding of 1/sqrt(k)
    Q = oracle.rotate(np.eye(k, dtype=np.float32), 1, k).astype(np.float64)
    np.testing.assert_allclose(Q @ Q.T, np.eye(k), atol=4e-7)


@pytest.mark.parametrize("k", KS)
def test_involution(oracle_lib, k):
    x = _ints(k, 7)
    np.testing.assert_array_equal(oracle.fwht_block(oracle.fwht_block(x)), k * x)


@pytest.mark.parametrize("k", KS)
def test_norm_const_is_nearest_fp32(oracle_lib, k):
    c = float(oracle.norm_const(k))
    exact = 1.0 / math.sqrt(k)
    # nearest fp32: its distance to 1/sqrt(k) is below half an fp32 ulp
    ulp = np.spacing(np.float32(c))
    assert abs(c - exact) <= 0.5 * float(ulp) * (1 + 1e-9)
    if k in (16, 64, 256):
        assert c == {16: 0.25, 64: 0.125, 256: 0.0625}[k]


@pytest.mark.parametrize("k", (16, 64))
def test_rotation_is_block_diagonal(oracle_lib, k):
    """Changing one input block changes only that block of the output."""
    x = synthetic.tiny_random((3, 4 * k), 1)
    y0 = oracle.rotate(x, 1, k)
    x2 = x.copy()
    x2[1, 2 * k:3 * k] += 1.0
    y1 = oracle.rotate(x2, 1, k)
    diff = y0 != y1
    assert diff[1, 2 * k:3 * k].any()
    diff[1, 2 * k:3 * k] = False
    assert not diff.any()


@pytest.mark.parametrize("k", (16, 128))
def test_rotate_rows_equals_rotate_cols_of_transpose(oracle_lib, k):
    x = synthetic.tiny_random((2 * k, 48), 2)
    np.testing.assert_array_equal(oracle.rotate(x, 0, k), oracle.rotate(np.ascontiguousarray(x.T), 1, k))


@pytest.mark.parametrize("k", KS)
def test_rotation_close_to_fp64_dense(oracle_lib, k):
    """fp32 butterflies vs fp64 dense H/sqrt(k): error within log2(k) fp32 roundings."""
    x = synthetic.tiny_random((4, 2 * k), 3)
    H = scipy.linalg.hadamard(k).astype(np.float64) / math.sqrt(k)
    want = np.concatenate([x[:, :k].astype(np.float64) @ H, x[:, k:].astype(np.float64) @ H], 1)
    got = oracle.rotate(x, 1, k)
    bound = (math.log2(k) + 2) * 2.0 ** -24 * np.abs(x).sum(1, keepdims=True) / math.sqrt(k)
    assert (np.abs(got - want) <= bound).all()


@pytest.mark.parametrize("k", (16, 32, 256))
def test_product_preserved(oracle_lib, k):
    """(X H)(W H)^T = X W^T: exact with integer inputs (unnormalised, k X W^T), and to fp32
    rounding after normalisation."""
    X = _ints((6, 2 * k), 11, -4, 4)
    W = _ints((5, 2 * k), 12, -4, 4)
    def unnorm(A):
        return np.concatenate([np.stack([oracle.fwht_block(r[b:b + k]) for r in A])
                               for b in range(0, A.shape[1], k)], 1)
    np.testing.assert_array_equal(unnorm(X).astype(np.int64) @ unnorm(W).astype(np.int64).T,
                                  k * (X.astype(np.int64) @ W.astype(np.int64).T))
    Xf = synthetic.tiny_random((6, 2 * k), 13)
    Wf = synthetic.tiny_random((5, 2 * k), 14)
    got = oracle.rotate(Xf, 1, k).astype(np.float64) @ oracle.rotate(Wf, 1, k).astype(np.float64).T
    want = Xf.astype(np.float64) @ Wf.astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5 * np.abs(want).max())


# ------------------------------------------------------------- randomized Hadamard (H_k D)

def _flags(n, seed):
    return np.random.default_rng(seed).integers(0, 2, size=n).astype(np.uint8)


@pytest.mark.parametrize("k", (16, 64, 256))
def test_signed_rotation_equals_dense_h_times_d(oracle_lib, k):
    """Integer inputs: the unnormalised signed rotation is exact, so rotate * sqrt(k) equals
    the dense integer product (x * s) H_k block by block, with s = 1 - 2 * neg."""
    x = _ints((3, 2 * k), 21, -8, 8)
    neg = _flags(2 * k, 22)
    s = 1 - 2 * neg.astype(np.int64)
    H = scipy.linalg.hadamard(k).astype(np.int64)
    xs = x.astype(np.int64) * s
    want = np.concatenate([xs[:, :k] @ H, xs[:, k:] @ H], 1)
    got = oracle.rotate(x, 1, k, neg=neg).astype(np.float64) / float(oracle.norm_const(k))
    np.testing.assert_allclose(got, want, rtol=2 ** -22, atol=0)


@pytest.mark.parametrize("k", (16, 128))
def test_signed_rotation_plain_and_all_negated(oracle_lib, k):
    """No flags is the plain rotation; flipping every position negates the result (H is
    linear, negation exact); the strided rotation uses the flags of its own positions."""
    x = synthetic.tiny_random((2 * k, 3 * k), 23)
    np.testing.assert_array_equal(oracle.rotate(x, 1, k, neg=np.zeros(3 * k)), oracle.rotate(x, 1, k))
    np.testing.assert_array_equal(oracle.rotate(x, 1, k, neg=np.ones(3 * k)), -oracle.rotate(x, 1, k))
    neg = _flags(2 * k, 24)
    np.testing.assert_array_equal(oracle.rotate(x, 0, k, neg=neg),
                                  oracle.rotate(np.ascontiguousarray(x.T), 1, k, neg=neg))


@pytest.mark.parametrize("k", (32, 256))
def test_signed_product_preserved(oracle_lib, k):
    """(X D H)(W D H)^T = X D D W^T = X W^T: exact for integer inputs (unnormalised,
    k X W^T), to fp32 rounding otherwise; with different signs on the two operands it is not."""
    neg = _flags(2 * k, 25)
    s = (1 - 2 * neg.astype(np.int64))
    X = _ints((6, 2 * k), 26, -4, 4)
    W = _ints((5, 2 * k), 27, -4, 4)
    def unnorm(A):
        As = (A.astype(np.int64) * s).astype(np.float32)
        return np.concatenate([np.stack([oracle.fwht_block(r[b:b + k]) for r in As])
                               for b in range(0, A.shape[1], k)], 1)
    np.testing.assert_array_equal(unnorm(X).astype(np.int64) @ unnorm(W).astype(np.int64).T,
                                  k * (X.astype(np.int64) @ W.astype(np.int64).T))
    Xf = synthetic.tiny_random((6, 2 * k), 28)
    Wf = synthetic.tiny_random((5, 2 * k), 29)
    got = oracle.rotate(Xf, 1, k, neg=neg).astype(np.float64) @ oracle.rotate(Wf, 1, k, neg=neg).astype(np.float64).T
    want = Xf.astype(np.float64) @ Wf.astype(np.float64).T
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-5 * np.abs(want).max())
    other = oracle.rotate(Wf, 1, k, neg=_flags(2 * k, 30)).astype(np.float64)
    assert np.abs(oracle.rotate(Xf, 1, k, neg=neg).astype(np.float64) @ other.T - want).max() > 1e-2 * np.abs(want).max()


def test_signed_quantize_matches_rotate_then_quantize(oracle_lib):
    x = synthetic.tiny_random((64, 128), 31)
    x[:, 5] *= 40.0
    neg = _flags(128, 32)
    for fmt in (oracle.INT8, oracle.FP8_E4M3):
        codes, scale = oracle.quantize(x, 1, 64, fmt, neg=neg)
        c2, s2 = oracle.quantize_rotated(oracle.rotate(x, 1, 64, neg=neg), fmt)
        np.testing.assert_array_equal(codes, c2)
        assert scale == s2
    with pytest.raises(ValueError):
        oracle.quantize(x, 1, 64, oracle.INT8, neg=np.zeros(64))


def test_rotate_rejects_bad_shapes(oracle_lib):
    with pytest.raises(oracle.OracleError):
        oracle.rotate(np.zeros((3, 24), np.float32), 1, 16)
    with pytest.raises(oracle.OracleError):
        oracle.rotate(np.zeros((3, 32), np.float32), 1, 8)


def test_bf16_source_widening(oracle_lib):
    x = synthetic.tiny_random((2, 32), 4)
    bits = synthetic.to_bf16_bits(x)
    widened = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(oracle.rotate(bits, 1, 16), oracle.rotate(widened, 1, 16))


# ------------------------------------------------------------------------- INT8 quantizer

def test_int8_quantizer_brute_force(oracle_lib):
    """Codes = clamp(round-half-even(fp32(y * fp32(127/a)))) with Python's round (RNE)."""
    y = synthetic.tiny_random((64, 64), 5, scale=3.0)
    codes, s = oracle.quantize_rotated(y, oracle.INT8)
    a = np.float32(np.abs(y).max())
    inv = np.float32(127.0) / a
    assert s == np.float32(a / np.float32(127.0))
    z = (y * inv).astype(np.float32)
    want = np.array([max(-127, min(127, round(float(v)))) for v in z.ravel()]).reshape(y.shape)
    np.testing.assert_array_equal(codes.view(np.int8), want)
    q = codes.view(np.int8)
    assert q.min() >= -127 and q.max() <= 127
    i = np.unravel_index(np.abs(y).argmax(), y.shape)
    assert abs(int(q[i])) == 127
    # round trip within half a step (plus fp32 slack on the scale)
    err = np.abs(y.astype(np.float64) - q.astype(np.float64) * float(s))
    assert err.max() <= 0.5 * float(s) * (1 + 1e-5)


def test_int8_ties_to_even(oracle_lib):
    y = np.array([[127.0, 2.5, 3.5, -2.5, -3.5, 0.5, -0.5, 1.5]], dtype=np.float32)
    codes, s = oracle.quantize_rotated(y, oracle.INT8)
    assert s == 1.0
    np.testing.assert_array_equal(codes.view(np.int8)[0], [127, 2, 4, -2, -4, 0, 0, 2])


def test_quantize_zero_and_nonfinite(oracle_lib):
    codes, s = oracle.quantize_rotated(np.zeros((4, 16), np.float32), oracle.INT8)
    assert s == 1.0 and not codes.any()
    codes, s = oracle.quantize(np.zeros((4, 16), np.float32), 1, 16, oracle.FP8_E4M3)
    assert s == 1.0 and not codes.any()
    for bad in (np.nan, np.inf, -np.inf):
        x = np.ones((2, 16), np.float32)
        x[1, 3] = bad
        with pytest.raises(oracle.OracleError) as e:
            oracle.quantize(x, 1, 16, oracle.INT8)
        assert e.value.status == oracle.ERR_NONFINITE


def test_quantize_single_outlier(oracle_lib):
    """One huge entry: after the rotation its block carries +-v/sqrt(k) everywhere, so the
    scale is v/sqrt(k)/127 and the outlier's block saturates to +-127 codes."""
    k = 16
    x = np.zeros((2, 64), np.float32)
    x[0, 20] = 1000.0
    codes, s = oracle.quantize(x, 1, k, oracle.INT8)
    assert s == np.float32(np.float32(1000.0 * 0.25) / np.float32(127))
    q = codes.view(np.int8)
    assert (np.abs(q[0, 16:32]) == 127).all()
    assert not q[0, :16].any() and not q[0, 32:].any() and not q[1].any()


# ------------------------------------------------------------------------- e4m3

def test_e4m3_spec_points(oracle_lib):
    for line in open(os.path.join(GOLDEN, "e4m3_points.txt")):
        if line.startswith("#") or not line.strip():
            continue
        code_s, val_s = line.split()
        code, val = int(code_s, 16), float(val_s)
        got = oracle.e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1, got) == math.copysign(1, val)
            assert oracle.e4m3_encode(val) == code


def test_e4m3_table_matches_torch(oracle_lib):
    table = oracle.e4m3_table()
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    np.testing.assert_array_equal(np.isnan(table), np.isnan(ref))
    ok = ~np.isnan(ref)
    np.testing.assert_array_equal(table[ok], ref[ok])


def test_e4m3_roundtrip_all_codes(oracle_lib):
    for c in range(256):
        if c in (0x7F, 0xFF):
            continue
        assert oracle.e4m3_encode(oracle.e4m3_decode(c)) == c


def _nearest_even_bruteforce(x, table):
    finite = [(c, table[c]) for c in range(128) if not math.isnan(table[c])]
    a = abs(x)
    if a >= 448:
        best = 0x7E
    else:
        d = [(abs(a - v), c) for c, v in finite]
        m = min(d)[0]
        cands = [c for dd, c in d if dd == m]
        best = min(cands) if len(cands) == 1 else [c for c in cands if c % 2 == 0][0]
    sign = 0x80 if (x < 0 or (x == 0 and math.copysign(1, x) < 0)) else 0
    return best | sign


def test_e4m3_encode_bruteforce_and_ties(oracle_lib):
    table = oracle.e4m3_table()
    vals = list(np.random.default_rng(9).uniform(-500, 500, 400).astype(np.float32))
    vals += list((np.random.default_rng(10).standard_normal(400) * 0.05).astype(np.float32))
    finite = sorted(v for v in table[:127] if not math.isnan(v))
    vals += [np.float32((finite[i] + finite[i + 1]) / 2) for i in range(len(finite) - 1)]
    vals += [np.float32(-v) for v in vals[-20:]]
    for v in vals:
        assert oracle.e4m3_encode(float(v)) == _nearest_even_bruteforce(float(v), table), v


def test_e4m3_encode_matches_torch_in_range(oracle_lib):
    v = np.random.default_rng(11).uniform(-448, 448, 20000).astype(np.float32)
    v[:200] *= 1e-4
    ref = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(float(x)) for x in v], dtype=np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_saturates(oracle_lib):
    for x, c in ((449.0, 0x7E), (464.0, 0x7E), (1e30, 0x7E), (-1e30, 0xFE), (-460.0, 0xFE)):
        assert oracle.e4m3_encode(x) == c


def test_fp8_quantizer_absmax_maps_to_448(oracle_lib):
    y = synthetic.tiny_random((32, 32), 6, scale=2.0)
    codes, s = oracle.quantize_rotated(y, oracle.FP8_E4M3)
    a = np.float32(np.abs(y).max())
    assert s == np.float32(a / np.float32(448.0))
    i = np.unravel_index(np.abs(y).argmax(), y.shape)
    assert codes[i] & 0x7F == 0x7E
    table = oracle.e4m3_table()
    dec = table[codes] * float(s)
    rel = np.abs(dec - y) / np.maximum(np.abs(y), 2 ** -6 * float(s))
    assert rel.max() <= 2 ** -4 * (1 + 1e-6)   # half of e4m3's 2^-3 relative spacing


# ------------------------------------------------------------------------- FP6 / FP4

# (fmt, exponent bits, mantissa bits): the minifloats below FP8 that HALO names (FP6) plus
# FP4; sign-magnitude with subnormals and no infinities or NaN.
MINIS = [(oracle.FP6_E3M2, 3, 2), (oracle.FP6_E2M3, 2, 3), (oracle.FP4_E2M1, 2, 1)]


def _mini_table(fmt):
    return [oracle.minifloat_decode(fmt, c) for c in range(1 << oracle.minifloat_bits(fmt))]


@pytest.mark.parametrize("fmt,eb,mb", MINIS)
def test_minifloat_value_structure(oracle_lib, fmt, eb, mb):
    """Positive codes decode strictly increasing from 0; the sign bit negates; the spacing is
    constant within each binade of 2^mb values and doubles from one binade to the next (the
    subnormals share the first normal binade's spacing)."""
    t = _mini_table(fmt)
    half = len(t) // 2
    pos = t[:half]
    assert pos[0] == 0.0 and all(b > a for a, b in zip(pos, pos[1:]))
    for c in range(half):
        assert t[c + half] == -t[c]
    steps = [b - a for a, b in zip(pos, pos[1:])]
    n = 1 << mb
    for i, st in enumerate(steps):  # step from code i to i + 1
        assert st == steps[0] * 2 ** max(0, i // n - 1), (fmt, i)
    assert oracle.minifloat_max(fmt) == pos[-1]


def test_minifloat_spec_points(oracle_lib):
    """Closed forms: e2m1 is exactly {0, 0.5, 1, 1.5, 2, 3, 4, 6}; e2m3 tops out at 7.5 with
    smallest subnormal 1/8; e3m2 tops out at 28 with smallest subnormal 1/16."""
    assert _mini_table(oracle.FP4_E2M1)[:8] == [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    t = _mini_table(oracle.FP6_E2M3)
    assert (t[1], t[31], t[8]) == (0.125, 7.5, 1.0)
    t = _mini_table(oracle.FP6_E3M2)
    assert (t[1], t[31], t[4]) == (0.0625, 28.0, 0.25)


def _mini_nearest_even(x, fmt):
    t = _mini_table(fmt)
    half = len(t) // 2
    a = abs(x)
    best = min(range(half), key=lambda c: abs(t[c] - a))
    d = abs(t[best] - a)
    ties = [c for c in range(half) if abs(t[c] - a) == d]
    if len(ties) > 1:
        best = [c for c in ties if c % 2 == 0][0]
    if a > t[half - 1]:
        best = half - 1
    sign = half if (x < 0 or (x == 0 and math.copysign(1, x) < 0)) else 0
    return best | sign


@pytest.mark.parametrize("fmt,eb,mb", MINIS)
def test_minifloat_encode_bruteforce_and_ties(oracle_lib, fmt, eb, mb):
    """Encode = brute-force nearest over every code, ties to the even code, at every code
    value, every midpoint (exact ties), just beside each midpoint, random values and beyond
    the maximum (saturation)."""
    t = _mini_table(fmt)
    pos = t[: len(t) // 2]
    vals = list(pos) + [(a + b) / 2 for a, b in zip(pos, pos[1:])]
    vals += [np.nextafter(np.float32(v), np.float32(100)) for v in vals] + [np.nextafter(np.float32(v), np.float32(-1)) for v in vals]
    mx = pos[-1]
    vals += list(np.random.default_rng(41).uniform(0, 1.3 * mx, 300).astype(np.float32)) + [mx * 1.01, mx * 5, 1e30]
    vals = [float(np.float32(v)) for v in vals]
    vals += [-v for v in vals] + [-0.0]
    for v in vals:
        assert oracle.minifloat_encode(fmt, v) == _mini_nearest_even(v, fmt), (fmt, v)


@pytest.mark.parametrize("fmt,eb,mb", MINIS)
def test_minifloat_quantizer_absmax_and_roundtrip(oracle_lib, fmt, eb, mb):
    """The absmax element maps to the largest code; every element decodes back to within half
    a step of its binade (relative 2^-(mb+1), or the subnormal step near zero)."""
    y = synthetic.tiny_random((48, 40), 7 + fmt, scale=3.0)
    codes, s = oracle.quantize_rotated(y, fmt)
    mx = np.float32(oracle.minifloat_max(fmt))
    a = np.float32(np.abs(y).max())
    assert s == np.float32(a / mx)
    i = np.unravel_index(np.abs(y).argmax(), y.shape)
    half = 1 << (eb + mb)
    assert codes[i] & (half - 1) == half - 1
    t = np.array(_mini_table(fmt))
    dec = t[codes] * float(s)
    sub_step = t[1] * float(s)
    err = np.abs(dec - y.astype(np.float64))
    bound = np.maximum(np.abs(y) * 2.0 ** -(mb + 1), sub_step / 2) * (1 + 1e-6)
    assert (err <= bound).all()
    assert (codes < 2 * half).all()


@pytest.mark.parametrize("fmt,eb,mb", MINIS)
def test_gemm_minifloat_exact_rational(oracle_lib, fmt, eb, mb):
    r = np.random.default_rng(43 + fmt)
    n = 1 << oracle.minifloat_bits(fmt)
    A = r.integers(0, n, size=(4, 40)).astype(np.uint8)
    B = r.integers(0, n, size=(3, 40)).astype(np.uint8)
    t = _mini_table(fmt)
    C = oracle.gemm(A, B, fmt)
    for i in range(4):
        for j in range(3):
            exact = sum(Fraction(t[A[i, l]]) * Fraction(t[B[j, l]]) for l in range(40))
            assert Fraction(C[i, j]) == exact


# ------------------------------------------------------------------------- GEMMs

def test_gemm_i8_triple_loop_and_numpy(oracle_lib):
    r = np.random.default_rng(12)
    A = r.integers(-127, 128, size=(5, 48)).astype(np.int8)
    B = r.integers(-127, 128, size=(7, 48)).astype(np.int8)
    C = oracle.gemm(A.view(np.uint8), B.view(np.uint8), oracle.INT8)
    loop = [[sum(int(A[i, l]) * int(B[j, l]) for l in range(48)) for j in range(7)] for i in range(5)]
    np.testing.assert_array_equal(C, np.array(loop))
    big_A = r.integers(-127, 128, size=(33, 300)).astype(np.int8)
    big_B = r.integers(-127, 128, size=(17, 300)).astype(np.int8)
    np.testing.assert_array_equal(oracle.gemm(big_A.view(np.uint8), big_B.view(np.uint8), oracle.INT8),
                                  big_A.astype(np.int64) @ big_B.astype(np.int64).T)
    rows = np.array([32, 0, 5])
    np.testing.assert_array_equal(oracle.gemm(big_A.view(np.uint8), big_B.view(np.uint8), oracle.INT8, rows),
                                  (big_A.astype(np.int64) @ big_B.astype(np.int64).T)[rows])


def test_gemm_f8_exact_rational(oracle_lib):
    r = np.random.default_rng(13)
    finite = [c for c in range(256) if c not in (0x7F, 0xFF)]
    A = r.choice(finite, size=(4, 40)).astype(np.uint8)
    B = r.choice(finite, size=(3, 40)).astype(np.uint8)
    table = oracle.e4m3_table()
    C = oracle.gemm(A, B, oracle.FP8_E4M3)
    for i in range(4):
        for j in range(3):
            exact = sum(Fraction(table[A[i, l]]) * Fraction(table[B[j, l]]) for l in range(40))
            assert Fraction(C[i, j]) == exact


# ------------------------------------------------------------------------- epilogue and bf16

def test_bf16_rounding_matches_torch(oracle_lib):
    v = np.random.default_rng(14).standard_normal(4000).astype(np.float32) * 100
    # exact ties: bf16 value + half a bf16 ulp
    b = torch.from_numpy(v[:500]).to(torch.bfloat16).float().numpy()
    ties = (b + np.spacing(b.astype(np.float32)) * 2 ** 15).astype(np.float32)
    v = np.concatenate([v, ties])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.bf16_from_f32(float(x)) for x in v], dtype=np.uint16)
    np.testing.assert_array_equal(got, ref)


def _bf16_exact(fr: Fraction) -> int:
    """Nearest-even bf16 of an exact rational, by search over neighbouring bf16 values."""
    f = float(fr)
    base = int(torch.tensor([f], dtype=torch.float32).to(torch.bfloat16).view(torch.int16).item()) & 0xFFFF
    cands = [(base + d) & 0xFFFF for d in (-1, 0, 1)]
    vals = [Fraction(float(oracle.bf16_bits_to_f32(np.array([c]))[0])) for c in cands]
    dist = [abs(v - fr) for v in vals]
    m = min(dist)
    best = [c for c, d in zip(cands, dist) if d == m]
    return best[0] if len(best) == 1 else [c for c in best if c % 2 == 0][0]


def test_epilogue_ref_and_fast(oracle_lib):
    r = np.random.default_rng(15)
    acc = r.integers(-2 ** 30, 2 ** 30, size=300).astype(np.int32)
    sa, sb = np.float32(0.0123), np.float32(3.7e-4)
    ref, fast = oracle.epilogue(acc, sa, sb)
    # fast formula == torch CPU fp32 ops in the same order
    t = (torch.from_numpy(acc).float() * (torch.tensor(sa) * torch.tensor(sb))).to(torch.bfloat16)
    np.testing.assert_array_equal(fast, t.view(torch.int16).numpy().view(np.uint16))
    for i in range(0, 300, 7):
        assert ref[i] == _bf16_exact(Fraction(int(acc[i])) * Fraction(float(sa)) * Fraction(float(sb)))
    diff = np.abs(oracle.bf16_bits_to_f32(ref).astype(np.float64) - oracle.bf16_bits_to_f32(fast))
    ulp = np.abs(oracle.bf16_bits_to_f32(ref)).astype(np.float64) * 2 ** -7
    assert (diff <= ulp).all()


# ------------------------------------------------------------------------- the layer

def _rel_fro(a, b):
    return np.linalg.norm(a - b) / np.linalg.norm(b)


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3))
def test_layer_wiring_tracks_unquantized_products(oracle_lib, fmt):
    """Each GEMM's dequantized output approximates its unquantized product; a wrong rotation
    dimension (transform not on the contraction) or a transposed operand breaks this: such
    mistakes give relative errors above 1, the correct wiring stays below 0.1 here (dW is
    the loosest: its contraction is only 64 tokens and X's outlier columns are not spread by
    a rotation along tokens)."""
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw(w)
    X, W, dY = (d[n].astype(np.float64) for n in ("X", "W", "dY"))
    k = w.k
    f = oracle.bf16_bits_to_f32
    tol = 0.1
    Y = oracle.linear_fwd(d["X"], d["W"], k, fmt)
    assert _rel_fro(f(Y["ref"]), X @ W.T) < tol
    dX = oracle.linear_bwd_dx(d["dY"], d["W"], k, fmt)
    assert _rel_fro(f(dX["ref"]), dY @ W) < tol
    dW = oracle.linear_bwd_dw(d["dY"], d["X"], k, fmt)
    assert _rel_fro(f(dW["ref"]), dY.T @ X) < tol
    assert Y["ref"].shape == (64, 128) and dX["ref"].shape == (64, 256) and dW["ref"].shape == (128, 256)


def test_hadamard_reduces_error_on_outliers(oracle_lib):
    """The method's premise (4-bit page section 3.2/3.3): on inputs with outlier channels the
    rotated INT8 product is more accurate than quantizing without rotation (k=1 reading)."""
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw(w)
    X, W = d["X"], d["W"]
    want = X.astype(np.float64) @ W.astype(np.float64).T
    rot = oracle.linear_fwd(X, W, 16, oracle.INT8)
    f = oracle.bf16_bits_to_f32
    qx, sx = oracle.quantize_rotated(X, oracle.INT8)
    qw, sw = oracle.quantize_rotated(W, oracle.INT8)
    plain_ref, _ = oracle.epilogue(oracle.gemm(qx, qw, oracle.INT8), sx, sw)
    assert _rel_fro(f(rot["ref"]), want) < 0.5 * _rel_fro(f(plain_ref), want)


# ------------------------------------------------------------------------- inputs

def test_synthetic_prefix_and_reproducible():
    w = synthetic.WORKLOADS[4]
    full = synthetic.draw_fp32(w, 0, M=64)
    part = synthetic.draw_fp32(w, 0, M=16)
    for n in ("X", "dY"):
        np.testing.assert_array_equal(full[n][:16], part[n])
    np.testing.assert_array_equal(full["W"], part["W"])
    again = synthetic.draw_fp32(w, 0, M=64)
    np.testing.assert_array_equal(full["X"], again["X"])
    assert len(full["outlier_cols"]) == 4   # 0.5% of 768
    assert len(synthetic.draw_fp32(w, 1, M=4)["outlier_cols"]) == 15   # 0.5% of 3072
    assert len(synthetic.draw_fp32(synthetic.WORKLOADS[1])["outlier_cols"]) == 4


def test_signed_layer_wiring(oracle_lib):
    """The layer with sign flags over each contraction dimension still tracks the unquantized
    product (the same D on both operands cancels); giving the two operands different flags
    does not."""
    from hadamard_rotated_precision_b200 import synthetic
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw_fp32(w)
    X, W, dY = d["X"].astype(np.float64), d["W"].astype(np.float64), d["dY"].astype(np.float64)
    k = w.k
    for name, fn, a, b, want, n in (("fwd", oracle.linear_fwd, d["X"], d["W"], X @ W.T, X.shape[1]),
                                    ("dx", oracle.linear_bwd_dx, d["dY"], d["W"], dY @ W, W.shape[0]),
                                    ("dw", oracle.linear_bwd_dw, d["dY"], d["X"], dY.T @ X, X.shape[0])):
        neg = synthetic.sign_flags(n, 3)
        got = oracle.bf16_bits_to_f32(fn(a, b, k, oracle.INT8, neg=neg)["ref"]).astype(np.float64)
        assert np.linalg.norm(got - want) / np.linalg.norm(want) < 0.1, name
    neg = synthetic.sign_flags(X.shape[1], 3)
    qa, sa = oracle.quantize(d["X"], 1, k, oracle.INT8, neg=neg)
    qb, sb = oracle.quantize(d["W"], 1, k, oracle.INT8, neg=1 - neg)
    acc = oracle.gemm(qa, qb, oracle.INT8).astype(np.float64) * float(sa) * float(sb)
    assert np.linalg.norm(acc - X @ W.T) / np.linalg.norm(X @ W.T) > 0.5


# ------------------------------------------------- rotated-output placement (forward codes reused)

def _blockdiag_h(n, k):
    """fp64 blockdiag(H_k) of size n (scipy's Sylvester construction), unnormalised."""
    return scipy.linalg.block_diag(*([scipy.linalg.hadamard(k).astype(np.float64)] * (n // k)))


@pytest.mark.parametrize("k", KS)
def test_derotate_output_one_hot_closed_form(oracle_lib, k):
    """E_ij -> c^2 h_i h_j^T on the (row block of i) x (column block of j): every butterfly is
    exact for a one-hot input, so the value is fp32(c * c) with the Sylvester sign
    (-1)^(popcount(i' & a) + popcount(j' & b)), zero outside the two blocks."""
    c = oracle.norm_const(k)
    mag = np.float32(c) * np.float32(c)
    H = scipy.linalg.hadamard(k)
    for (i, j) in ((0, 0), (k + 3 % k, 1), (2 * k - 1, k // 2), (5 % k, 2 * k - 1)):
        Z = np.zeros((2 * k, 3 * k), dtype=np.float32)
        Z[i, j] = 1.0
        got = oracle.derotate_output(Z, k)
        want = np.zeros_like(Z)
        r0, c0 = (i // k) * k, (j // k) * k
        want[r0:r0 + k, c0:c0 + k] = mag * np.outer(H[i % k], H[j % k]).astype(np.float32)
        np.testing.assert_array_equal(got, want)


@pytest.mark.parametrize("k", KS)
def test_derotate_output_close_to_dense(oracle_lib, k):
    """Against the fp64 product H Z H / k with scipy's block-diagonal Hadamard matrices: equal
    up to fp32 rounding of log2(k) butterfly stages per side."""
    rng = np.random.default_rng(k)
    Z = rng.standard_normal((2 * k, 3 * k)).astype(np.float32)
    want = _blockdiag_h(2 * k, k) @ Z.astype(np.float64) @ _blockdiag_h(3 * k, k) / k
    got = oracle.derotate_output(Z, k).astype(np.float64)
    assert np.abs(got - want).max() < 1e-4


@pytest.mark.parametrize("k", (16, 128))
def test_derotate_output_involution(oracle_lib, k):
    rng = np.random.default_rng(7)
    Z = rng.standard_normal((k, 2 * k)).astype(np.float32)
    back = oracle.derotate_output(oracle.derotate_output(Z, k), k)
    assert np.abs(back - Z).max() < 1e-5


def test_dequant_f32_and_bf16_rounding(oracle_lib):
    """dequant_f32 is the fp32 product with the fp32 product of the scales (numpy's IEEE
    single arithmetic), f32_to_bf16 agrees with torch's round-to-nearest-even conversion."""
    rng = np.random.default_rng(3)
    acc = rng.integers(-2**24, 2**24, size=1000).astype(np.int32)
    sa, sb = np.float32(0.0123), np.float32(3.7e-3)
    np.testing.assert_array_equal(oracle.dequant_f32(acc, sa, sb), acc.astype(np.float32) * (sa * sb))
    x = (rng.standard_normal(4096) * 10.0 ** rng.integers(-30, 30, 4096)).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.f32_to_bf16(x), want)


def _reuse_case(fmt):
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw(w)
    k = w.k
    wq, sw = oracle.quantize(d["W"], 1, k, fmt)    # forward's W codes, rotated along K
    xq, sx = oracle.quantize(d["X"], 0, k, fmt)    # saved X codes, rotated along M
    return w, d, k, wq, sw, xq, sx


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3))
def test_reuse_backward_tracks_unquantized_products(oracle_lib, fmt):
    """dX from dY's token-rotated codes and the forward's K-rotated weight codes approximates
    dY W once both rotations are undone on the output; leaving out either de-rotation (a
    mistake planted here, on the CPU) or transposing the weight codes gives errors near 1."""
    w, d, k, wq, sw, xq, sx = _reuse_case(fmt)
    X, W, dY = (d[n].astype(np.float64) for n in ("X", "W", "dY"))
    f = oracle.bf16_bits_to_f32
    r = oracle.linear_bwd_reuse(d["dY"], xq, sx, wq, sw, k, fmt)
    assert r["dx"].shape == (64, 256) and r["dw"].shape == (128, 256)
    assert _rel_fro(f(r["dx"]), dY @ W) < 0.1
    assert _rel_fro(f(r["dw"]), dY.T @ X) < 0.1
    acc = oracle.gemm(np.ascontiguousarray(r["g"].T), np.ascontiguousarray(wq.T), fmt)
    z = oracle.dequant_f32(acc, r["s_g"], sw)
    only_cols = oracle.rotate(z, 1, k)
    only_rows = np.ascontiguousarray(oracle.rotate(z, 0, k).T)
    for bad in (z, only_cols, only_rows):
        assert _rel_fro(bad.astype(np.float64), dY @ W) > 0.5
    wrong = oracle.linear_bwd_dx_reuse(r["g"], r["s_g"], np.ascontiguousarray(np.flip(wq, 0)), sw, k, fmt)
    assert _rel_fro(f(wrong["out"]), dY @ W) > 0.5


def test_reuse_dw_is_the_standard_dw(oracle_lib):
    """The reuse placement's dW is the HALO-2 dW: same dY codes along M, same X codes."""
    w, d, k, wq, sw, xq, sx = _reuse_case(oracle.INT8)
    r = oracle.linear_bwd_reuse(d["dY"], xq, sx, wq, sw, k, oracle.INT8)
    np.testing.assert_array_equal(r["dw"], oracle.linear_bwd_dw(d["dY"], d["X"], k, oracle.INT8)["fast"])


def test_reuse_dx_row_block_sampling(oracle_lib):
    """Sampling whole k-row blocks gives exactly those rows of the full result."""
    w, d, k, wq, sw, xq, sx = _reuse_case(oracle.INT8)
    r = oracle.linear_bwd_reuse(d["dY"], xq, sx, wq, sw, k, oracle.INT8)
    part = oracle.linear_bwd_dx_reuse(r["g"], r["s_g"], wq, sw, k, oracle.INT8, rows=[2 * k, 0])
    np.testing.assert_array_equal(part["out"], np.concatenate([r["dx"][2 * k:3 * k], r["dx"][:k]]))


# ------------------------------------------------- next layer's rotation in the GEMM's epilogue

@pytest.mark.parametrize("k", (16, 128))
def test_gemm_rotout_close_to_dense(oracle_lib, k):
    """The dequantized product rotated along its columns equals the fp64 dense product
    (A B^T s_a s_b) blockdiag(H_k) / sqrt(k) up to fp32 rounding."""
    rng = np.random.default_rng(k)
    A = rng.integers(-127, 128, size=(48, 96)).astype(np.int8).view(np.uint8)
    B = rng.integers(-127, 128, size=(2 * k, 96)).astype(np.int8).view(np.uint8)
    sa, sb = np.float32(0.013), np.float32(0.0021)
    want = (A.view(np.int8).astype(np.float64) @ B.view(np.int8).astype(np.float64).T) * float(sa * sb)
    want = want @ _blockdiag_h(2 * k, k) / math.sqrt(k)
    got = oracle.gemm_rotout(A, B, sa, sb, oracle.INT8, k).astype(np.float64)
    assert np.abs(got - want).max() <= 1e-5 * np.abs(want).max()


def test_next_layer_flow_tracks_two_layer_product(oracle_lib):
    """Layer 1's output rotated in its epilogue and quantized as it is, times layer 2's weight
    codes rotated along the same dimension, approximates X W1^T W2^T; leaving out the epilogue
    rotation (a planted mistake) does not."""
    w = synthetic.WORKLOADS[1]
    d = synthetic.draw_fp32(w)
    X, W1 = d["X"], d["W"]                                       # [64][256], [128][256]
    W2 = synthetic.tiny_random((96, 128), 4, scale=0.05)          # the next layer, 128 -> 96
    k = 16
    qx, sx = oracle.quantize(X, 1, k, oracle.INT8)
    qw1, sw1 = oracle.quantize(W1, 1, k, oracle.INT8)
    y_rot = oracle.gemm_rotout(qx, qw1, sx, sw1, oracle.INT8, k)   # [64][128], rotated along N
    qy, sy = oracle.quantize_rotated(y_rot, oracle.INT8)
    qw2, sw2 = oracle.quantize(W2, 1, k, oracle.INT8)
    _, fast = oracle.epilogue(oracle.gemm(qy, qw2, oracle.INT8), sy, sw2)
    want = X.astype(np.float64) @ W1.astype(np.float64).T @ W2.astype(np.float64).T
    assert _rel_fro(oracle.bf16_bits_to_f32(fast).astype(np.float64), want) < 0.1
    y_plain = oracle.dequant_f32(oracle.gemm(qx, qw1, oracle.INT8), sx, sw1)
    qp, sp = oracle.quantize_rotated(y_plain, oracle.INT8)
    bad = oracle.gemm(qp, qw2, oracle.INT8).astype(np.float64) * float(sp) * float(sw2)
    assert _rel_fro(bad, want) > 0.5


# ------------------------------------------------------------------ packed minifloat layout

def _lowp_pack_fixture():
    path = os.path.join(os.path.dirname(__file__), "golden", "lowp_pack16.txt")
    out = []
    with open(path) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            bits, codes, chunk = (p.strip() for p in line.split("|"))
            out.append((int(bits), [int(c) for c in codes.split()], bytes(int(b, 16) for b in chunk.split())))
    return out


def test_device_codes_packed_layout_fixture():
    """oracle.device_codes packs FP6 / FP4 codes as the hand-derived chunks of the fixture
    (16 codes per 16-byte chunk, LSB first, zero tail), for every minifloat format of the bit
    width, and leaves INT8 / FP8 codes as they are."""
    cases = _lowp_pack_fixture()
    assert len(cases) == 3
    for bits, codes, chunk in cases:
        fmts = (oracle.FP6_E3M2, oracle.FP6_E2M3) if bits == 6 else (oracle.FP4_E2M1,)
        for fmt in fmts:
            got = oracle.device_codes(np.array([codes], dtype=np.uint8), fmt)
            assert got.shape == (1, 16) and got.tobytes() == chunk, (fmt, got.tobytes().hex())
    x = np.arange(64, dtype=np.uint8).reshape(2, 32)
    for fmt in (oracle.INT8, oracle.FP8_E4M3):
        assert np.array_equal(oracle.device_codes(x, fmt), x)


def test_device_codes_packed_chunk_order():
    """Chunks follow the code groups in order along the rotated dimension and rows stay rows:
    a 2 x 32 array of FP4 codes is four fixture-style chunks, group by group."""
    (_, c6, ch6), _, (_, c4, ch4) = _lowp_pack_fixture()
    rows = np.array([c4 + [0] * 16, [0] * 16 + c4], dtype=np.uint8)
    got = oracle.device_codes(rows, oracle.FP4_E2M1)
    zero = bytes(16)
    assert got[0].tobytes() == ch4 + zero and got[1].tobytes() == zero + ch4
    rows6 = np.array([c6 + c6], dtype=np.uint8)
    assert oracle.device_codes(rows6, oracle.FP6_E2M3)[0].tobytes() == ch6 + ch6
