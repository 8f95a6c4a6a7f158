"""CPU-only checks of the C ABI library: it builds, loads, exports every symbol the header
declares, and rejects bad arguments synchronously (these paths return before any CUDA call,
so no GPU is needed; fake but 16-byte-aligned addresses are never dereferenced)."""
import ctypes
import os
import re

import numpy as np
import pytest

import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hq.h")

FAKE = 0x10000      # aligned, never dereferenced: every call below fails validation first
FAKE_MIS = 0x10002  # misaligned


@pytest.fixture(scope="module")
def L():
    build.build()
    return hq.lib()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"HQ_API\s+[\w\s\*]+?\b(hq_\w+)\s*\(", text)))


def test_exports_every_declared_symbol(L):
    names = header_functions()
    assert len(names) >= 11
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(hq.EXPORTS)


def test_status_strings_and_version(L):
    for s in range(10):
        assert hq.hq_status_string(s)
    assert hq.hq_version() >= 100


def test_workspace_sizes(L):
    q = hq.hq_quantize_workspace_bytes()
    assert q >= 4096 * 4
    M, K, N = 4096, 4096, 11008
    need = hq.hq_linear_workspace_bytes(M, K, N)
    assert need >= max(M * K + N * K, M * N + K * N, N * M + K * M) + q
    assert hq.hq_linear_workspace_bytes(-1, 2, 3) == 0
    # one size for every layer-level call of the shape, whatever the format
    one = hq.hq_workspace_bytes(M, K, N, "int8")
    for f in ("hq_linear_workspace_bytes", "hq_linear_fwd_bwd_workspace_bytes", "hq_linear_fwd_save_workspace_bytes",
              "hq_linear_bwd_workspace_bytes", "hq_linear_fwd_keep_workspace_bytes",
              "hq_linear_bwd_reuse_workspace_bytes", "hq_linear_bwd_dx_reuse_workspace_bytes"):
        assert one >= getattr(L, f)(M, K, N), f
    assert all(hq.hq_workspace_bytes(M, K, N, f) == one for f in ("fp8", "fp6_e3m2", "fp6_e2m3", "fp4_e2m1"))
    assert L.hq_workspace_bytes(M, K, N, 5) == 0 and L.hq_workspace_bytes(-1, K, N, 0) == 0


def test_mma_peak_argument_errors(L):
    assert L.hq_mma_peak(2, 16, None, None) == 1   # FP6: the probe runs INT8 / FP8 only
    assert L.hq_mma_peak(0, 0, None, None) == 1
    assert L.hq_mma_peak(1, (1 << 24) + 1, None, None) == 1


def _q(L, src=FAKE, dt=hq.HQ_BF16, rows=64, cols=256, dim=1, k=16, fmt=0, codes=FAKE, scale=FAKE,
       ws=FAKE, wsb=1 << 20):
    return L.hq_quantize(src, dt, rows, cols, dim, k, fmt, codes, scale, ws, wsb, None)


def test_quantize_argument_errors(L):
    assert _q(L, dt=7) == 3
    assert _q(L, k=24) == 1
    assert _q(L, k=512) == 1
    assert _q(L, dim=2) == 1
    assert _q(L, fmt=5) == 1
    assert _q(L, fmt=-1) == 1
    for f in (2, 3, 4):  # FP6 e3m2 / e2m3 and FP4 e2m1 pass the format check: a misaligned
        assert _q(L, fmt=f, codes=FAKE_MIS) == 4  # codes pointer is what fails (no launch)
    assert _q(L, rows=-1) == 1
    assert _q(L, scale=None) == 1
    assert _q(L, src=None) == 1
    assert _q(L, cols=250) == 2                      # not a multiple of k along dim 1
    assert _q(L, dim=0, rows=60) == 2                # not a multiple of k along dim 0
    assert _q(L, dim=0, rows=64, cols=24) == 2       # other dim not a multiple of 16
    assert _q(L, src=FAKE_MIS) == 4
    assert _q(L, codes=FAKE_MIS) == 4
    assert _q(L, ws=None) == 8
    assert _q(L, wsb=16) == 8
    assert _q(L, ws=FAKE_MIS) == 4


def _g(L, A=FAKE, sa=FAKE, B=FAKE, sb=FAKE, M=128, N=256, K=128, fmt=0, out_kind=0, out=FAKE):
    return L.hq_gemm(A, sa, B, sb, M, N, K, fmt, out_kind, out, None)


def test_gemm_argument_errors(L):
    assert _g(L, fmt=6) == 1
    assert _g(L, out_kind=2) == 1
    assert _g(L, M=-1) == 1
    assert _g(L, out=None) == 1
    assert _g(L, A=None) == 1
    assert _g(L, sa=None) == 1                # bf16 output needs the scales
    assert _g(L, K=40) == 2
    assert _g(L, N=100) == 2
    assert _g(L, K=133152) == 2               # INT8 accumulator bound (127^2 K < 2^31)
    assert _g(L, M=1 << 31) == 2
    assert _g(L, A=FAKE_MIS) == 4
    assert _g(L, out=FAKE_MIS) == 4
    assert _g(L, M=0) == 0                    # empty: nothing to do, no launch
    assert _g(L, N=0) == 0


def _lin(L, name, M=256, K=512, N=256, k=64, dt=hq.HQ_BF16, fmt=0, out=FAKE, ws=FAKE, wsb=1 << 30):
    return getattr(L, name)(FAKE, FAKE, dt, M, K, N, k, fmt, out, ws, wsb, None)


@pytest.mark.parametrize("name", ("hq_linear_fwd", "hq_linear_bwd_dx", "hq_linear_bwd_dw"))
def test_linear_argument_errors(L, name):
    assert _lin(L, name, dt=9) == 3
    assert _lin(L, name, k=8) == 1
    assert _lin(L, name, fmt=5) == 1
    assert _lin(L, name, M=100) == 2
    assert _lin(L, name, K=100) == 2
    assert _lin(L, name, N=100) == 2
    assert _lin(L, name, out=None) == 1
    assert _lin(L, name, out=FAKE_MIS) == 4
    assert _lin(L, name, ws=None) == 8
    assert _lin(L, name, wsb=1024) == 8
    big = 133248  # multiple of 64 above the INT8 contraction bound
    if name == "hq_linear_fwd":
        assert _lin(L, name, K=big) == 2
    elif name == "hq_linear_bwd_dx":
        assert _lin(L, name, N=big) == 2
    else:
        assert _lin(L, name, M=big) == 2


def test_dual_and_step_argument_errors(L):
    q = lambda **kw: L.hq_quantize_dual(kw.get("src", FAKE), kw.get("dt", hq.HQ_BF16), kw.get("rows", 256),
                                        kw.get("cols", 256), kw.get("k", 64), kw.get("fmt", 0),
                                        kw.get("cc", FAKE), kw.get("sc", FAKE), kw.get("cr", FAKE),
                                        kw.get("sr", FAKE), kw.get("ws", FAKE), kw.get("wsb", 1 << 20), None)
    assert q(dt=4) == 3
    assert q(k=48) == 1
    assert q(sr=None) == 1
    assert q(rows=100) == 2
    assert q(cols=96) == 2
    assert q(cr=FAKE_MIS) == 4
    assert q(ws=None) == 8
    assert q(wsb=100) == 8
    assert hq.hq_quantize_dual_workspace_bytes() >= 2 * hq.hq_quantize_workspace_bytes()
    f = lambda **kw: L.hq_linear_fwd_bwd(FAKE, FAKE, FAKE, kw.get("dt", hq.HQ_BF16), kw.get("M", 256),
                                         kw.get("K", 512), kw.get("N", 256), kw.get("k", 64), 0,
                                         kw.get("Y", FAKE), FAKE, FAKE, kw.get("ws", FAKE),
                                         kw.get("wsb", 1 << 34), None)
    assert f(dt=5) == 3
    assert f(k=20) == 1
    assert f(M=100) == 2
    assert f(M=0) == 2
    assert f(Y=None) == 1
    assert f(Y=FAKE_MIS) == 4
    assert f(ws=None) == 8
    assert f(wsb=1000) == 8
    M, K, N = 4096, 4096, 11008
    assert hq.hq_linear_fwd_bwd_workspace_bytes(M, K, N) >= 2 * (M * K + N * K + M * N)


def test_saved_codes_flow_argument_errors(L):
    fs = lambda **kw: L.hq_linear_fwd_save(FAKE, FAKE, kw.get("dt", hq.HQ_BF16), kw.get("M", 256),
                                           kw.get("K", 512), kw.get("N", 256), kw.get("k", 64), 0,
                                           kw.get("Y", FAKE), kw.get("xqt", FAKE), kw.get("sx", FAKE),
                                           kw.get("ws", FAKE), kw.get("wsb", 1 << 34), None)
    assert fs(dt=2) == 3
    assert fs(k=12) == 1
    assert fs(M=96) == 2                     # tokens not a multiple of k: no rotation along M
    assert fs(N=0) == 2
    assert fs(xqt=None) == 1
    assert fs(sx=None) == 1
    assert fs(xqt=FAKE_MIS) == 4
    assert fs(sx=FAKE + 2) == 4
    assert fs(ws=None) == 8
    assert fs(wsb=4096) == 8
    b = lambda **kw: L.hq_linear_bwd(FAKE, FAKE, kw.get("xqt", FAKE), kw.get("sx", FAKE),
                                     kw.get("dt", hq.HQ_BF16), kw.get("M", 256), kw.get("K", 512),
                                     kw.get("N", 256), kw.get("k", 64), kw.get("fmt", 1),
                                     kw.get("dX", FAKE), kw.get("dW", FAKE), kw.get("ws", FAKE),
                                     kw.get("wsb", 1 << 34), None)
    assert b(dt=3) == 3
    assert b(fmt=9) == 1
    assert b(K=80) == 2
    assert b(M=133248, K=128, N=128, fmt=0) == 2   # INT8 contraction bound on the dW GEMM
    assert b(xqt=None) == 1
    assert b(dW=None) == 1
    assert b(dX=FAKE_MIS) == 4
    assert b(ws=None) == 8
    assert b(wsb=4096) == 8
    M, K, N = 4096, 4096, 11008
    assert hq.hq_linear_fwd_save_workspace_bytes(M, K, N) >= M * K + N * K
    assert hq.hq_linear_bwd_workspace_bytes(M, K, N) >= 2 * M * N + K * N
    assert hq.hq_linear_bwd_workspace_bytes(-1, 1, 1) == 0


def test_python_binding_rejects_cpu_tensors(L):
    import torch
    with pytest.raises(TypeError):
        hq.hq_quantize(torch.zeros(16, 16), 1, 16, "int8")
    with pytest.raises(TypeError):
        hq.hq_linear_fwd(torch.zeros(16, 16), torch.zeros(16, 16), 16, "int8")
    with pytest.raises(TypeError):
        hq.hq_linear_fwd_save(torch.zeros(16, 16), torch.zeros(16, 16), 16, "int8")


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    monkeypatch.setattr(hq, "_lib", None)
    monkeypatch.setattr(hq, "LIB_PATH", str(tmp_path / "libhq.so"))
    with pytest.raises(ImportError):
        hq.lib()


def test_rht_argument_errors(L):
    """The randomized variant's entry points: the plain checks, plus 16-byte-aligned flags."""
    q = lambda **kw: L.hq_quantize_rht(kw.get("src", FAKE), hq.HQ_BF16, 256, 256, kw.get("dim", 1), 64, 0,
                                       kw.get("neg", FAKE), FAKE, FAKE, FAKE, 1 << 20, None)
    assert q(neg=FAKE_MIS) == 4
    assert q(dim=2) == 1
    assert q(src=None) == 1
    dq = lambda **kw: L.hq_quantize_dual_rht(FAKE, hq.HQ_BF16, 256, kw.get("cols", 256), 64, 0,
                                             kw.get("nc", FAKE), kw.get("nr", FAKE), FAKE, FAKE, FAKE, FAKE,
                                             FAKE, 1 << 20, None)
    assert dq(nc=FAKE_MIS) == 4
    assert dq(nr=FAKE_MIS) == 4
    assert dq(cols=96) == 2
    f = lambda **kw: L.hq_linear_fwd_bwd_rht(FAKE, FAKE, FAKE, hq.HQ_BF16, 256, 512, 256, 64, 0,
                                             kw.get("nk", FAKE), kw.get("nn", FAKE), kw.get("nm", FAKE),
                                             FAKE, FAKE, FAKE, FAKE, kw.get("wsb", 1 << 34), None)
    assert f(nk=FAKE_MIS) == 4
    assert f(nn=FAKE_MIS) == 4
    assert f(nm=FAKE_MIS) == 4
    assert f(wsb=1000) == 8


def test_sign_flag_draws():
    """The randomized variant's flags are seeded draws of 0/1 (about half set), reproducible."""
    from hadamard_rotated_precision_b200 import synthetic
    a = synthetic.sign_flags(4096, 9)
    assert a.dtype == np.uint8 and set(np.unique(a)) <= {0, 1}
    assert 0.45 < a.mean() < 0.55
    assert np.array_equal(a, synthetic.sign_flags(4096, 9))
    assert not np.array_equal(a, synthetic.sign_flags(4096, 10))


def test_split_pass_argument_errors(L):
    """hq_quantize_absmax / hq_quantize_codes: the source checks of hq_quantize, a non-null
    4-byte-aligned absmax scalar, 16-byte-aligned flags (all rejected before any launch)."""
    a = lambda **kw: L.hq_quantize_absmax(kw.get("src", FAKE), hq.HQ_BF16, 256, 256, kw.get("dim", 1),
                                          kw.get("k", 64), kw.get("neg", None), kw.get("am", FAKE), FAKE,
                                          1 << 20, None)
    assert a(am=None) == 1
    assert a(am=FAKE + 2) == 4
    assert a(k=48) == 1
    assert a(neg=FAKE_MIS) == 4
    assert a(src=FAKE_MIS) == 4
    c = lambda **kw: L.hq_quantize_codes(FAKE, hq.HQ_BF16, 256, 256, 1, 64, kw.get("fmt", 0), None,
                                         kw.get("am", FAKE), kw.get("codes", FAKE), FAKE, None)
    assert c(am=None) == 1
    assert c(am=FAKE + 2) == 4
    assert c(fmt=7) == 1
    assert c(codes=FAKE_MIS) == 4


def test_reuse_flow_argument_errors(L):
    """The forward that keeps W's codes and the backward that reuses them reject bad arguments
    before any launch; the reuse GEMM takes 8-bit formats only (FP6 / FP4 are HQ_ERR_ARG)."""
    fk = lambda **kw: L.hq_linear_fwd_keep(FAKE, FAKE, hq.HQ_BF16, kw.get("M", 256), kw.get("K", 512),
                                           kw.get("N", 256), kw.get("k", 64), kw.get("fmt", 0), FAKE, FAKE, FAKE,
                                           kw.get("wq", FAKE), kw.get("sw", FAKE), kw.get("ws", FAKE),
                                           kw.get("wsb", 1 << 34), None)
    assert fk(wq=None) == 1
    assert fk(sw=None) == 1
    assert fk(wq=FAKE_MIS) == 4
    assert fk(sw=FAKE + 1) == 4
    assert fk(M=96) == 2
    assert fk(ws=None) == 8
    assert fk(wsb=16) == 8
    dx = lambda **kw: L.hq_linear_bwd_dx_reuse(kw.get("g", FAKE), kw.get("sg", FAKE), kw.get("wq", FAKE), FAKE,
                                               kw.get("M", 256), kw.get("K", 512), kw.get("N", 200),
                                               kw.get("k", 64), kw.get("fmt", 0), kw.get("dX", FAKE),
                                               kw.get("ws", FAKE), kw.get("wsb", 1 << 34), None)
    for fmt in (2, 3, 4, 7):
        assert dx(fmt=fmt) == 1
    assert dx(k=48) == 1
    assert dx(M=96) == 2          # M rotated: multiple of k
    assert dx(K=32) == 2          # K rotated: multiple of k
    assert dx(N=0) == 2
    assert dx(N=133200) == 2      # INT8 contraction bound
    assert dx(g=None) == 1
    assert dx(dX=None) == 1
    assert dx(wq=FAKE_MIS) == 4
    assert dx(sg=FAKE + 2) == 4
    assert dx(ws=None) == 8
    assert dx(wsb=256 * 512 * 4 - 1) == 8
    assert dx(ws=FAKE_MIS) == 4
    br = lambda **kw: L.hq_linear_bwd_reuse(FAKE, kw.get("dt", hq.HQ_BF16), kw.get("xqt", FAKE), FAKE,
                                            kw.get("wq", FAKE), kw.get("sw", FAKE), kw.get("M", 256),
                                            kw.get("K", 512), kw.get("N", 256), 64, kw.get("fmt", 1),
                                            kw.get("dX", FAKE), kw.get("dW", FAKE), kw.get("ws", FAKE),
                                            kw.get("wsb", 1 << 34), None)
    assert br(dt=5) == 3
    assert br(fmt=2) == 1
    assert br(N=200) == 2         # the layer calls keep every dimension a multiple of k
    assert br(wq=None) == 1
    assert br(dW=None) == 1
    assert br(sw=FAKE + 2) == 4
    assert br(ws=None) == 8
    assert br(wsb=4096) == 8
    M, K, N = 4096, 4096, 11008
    assert hq.hq_linear_fwd_keep_workspace_bytes(M, K, N) >= M * K
    assert hq.hq_linear_fwd_keep_workspace_bytes(M, K, N) < hq.hq_linear_fwd_save_workspace_bytes(M, K, N)
    assert hq.hq_linear_bwd_dx_reuse_workspace_bytes(M, K, N) >= 4 * M * K
    assert hq.hq_linear_bwd_reuse_workspace_bytes(M, K, N) >= N * M + 4 * M * K
    assert hq.hq_linear_bwd_reuse_workspace_bytes(-1, 1, 1) == 0


def test_rotout_and_prerotated_argument_errors(L):
    g = lambda **kw: L.hq_gemm_rotout(kw.get("A", FAKE), kw.get("sa", FAKE), FAKE, FAKE, kw.get("M", 256),
                                      kw.get("N", 512), kw.get("K", 256), kw.get("k", 128), kw.get("fmt", 0),
                                      kw.get("out", FAKE), None)
    for fmt in (2, 3, 4, 9):
        assert g(fmt=fmt) == 1
    assert g(k=100) == 1
    assert g(N=384, k=256) == 2     # N not a multiple of k
    assert g(K=24) == 2             # contraction not a multiple of 16
    assert g(sa=None) == 1          # the dequantized output needs both scales
    assert g(out=None) == 1
    assert g(A=FAKE_MIS) == 4
    assert g(M=0) == 0 and g(N=0) == 0
    q = lambda **kw: L.hq_quantize_prerotated(kw.get("y", FAKE), kw.get("rows", 64), kw.get("cols", 256),
                                              kw.get("fmt", 1), kw.get("codes", FAKE), kw.get("scale", FAKE),
                                              kw.get("ws", FAKE), kw.get("wsb", 1 << 20), None)
    assert q(fmt=3) == 1
    assert q(rows=-1) == 1
    assert q(cols=24) == 2
    assert q(y=None) == 1
    assert q(scale=None) == 1
    assert q(codes=FAKE_MIS) == 4
    assert q(scale=FAKE + 2) == 4
    assert q(ws=None) == 8
    assert q(wsb=16) == 8
    assert hq.hq_quantize_prerotated_workspace_bytes() == hq.hq_quantize_workspace_bytes()


def test_gemm_ws_arguments_and_sizes(L):
    g = lambda **kw: L.hq_gemm_ws(FAKE, FAKE, FAKE, FAKE, 256, 256, kw.get("K", 256), kw.get("fmt", 0), 0,
                                  kw.get("out", FAKE), kw.get("ws", FAKE), 1 << 20, None)
    assert g(fmt=7) == 1
    assert g(K=24) == 2
    assert g(out=None) == 1
    assert g(ws=FAKE_MIS) == 4
    # the Llama up-projection's dX GEMM splits its last wave, its forward GEMM does not
    assert hq.hq_gemm_workspace_bytes(4096, 4096, 11008) >= 2 * 34 * 256 * 256 * 4
    assert hq.hq_gemm_workspace_bytes(4096, 11008, 4096) == 0
    assert hq.hq_gemm_workspace_bytes(-1, 1, 1) == 0


def test_split_rule_through_workspace_sizes(L):
    """The GEMM's split choice, seen through the scratch it asks for (74 CTA pairs, 256 x 256
    tiles): a last wave at most half full after at most three full waves, with 64 or more
    128-deep k-blocks, splits only its own tiles; a GEMM with too few tiles splits all of them;
    everything else needs no scratch."""
    tile_half = 256 * 256 * 4  # one half's fp32 / int32 partial of one tile
    ws = hq.hq_gemm_workspace_bytes
    # 4096 x 4096 x 11008: 256 tiles = 3 waves + 34, 86 k-blocks -> the 34 tail tiles split
    assert 2 * 34 * tile_half <= ws(4096, 4096, 11008) < 2 * 35 * tile_half + 4096
    assert ws(4096, 4096, 4096) == 0       # 32 k-blocks: the split would cost more than it saves
    assert ws(4096, 11008, 4096) == 0      # 688 tiles = 9 full waves + 22: not split
    assert ws(8192, 4096, 4096) == 0       # 512 tiles: the last wave is 68 of 74, more than half
    # 3072 x 768 x 12608: 36 tiles for 74 pairs -> every tile split in two
    assert ws(3072, 768, 12608) >= 2 * 36 * tile_half
    assert ws(128, 4096, 11008) == 0       # fewer than 256 rows: single-CTA kernel, no split
