"""GPU checks of the split quantization passes used by quantized FSDP communication: the
absmax pass alone equals the oracle's absmax; slices of a tensor quantized with the maximum of
their absmax values concatenate to the whole tensor's codes and scale, bit for bit (the ranks'
collectives are simulated here on one GPU; their flow runs on gloo ranks in test_fsdp_host)."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq
from hadamard_rotated_precision_b200 import synthetic
from _helpers import to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_lib):
    from hadamard_rotated_precision_b200 import build
    build.build()
    assert torch.cuda.is_available()
    hq.lib()
    yield
    assert hq.hq_get_error() == 0


def _weights(dtype):
    w = synthetic.tiny_random((4 * 512, 1024), 31, scale=0.02)
    w[:, 11] *= 50.0
    return synthetic.to_bf16_bits(w) if dtype == "bf16" else w


@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("dim,k", [(1, 256), (1, 16), (0, 64), (0, 256)])
def test_absmax_pass_alone(dtype, dim, k):
    W = _weights(dtype)
    a = hq.hq_quantize_absmax(to_device(W), dim, k)
    assert a.cpu().numpy()[0] == oracle.absmax(oracle.rotate(W, dim, k))


@pytest.mark.parametrize("fmt", (oracle.INT8, oracle.FP8_E4M3, oracle.FP6_E3M2, oracle.FP4_E2M1))
@pytest.mark.parametrize("dtype", ("f32", "bf16"))
@pytest.mark.parametrize("dim,k", [(1, 256), (0, 64)])
def test_four_slices_equal_whole(fmt, dtype, dim, k):
    """Four row slices (each a multiple of k rows when the rotation runs along the rows)."""
    W = _weights(dtype)
    Wd = to_device(W)
    whole_codes, whole_scale = hq.hq_quantize(Wd, dim, k, fmt)
    slices = torch.chunk(Wd, 4, dim=0)
    a = torch.stack([hq.hq_quantize_absmax(s, dim, k) for s in slices]).max().reshape(1)
    parts = [hq.hq_quantize_codes(s, dim, k, fmt, a) for s in slices]
    cat = torch.cat([c for c, _ in parts], dim=0 if dim == 1 else 1)
    assert torch.equal(cat, whole_codes)
    for _, sc in parts:
        assert torch.equal(sc, whole_scale)
    want, want_scale = oracle.quantize(W, dim, k, fmt)
    assert np.array_equal(cat.cpu().numpy(), oracle.device_codes(want, fmt))


def test_sharded_helpers_single_process():
    """Without a process group the sharded quantization is the plain one, and the quantized
    all-gather returns this rank's (whole) codes."""
    W = to_device(_weights("bf16"))
    c, s = hq.hq_quantize_sharded(W, 1, 128, "int8")
    c0, s0 = hq.hq_quantize(W, 1, 128, "int8")
    assert torch.equal(c, c0) and torch.equal(s, s0)
    g, gs = hq.hq_fsdp_all_gather(W, 128, "fp8")
    g0, gs0 = hq.hq_quantize(W, 1, 128, "fp8")
    assert torch.equal(g, g0) and torch.equal(gs, gs0)


def test_codes_pass_special_absmax():
    """absmax 0: zero codes and scale 1; absmax +inf: HQ_ERR_NONFINITE, NaN scale."""
    W = to_device(_weights("bf16"))
    c, s = hq.hq_quantize_codes(W, 1, 64, "int8", torch.zeros(1, device="cuda"))
    assert int(c.count_nonzero()) == 0 and s.item() == 1.0
    assert hq.hq_get_error() == 0
    c, s = hq.hq_quantize_codes(W, 1, 64, "int8", torch.full((1,), float("inf"), device="cuda"))
    assert hq.hq_get_error() == 5
    assert not np.isfinite(s.cpu().numpy()[0])


@pytest.mark.gpu
@pytest.mark.parametrize("fmt", ("int8", "fp8"))
def test_fsdp_forward_flow_one_gpu(fmt):
    """The quantized-FSDP forward flow (gathers on a communication stream, prefetched one layer
    ahead) on one GPU, where each rank's shard is the whole weight: every layer's output equals
    hq_linear_fwd bit for bit."""
    from hadamard_rotated_precision_b200 import synthetic
    k = 64
    xs, ws = [], []
    for i in range(3):
        K, N, M = 256 * (i + 1), 128 * (i + 2), 512
        X = synthetic.tiny_random((M, K), 500 + i)
        X[:, 3] *= 40.0
        xs.append(to_device(synthetic.to_bf16_bits(X)))
        ws.append(to_device(synthetic.to_bf16_bits(synthetic.tiny_random((N, K), 600 + i, scale=0.02))))
    ys = hq.hq_fsdp_forward(ws, xs, k, fmt)
    torch.cuda.synchronize()
    for i, (x, w, y) in enumerate(zip(xs, ws, ys)):
        want = hq.hq_linear_fwd(x, w, k, fmt)
        assert torch.equal(y.view(torch.int16), want.view(torch.int16)), f"layer {i}"
    assert hq.hq_get_error() == 0
