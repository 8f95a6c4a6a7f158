"""GPU checks of the GEMM's split contraction (hq_gemm_ws): the last wave's tiles, or all
tiles of a GEMM with too few of them, computed as two halves of the k-blocks whose partials are
added once.  INT8 results equal the unsplit GEMM's bit for bit (integer partials); FP8 ones
stay within the 2e-3 bound of the oracle's exact product on sampled rows."""
import numpy as np
import pytest
import torch

import oracle
import hadamard_rotated_precision_b200 as hq

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _setup(oracle_lib):
    from hadamard_rotated_precision_b200 import build
    build.build()
    assert torch.cuda.is_available()
    hq.lib()
    yield
    assert hq.hq_get_error() == 0


def _codes(shape, seed, fp8):
    g = torch.Generator(device="cuda").manual_seed(seed)
    c = torch.randint(-127, 128, shape, generator=g, device="cuda", dtype=torch.int32).to(torch.int8).view(torch.uint8)
    return c & 0x77 if fp8 else c  # finite e4m3 codes of magnitude <= 240


# (M, N, K): the dX GEMM of the Llama up-projection (last wave split), a GEMM with few tiles
# and a long contraction (every tile split), and one that never splits
@pytest.mark.parametrize("M,N,K", [(4096, 4096, 11008), (3072, 768, 12608), (4096, 11008, 4096)])
@pytest.mark.parametrize("fmt", ("int8", "fp8"))
def test_split_matches_unsplit(M, N, K, fmt):
    fp8 = fmt == "fp8"
    A, B = _codes((M, K), 1, fp8), _codes((N, K), 2, fp8)
    s = torch.full((1,), 1e-3, device="cuda")
    plain = hq.hq_gemm(A, s, B, s, fmt)
    nbytes = hq.hq_gemm_workspace_bytes(M, N, K)
    ws = torch.empty(max(16, nbytes), dtype=torch.uint8, device="cuda")
    split = hq.hq_gemm(A, s, B, s, fmt, workspace=ws)
    again = hq.hq_gemm(A, s, B, s, fmt, workspace=ws)  # counters left ready for the next call
    torch.cuda.synchronize()
    assert torch.equal(split, again)
    if not fp8:
        assert torch.equal(plain, split)
    else:
        rows = np.array([0, 255, 256, M // 2, M - 1])
        acc = oracle.gemm(A.cpu().numpy(), B.cpu().numpy(), oracle.FP8_E4M3, rows)
        ref, _ = oracle.epilogue(acc, 1e-3, 1e-3)
        r = oracle.bf16_bits_to_f32(ref).astype(np.float64)
        got = split[torch.from_numpy(rows).cuda()].float().cpu().numpy().astype(np.float64)
        assert np.linalg.norm(got - r) / np.linalg.norm(r) <= 2e-3
    if (M, N, K) == (4096, 11008, 4096):
        assert nbytes == 0
    else:
        assert nbytes > 0
