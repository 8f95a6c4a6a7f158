"""The dense tensor-core probe (hq_mma_peak), which the benchmark divides the GEMMs' throughput
by: it runs to completion, reports no device error, and its INT8 / FP8 rates lie in the range a
B200 can deliver (below the nominal dense figure at the maximum SM clock, 16384 operations per
clock per SM x 148 SMs x 1.965 GHz = 4.77 POPS, and well above half of it)."""
import pytest
import torch

import hadamard_rotated_precision_b200 as hq

pytestmark = pytest.mark.gpu

OPS_PER_MMA = 2 * 256 * 256 * 32  # one CTA-pair instruction: M = 256, N = 256, K = 32


@pytest.mark.parametrize("fmt", ("int8", "fp8"))
def test_mma_peak_probe(fmt):
    from hadamard_rotated_precision_b200 import build
    build.build()
    for _ in range(2):
        hq.hq_mma_peak(fmt, 256)
    best = 0.0
    for _ in range(3):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        pairs = hq.hq_mma_peak(fmt, 4096)
        b.record()
        torch.cuda.synchronize()
        best = max(best, pairs * 4096 * 4 * OPS_PER_MMA / (a.elapsed_time(b) * 1e-3) / 1e12)
    assert hq.hq_get_error() == 0
    assert pairs == torch.cuda.get_device_properties(0).multi_processor_count // 2
    assert 2000.0 < best < 4800.0, best
