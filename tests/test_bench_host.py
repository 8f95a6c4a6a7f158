"""CPU checks of bench.py's host helpers: the measured peaks it divides by, and the per-launch
DRAM traffic it reports for the GEMM, which is only valid while the committed ncu capture was
taken on the current kernel source (a changed kernel must be captured again)."""
import json
import os

import bench


def test_measured_peaks_loaded():
    p = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        assert p["src"] == "measured"
    assert p["hbm"] > 1000 and p["bf16"] > 100


def test_recorded_gemm_traffic_matches_current_source():
    with open(bench.TRAFFIC_FILE) as f:
        d = json.load(f)
    key = bench.ROOFLINE_GEMM_KEY
    e = d[key]
    assert e["source_sha"] == bench.file_digest(bench.GEMM_SRC), \
        "the GEMM kernel changed since its ncu capture: capture it again and update profiles/traffic.json"
    t = bench.recorded_traffic(key)
    # at least the operands once (A 100.7 MB + B 33.6 MB), at most operands + the bf16 output
    # (100.7 MB) + a few re-reads
    assert 134e6 <= t <= 2.0 * (134.3e6 + 100.7e6)
    assert os.path.exists(os.path.join(bench.ROOT, e["capture"]))


def test_unknown_traffic_kind_is_null():
    assert bench.recorded_traffic("no_such_kernel") is None
