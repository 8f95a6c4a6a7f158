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
    e = d["gemm_pair_int8_llama_up_proj"]
    assert e["source_sha"] == bench.file_digest(bench.GEMM_SRC), \
        "the GEMM kernel changed since its ncu capture: capture it again and update profiles/traffic.json"
    t = bench.recorded_traffic("gemm_pair_int8_llama_up_proj")
    # at least the operands once (A 16.8 MB + B 45.1 MB), at most operands + the bf16 output
    assert 62e6 <= t <= 62.0e6 + 90.2e6 + 1e6
    assert os.path.exists(os.path.join(bench.ROOT, e["capture"]))


def test_unknown_traffic_kind_is_null():
    assert bench.recorded_traffic("no_such_kernel") is None
