"""The bench's host-side helpers on the CPU: the DRAM-traffic figures it
reports come from committed capture summaries whose recorded source sha256
must match the kernel sources as committed (an edit of the kernel without a
new capture turns the figure into null, and this test into a failure), and
the workload tables are consistent."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def test_traffic_captures_describe_the_committed_kernel():
    for (kind, workload), (path, _) in bench.TRAFFIC_PROFILES.items():
        if not os.path.exists(os.path.join(ROOT, path)):
            continue   # a capture not taken yet reports null
        value, src = bench.captured_traffic(kind, workload)
        assert value is not None and value > 0, (kind, workload, src)


def test_no_capture_means_null():
    assert bench.captured_traffic("attention", "attention")[0] is None
    assert bench.captured_traffic("gemm", "attention")[0] is None


def test_tensor_peak_follows_the_clock():
    assert bench.tensor_peak_kind({"sm_mhz": 1940.0, "sm_max_mhz": 1965.0}) == (True, "burst")
    assert bench.tensor_peak_kind({"sm_mhz": 1350.0, "sm_max_mhz": 1965.0}) == (False, "sustained")
    assert bench.tensor_peak_kind({"sm_mhz": None, "sm_max_mhz": None}) == (False, "sustained")


def test_workload_tables():
    assert bench.data_of("tower_fp8") == "tower" and bench.data_of("lfm_frontend") == "frontend"
    assert bench.data_of("ragged") == "ragged"
    assert bench.data_of("lfm_encoder") == "tower" and bench.data_of("lfm_ragged") == "ragged"
    for w in ("tower", "tower_fp8", "ragged", "frontend", "lfm_frontend", "lfm_encoder", "lfm_ragged", "attention",
              "resample"):
        d = bench.workload_desc(w, {"parallelism": "replicas x1"})
        assert d["workload"].startswith(w + ":") and "l2" in d


def test_peaks_are_positive():
    p = bench.peaks()
    assert p["hbm_gbs"] > 0 and p["bf16_tflops"] > 0 and p["bf16_tflops_sustained"] > 0
    assert p["source"] in ("measured", "fallback")
