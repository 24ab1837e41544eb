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
    for kind in ("gemm", "gemm_fp8"):
        value, src = bench.captured_traffic(kind)
        assert value is not None and value > 0, (kind, src)
        assert os.path.exists(os.path.join(ROOT, src))


def test_no_capture_means_null():
    assert bench.captured_traffic("attention")[0] is None


def test_workload_tables():
    assert bench.data_of("tower_fp8") == "tower" and bench.data_of("lfm_frontend") == "frontend"
    assert bench.data_of("ragged") == "ragged"
    for w in ("tower", "tower_fp8", "ragged", "frontend", "lfm_frontend", "attention", "resample"):
        d = bench.workload_desc(w, {"parallelism": "replicas x1"})
        assert d["workload"].startswith(w + ":") and "l2" in d


def test_peaks_are_positive():
    p = bench.peaks()
    assert p["hbm_gbs"] > 0 and p["bf16_tflops"] > 0 and p["bf16_tflops_sustained"] > 0
    assert p["source"] in ("measured", "fallback")
