"""Host-side helpers of bench.py that need no GPU: the DRAM traffic scaled from the
committed small-case captures, and the roofline denominators."""

import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from long_context_sparse_05_b200 import workloads  # noqa: E402


def test_profiled_traffic_is_linear_in_the_entries_of_the_launch():
    for w in (workloads.CSA_DECODE_64K, workloads.CSA_DECODE_1M):
        full = bench.profiled_traffic(w, "index_scores")
        unit, per = bench.PROFILED_TRAFFIC[("index_scores", w.idx_dtype)]
        assert unit == "entries"
        assert full == round(per * w.b * w.E)
        # a shape override (as --batch / --context give) scales the figure, not reuses it
        half = workloads.shrink(w, b=w.b // 2)
        assert abs(bench.profiled_traffic(half, "index_scores") - full / 2) <= 1
        short = workloads.shrink(w, n=w.n // 4)
        assert abs(bench.profiled_traffic(short, "index_scores") - full / 4) <= 1


def test_profiled_traffic_per_entry_is_close_to_the_algorithmic_bytes():
    # key bytes per entry: FP8 128 codes + one fp32 scale, NVFP4 64 packed codes + 8 scales;
    # the captures add the query side and rounding, a few percent at most
    assert 132.0 <= bench.PROFILED_TRAFFIC[("index_scores", "fp8")][1] <= 132.0 * 1.05
    assert 72.0 <= bench.PROFILED_TRAFFIC[("index_scores", "nvfp4")][1] <= 72.0 * 1.05


def test_profiled_attention_traffic_is_per_query_and_near_the_rows_read():
    # 64K decode attention: 640 rows of 1 KiB and the 64 KiB query heads per query (the
    # output's writes stay in L2 in the capture), plus a few percent: the query's selection
    # list, and the lines of the merge records (written to L2 just before the cluster
    # barrier) that the cold-cache capture reads back from DRAM
    w = workloads.CSA_DECODE_64K
    if ("sparse_attn", w.name) not in bench.PROFILED_TRAFFIC:
        pytest.skip("no capture of the current attention kernel")
    unit, per = bench.PROFILED_TRAFFIC[("sparse_attn", w.name)]
    assert unit == "queries"
    alg = 640 * 1024 + 64 * 1024
    assert 0.97 * alg <= per <= 1.08 * alg
    assert bench.profiled_traffic(w, "sparse_attn") == round(per * w.b)
    assert abs(bench.profiled_traffic(workloads.shrink(w, b=4), "sparse_attn") - 4 * per) <= 1


def test_no_traffic_without_a_capture():
    assert bench.profiled_traffic(workloads.HCA_DECODE_1M, "sparse_attn") is None


def test_peaks_name_their_source():
    p = bench.load_peaks()
    assert p["src"] in ("measured", "fallback")
    assert p["hbm"] > 1000 and p["bf16"] > 100
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        assert p["src"] == "measured"
