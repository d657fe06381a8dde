"""Host-side pieces of bench.py that need no GPU: the constants it shares with the
library (its roofline splits the algorithmic bytes between the two delta kernels with
the library's many-token rule) and the traffic record that must go stale with the
kernel's sources."""

import os
import re
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "tenant_serving_b200", "csrc")


def _define(path, name):
    src = open(os.path.join(CSRC, path)).read()
    m = re.search(r"#define\s+%s\s+(\d+)" % name, src)
    assert m, name
    return int(m.group(1))


def test_many_token_threshold_comes_from_the_library():
    from tenant_serving_b200 import build
    build.build()
    assert bench.tc_min_tokens() == _define("bd_apply.cu", "BD_TC_MIN_TOKENS")
    assert not hasattr(bench, "TC_MIN_TOKENS")  # no copy of the value to go stale


def test_traffic_record_is_tied_to_the_kernel_sources(tmp_path, monkeypatch):
    rec = bench.NCU_TRAFFIC["delta_lut"]
    assert bench.ncu_traffic("nonexistent_kernel") is None  # no record, no number
    got = bench.ncu_traffic("delta_lut")
    assert got in (None, rec["bytes_per_launch"])
    # a source that differs from the captured one gives no traffic number
    fake = dict(rec, sha256_16="0" * 16)
    monkeypatch.setitem(bench.NCU_TRAFFIC, "delta_lut", fake)
    assert bench.ncu_traffic("delta_lut") is None


def test_fused_layer_has_the_projection_rows():
    from workloads import LLAMA3_8B_FUSED, LLAMA3_8B_PROJECTIONS
    rows = lambda t: sum(o * i for _, o, i in t)  # noqa: E731
    assert rows(LLAMA3_8B_FUSED) == rows(LLAMA3_8B_PROJECTIONS)


def test_cpu_baseline_sample_is_bounded_and_positive():
    import time
    t0 = time.perf_counter()
    value, cores, desc = bench.oracle_sample(0.2)
    assert value > 0 and cores >= 1 and "oracle" in desc
    assert time.perf_counter() - t0 < 60


def test_both_arms_report_the_same_config():
    class A:  # the fields serving_config reads
        layers, tenants, batch = 32, 100, 512
    cfg = bench.serving_config(A, 1)
    assert cfg["batch"] == 512 and cfg["tenants"] == 100 and "fused" in cfg["workload"]
    assert bench.serving_config(A, 8)["parallelism"] == "replicas x8"
