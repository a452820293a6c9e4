"""Host-side pieces of bench.py that decide what the bench line reports:
the ncu traffic figure is attached only while the profiled source is the
current one, the CTA imbalance ratio, the whole-job value of weak scaling,
and the records that name the workload and the CPU baseline.  No GPU."""
import json
import os

import numpy as np
import pytest

import bench
from block_sparse_spatiotemporal_b200.inputs import WORKLOADS


def test_traffic_only_for_the_profiled_source(monkeypatch):
    path = os.path.join(bench.ROOT, "profiles", "fine_tc_wan480p.json")
    with open(path) as f:
        rec = json.load(f)
    assert rec["dram_bytes_per_launch"] == rec["dram_bytes_read"] + rec["dram_bytes_write"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: rec["kernel_source_hash"])
    assert bench.profiled_traffic("wan480p") == rec["dram_bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda: "0" * 16)
    assert bench.profiled_traffic("wan480p") is None
    assert bench.profiled_traffic("no_such_workload") is None


def test_kernel_source_hash_covers_the_work_list_order():
    # the fine kernel, its helpers, and the files that order its work list
    h = bench.kernel_source_hash()
    assert len(h) == 16 and int(h, 16) >= 0


class _FakeLib:
    def __init__(self, times):
        self.times = np.asarray(times, dtype=np.int64)

    def profile_cta_times(self, shape, ws, rope=None):
        return self.times


def test_sm_imbalance_is_max_over_mean_busy_time():
    # busy times 100, 110, 90 ns: mean 100, max 110
    got = bench.sm_imbalance(_FakeLib([[0, 100], [0, 110], [5, 95]]), None, None)
    assert got["ctas"] == 3
    assert got["max_over_mean"] == pytest.approx(1.1)
    assert got["max_busy_us"] == pytest.approx(0.110)
    assert got["min_busy_us"] == pytest.approx(0.090)
    assert got["launch_span_us"] == pytest.approx(0.110)
    assert bench.sm_imbalance(_FakeLib(np.zeros((0, 2))), None, None) is None


def test_whole_job_value_counts_every_rank():
    # 2 TFLOP per rank in 4 ms: 500 TFLOP/s a rank, 2000 over four ranks
    assert bench.whole_job_value(1, 2e12, 4.0) == pytest.approx(500.0)
    assert bench.whole_job_value(4, 2e12, 4.0) == pytest.approx(2000.0)


def test_workload_config_names_the_workload_and_its_shape():
    class A:
        subblock = False
    wl = WORKLOADS["wan480p"]
    cfg = bench.workload_config(wl, A(), world=2)
    assert cfg["workload"] == "wan480p" and cfg["grid"] == [20, 32, 52]
    assert cfg["tokens"] == 33280 and cfg["heads"] == 40 and cfg["head_dim"] == 128
    assert cfg["top_p"] == 0.95 and cfg["k_min"] == 8
    assert cfg["parallelism"] == "replica x2"
    assert "larger than L2" in cfg["l2"]
    A.subblock = True
    assert bench.workload_config(wl, A())["scoring"].startswith("sub-block")


def test_cpu_baseline_record():
    res = {"flops": 2e12, "est_s": 1000.0, "threads": 16, "desc": "sample",
           "stage_s": {"coarse": 2.0, "fine": 998.0}}
    rec = bench.cpu_baseline_of(res)
    assert rec["kind"] == "oracle" and rec["cores"] == 16 and rec["sample"] == "sample"
    assert rec["value"] == pytest.approx(2e12 / 1000.0 / 1e12)
    assert rec["est_ms_per_step"] == pytest.approx(1e6)
    assert rec["stage_ms"] == {"coarse": 2000.0, "fine": 998000.0}
    assert "estimate" in rec["ms_is"]


def test_pair_flops():
    assert bench.pair_flops(128) == 4 * 64 * 64 * 128
