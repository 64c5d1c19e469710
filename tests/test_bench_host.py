"""Host-side logic of bench.py (no GPU): metric names, the CPU oracle sample,
and the reference arm's JSON line on the small dense workload."""

from __future__ import annotations

import json
import os
import subprocess
import sys

import bench
import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_metric_names_follow_the_workload_kind():
    assert bench.metric_for(bench.DEFAULT_WORKLOAD, False) == bench.METRIC
    for name in ("tiny_64x48_d24_i8", "dense_512x384_pts3_f32", "pair_512x384_pts3_f32"):
        dense = synth.make_workload(name).dense
        metric = bench.metric_for(name, dense)
        assert metric.startswith("dense mutual") == dense, (name, metric)


def test_dense_oracle_sample_is_clamped_to_the_map():
    w = synth.make_workload("tiny_64x48_d24_i8")
    found, dt, threads, desc = bench.oracle_sample(w, 10 ** 6)
    n = w.pairs[0].H1 * w.pairs[0].W1
    assert 0 < found <= n and dt > 0 and threads >= 1
    assert f"first {n} image-1 pixels" in desc


def test_reference_arm_prints_one_json_line():
    out = subprocess.run(
        [sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "0",
         "--workload", "tiny_64x48_d24_i8"],
        cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [x for x in out.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    j = json.loads(lines[0])
    assert j["impl"] == "reference" and j["value"] > 0 and j["steps"] == 1
    assert j["metric"].startswith("dense mutual")
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"]["h2d_bytes_per_step"] == 0 and j["e2e"]["d2h_bytes_per_step"] == 0


def test_gpus_n_starts_n_ranks_that_reduce_over_gloo():
    """``bench.py --gpus 2`` outside a launcher starts two ranks itself (local
    rendezvous); their sum and max reductions reach rank 0, which alone
    prints, with n_gpus equal to the rank count."""
    out = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--selftest-launcher"],
                         cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [json.loads(x) for x in out.stdout.splitlines() if x.startswith("{")]
    assert lines == [{"selftest": "launcher", "n_gpus": 2, "rank_sum": 3.0, "rank_max": 1.0}]


def test_headline_nests_the_other_configurations_by_default():
    old = sys.argv
    try:
        sys.argv = ["bench.py"]
        a = bench.parse_args()
        assert a.workload == bench.DEFAULT_WORKLOAD and a.gpus == 1
        assert a.also.split(",") == bench.NESTED_DEFAULT
        sys.argv = ["bench.py", "--workload", "pair_512x384_d24_bf16"]
        assert bench.parse_args().also == ""
        sys.argv = ["bench.py", "--also", ""]
        assert bench.parse_args().also == ""
    finally:
        sys.argv = old
    assert set(bench.NESTED_DEFAULT) <= set(synth.CONFIGS)
    p = bench.percentiles([float(x) for x in range(1, 101)])
    assert (p["p10"], p["p50"], p["p90"]) == (11.0, 51.0, 91.0)
