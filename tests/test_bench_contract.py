"""The bench's JSON contract on the host: the reference arm's line and the
config of the main line (the GPU arm itself runs on a B200)."""
import argparse
import json

import pytest

import bench


def test_reference_arm_prints_one_complete_line(capsys):
    args = argparse.Namespace(steps=1, warmup=0, gpus=1, impl="reference", layout="paired")
    assert bench.run_reference(args, world=1, rank=0) == 0
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1
    d = json.loads(out[0])
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "GB/s"
    assert d["value"] > 0 and d["higher_is_better"] is True and d["n_gpus"] == 1
    assert d["steps"] == 1 and d["data"] == "synthetic" and d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert "workload" in d["config"] and "model" not in d["config"]


def test_decode_config_names_the_workload():
    args = argparse.Namespace(gpus=2, layout="paired")
    c = bench.decode_config(args, 43)
    assert c["N"] == 4096 and c["K"] == 4096 and c["M"] == 1 and c["bits"] == bench.HEADLINE_BITS
    assert c["pool_matrices"] == 43 and "L2" in c["l2"] and "replicas x2" == c["parallelism"]
    assert "x_ready" in c["launches"] and c["layout"].startswith("paired")


def test_cpu_baseline_reports_its_sample():
    cb = bench.cpu_baseline(seconds=0.0)
    assert cb["unit"] == "GB/s" and cb["value"] > 0 and cb["kind"] == "oracle"
    assert "rows" in cb["sample"] and "cores" in cb["sample"]


@pytest.mark.parametrize("world,units,ms,want", [(1, 100, 2.0, 5e4), (4, 100, 2.0, 2e5), (8, 1, 0.5, 16e3)])
def test_whole_job_rate(world, units, ms, want):
    assert bench.whole_job_rate(world, units, ms) == pytest.approx(want)
