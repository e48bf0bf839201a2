"""The benchmark's command line on a machine without a GPU: the reference
arm (the CPU oracle) prints one JSON line with the fields the benchmark
contract asks for, labelled like the GPU arm's line of the same workload."""
import json
import os
import subprocess
import sys

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return json.loads(out.stdout.strip().splitlines()[-1])


@pytest.mark.parametrize("workload", ["tiny_gdn", "tiny_relu"])
def test_reference_arm_prints_the_contract_line(workload):
    d = _run("--impl", "reference", "--workload", workload, "--steps", "2", "--warmup", "1")
    assert d["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["metric"] == bench.METRIC and d["unit"] == "latent frames/s"
    assert d["higher_is_better"] is True and d["n_gpus"] == 1 and d["steps"] == 2
    assert d["value"] > 0 and d["vs_baseline"] is None
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"]
    assert "oracle on" in cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0
    assert d["config"]["workload"] == "tiny_fp32_B1_H2_D32_F8_S64"


def test_workload_labels_of_the_variants():
    assert bench.workload_label("gdn_720p_60s_B1", "gdn") == "gdn_720p_60s_B1"
    assert bench.workload_label("gdn_720p_60s_B1", "gdn_reverse") == "gdn_720p_60s_B1_reverse8"
    assert bench.workload_label("gdn_720p_60s_B1", "gdn_token_beta") == "gdn_720p_60s_B1_token_beta"


def test_every_bench_workload_names_a_synthetic_workload():
    import synth
    for name, (wname, mode) in bench.WORKLOADS.items():
        spec = synth.workload(wname)
        assert mode in ("relu", "gdn", "gdn_reverse", "gdn_token_beta", "gdn_prep"), name
        assert spec.F > 0 and spec.S > 0


def test_gpus_n_launches_n_ranks_and_reports_them():
    """`bench.py --gpus 2` starts two ranks itself (torchrun on this node);
    rank 0 prints the one line, with n_gpus equal to the ranks that ran."""
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_gdn", "--gpus", "2", "--steps", "1",
                          "--warmup", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [ln for ln in out.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, out.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2


def test_world_size_that_disagrees_with_gpus_is_an_error():
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_gdn", "--gpus", "4", "--steps", "1"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode != 0 and "WORLD_SIZE" in out.stderr
