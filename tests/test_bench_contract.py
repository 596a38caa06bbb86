"""bench.py's command-line contract on a CPU host: the reference arm (the oracle on the host
cores) prints one JSON line with the required keys, ranks other than 0 exit without work, and
fewer than 3 warm-up steps are refused."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, cwd=ROOT,
                          env=e, capture_output=True, text=True, timeout=600)


import pytest


@pytest.mark.parametrize("workload", ["opt-125m", "quadratic"])
def test_reference_arm_prints_one_contract_line(workload):
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", workload])
    assert r.returncode == 0, r.stderr[-500:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["steps"] == 1 and line["warmup"] == 3
    assert line["value"] > 0 and line["higher_is_better"] is True
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["e2e"]["value"] == line["value"] and line["e2e"]["unit"] == line["unit"]
    assert "workload" in line["config"]
    assert line["extrapolated"] is True and line["timed_region_s"] > 0
    # the reference line names the same config as the GPU arm's line
    sys.path.insert(0, ROOT)
    import bench
    want = (bench.quad_config(1) if workload == "quadratic" else
            bench.decoder_config(workload, bench.decoder_workload(workload), line["config"]["params"], 1))
    assert line["config"] == want


def test_default_workload_is_the_opt30b_step():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.DEFAULT_WORKLOAD == "opt-30b"
    w = bench.decoder_workload("opt-30b")
    assert (w["batch"], w["seq"], w["n_micro"], w["n_pert"]) == (8, 2048, 1, 16)
    cfg = bench.decoder_cfg("opt-30b")
    assert (cfg["n_layers"], cfg["d_model"], cfg["n_heads"], cfg["d_ffn"]) == (48, 7168, 56, 28672)


def test_reference_arm_other_ranks_exit_quietly():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "3", "--workload", "opt-125m"],
             env={"RANK": "1", "LOCAL_RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_warmup_below_three_is_refused():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "2"])
    assert r.returncode != 0
