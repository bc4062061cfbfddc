"""Host side of bench.py, no GPU: the reference arm.

`bench.py --impl reference` times the CPU oracle (the plain definition of
each op) on the host's cores and prints one JSON line with the same metric,
unit and direction as the GPU arm, plus the cpu_baseline and e2e objects
that describe that run.  Under torchrun only rank 0 works and prints; the
other ranks exit 0 at once.
"""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=e, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    p = run_bench(["--impl", "reference", "--workload", "twoshot_160k", "--steps", "2", "--warmup", "1"])
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    sys.path.insert(0, ROOT)
    import bench

    assert d["impl"] == "reference"
    assert d["metric"] == bench.METRIC and d["unit"] == "GB/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["config"] == bench.twoshot_160k_cfg(4)  # the GPU arm's workload description
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == "GB/s" and cb["cores"] >= 1
    assert "sample" in cb
    assert d["e2e"] == {"value": d["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_exit_quietly():
    p = run_bench(["--impl", "reference", "--workload", "twoshot_160k", "--steps", "1", "--warmup", "0"],
                  env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert p.returncode == 0, p.stderr[-2000:]
    assert p.stdout.strip() == ""


def test_reference_arm_rejects_a_workload_it_has_no_oracle_step_for():
    p = run_bench(["--impl", "reference", "--workload", "moe", "--steps", "1", "--warmup", "0"])
    assert p.returncode != 0
    assert "supports tp_decode and twoshot_160k" in p.stderr
