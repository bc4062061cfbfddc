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
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["unit"] == "GB/s"
    assert cb["cores"] == bench.oracle_workers() and cb["single_thread_value"] > 0
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
    assert "supports full_step, tp_decode, twoshot_160k" in p.stderr


def test_reference_arm_default_is_the_gpu_arms_default_workload():
    sys.path.insert(0, ROOT)
    import bench

    p = run_bench(["--impl", "reference", "--steps", "1", "--warmup", "0"])
    assert p.returncode == 0, p.stderr[-2000:]
    d = json.loads([ln for ln in p.stdout.splitlines() if ln.startswith("{")][0])
    assert d["config"] == bench.full_step_cfg(8)
    assert d["cpu_baseline"]["cores"] == bench.oracle_workers()


def test_oracle_pieces_give_the_whole_ops_bits():
    """The oracle's timing cuts each op into pieces that separate workers run;
    for every op whose result is defined element by element (or token by
    token), the pieces' results put together are the one-piece result, bit
    for bit: each element keeps its rank order, each packet line its bytes,
    each token its combine.  Checked on the default workload at 1/256 size."""
    import numpy as np

    sys.path.insert(0, ROOT)
    import bench
    import oracle

    whole, _, _ = bench.host_full_step(oracle, parts=1, frac=256)
    split, _, _ = bench.host_full_step(oracle, parts=3, frac=256)
    run = bench.HOST_TASKS
    checked = set()
    for w, s_ in zip(whole, split):
        assert w.name == s_.name and w.alg_bytes == s_.alg_bytes and len(w.pieces) == 1
        one = run[w.kind](oracle, w.pieces[0], w.params)
        parts = [run[s_.kind](oracle, pc, s_.params) for pc in s_.pieces]
        kind = w.kind
        if kind in ("all_reduce", "reduce_scatter", "scatter") and w.params.get("algo") != "ring":
            for q in range(len(one)):
                assert np.array_equal(np.concatenate([pr[q] for pr in parts]), one[q]), (w.name, q)
        elif kind == "reduce":
            assert np.array_equal(np.concatenate(parts), one), w.name
        elif kind == "all_gather":
            n = len(one)
            e = one[0].size // n
            got = np.concatenate([np.asarray(pr[0]).reshape(n, -1) for pr in parts], axis=1).reshape(-1)
            assert np.array_equal(got, one[0]) and e * n == got.size, w.name
        elif kind == "pack":
            for r in range(len(one)):
                assert np.array_equal(np.concatenate([pr[r] for pr in parts]), one[r]), (w.name, r)
        elif kind == "all_reduce_packed":
            proto = w.params["proto"]

            def payload(res, count):
                return oracle.unpack(res[0][0], count * 2, proto, 1)[0]

            counts = [int(pc["count"][0]) for pc in s_.pieces]
            got = np.concatenate([payload(pr, c) for pr, c in zip(parts, counts)])
            assert np.array_equal(got, payload(one, int(w.pieces[0]["count"][0]))), w.name
            assert one[1] == 0 and all(pr[1] == 0 for pr in parts)
        elif kind == "moe_combine":
            for src in range(len(one)):
                assert np.array_equal(np.concatenate([pr[src] for pr in parts]), one[src]), (w.name, src)
        else:
            continue
        checked.add(kind)
    assert checked == {"all_reduce", "reduce_scatter", "scatter", "reduce", "all_gather", "pack",
                       "all_reduce_packed", "moe_combine"}
