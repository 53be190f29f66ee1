"""bench.py's reference arm (the oracle timed on the host cores) on the CPU: one JSON line with the
contract's keys, and under torchrun only rank 0 prints it (the other ranks exit 0 without work); the
step-time spread (median, 10th / 90th percentiles) that every bench line carries."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_ref(extra_env=None):
    env = dict(os.environ)
    env.update(extra_env or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "2", "--warmup", "3", "--workload", SMALL],
                          capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)


SMALL = "causal_b1_h2_n128_d64_fp16"


def test_reference_arm_prints_one_contract_line():
    """Whole steps of the named workload are timed, so steps x ms_per_step fits inside the run,
    and the line carries the same config as the GPU arm's."""
    import time
    t0 = time.perf_counter()
    r = run_ref({"RANK": "0", "WORLD_SIZE": "1"})
    wall_ms = (time.perf_counter() - t0) * 1e3
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config", "impl",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    sys.path.insert(0, ROOT)
    import bench
    assert d["config"] == bench.main_config(SMALL, 1)
    assert d["steps"] * d["ms_per_step"] < wall_ms
    assert "whole steps" in d["cpu_baseline"]["sample"]


def test_reference_arm_other_ranks_exit_quietly():
    r = run_ref({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""


def test_step_time_spread_is_median_and_deciles():
    """The per-workload spread the bench reports: median and 10th / 90th percentiles by linear
    interpolation between order statistics, independent of the order the steps ran in."""
    sys.path.insert(0, ROOT)
    import bench
    r = bench.spread([10.0, 1.0, 9.0, 2.0, 8.0, 3.0, 7.0, 4.0, 6.0, 5.0])
    assert r == {"ms_median": 5.5, "ms_p10": 1.9, "ms_p90": 9.1}
    assert bench.spread([2.0]) == {"ms_median": 2.0, "ms_p10": 2.0, "ms_p90": 2.0}
    assert bench.spread([]) == {}


def test_every_gpu_line_is_timed_at_one_gpu():
    """The workload loops of the GPU arm (prefill, decode, backward) run at any world size: only
    the splits-over-GPUs decode line may depend on there being more than one GPU."""
    import ast
    src = open(os.path.join(ROOT, "bench.py")).read()
    tree = ast.parse(src)
    parents = {}
    for node in ast.walk(tree):
        for child in ast.iter_child_nodes(node):
            parents[child] = node
    loops = [n for n in ast.walk(tree) if isinstance(n, ast.For) and isinstance(n.iter, ast.Name)
             and n.iter.id == "BACKWARD_WORKLOADS"]
    assert loops, "the backward workloads are timed in a loop over BACKWARD_WORKLOADS"
    for loop in loops:
        node = loop
        while node in parents:
            node = parents[node]
            if isinstance(node, ast.If):
                names = {n.id for n in ast.walk(node.test) if isinstance(n, ast.Name)}
                assert "world" not in names, "the backward lines must not need more than one GPU"
