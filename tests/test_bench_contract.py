"""bench.py's JSON line: the keys and types the benchmark contract asks for.

The reference arm (the oracle on the host cores) runs anywhere; the GPU arm
(replicas, from a CUDA graph, and the sharded step on one NCCL rank) runs on
a B200 only. All run bench.py as a subprocess on the tiny set.
"""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
BASE_KEYS = {"metric": str, "value": float, "unit": str, "n_gpus": int, "steps": int, "warmup": int,
             "ms_per_step": float, "higher_is_better": bool, "scaling": str, "dtype": str, "data": str,
             "config": dict}


def _run(args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py")] + args, capture_output=True, text=True,
                       timeout=900, cwd=ROOT, env=e)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    return lines


def _check_base(d, steps, warmup):
    for k, t in BASE_KEYS.items():
        assert k in d, k
        assert isinstance(d[k], t) or (t is float and isinstance(d[k], int)), (k, d[k])
    assert d["steps"] == steps and d["warmup"] == warmup
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["higher_is_better"] is True and d["scaling"] == "weak"
    assert "vs_baseline" in d
    assert d["config"]["workload"].startswith("tiny")


def test_reference_arm_line():
    (line,) = _run(["--impl", "reference", "--workload", "tiny", "--steps", "2", "--warmup", "1"])
    d = json.loads(line)
    _check_base(d, 2, 1)
    assert d["impl"] == "reference" and d["dtype"] == "f64"
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == d["value"] and cb["sample"]
    e = d["e2e"]
    assert e["value"] == d["value"] and e["unit"] == d["unit"]
    assert e["h2d_bytes_per_step"] == 0 and e["d2h_bytes_per_step"] == 0


def test_reference_arm_other_ranks_print_nothing():
    lines = _run(["--impl", "reference", "--workload", "tiny", "--steps", "1", "--warmup", "1"],
                 env={"RANK": "1", "WORLD_SIZE": "2", "LOCAL_RANK": "1"})
    assert lines == []


@pytest.mark.gpu
@pytest.mark.parametrize("graph", [False, True])
def test_gpu_arm_line(graph):
    (line,) = _run(["--workload", "tiny", "--steps", "3", "--warmup", "3"] + (["--graph"] if graph else []))
    d = json.loads(line)
    _check_base(d, 3, 3)
    assert d["n_gpus"] == 1 and d["dtype"] == "bf16"
    lo, hi = d["ms_per_step_range"]
    assert 0 < lo <= d["ms_per_step_median"] <= hi
    r = d["roofline"]
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] > 0 and r["peak"] > 0 and abs(r["frac"] - r["achieved"] / r["peak"]) < 1e-9
    assert "traffic" in r
    e = d["e2e"]
    assert e["value"] > 0 and e["unit"] == d["unit"] and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == 3 * 13  # per step: 1 AdamW, momentum, finalize, 5 x (Gram + apply)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(d["clocks"])
    assert "L2" in d["config"]["l2"]


@pytest.mark.gpu
def test_gpu_arm_line_sharded():
    # one NCCL rank: the sharded step (reduce-scatter, local update, all-gather)
    (line,) = _run(["--workload", "tiny", "--steps", "3", "--warmup", "3", "--sharded", "--no-cpu-baseline"])
    d = json.loads(line)
    assert d["scaling"] == "strong" and d["config"]["parallelism"].startswith("sharded dp1")
    assert d["value"] > 0 and d["n_gpus"] == 1
    assert d["gpu_launches"] == 3 * 13  # a Muon bucket (12 launches) and an AdamW bucket (1)
    e = d["e2e"]
    assert e["value"] > 0 and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] == 4
    assert d["roofline"]["achieved"] > 0
