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


def _ncu_csv(path, launches):
    # an ncu --csv launch list: preamble lines, a header, one row per launch and metric
    head = ('"ID","Process ID","Process Name","Host Name","Kernel Name","Context","Stream","Block Size",'
            '"Grid Size","Device","CC","Section Name","Metric Name","Metric Unit","Metric Value"\n')
    with open(path, "w") as f:
        f.write("==PROF== Connected to process 1 (python)\n" + head)
        for i, (kern, rd, wr, unit) in enumerate(launches):
            for name, v in (("dram__bytes_read.sum", rd), ("dram__bytes_write.sum", wr),
                            ("gpu__time_duration.sum", "1,000")):
                u = "nsecond" if name.startswith("gpu__") else unit
                f.write(f'"{i}","1","python","h","{kern}","1","7","(320, 1, 1)","(148, 1, 1)","0","10.0",'
                        f'"Command line profiler metrics","{name}","{u}","{v}"\n')


def test_traffic_record_writer_scales_captures_to_the_7b_step(tmp_path, monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    import synth
    sq = tmp_path / "sq.csv"
    rc = tmp_path / "rc.csv"
    # square8: two Newton-Schulz launches (MB units) and a launch of another kernel that must be ignored
    _ncu_csv(sq, [("void ns_tc_kernel<0, 1>(NsLaunch)", "300", "100", "Mbyte"),
                  ("void adamw_kernel(Args)", "999", "999", "Mbyte"),
                  ("void ns_tc_kernel<3, 1>(NsLaunch)", "1,200,000,000", "400,000,000", "byte")])
    # rect8: three launches
    _ncu_csv(rc, [("void ns_tc_kernel<0, 1>(NsLaunch)", "1.5", "0.5", "Gbyte")] * 3)
    log = tmp_path / "b.log"
    line = {"config": {"workload": "7b: 32 layers"},
            "kernels": {"ns_gram": {"launches_per_step": 26.0}, "ns_final": {"launches_per_step": 10.0},
                        "momentum": {"launches_per_step": 3.0}}}
    log.write_text("noise\n" + json.dumps(line) + "\n")
    rec_path = tmp_path / "rec.json"
    monkeypatch.setattr(bench, "NS_TRAFFIC_RECORD", str(rec_path))
    bench.write_traffic_record(str(sq), str(rc), str(log))
    rec = json.loads(rec_path.read_text())
    w = rec["workloads"]
    assert w["square8"] == {"bytes_per_launch": (4e8 + 1.6e9) / 2, "ns_launches_per_step": 2}
    assert w["rect8"] == {"bytes_per_launch": 2e9, "ns_launches_per_step": 3}
    # 7b: 128 square and 96 rectangular units; each 8-matrix chain's traffic per unit
    hidden = [t for t in synth.WORKLOADS["7b"]().tensors if t.role == synth.ROLE_HIDDEN and len(t.shape) == 2]
    assert len(hidden) == 224
    step = 128 * 2e9 / 8 + 96 * 6e9 / 8
    assert w["7b"]["ns_launches_per_step"] == 36
    assert w["7b"]["bytes_per_launch"] == pytest.approx(step / 36, rel=1e-12)
    # read back while the kernel sources match; not for another launch structure
    assert bench.ns_traffic("7b", 36) == pytest.approx(step / 36, rel=1e-12)
    assert bench.ns_traffic("7b", 35) is None
    rec["kernel_sha16"] = "0" * 16
    rec_path.write_text(json.dumps(rec))
    assert bench.ns_traffic("7b", 36) is None


def test_committed_traffic_record_matches_the_kernel_sources():
    # the per-launch DRAM record must belong to the kernel sources in the tree,
    # or bench.py prints no traffic: re-capture it after changing the kernel
    sys.path.insert(0, ROOT)
    import bench
    with open(os.path.join(ROOT, bench.NS_TRAFFIC_RECORD)) as f:
        rec = json.load(f)
    assert rec["kernel_sha16"] == bench.ns_kernel_sha16()
    assert rec["workloads"]["7b"]["ns_launches_per_step"] > 0
    assert 1.0 < rec["workloads"]["7b"]["bytes_per_launch"] / 2.38e9 < 1.5  # within 1-1.5x the algorithmic bytes
