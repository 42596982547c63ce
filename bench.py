#!/usr/bin/env python
"""Benchmark of one MuonAdamW optimizer step on a B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 7b|d20|square|aspect|tiny|square8]
                    [--impl ours|reference] [--no-e2e] [--no-cpu-baseline] [--graph] [--sharded]
                    [--coeffs a,b,c;...]

A step is one muonadamw_step over a synthetic parameter set (with --graph,
the same step replayed from a CUDA graph). Each step runs AdamW on every
0-D/1-D tensor and on the embedding/unembedding, and the momentum/norm pass
plus 5 Newton-Schulz iterations on every hidden matrix, with the final decay
and apply. The default workload is the 7B-shaped set. Its inputs (params,
grads, state: ~70 GB) are far larger than the 126 MB L2, so no flush is
needed between steps; sets smaller than twice the L2 get a 512 MB write
between timed steps, outside their events.

Printed (rank 0): one JSON line with the metric (params/s), ms per step (the
mean over the K timed steps, plus the median and range of the per-step times), the
end-to-end number through the C ABI with host buffers, the roofline of the
dominant kernel (Newton-Schulz GEMMs, measured live with CUDA events on their
launch stream), the clocks seen during the timed region, and a CPU baseline
(the fp64 oracle on a bounded sample, host cores).

``--sharded`` times the sharded data-parallel step instead (DistMuonAdamW:
the ranks share one step of the set, so its scaling is strong; with one GPU
the collectives move each bucket onto itself).

``--impl reference`` times that same oracle (there is no other implementation
of this method to run) on a bounded sample per step and prints the same line
with ``"impl": "reference"``.
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "MuonAdamW step ms & params/s; NS TFLOP/s vs bf16 peak; AdamW GB/s vs HBM"
UNIT = "params/s"

# Sources of the Newton-Schulz kernel: a DRAM-traffic record (ncu's
# dram__bytes_read.sum + dram__bytes_write.sum per launch) applies only to the
# kernel built from exactly these files.
NS_KERNEL_SOURCES = ("adamw_hybrid_optimizer_muon_b200/csrc/ns_tc.cu", "adamw_hybrid_optimizer_muon_b200/csrc/common.cuh")
NS_TRAFFIC_RECORD = os.path.join("profiles", "ns_tc_kernel_traffic.json")


def ns_kernel_sha16():
    import hashlib
    h = hashlib.sha256()
    for rel in NS_KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ns_traffic(workload, ns_launches_per_step):
    """DRAM bytes per Newton-Schulz launch of this workload from the committed
    capture record, or None: when there is no record for the workload, when it
    was taken on other kernel sources, or for another launch structure."""
    path = os.path.join(ROOT, NS_TRAFFIC_RECORD)
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_sha16") != ns_kernel_sha16():
        return None
    w = rec.get("workloads", {}).get(workload)
    if not w or w.get("ns_launches_per_step") != ns_launches_per_step:
        return None
    return float(w["bytes_per_launch"])


def _ncu_ns_launch_bytes(csv_path):
    """DRAM bytes (read + write) of each ns_tc_kernel launch in an ncu --csv
    launch list taken with --metrics dram__bytes_read.sum,dram__bytes_write.sum."""
    import csv
    scale = {"byte": 1.0, "Kbyte": 1e3, "Mbyte": 1e6, "Gbyte": 1e9, "Tbyte": 1e12}
    with open(csv_path) as f:
        lines = [ln for ln in f if ln.startswith('"')]
    per = {}
    for r in csv.DictReader(lines):
        if "ns_tc_kernel" not in r["Kernel Name"]:
            continue
        if r["Metric Name"] in ("dram__bytes_read.sum", "dram__bytes_write.sum"):
            v = float(r["Metric Value"].replace(",", "")) * scale[r["Metric Unit"]]
            per[int(r["ID"])] = per.get(int(r["ID"]), 0.0) + v
    return [per[k] for k in sorted(per)]


def write_traffic_record(square_csv, rect_csv, bench_7b_log):
    """Write the DRAM-traffic record for the current kernel sources from ncu
    launch lists of one step of the square8 and rect8 workloads (every
    ns_tc_kernel launch of the step) and a bench.py line of the 7b workload
    (for its Newton-Schulz launches per step). The 7b figure scales the two
    8-matrix chains' traffic per unit to the 7b step's units: square units
    take the 4096 x 4096 chain, the 4096 x 11008 and 11008 x 4096 units the
    rectangular one (their chains differ only in the transposition of the
    momentum pass and of the final store)."""
    sq, rc = _ncu_ns_launch_bytes(square_csv), _ncu_ns_launch_bytes(rect_csv)
    n_sq = len(synth.WORKLOADS["square8"]().tensors)
    n_rc = len(synth.WORKLOADS["rect8"]().tensors)
    units = {}
    for t in synth.WORKLOADS["7b"]().tensors:
        if t.role == synth.ROLE_HIDDEN and len(t.shape) == 2:
            units[tuple(sorted(t.shape))] = units.get(tuple(sorted(t.shape)), 0) + 1
    u_sq, u_rc = units.get((4096, 4096), 0), units.get((4096, 11008), 0)
    if set(units) - {(4096, 4096), (4096, 11008)}:
        raise SystemExit(f"7b hidden matrices of shapes this record does not cover: {sorted(units)}")
    with open(bench_7b_log) as f:
        line = json.loads([ln for ln in f if ln.startswith("{")][-1])
    if not line["config"]["workload"].startswith("7b"):
        raise SystemExit("the bench line is not the 7b workload's")
    n7 = int(round(sum(line["kernels"][c]["launches_per_step"]
                       for c in ("ns_gram", "ns_apply", "ns_gramsq", "ns_final") if c in line["kernels"])))
    step_7b = u_sq * sum(sq) / n_sq + u_rc * sum(rc) / n_rc
    rec = {
        "kernel_sha16": ns_kernel_sha16(),
        "source": "ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum,gpu__time_duration.sum (one pass), "
                  "every ns_tc_kernel launch of one step of bench.py --workload square8 and --workload rect8",
        "workloads": {
            "square8": {"bytes_per_launch": sum(sq) / len(sq), "ns_launches_per_step": len(sq)},
            "rect8": {"bytes_per_launch": sum(rc) / len(rc), "ns_launches_per_step": len(rc)},
            "7b": {"bytes_per_launch": step_7b / n7, "ns_launches_per_step": n7,
                   "derivation": f"per-unit traffic of the 8-matrix chains scaled to the 7B step's units: "
                                 f"{u_sq} x (4096 x 4096 chain) + {u_rc} x (4096 x 11008 chain, wide and tall "
                                 f"alike), over its {n7} Newton-Schulz launches"},
        },
    }
    with open(os.path.join(ROOT, NS_TRAFFIC_RECORD), "w") as f:
        json.dump(rec, f, indent=1)
    print(json.dumps({"square8_per_launch": sq, "rect8_per_launch": rc, "7b_step_bytes": step_7b,
                      "7b_ns_launches": n7}))


def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def free_port():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join("/tmp", f"ma_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.fh,
                                         stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def gpu_id_for(device_index):
    import torch
    try:
        uuid = str(torch.cuda.get_device_properties(device_index).uuid)
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            return vis.split(",")[device_index]
        return device_index


# ----------------------------------------------------------------------------- oracle timing (CPU baseline)

def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = [i for i in threadpool_info() if i.get("user_api") == "blas"]
        if info:
            return int(info[0]["num_threads"])
    except Exception:
        pass
    return os.cpu_count()


def oracle_sample(wl, n_matrices=1):
    """A bounded slice of the workload for the oracle: n_matrices Muon matrices of
    the most common shape plus AdamW elements in the workload's AdamW:Muon
    proportion."""
    import oracle
    kinds = oracle.partition([(t.shape, t.role) for t in wl.tensors])
    muon = [i for i, k in enumerate(kinds) if k == 0]
    adamw = [i for i, k in enumerate(kinds) if k == 1]
    shapes = {}
    for i in muon:
        shapes.setdefault(wl.tensors[i].shape, []).append(i)
    mis = max(shapes.values(), key=len)[:n_matrices] if muon else []
    n_muon = sum(wl.tensors[i].numel for i in muon)
    n_adamw = sum(wl.tensors[i].numel for i in adamw)
    mat = sum(wl.tensors[i].numel for i in mis)
    k_adamw = int(round(n_adamw * mat / n_muon)) if n_muon else min(n_adamw, 4_000_000)
    return mis, adamw, k_adamw


def time_oracle_step(wl, mis, adamw, k_adamw, step=2):
    import oracle
    elapsed = 0.0
    params = 0
    for mi in mis:
        spec = wl.tensors[mi]
        g = wl.groups[spec.group].muon
        W = synth.initial_weight(spec, mi)
        G = synth.gradient(wl, mi, step)
        M = np.zeros(spec.shape)
        t0 = time.perf_counter()
        oracle.muon_update(W, G, M, g.lr, g.beta, g.weight_decay, g.nesterov, g.ns_steps, g.coeffs, g.eps,
                           g.scale_mode, g.heads)
        elapsed += time.perf_counter() - t0
        params += spec.numel
    left = k_adamw
    for i in adamw:
        if left <= 0:
            break
        spec = wl.tensors[i]
        n = min(spec.numel, left)
        r = synth.rng(i, step, synth.STREAM_GRAD)
        p = (r.standard_normal(n) * 0.02)
        gr = r.standard_normal(n) * 1e-3
        a = wl.groups[spec.group].adamw
        t0 = time.perf_counter()
        oracle.adamw_update(p, gr, np.zeros(n), np.zeros(n), step, a.lr, a.beta1, a.beta2, a.eps, a.weight_decay)
        elapsed += time.perf_counter() - t0
        params += n
        left -= n
    return params, elapsed


def cpu_baseline(wl, n_matrices=4):
    mis, adamw, k = oracle_sample(wl, n_matrices)
    params, secs = time_oracle_step(wl, mis, adamw, k)
    desc = (f"oracle fp64 on {len(mis)} Muon matrices {wl.tensors[mis[0]].shape} + {k} AdamW elements "
            f"({params} params, {secs:.1f} s)") if mis else f"oracle fp64 on {params} AdamW elements"
    return {"value": params / secs, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": desc}


# ----------------------------------------------------------------------------- reference arm

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    wl = synth.WORKLOADS[args.workload]()
    mis, adamw, k = oracle_sample(wl)
    for _ in range(args.warmup):
        time_oracle_step(wl, mis, adamw, k)
    tot_params, tot_s = 0, 0.0
    for _ in range(args.steps):
        p, s = time_oracle_step(wl, mis, adamw, k)
        tot_params += p
        tot_s += s
    value = tot_params / tot_s
    sample = (f"per step: oracle fp64 on 1 Muon matrix {wl.tensors[mis[0]].shape} + {k} AdamW elements"
              if mis else f"per step: oracle fp64 on {k} AdamW elements")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * tot_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": workload_config(wl, args.gpus),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


L2_BYTES = 126 << 20


def small_inputs(wl):
    """Whether one step's data (fp32 params and state, bf16 grads) fits in twice the L2."""
    return wl.numel * 14 < 2 * L2_BYTES


def _descs_for(wl, ma):
    """Host-only tensor descriptors of a workload (shapes and roles) for ma_partition."""
    out = []
    for t in wl.tensors:
        d = ma.Tensor()
        d.ndim = len(t.shape)
        for k, v in enumerate(t.shape[:2]):
            d.shape[k] = v
        d.role = t.role
        out.append(d)
    return out


def workload_config(wl, n_gpus):
    import oracle
    kinds = oracle.partition([(t.shape, t.role) for t in wl.tensors])
    l2 = ("inputs smaller than L2: a 512 MB buffer is written between timed steps, outside their events"
          if small_inputs(wl) else "inputs larger than L2 (no flush needed)")
    return {"workload": f"{wl.name}: {wl.description}", "params": wl.numel,
            "muon_matrices": kinds.count(0), "adamw_tensors": kinds.count(1),
            "ns_steps": wl.groups[0].muon.ns_steps if wl.groups[0].kind == 0 else None,
            "ns_coeffs": [list(c) for c in wl.groups[0].muon.coeffs] if wl.groups[0].kind == 0 else None,
            "l2": l2, "parallelism": f"replicas x{n_gpus}"}


# ----------------------------------------------------------------------------- our arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="7b", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="time the step replayed from a CUDA graph (muonadamw_step_graph); the per-kernel "
                         "profile then comes from an extra, untimed pass of eager steps")
    ap.add_argument("--sharded", action="store_true",
                    help="time the sharded data-parallel step (DistMuonAdamW: reduce-scatter of the gradients, "
                         "each rank's share of the update, all-gather of the parameters) instead of N replicas")
    ap.add_argument("--coeffs", default=None,
                    help="Newton-Schulz polynomial per iteration, 'a,b,c[;a,b,c...]' (default: the cubic 1.5,-0.5,0)")
    ap.add_argument("--momentum-overlap", action="store_true",
                    help="run each Muon sub-batch's momentum pass on a side stream under the previous sub-batch's "
                         "Newton-Schulz chain (ma_set_momentum_overlap; off by default, slower on a B200)")
    ap.add_argument("--write-traffic-record", nargs=3, metavar=("SQUARE8_CSV", "RECT8_CSV", "BENCH_7B_LOG"),
                    default=None, help="host only: write the Newton-Schulz DRAM-traffic record for the current "
                                       "kernel sources from ncu launch lists and a 7b bench line, then exit")
    args = ap.parse_args()
    if args.write_traffic_record:
        return write_traffic_record(*args.write_traffic_record)
    rank, world, local = env_int("RANK", 0), env_int("WORLD_SIZE", 1), env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist

    import adamw_hybrid_optimizer_muon_b200 as ma
    import synth.device as sdev

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if args.sharded and args.graph:
        raise SystemExit("--sharded steps run collectives and are not captured in a graph")
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    elif args.sharded:  # one rank: a process group of its own
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{free_port()}", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    wl = synth.WORKLOADS[args.workload]()
    if args.coeffs:
        co = tuple(tuple(float(x) for x in t.split(",")) for t in args.coeffs.split(";"))
        for g in wl.groups:
            if g.kind == synth.KIND_MUON:
                g.muon.coeffs = co
                if len(co) > 1:
                    g.muon.ns_steps = len(co)
    params = sdev.weights(wl, device=dev, base=rank)
    grads = sdev.gradients(wl, 1, device=dev, base=rank)
    groups = []
    for g in wl.groups:
        if g.kind == synth.KIND_MUON:
            h = g.muon
            groups.append(("muon", ma.muon_hparams(h.lr, h.beta, h.weight_decay, h.eps, h.nesterov, h.ns_steps,
                                                   h.coeffs, h.scale_mode, h.heads, h.precision)))
        else:
            h = g.adamw
            groups.append(("adamw", ma.adamw_hparams(h.lr, h.beta1, h.beta2, h.eps, h.weight_decay, 1)))
    table = [(p, t.role, t.group) for p, t in zip(params, wl.tensors)]
    ma.ma_set_momentum_overlap(args.momentum_overlap)  # read when the plans are made
    if args.sharded:
        from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW
        gdts = {g.dtype for g in grads}
        if len(gdts) != 1:
            raise SystemExit("--sharded needs one gradient dtype across the workload")
        opt = DistMuonAdamW(table, groups, grad_dtype=gdts.pop())
        for gv, g in zip(opt.grads, grads):
            gv.copy_(g)
        del grads, params, table
        grads = None

        def do_step():
            opt.step()
    else:
        opt = ma.MuonAdamW(table, groups)

        def do_step():
            opt.step(grads, graph=args.graph)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        do_step()
    torch.cuda.synchronize(dev)
    st = ma.ma_device_status(stream)
    if st != ma.MA_OK:
        raise SystemExit(f"device status after warm-up: {st}")

    # ---- timed region: K steps, inputs resident in HBM
    clocks = ClockSampler(gpu_id_for(local))
    clocks.start()
    time.sleep(0.5)
    barrier()
    torch.cuda.synchronize(dev)
    ma.ma_profile_enable(not args.graph)
    if small_inputs(wl):
        # flush L2 between steps; each step is timed by its own pair of events
        flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            do_step()
            b.record(stream)
        torch.cuda.synchronize(dev)
        per_step = [a.elapsed_time(b) for a, b in evs]
        step_ms = sum(per_step)
        del flush
    else:
        # one event before each step and one after the last: the steps run
        # back to back, and each one's time is read between its two events
        evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
        evs[0].record(stream)
        for i in range(args.steps):
            do_step()
            evs[i + 1].record(stream)
        torch.cuda.synchronize(dev)
        per_step = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
        step_ms = evs[0].elapsed_time(evs[-1])
    barrier()
    clk = clocks.stop()
    if args.graph:  # graph replays record no per-kernel events: profile eager steps, untimed
        ma.ma_profile_enable(True)
        for _ in range(args.steps):
            opt.step(grads)
        torch.cuda.synchronize(dev)
    ma.ma_profile_enable(False)
    prof = ma.ma_profile_collect()
    ms = step_ms / args.steps
    launches_per_step = opt.launches
    if world > 1:
        tt = torch.tensor([ms], device=dev, dtype=torch.float64)
        dist.all_reduce(tt, op=dist.ReduceOp.MAX)
        ms = float(tt.item())
    st = ma.ma_device_status(stream)
    if st != ma.MA_OK:
        raise SystemExit(f"device status after the timed steps: {st}")
    n_params = wl.numel
    # replicas: each rank steps its own copy of the set (weak scaling); sharded:
    # the ranks share one step of the set (strong scaling)
    jobs = 1 if args.sharded else world
    value = jobs * n_params / (ms / 1000.0)

    # ---- end to end through the public API: every step the gradients come from
    # pinned host memory (copied by the library on its own stream, overlapped with
    # the compute), then the device status word (the step's result) is read back
    e2e = None
    if not args.no_e2e and args.sharded:
        # the gradients of the whole set arrive in the flat gradient buffer from
        # pinned host memory every step (bucket by bucket on a side stream, each
        # bucket's reduce-scatter starting when its copy lands); the status word
        # is read back after it
        host_flat = torch.empty(opt.flat_grad.shape, dtype=opt.flat_grad.dtype, pin_memory=True)
        host_flat.copy_(opt.flat_grad)
        h2d = host_flat.numel() * host_flat.element_size()
        k_e2e = max(1, min(args.steps, 5))
        status = torch.full((k_e2e,), -1, dtype=torch.int32, pin_memory=True)
        barrier()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(k_e2e):
            opt.step_from_host(host_flat)
            ma.ma_device_status_async(status.data_ptr() + 4 * i, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        if int(status.abs().max()) != ma.MA_OK:
            raise SystemExit(f"device status error in the end-to-end loop: {status.tolist()}")
        ems = e0.elapsed_time(e1) / k_e2e
        if world > 1:
            tt = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ems = float(tt.item())
        e2e = {"value": n_params / (ems / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": 4, "ms_per_step": ems,
               "path": "DistMuonAdamW.step_from_host (pinned host gradients copied bucket by bucket, overlapped "
                       "with the reductions and updates; each step's status word read back asynchronously)"}
        del host_flat
    elif not args.no_e2e:
        host_grads = [torch.empty(g.shape, dtype=g.dtype, pin_memory=True) for g in grads]
        for hg, g in zip(host_grads, grads):
            hg.copy_(g)
        h2d = sum(g.numel() * g.element_size() for g in grads)
        k_e2e = max(1, min(args.steps, 5))
        opt.step_from_host(host_grads, grads)  # untimed: creates the copy stream and events
        torch.cuda.synchronize(dev)
        barrier()
        torch.cuda.synchronize(dev)
        # every step's result (the status word) is read back into pinned host
        # memory without stalling the host; all of them are checked afterwards
        status = torch.full((k_e2e,), -1, dtype=torch.int32, pin_memory=True)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for i in range(k_e2e):
            opt.step_from_host(host_grads, grads)
            ma.ma_device_status_async(status.data_ptr() + 4 * i, stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        barrier()
        if int(status.abs().max()) != ma.MA_OK:
            raise SystemExit(f"device status error in the end-to-end loop: {status.tolist()}")
        ems = e0.elapsed_time(e1) / k_e2e
        if world > 1:
            tt = torch.tensor([ems], device=dev, dtype=torch.float64)
            dist.all_reduce(tt, op=dist.ReduceOp.MAX)
            ems = float(tt.item())
        e2e = {"value": world * n_params / (ems / 1000.0), "unit": UNIT, "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": 4, "ms_per_step": ems,
               "path": "muonadamw_step_from_host (pinned host gradients, copies overlapped with compute; "
                       "each step's status word read back asynchronously)"}
        del host_grads

    if rank == 0:
        peaks = load_peaks()
        ns_cls = ("ns_gram", "ns_apply", "ns_gramsq", "ns_final")
        ns_ms = sum(prof[c]["ms"] for c in ns_cls)
        ns_fl = sum(prof[c]["flops"] for c in ns_cls)
        ns_bytes = sum(prof[c]["bytes"] for c in ns_cls)
        ns_launches = sum(prof[c]["launches"] for c in ns_cls)
        ns_tflops = ns_fl / (ns_ms / 1000.0) / 1e12 if ns_ms > 0 else None
        # The sustained (power-capped) GEMM peak applies when the power cap held
        # the SM clock down during the timed region; at full clock, the burst one.
        capped = bool(clk and clk.get("sm_mhz") and clk.get("sm_max_mhz")
                      and clk["sm_mhz"] < 0.95 * clk["sm_max_mhz"])
        peak_t = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
        # the flops the pages' iteration itself would take (N Grams, symmetric,
        # and N applies per matrix); the achieved rate counts the flops executed,
        # which the Gram-space chain of wide matrices makes fewer
        direct = 0.0
        for t, kd in zip(wl.tensors, ma.ma_partition(_descs_for(wl, ma))):
            if kd != ma.MA_MUON:
                continue
            g = wl.groups[t.group].muon
            rh = t.shape[0] // g.heads
            m_, n_ = min(rh, t.shape[1]), max(rh, t.shape[1])
            direct += g.heads * g.ns_steps * (m_ * (m_ + 1) * n_ + 2 * m_ * m_ * n_)
        roofline = {"kernel": "ns_tc_kernel (Newton-Schulz Gram + apply, tcgen05)", "bound": "tensor",
                    "achieved": ns_tflops, "peak": peak_t, "unit": "TFLOP/s",
                    "frac": ns_tflops / peak_t if ns_tflops else None,
                    "peak_kind": f"bf16 dense, {'sustained' if capped else 'burst'} ({peaks['source']})",
                    "traffic": ns_traffic(args.workload, ns_launches / args.steps),
                    "traffic_algorithmic": ns_bytes / max(1, ns_launches),
                    "launches": ns_launches, "avg_launch_ms": ns_ms / max(1, ns_launches),
                    "flops_per_launch": ns_fl / max(1, ns_launches),
                    "flops_per_step_executed": ns_fl / args.steps, "flops_per_step_direct_iteration": direct}
        kernels = {}
        for c in ma.PROF_CLASSES:
            pc = prof[c]
            if pc["launches"] == 0:
                continue
            d = {"ms_per_step": pc["ms"] / args.steps, "launches_per_step": pc["launches"] / args.steps}
            if pc["flops"] > 0:
                d["tflops"] = pc["flops"] / (pc["ms"] / 1000.0) / 1e12
            if pc["bytes"] > 0 and pc["flops"] > 0:
                d["algorithmic_gbs"] = pc["bytes"] / (pc["ms"] / 1000.0) / 1e9  # tensor-bound: context only
            elif pc["bytes"] > 0:
                d["gbs"] = pc["bytes"] / (pc["ms"] / 1000.0) / 1e9
                d["frac_hbm"] = d["gbs"] / peaks["hbm_gbs"]
            if c == "momentum_side":
                d["note"] = ("momentum passes and their norm finalizes run on a side stream, one block per SM "
                             "beside the Newton-Schulz CTAs of the previous sub-batch: their time is hidden, "
                             "not a bandwidth target")
            kernels[c] = d
        config = workload_config(wl, world)
        if args.momentum_overlap:
            config["momentum_overlap"] = "momentum passes on a side stream under the previous sub-batch's chain"
        if args.sharded:
            config["parallelism"] = (f"sharded dp{world}: reduce-scatter, each rank's share of the update, "
                                     f"all-gather ({len(opt.buckets)} buckets)")
        line = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms,
                "ms_per_step_median": statistics.median(per_step),
                "ms_per_step_range": [min(per_step), max(per_step)], "higher_is_better": True,
                "scaling": "strong" if args.sharded else "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,0.02^2) weights, "
                "N(0,1e-3^2) bf16 grads)", "config": config,
                "e2e": e2e, "gpu_launches": launches_per_step * args.steps, "roofline": roofline,
                "kernels": kernels, "clocks": clk,
                "precision": {"ns_operands": "bf16", "accumulate": "fp32", "state": "fp32"}}
        if world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(wl)
        print(json.dumps(line))
    if args.sharded:
        opt.close()
    else:
        opt._plan.close()
    if dist.is_initialized():
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
