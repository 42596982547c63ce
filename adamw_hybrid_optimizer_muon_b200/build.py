"""Build the MuonAdamW CUDA library in-tree for sm_100a.

    python -m adamw_hybrid_optimizer_muon_b200.build [--verbose] [--force]

Compiles every ``csrc/*.cu`` with nvcc (``-gencode arch=compute_100a,code=sm_100a``)
into ``lib/libmuonadamw.so``, and once more with ``-DMA_DEBUG`` into
``lib/libmuonadamw_debug.so``: the debug build checks every hand-computed device
index against the extent of its buffer (a failed check records MA_ERR_BOUNDS
and skips the access) and otherwise computes the same bits. Each object is
rebuilt only when a source or header is newer than it; the objects compile in
parallel. nvcc cross-compiles, so no GPU is needed.
"""
from __future__ import annotations

import concurrent.futures
import glob
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJ = os.path.join(HERE, "_build")
LIB_DIR = os.path.join(HERE, "lib")
LIB = os.path.join(LIB_DIR, "libmuonadamw.so")
LIB_DEBUG = os.path.join(LIB_DIR, "libmuonadamw_debug.so")
VARIANTS = (("release", LIB, []), ("debug", LIB_DEBUG, ["-DMA_DEBUG"]))

ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC", "-Xcompiler", "-O3",
         "--expt-relaxed-constexpr", "-I" + os.path.join(ROOT, "include")]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _headers():
    return glob.glob(os.path.join(CSRC, "*.cuh")) + glob.glob(os.path.join(CSRC, "*.h")) + \
        glob.glob(os.path.join(ROOT, "include", "*.h"))


def build(verbose: bool = False, force: bool = False) -> str:
    """Build both libraries; returns the release library's path."""
    os.makedirs(LIB_DIR, exist_ok=True)
    srcs = sorted(glob.glob(os.path.join(CSRC, "*.cu")))
    hdr_mtime = max([os.path.getmtime(h) for h in _headers()] + [0.0])
    jobs = []  # (source, object, extra flags)
    objs = {}
    for name, _, extra in VARIANTS:
        odir = os.path.join(OBJ, name)
        os.makedirs(odir, exist_ok=True)
        objs[name] = []
        for src in srcs:
            obj = os.path.join(odir, os.path.basename(src)[:-3] + ".o")
            objs[name].append(obj)
            if force or not os.path.exists(obj) or os.path.getmtime(obj) < max(os.path.getmtime(src), hdr_mtime):
                jobs.append((src, obj, extra))

    def compile_one(job):
        src, obj, extra = job
        cmd = [nvcc()] + ARCH + FLAGS + extra + (["-Xptxas", "-v"] if verbose else []) + ["-c", src, "-o", obj]
        return job, subprocess.run(cmd, capture_output=True, text=True)

    workers = max(1, min(len(jobs), os.cpu_count() or 1))
    failed = []
    with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as pool:
        for (src, obj, extra), res in pool.map(compile_one, jobs):
            if verbose or res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
            if res.returncode != 0:
                failed.append(os.path.basename(src) + (" (debug)" if extra else ""))
    if failed:
        raise RuntimeError("nvcc failed on " + ", ".join(failed))
    for name, lib_path, _ in VARIANTS:
        o = objs[name]
        if force or not os.path.exists(lib_path) or os.path.getmtime(lib_path) < max(os.path.getmtime(x) for x in o):
            cmd = [nvcc()] + ARCH + ["-shared", "-Xcompiler", "-fPIC", "-o", lib_path] + o
            res = subprocess.run(cmd, capture_output=True, text=True)
            if res.returncode != 0:
                sys.stderr.write(res.stdout + res.stderr)
                raise RuntimeError(f"link failed ({name})")
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, force="--force" in sys.argv))
