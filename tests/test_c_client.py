"""The C ABI from plain C: tests/c_client/abi_client.c, compiled with the
system C compiler against include/muonadamw.h and linked against the built
library, exercises the host-only entry points (partition, owners, the
sharded layout, struct sizes, argument checks). No GPU is needed."""
import os
import shutil
import subprocess

import pytest

import adamw_hybrid_optimizer_muon_b200 as ma

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_plain_c_client(tmp_path):
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    ma.lib()  # the library must exist (LibraryMissing otherwise)
    lib_dir = os.path.dirname(ma.LIB_PATH)
    exe = str(tmp_path / "abi_client")
    src = os.path.join(ROOT, "tests", "c_client", "abi_client.c")
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), src,
                        "-L", lib_dir, "-lmuonadamw", f"-Wl,-rpath,{lib_dir}", "-o", exe],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
