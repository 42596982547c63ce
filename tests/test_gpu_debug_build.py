"""The debug build (guarded device indexing) against the release build.

libmuonadamw_debug.so checks every hand-computed device index against the
extent of its buffer before the access; a failed check records
MA_ERR_BOUNDS in the status word. tests/debug_cases.py runs the same seeded
steps under each library in a process of its own: the debug run must end
with status OK in every case (no guarded index fell outside its buffer) and
produce the release run's results bit for bit (the guards change no
arithmetic).
"""
import os
import subprocess
import sys

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(tmp_path, which):
    out = tmp_path / f"{which}.npz"
    env = dict(os.environ)
    env["MA_LIBRARY"] = which
    env["PYTHONPATH"] = ROOT + os.pathsep + env.get("PYTHONPATH", "")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_cases.py"), str(out)], env=env,
                       capture_output=True, text=True, timeout=900, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    return np.load(out)


def test_debug_build_guards_hold_and_match_release_bit_for_bit(tmp_path):
    rel = _run(tmp_path, "release")
    dbg = _run(tmp_path, "debug")
    assert int(rel["debug_build"]) == 0 and int(dbg["debug_build"]) == 1
    assert set(rel.files) == set(dbg.files)
    for k in sorted(dbg.files):
        if k.endswith("_status"):
            assert int(dbg[k]) == 0, f"{k}: status {int(dbg[k])} in the debug build"
            assert int(rel[k]) == 0, f"{k}: status {int(rel[k])}"
        elif k != "debug_build":
            assert np.array_equal(rel[k], dbg[k]), f"{k} differs between the builds"
