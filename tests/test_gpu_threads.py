"""First calls on a device from two host threads at once.

The library caches per-device facts on the host (the status word's address,
the SM count, the Newton-Schulz kernels' shared-memory attribute and
occupancy, the allocation-free scratch's address). Two threads that make
their first call at the same moment must both get a complete set-up: every
launch sees its kernel's attributes already set. The test runs in a fresh
interpreter, so that the calls it makes really are the process's first, and
checks the two threads' results bit for bit against the same calls made
again one after the other.
"""
import os
import subprocess
import sys
import textwrap

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

CHILD = textwrap.dedent("""
    import sys, threading
    sys.path.insert(0, {root!r})
    import torch
    import adamw_hybrid_optimizer_muon_b200 as ma

    torch.cuda.set_device(0)
    g = torch.Generator(device="cuda").manual_seed(5)
    shape = (512, 1024)
    hp = ma.muon_hparams()
    W0 = [torch.randn(shape, device="cuda", generator=g) * 0.02 for _ in range(4)]
    G = [(torch.randn(shape, device="cuda", generator=g) * 1e-3).bfloat16() for _ in range(4)]
    need = ma.muon_workspace_bytes(2, *shape, hp)
    streams = [torch.cuda.Stream() for _ in range(2)]
    torch.cuda.synchronize()

    def run(W, M, ws, k, noalloc):
        if noalloc:
            ma.muon_step_batched_noalloc(W, G[2 * k:2 * k + 2], M, hp, stream=streams[k])
        else:
            ma.muon_step_batched(W, G[2 * k:2 * k + 2], M, hp, ws, stream=streams[k])

    for noalloc in (False, True):
        Wt = [w.clone() for w in W0]
        Mt = [torch.zeros(shape, device="cuda") for _ in range(4)]
        ws = [torch.empty(need, dtype=torch.uint8, device="cuda") for _ in range(2)]
        torch.cuda.synchronize()
        start = threading.Barrier(2)
        errors = []

        def worker(k):
            try:
                start.wait()
                # thread 0 takes the workspace path, thread 1 the allocation-free
                # one in the second round (one caller of the shared scratch at a time)
                run(Wt[2 * k:2 * k + 2], Mt[2 * k:2 * k + 2], ws[k], k, noalloc and k == 1)
            except Exception as e:  # reported by the parent
                errors.append(repr(e))

        th = [threading.Thread(target=worker, args=(k,)) for k in range(2)]
        for t in th:
            t.start()
        for t in th:
            t.join()
        torch.cuda.synchronize()
        assert not errors, errors
        assert ma.ma_device_status() == ma.MA_OK
        # the same calls again, one after the other, from fresh copies
        Ws = [w.clone() for w in W0]
        Ms = [torch.zeros(shape, device="cuda") for _ in range(4)]
        for k in range(2):
            run(Ws[2 * k:2 * k + 2], Ms[2 * k:2 * k + 2], ws[k], k, noalloc and k == 1)
        torch.cuda.synchronize()
        for a, b in zip(Wt + Mt, Ws + Ms):
            assert torch.equal(a, b)
    print("threads ok")
""")


def test_first_calls_from_two_threads_at_once():
    res = subprocess.run([sys.executable, "-c", CHILD.format(root=ROOT)], capture_output=True, text=True,
                         timeout=600)
    assert res.returncode == 0, res.stdout + res.stderr
    assert "threads ok" in res.stdout
