"""The allocation-free Muon entry point against the workspace one.

muon_step_batched_noalloc is for callers that cannot call cudaMalloc (framework
plugins that own the device allocator and pass no scratch buffer, processes
that reserve all memory up front, loops that cannot take cudaMalloc's
device-wide synchronisation). It must give the same results as
muon_step_batched on the same inputs, within the tolerances the other tests
use, on two calls in a row (the second call finds the first call's leftovers
in the shared scratch array). Both entry points run the same kernels in the
same order on the same inputs, so their results agree bit for bit, and the
allocation-free result is also checked against the oracle directly. This file is collected last, so a failure here
comes after every other test has run. It passes on its own in a fresh process
as well.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import (TOL_BF16, TOL_F32, bf16_round, check_muon, check_state, dev_f32, dev_grad, f32, host,
                         momentum_terms)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape,heads,precision", [((256, 512), 1, 0), ((512, 256), 1, 0), ((256, 512), 4, 0),
                                                   ((200, 136), 1, 1)])
def test_noalloc_matches_workspace_entry_point(shape, heads, precision):
    R, C = shape
    batch = 2
    hp = ma.muon_hparams(heads=heads, precision=precision)
    need = ma.muon_workspace_bytes(batch, R, C, hp)
    assert 0 < need <= ma.STATIC_SCRATCH_BYTES
    r = np.random.default_rng(77)
    W0 = [(r.standard_normal(shape) * 0.02).astype(np.float32) for _ in range(batch)]
    Wa, Ma = [dev_f32(w) for w in W0], [torch.zeros(shape, device="cuda") for _ in range(batch)]
    Wb, Mb = [dev_f32(w) for w in W0], [torch.zeros(shape, device="cuda") for _ in range(batch)]
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    tol = TOL_F32 if precision else TOL_BF16
    for _ in range(2):  # two calls in a row
        g = [bf16_round(r.standard_normal(shape) * 1e-3) for _ in range(batch)]
        G = [dev_grad(x, "bf16") for x in g]
        before_w = [host(w) for w in Wb]
        before_m = [host(m) for m in Mb]
        ma.muon_step_batched(Wa, G, Ma, hp, ws)
        ma.muon_step_batched_noalloc(Wb, G, Mb, hp)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        # the same kernels in the same order on the same inputs: the same bits
        for wa, wb, ma_, mb in zip(Wa, Wb, Ma, Mb):
            assert torch.equal(wa, wb) and torch.equal(ma_, mb)
        # and the allocation-free result on its own against the oracle
        for w0, m0, gk, wb, mb in zip(before_w, before_m, g, Wb, Mb):
            rw, rm = oracle.muon_update(w0, gk, m0, f32(0.02), f32(0.95), f32(0.01), True, 5, ((1.5, -0.5, 0.0),),
                                        f32(1e-7), 0, heads)
            check_muon(w0, host(wb), rw, f32(0.02), f32(0.01), tol, what="noalloc vs oracle")
            check_state(host(mb), rm, momentum_terms(m0, gk, f32(0.95)), what="momentum")


def test_noalloc_rejects_steps_larger_than_its_scratch():
    R, C = 4096, 8192
    hp = ma.muon_hparams()
    assert ma.muon_workspace_bytes(1, R, C, hp) > ma.STATIC_SCRATCH_BYTES
    W = [torch.zeros((R, C), device="cuda")]
    M = [torch.zeros((R, C), device="cuda")]
    G = [torch.zeros((R, C), device="cuda", dtype=torch.bfloat16)]
    with pytest.raises(ma.MAError) as e:
        ma.muon_step_batched_noalloc(W, G, M, hp)
    assert e.value.code == ma.MA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert float(M[0].abs().sum()) == 0.0  # rejected before any launch


def test_noalloc_scratch_limit_is_where_the_rejection_starts():
    # the largest workspace the array takes is STATIC_SCRATCH_BYTES: a batch whose
    # workspace fits runs, the next larger batch of the same shape is rejected
    R, C = 2048, 2048
    hp = ma.muon_hparams()
    b = 1
    while ma.muon_workspace_bytes(b + 1, R, C, hp) <= ma.STATIC_SCRATCH_BYTES:
        b += 1
    assert ma.muon_workspace_bytes(b, R, C, hp) <= ma.STATIC_SCRATCH_BYTES < ma.muon_workspace_bytes(b + 1, R, C, hp)
    mk = lambda n: ([torch.zeros((R, C), device="cuda") for _ in range(n)],  # noqa: E731
                    [torch.zeros((R, C), device="cuda", dtype=torch.bfloat16) for _ in range(n)],
                    [torch.zeros((R, C), device="cuda") for _ in range(n)])
    W, G, M = mk(b + 1)
    with pytest.raises(ma.MAError) as e:
        ma.muon_step_batched_noalloc(W, G, M, hp)
    assert e.value.code == ma.MA_ERR_WORKSPACE
    W, G, M = mk(b)
    ma.muon_step_batched_noalloc(W, G, M, hp)  # zero gradients: the step only decays W (here zero)
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
