"""The CUDA-graph step (muonadamw_step_graph) against the eager step, bit for bit.

Two optimizers start from the same parameters; one steps eagerly, the other
through the graph path. Between steps the AdamW hyperparameters and step
(patched into the captured AdamW launches), the Muon lr and weight decay
(patched into the captured final applies), and the Muon coefficients (a new
capture) change. Every parameter and state buffer must stay identical.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import bf16_round, dev_f32, dev_grad

pytestmark = pytest.mark.gpu

H, E = ma.ROLE_HIDDEN, ma.ROLE_EMBED
# (shape, role, group, grad dtype): pair tiles (m = 256), single-CTA tiles
# (m = 128, and 64-row head slices), a tall matrix, an fp32-mode group,
# AdamW matrices, vectors and a 0-D scalar
TABLE = [((256, 512), H, 0, "bf16"), ((128, 384), H, 0, "bf16"), ((512, 256), H, 0, "f32"),
         ((256, 512), H, 1, "bf16"), ((192, 128), H, 2, "f32"), ((1000, 64), E, 3, "bf16"),
         ((300,), H, 3, "bf16"), ((), H, 4, "f32")]


def _groups(k):
    """Hyperparameters of step k: 2 changes AdamW values (patched), 3 the Muon lr
    and weight decay on the tensor-core path (patched), 4 the fp32-mode lr and
    5 the coefficients (both re-capture), 6 nothing."""
    m0 = dict(lr=0.02, weight_decay=0.01)
    m1 = dict(lr=0.01, weight_decay=0.05, heads=4)
    m2 = dict(lr=0.02, precision=1)
    a0 = dict(lr=0.01, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01)
    a1 = dict(lr=0.003, beta1=0.9, beta2=0.99, eps=1e-8, weight_decay=0.0)
    if k >= 2:
        a0["lr"], a1["beta2"] = 0.005, 0.98
    if k >= 3:
        m0.update(lr=0.015, weight_decay=0.02)
        m1["lr"] = 0.02
    if k >= 4:
        m2["lr"] = 0.01
    if k >= 5:
        m0["coeffs"] = ((2.0, -1.5, 0.5), (1.5, -0.5, 0.0), (1.5, -0.5, 0.0), (1.5, -0.5, 0.0), (1.5, -0.5, 0.0))
    return [("muon", ma.muon_hparams(**m0)), ("muon", ma.muon_hparams(**m1)), ("muon", ma.muon_hparams(**m2)),
            ("adamw", ma.adamw_hparams(**a0)), ("adamw", ma.adamw_hparams(**a1))]


CAPTURES_AFTER = {1: 1, 2: 1, 3: 1, 4: 2, 5: 3, 6: 3}


def _make(P0):
    params = [dev_f32(p) for p in P0]
    opt = ma.MuonAdamW([(p, role, g) for p, (_, role, g, _) in zip(params, TABLE)], _groups(1))
    return params, opt


def _set_groups(opt, k):
    for g, (kind, hp) in zip(opt.groups, _groups(k)):
        if kind == "muon":
            g.muon = hp
        else:
            g.adamw = hp  # the step counter is set again by the next step()


def test_graph_step_equals_eager_step():
    r = np.random.default_rng(77)
    P0 = [(r.standard_normal(s) * 0.02).astype(np.float32) for s, *_ in TABLE]
    pa, eager = _make(P0)
    pb, graph = _make(P0)
    side = torch.cuda.Stream()
    # fixed gradient buffers: a plan (and its graph) belongs to one set of pointers
    ga = [dev_grad(np.zeros(s), dt) for s, _, _, dt in TABLE]
    gb = [dev_grad(np.zeros(s), dt) for s, _, _, dt in TABLE]
    for step in range(1, 7):
        G = [bf16_round(r.standard_normal(s) * 1e-3) for s, *_ in TABLE]
        for a, b, g, (_, _, _, dt) in zip(ga, gb, G, TABLE):
            a.copy_(dev_grad(g, dt))
            b.copy_(a)
        _set_groups(eager, step)
        _set_groups(graph, step)
        eager.step(ga)
        gd = gb
        if step == 6:  # replay on another stream than the capture's and the default one
            side.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(side):
                graph.step(gd, stream=side.cuda_stream, graph=True)
            torch.cuda.current_stream().wait_stream(side)
        else:
            graph.step(gd, graph=True)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for i, (x, y) in enumerate(zip(pa, pb)):
            assert torch.equal(x, y), f"step {step}: parameter {i}"
        for i, ((s0, s1), (t0, t1)) in enumerate(zip(eager.state, graph.state)):
            assert torch.equal(s0, t0) and (s1 is None or torch.equal(s1, t1)), f"step {step}: state {i}"
        assert graph.launches == eager.launches
        assert graph.graph_captures == CAPTURES_AFTER[step], f"step {step}"


def test_graph_patches_the_deep_final_apply():
    # matrices with m >= 2048 only, so that the final applies take the deep
    # variant (5-stage ring): a square one (a*X term) and a wide one
    # (Gram-space chain, a = 0); lr and decay change every step and must be
    # patched into the deep kernel's parameter block, with no re-capture
    table = [((2048, 2048), H, 0), ((2048, 2560), H, 0)]
    r = np.random.default_rng(78)
    P0 = [(r.standard_normal(s) * 0.02).astype(np.float32) for s, *_ in table]
    lrs = [(0.02, 0.01), (0.015, 0.02), (0.01, 0.0)]

    def make():
        params = [dev_f32(p) for p in P0]
        return params, ma.MuonAdamW([(p, role, g) for p, (_, role, g) in zip(params, table)],
                                    [("muon", ma.muon_hparams(lr=lrs[0][0], weight_decay=lrs[0][1]))])

    pa, eager = make()
    pb, graph = make()
    ga = [dev_grad(np.zeros(s), "bf16") for s, *_ in table]
    gb = [dev_grad(np.zeros(s), "bf16") for s, *_ in table]
    for step, (lr, wd) in enumerate(lrs, start=1):
        G = [bf16_round(r.standard_normal(s) * 1e-3) for s, *_ in table]
        for a, b, g in zip(ga, gb, G):
            a.copy_(dev_grad(g, "bf16"))
            b.copy_(a)
        for opt in (eager, graph):
            opt.groups[0].muon = ma.muon_hparams(lr=lr, weight_decay=wd)
        eager.step(ga)
        graph.step(gb, graph=True)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for i, (x, y) in enumerate(zip(pa, pb)):
            assert torch.equal(x, y), f"step {step}: parameter {i}"
        assert graph.graph_captures == 1
