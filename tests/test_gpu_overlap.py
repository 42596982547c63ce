"""Momentum passes on a side stream, under the Newton-Schulz chain of the
sub-batch before them, against separate calls, bit for bit.

With momentum overlap on (ma_set_momentum_overlap; off by default), a plan
whose step has several Muon sub-batches splits its workspace in two halves.
Each sub-batch then has its momentum pass (flat for wide matrices,
transposing for tall ones) run on the plan's side stream, one block per SM
beside the Newton-Schulz CTAs of the sub-batch before it. Every kernel does
the same arithmetic as in a call of its own, so the parameters and momentum
must equal those of one muon_step_batched call per matrix, eagerly and
replayed from a CUDA graph.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import bf16_round, dev_f32, dev_grad

pytestmark = pytest.mark.gpu

H = ma.ROLE_HIDDEN
# wide (flat) and tall (transposing) buckets, interleaved in table order
TABLE = [((512, 1024), 0)] * 5 + [((1024, 512), 0)] * 3 + [((384, 768), 1)] * 4 + [((2048,), 2)]


def _groups():
    return [("muon", ma.muon_hparams(lr=0.02, weight_decay=0.01)),
            ("muon", ma.muon_hparams(lr=0.01, weight_decay=0.02)),
            ("adamw", ma.adamw_hparams(lr=0.01))]


def _cap():
    # halves that hold two of the largest matrices: sub-batches of two, many segments
    hp = ma.muon_hparams()
    return 2 * max(ma.muon_workspace_bytes(2, 512, 1024, hp), ma.muon_workspace_bytes(2, 1024, 512, hp))


@pytest.fixture
def overlap_on():
    ma.ma_set_momentum_overlap(True)
    yield
    ma.ma_set_momentum_overlap(False)


@pytest.mark.parametrize("graph", [False, True])
def test_side_stream_momentum_matches_separate_calls(graph, overlap_on):
    r = np.random.default_rng(41)
    P0 = [(r.standard_normal(s) * 0.02).astype(np.float32) for s, _ in TABLE]
    pa = [dev_f32(p) for p in P0]
    opt = ma.MuonAdamW([(p, H, g) for p, (_, g) in zip(pa, TABLE)], _groups(), ws_cap=_cap())
    pb = [dev_f32(p) for p in P0]
    mb = [torch.zeros_like(p) for p in pb]
    vb = [torch.zeros_like(p) for p in pb]
    gdev = [torch.zeros(s, device="cuda", dtype=torch.bfloat16) for s, _ in TABLE]
    groups = _groups()
    for step in (1, 2, 3):
        for gd, (s, _) in zip(gdev, TABLE):
            gd.copy_(dev_grad(bf16_round(r.standard_normal(s) * 1e-3), "bf16"))
        opt.step(gdev, graph=graph)
        if step == 1:
            assert "two halves" in opt.describe()
        for i, ((s, g), p, m, v, gd) in enumerate(zip(TABLE, pb, mb, vb, gdev)):
            kind, hp = groups[g]
            if kind == "muon":
                ws = torch.empty(ma.muon_workspace_bytes(1, *s, hp), dtype=torch.uint8, device="cuda")
                ma.muon_step_batched([p], [gd], [m], hp, ws)
            else:
                hp.step = step
                ma.adamw_step_fused([p], [gd], [m], [v], hp)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for i, (x, y) in enumerate(zip(pa, pb)):
            assert torch.equal(x, y), f"step {step} tensor {i}"
        for i, ((s0, _), m) in enumerate(zip(opt.state, mb)):
            assert torch.equal(s0, m), f"step {step} state {i}"
    assert opt.graph_captures == (1 if graph else 0)
