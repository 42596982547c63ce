"""The sharded data-parallel step on the GPU, as one NCCL rank.

With one rank the reduce-scatter and the all-gather move each bucket onto
itself, so ``DistMuonAdamW`` must give, bit for bit, what ``MuonAdamW`` gives
on the same table: each tensor's arithmetic does not depend on the plan (or
the launch) it runs in, and an average over one rank is the value itself.
The table has several buckets (a small segment cap), Muon classes of one and
of several matrices, a per-head group, bf16 gradients, an embedding, 1-D and
0-D tensors. The first step is also checked against the oracle, and the
step with gradients copied from pinned host memory against the
device-resident one, bit for bit. Multi-rank runs of the same code are the
gloo tests (the collectives are the only difference).
"""
import datetime
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist

import oracle
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import TOL_BF16, bf16_round, check_muon, dev_f32, dev_grad, f32, host

pytestmark = pytest.mark.gpu

H, E = ma.ROLE_HIDDEN, ma.ROLE_EMBED
TABLE = [((1000, 64), E, 2), ((256, 512), H, 0), ((256, 512), H, 0), ((256, 512), H, 0),
         ((384, 128), H, 0), ((512, 256), H, 1), ((96,), H, 2), ((), H, 3), ((7,), H, 3), ((256, 512), H, 0)]


def _groups():
    return [("muon", ma.muon_hparams(lr=0.02, weight_decay=0.01)),
            ("muon", ma.muon_hparams(lr=0.01, heads=4, nesterov=False, scale_mode=1)),
            ("adamw", ma.adamw_hparams(lr=0.01, weight_decay=0.01)),
            ("adamw", ma.adamw_hparams(lr=0.003, weight_decay=0.0))]


@pytest.fixture
def one_rank_group():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=120))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_one_rank_matches_muonadamw_bit_for_bit(one_rank_group):
    from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW

    r = np.random.default_rng(77)
    P0 = [np.asarray(r.standard_normal(s) * 0.02, dtype=np.float32) for s, _, _ in TABLE]
    pa = [dev_f32(p) for p in P0]
    pb = [dev_f32(p) for p in P0]
    ref = ma.MuonAdamW([(p, role, g) for p, (_, role, g) in zip(pa, TABLE)], _groups())
    opt = DistMuonAdamW([(p, role, g) for p, (_, role, g) in zip(pb, TABLE)], _groups(),
                        grad_dtype=torch.bfloat16, seg_cap=1 << 16)
    try:
        assert len(opt.buckets) >= 4
        G = [dev_grad(bf16_round(r.standard_normal(s) * 1e-3), "bf16") for s, _, _ in TABLE]
        for step in (1, 2, 3):
            if step > 1:
                G = [dev_grad(bf16_round(r.standard_normal(s) * 1e-3), "bf16") for s, _, _ in TABLE]
            before = [host(p) for p in pb]
            for gv, g in zip(opt.grads, G):
                gv.copy_(g)
            kept = opt.flat_grad.clone()
            ref.step(G)
            opt.step()
            torch.cuda.synchronize()
            assert ma.ma_device_status() == ma.MA_OK
            assert torch.equal(kept, opt.flat_grad)
            for i, (a, b) in enumerate(zip(pa, pb)):
                assert torch.equal(a, b), f"step {step} tensor {i}"
            for pc in opt.pieces():
                s0 = ref.state[pc.index][0].reshape(-1)[pc.lo:pc.hi]
                assert torch.equal(pc.state0.reshape(-1), s0)
                if pc.state1 is not None:
                    assert torch.equal(pc.state1, ref.state[pc.index][1].reshape(-1)[pc.lo:pc.hi])
            if step == 1:  # and against the oracle, for the Muon matrices of group 0
                hp = dict(lr=f32(0.02), beta=f32(0.95), weight_decay=f32(0.01), nesterov=True, steps=5,
                          coeffs=((1.5, -0.5, 0.0),), eps=f32(1e-7))
                for i, (s, _, g) in enumerate(TABLE):
                    if g != 0:
                        continue
                    rw, _ = oracle.muon_update(before[i], host(G[i]), np.zeros(s), **hp)
                    check_muon(before[i], host(pb[i]), rw, hp["lr"], hp["weight_decay"], TOL_BF16,
                               what=f"tensor {i}")
    finally:
        opt.close()
        ref._plan.close()


def test_one_rank_step_from_host_matches_step(one_rank_group):
    # gradients from pinned host memory, copied bucket by bucket on a side
    # stream: the same bits as the device-resident step
    from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW

    r = np.random.default_rng(78)
    P0 = [np.asarray(r.standard_normal(s) * 0.02, dtype=np.float32) for s, _, _ in TABLE]
    pa = [dev_f32(p) for p in P0]
    pb = [dev_f32(p) for p in P0]
    oa = DistMuonAdamW([(p, role, g) for p, (_, role, g) in zip(pa, TABLE)], _groups(),
                       grad_dtype=torch.bfloat16, seg_cap=1 << 16)
    ob = DistMuonAdamW([(p, role, g) for p, (_, role, g) in zip(pb, TABLE)], _groups(),
                       grad_dtype=torch.bfloat16, seg_cap=1 << 16)
    host_flat = torch.zeros(ob.flat_grad.shape, dtype=torch.bfloat16, pin_memory=True)
    hv = ob.host_views(host_flat)
    try:
        for step in (1, 2, 3):
            G = [dev_grad(bf16_round(r.standard_normal(s) * 1e-3), "bf16") for s, _, _ in TABLE]
            for gv, h, g in zip(oa.grads, hv, G):
                gv.copy_(g)
                h.copy_(g.cpu())
            oa.step()
            ob.step_from_host(host_flat)
            # the caller refills its pinned buffer as soon as the copies have
            # read it, while the step may still run (every tensor's range; the
            # alignment gaps between tensors keep their zeros)
            ob.host_copies_done.synchronize()
            for h in hv:
                h.fill_(1e3)
            torch.cuda.synchronize()
            assert ma.ma_device_status() == ma.MA_OK
            assert torch.equal(oa.flat_grad, ob.flat_grad)
            for i, (a, b) in enumerate(zip(pa, pb)):
                assert torch.equal(a, b), f"step {step} tensor {i}"
    finally:
        oa.close()
        ob.close()

