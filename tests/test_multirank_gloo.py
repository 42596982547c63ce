"""Multi-rank host logic on CPU: world_size 2 gloo ranks.

Each rank computes the owner of every tensor with ma_assign_owners and keeps
its own share. The ranks then exchange what they own. Every tensor must be
owned exactly once across ranks, and every rank must compute the same owner
table (deterministic, no communication needed to agree).
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import synth
import adamw_hybrid_optimizer_muon_b200 as ma


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _descs_groups(name):
    wl = synth.WORKLOADS[name]()
    descs = []
    for t in wl.tensors:
        d = ma.Tensor()
        d.ndim = len(t.shape)
        for i, s in enumerate(t.shape[:2]):
            d.shape[i] = s
        d.role = t.role
        d.group = t.group
        descs.append(d)
    groups = []
    for g in wl.groups:
        G = ma.Group()
        G.kind = g.kind
        if g.kind == ma.MA_MUON:
            G.muon = ma.muon_hparams(heads=g.muon.heads)
        else:
            G.adamw = ma.adamw_hparams()
        groups.append(G)
    return descs, groups


def _worker(rank, world, port, name, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        descs, groups = _descs_groups(name)
        owners = ma.ma_assign_owners(descs, groups, world)
        mine = torch.tensor([i for i, o in enumerate(owners) if o == rank] or [-1], dtype=torch.int64)
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([mine.numel()], dtype=torch.int64))
        maxn = int(max(s.item() for s in sizes))
        padded = torch.full((maxn,), -2, dtype=torch.int64)
        padded[:mine.numel()] = mine
        gathered = [torch.zeros(maxn, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(gathered, padded)
        tables = [torch.zeros(len(owners), dtype=torch.int32) for _ in range(world)]
        dist.all_gather(tables, torch.tensor(owners, dtype=torch.int32))
        if rank == 0:
            owned = [int(x) for g in gathered for x in g.tolist() if x >= 0]
            same = all(torch.equal(tables[0], t) for t in tables)
            q.put((sorted(owned) == list(range(len(owners))), len(owned) == len(set(owned)), same))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("name", ["7b", "d20"])
def test_owner_assignment_two_gloo_ranks(name):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, name, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    covered, disjoint, same = q.get(timeout=10)
    assert covered and disjoint and same
