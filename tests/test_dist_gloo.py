"""The sharded data-parallel step on CPU ranks (gloo), and its layout.

``ma_shard_layout`` (host-only) is checked for its invariants on the
benchmark tables and on random ones: every tensor placed once, aligned and
disjoint; a Muon matrix whole inside its owner's segment; an AdamW bucket's
segments covering its tensors; no padding where the class counts divide by
the world size.

``DistMuonAdamW`` is then run on 2 and 3 gloo ranks with its local update
replaced by the oracle (CPU ranks cannot run the library's kernels). Every
rank's parameters must equal a single-process oracle step on the averaged
gradients, bit for bit: on 2 ranks with any gradients (an average of two
fp32 values has one rounding, whatever the reduction order), on 3 with
gradients whose partial sums are all exact. The
table mixes Muon classes whose counts do not divide by the world size (mixed
buckets), a per-head group, an embedding that straddles AdamW segments, 1-D
and 0-D tensors, and a small segment cap so that there are many buckets.
The gradients must be left as they were, the initial parameters must come
from rank 0, and each rank must hold only its share of the optimizer state.
The second step takes its gradients from a host buffer (step_from_host). A
run resumed from a state_dict after its first step must match the
uninterrupted run bit for bit. Two mistakes planted in the exchange (a sum
instead of an average, a missing all-gather) must each break the comparison.
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth
import adamw_hybrid_optimizer_muon_b200 as ma

H, E = ma.ROLE_HIDDEN, ma.ROLE_EMBED


def _desc(shape, role, group):
    t = ma.Tensor()
    t.ndim = len(shape)
    for d, s in enumerate(shape[:2]):
        t.shape[d] = s
    t.role, t.group = role, group
    return t


def _wl_descs_groups(name):
    wl = synth.WORKLOADS[name]()
    descs = [_desc(t.shape, t.role, t.group) for t in wl.tensors]
    groups = []
    for g in wl.groups:
        G = ma.Group()
        G.kind = g.kind
        if g.kind == ma.MA_MUON:
            G.muon = ma.muon_hparams(heads=g.muon.heads)
        else:
            G.adamw = ma.adamw_hparams()
        groups.append(G)
    return wl, descs, groups


def _numel(shape):
    return int(np.prod(shape)) if len(shape) else 1


def _align(x):
    return (x + ma.SHARD_ALIGN - 1) // ma.SHARD_ALIGN * ma.SHARD_ALIGN


def _check_layout(shapes, kinds, slots, buckets, total, world, seg_cap):
    A = ma.SHARD_ALIGN
    assert len(slots) == len(shapes)
    covered = np.zeros(total, dtype=np.int32) if total <= 1 << 24 else None
    firsts = []
    members = [[] for _ in buckets]
    for i, ((b, owner, off), shape, kind) in enumerate(zip(slots, shapes, kinds)):
        assert 0 <= b < len(buckets)
        members[b].append(i)
        bk, count, start, seg = buckets[b]
        assert bk == kind
        n = _numel(shape)
        assert off % A == 0
        if kind == ma.MA_MUON:
            assert 0 <= owner < world
            lo = start + owner * seg
            assert lo <= off and off + n <= lo + seg, "Muon matrix outside its owner's segment"
        else:
            assert owner == -1
            assert start <= off and off + n <= start + world * seg
        if covered is not None:
            covered[off:off + n] += 1
    if covered is not None:
        assert covered.max(initial=0) <= 1, "two tensors overlap"
    prev_end = 0
    for b, (kind, count, start, seg) in enumerate(buckets):
        assert count == len(members[b]) and count >= 1
        assert start == prev_end and start % A == 0 and seg % A == 0
        prev_end = start + world * seg
        firsts.append(min(members[b]))
        sizes = [_align(_numel(shapes[i])) for i in members[b]]
        if kind == ma.MA_ADAMW:
            assert seg == _align(-(-sum(sizes) // world))
            # closes before the tensor that would pass the cap
            if count > 1:
                assert -(-sum(sizes[:-1]) // world) <= seg_cap
        else:
            loads = [0] * world
            for i in members[b]:
                loads[slots[i][1]] += _align(_numel(shapes[i]))
            assert seg == max(loads)
    assert prev_end == total
    assert firsts == sorted(firsts)


@pytest.mark.parametrize("name,world,cap", [("7b", 1, 1 << 27), ("7b", 2, 1 << 27), ("7b", 8, 1 << 27),
                                            ("7b", 8, 1 << 30), ("d20", 3, 1 << 24), ("d20", 8, 1 << 22),
                                            ("aspect", 4, 1 << 26), ("tiny", 2, 1 << 20), ("square", 8, 1 << 26)])
def test_shard_layout_invariants(name, world, cap):
    wl, descs, groups = _wl_descs_groups(name)
    kinds = ma.ma_partition(descs)
    slots, buckets, total = ma.ma_shard_layout(descs, groups, world, cap)
    _check_layout([t.shape for t in wl.tensors], kinds, slots, buckets, total, world, cap)
    assert (slots, buckets, total) == ma.ma_shard_layout(descs, groups, world, cap)  # deterministic


@pytest.mark.parametrize("world", [1, 2, 4, 8])
def test_shard_layout_7b_muon_buckets_have_no_padding(world):
    # every Muon class of the 7B table (128, 64 and 32 matrices) divides by
    # 1, 2, 4 and 8 ranks; AdamW buckets pad at most to the next 64 x world
    wl, descs, groups = _wl_descs_groups("7b")
    slots, buckets, total = ma.ma_shard_layout(descs, groups, world, 1 << 27)
    used = [0] * len(buckets)
    for (b, _, _), t in zip(slots, wl.tensors):
        used[b] += _align(t.numel)
    for (kind, _, _, seg), u in zip(buckets, used):
        if kind == ma.MA_MUON:
            assert seg * world == u
        else:
            assert u <= seg * world < u + ma.SHARD_ALIGN * world


def test_shard_layout_mixed_bucket_packs_largest_first():
    # three classes with one matrix each on 2 ranks: one mixed bucket, the
    # largest matrix alone on rank 0, the two smaller on rank 1
    shapes = [(64, 256), (128, 256), (64, 128)]
    descs = [_desc(s, H, 0) for s in shapes]
    g = ma.Group()
    g.kind = ma.MA_MUON
    g.muon = ma.muon_hparams()
    slots, buckets, total = ma.ma_shard_layout(descs, [g], 2, 1 << 20)
    assert len(buckets) == 1 and buckets[0][:2] == (ma.MA_MUON, 3)
    assert [s[1] for s in slots] == [1, 0, 1]
    assert buckets[0][3] == 128 * 256
    assert slots[0][2] == 128 * 256 and slots[2][2] == 128 * 256 + 64 * 256  # order of appearance in a segment


def test_shard_layout_random_tables():
    r = np.random.default_rng(11)
    for _ in range(60):
        n = int(r.integers(1, 30))
        world = int(r.integers(1, 9))
        cap = int(r.choice([64, 1000, 5000, 1 << 20]))
        shapes, descs, kinds = [], [], []
        for _ in range(n):
            nd = int(r.integers(0, 3))
            shape = tuple(int(x) for x in r.choice([0, 1, 3, 8, 16, 40], size=nd))
            role = int(r.choice([H, H, E]))
            kind = ma.MA_MUON if nd == 2 and role == H else ma.MA_ADAMW
            shapes.append(shape)
            kinds.append(kind)
            descs.append(_desc(shape, role, 0 if kind == ma.MA_MUON else 1))
        gm, ga = ma.Group(), ma.Group()
        gm.kind, gm.muon = ma.MA_MUON, ma.muon_hparams()
        ga.kind, ga.adamw = ma.MA_ADAMW, ma.adamw_hparams()
        slots, buckets, total = ma.ma_shard_layout(descs, [gm, ga], world, cap)
        _check_layout(shapes, kinds, slots, buckets, total, world, cap)


def test_shard_layout_errors():
    g = ma.Group()
    g.kind, g.muon = ma.MA_MUON, ma.muon_hparams()
    d = [_desc((8, 8), H, 0)]
    for args, code in [((d, [g], 0, 64), ma.MA_ERR_ARG), ((d, [g], 2, 0), ma.MA_ERR_ARG),
                       (([_desc((8, 8), H, 1)], [g], 2, 64), ma.MA_ERR_ARG),
                       (([_desc((8,), H, 0)], [g], 2, 64), ma.MA_ERR_ARG),       # AdamW tensor in a Muon group
                       (([_desc((8, 8, 8), H, 0)], [g], 2, 64), ma.MA_ERR_UNSUPPORTED),
                       (([_desc((-1, 8), H, 0)], [g], 2, 64), ma.MA_ERR_SHAPE)]:
        with pytest.raises(ma.MAError) as e:
            ma.ma_shard_layout(*args)
        assert e.value.code == code
    assert ma.ma_shard_layout([], [g], 4, 64) == ([], [], 0)


# ---------------------------------------------------------------------------- the step on gloo ranks

TABLE = [  # (shape, role, group)
    ((1000, 64), E, 2),     # embedding: AdamW, straddles segments
    ((48, 96), H, 0), ((48, 96), H, 0), ((48, 96), H, 0),     # 3 of a class: mixed leftovers on 2 ranks
    ((96, 40), H, 0),       # transposed path (R > C)
    ((64, 96), H, 1), ((64, 96), H, 1),                      # per-head group (4 heads of 16 x 96)
    ((96,), H, 2), ((), H, 3), ((7,), H, 3),
    ((48, 96), H, 0),
    ((40, 96), H, 0),
    ((0, 16), H, 0), ((0,), H, 2),                           # empty tensors: placed, never updated
]


def _groups():
    return [("muon", ma.muon_hparams(lr=0.02, weight_decay=0.01)),
            ("muon", ma.muon_hparams(lr=0.01, heads=4, nesterov=False, scale_mode=1)),
            ("adamw", ma.adamw_hparams(lr=0.01, weight_decay=0.01)),
            ("adamw", ma.adamw_hparams(lr=0.003, weight_decay=0.0))]


Q = 2.0 ** -20


def _grads(step, rank, world):
    """Rank ``rank``'s gradients. On 2 ranks, any fp32 values (their average
    has a single rounding). On more, multiples of 2^-20 below 2^-8 whose sum
    over the ranks is world * K * 2^-20: every partial sum is exact in fp32,
    so the average is exactly K * 2^-20 whatever the order of reduction."""
    out = []
    for i, (s, _, _) in enumerate(TABLE):
        if world == 2:
            g = np.random.default_rng([step, rank, i]).standard_normal(s) * 1e-3
        else:
            r = np.random.default_rng([step, i])
            K = r.integers(-1000, 1001, size=s)
            parts = [r.integers(-1000, 1001, size=s) for _ in range(world - 1)]
            parts.append(world * K - sum(parts))
            g = parts[rank] * Q
        out.append(np.asarray(g, dtype=np.float32))
    return out


def _average(step, world):
    if world == 2:
        a, b = _grads(step, 0, 2), _grads(step, 1, 2)
        return [((torch.from_numpy(x) + torch.from_numpy(y)) / 2).numpy() for x, y in zip(a, b)]
    return [np.asarray(np.random.default_rng([step, i]).integers(-1000, 1001, size=s) * Q, dtype=np.float32)
            for i, (s, _, _) in enumerate(TABLE)]


def _oracle_update(group, W, g, s0, s1, step):
    """The oracle's update of one tensor (or piece) in place of the library's."""
    if group.kind == ma.MA_MUON:
        h = group.muon
        coeffs = [tuple(float(c) for c in h.coeffs[k]) for k in range(h.n_coeffs)]
        W1, m1 = oracle.muon_update(W, g, s0, h.lr, h.beta, h.weight_decay, bool(h.nesterov), h.ns_steps,
                                    coeffs, h.eps, h.scale_mode, h.heads, bool(h.cautious))
        return W1.astype(np.float32), m1.astype(np.float32), None
    h = group.adamw
    p1, m1, v1 = oracle.adamw_update(W, g, s0, s1, step, h.lr, h.beta1, h.beta2, h.eps, h.weight_decay)
    return p1.astype(np.float32), m1.astype(np.float32), v1.astype(np.float32)


class _DoneWork:
    def wait(self):
        return True


def _plant(mutation):
    """A planted mistake in the exchange (for the test that the comparison catches it)."""
    if mutation == "sum":  # gradients summed instead of averaged
        orig = dist.reduce_scatter_tensor

        def reduce_scatter_sum(out, inp, op=None, group=None, async_op=False):
            return orig(out, inp, op=dist.ReduceOp.SUM, group=group, async_op=async_op)
        dist.reduce_scatter_tensor = reduce_scatter_sum
    elif mutation == "no_gather":  # updated segments never leave their rank
        def skip_gather(out, inp, group=None, async_op=False):
            return _DoneWork()
        dist.all_gather_into_tensor = skip_gather


def _worker(rank, world, port, q, mutation=None):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    _plant(mutation)
    try:
        from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW

        class OracleDist(DistMuonAdamW):
            def _local_step(self, b):
                for pc in self.buckets[b].pieces:
                    grp = self.groups[pc.group]
                    s1 = None if pc.state1 is None else pc.state1.numpy()
                    W1, a, v = _oracle_update(grp, pc.param.numpy(), pc.grad.numpy(), pc.state0.numpy(), s1,
                                              grp.adamw.step)
                    pc.param.copy_(torch.from_numpy(W1))
                    pc.state0.copy_(torch.from_numpy(a))
                    if v is not None:
                        pc.state1.copy_(torch.from_numpy(v))

        init = np.random.default_rng(5 + rank)  # rank 1's own start must be replaced by rank 0's
        params = [torch.from_numpy(np.asarray(init.standard_normal(s) * 0.02, dtype=np.float32)) for s, _, _ in TABLE]
        opt = OracleDist([(p, role, g) for p, (_, role, g) in zip(params, TABLE)], _groups(),
                         seg_cap=2048)
        start = [p.clone() for p in params]
        out = {"start": [p.numpy().copy() for p in start], "steps": [], "state_elems": opt.state0.numel(),
               "nbuckets": len(opt.buckets), "pieces": [(pc.index, pc.lo, pc.hi) for pc in opt.pieces()]}
        host_flat = torch.zeros_like(opt.flat_grad)
        for step in (1, 2):
            G = _grads(step, rank, world)
            if step == 1:
                for g, v in zip(opt.grads, G):
                    g.copy_(torch.from_numpy(v))
                flat_before = opt.flat_grad.clone()
                opt.step()
            else:  # the second step takes its gradients from a host buffer
                for h, v in zip(opt.host_views(host_flat), G):
                    h.copy_(torch.from_numpy(v))
                opt.step_from_host(host_flat)
                flat_before = host_flat
            out["steps"].append({"params": [p.numpy().copy() for p in params],
                                 "grads_kept": bool(torch.equal(flat_before, opt.flat_grad)),
                                 "views": all(p.data_ptr() == opt.flat_param[s[2]:].data_ptr()
                                              for p, s in zip(params, opt.slots) if p.numel())})
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def _reference(world, start):
    groups = ma.group_table(_groups())
    P = [s.copy() for s in start]
    S0 = [np.zeros(s, np.float32) for s, _, _ in TABLE]
    S1 = [np.zeros(s, np.float32) for s, _, _ in TABLE]
    out = []
    for step in (1, 2):
        avg = _average(step, world)
        for i, (s, _, g) in enumerate(TABLE):
            if _numel(s) == 0:
                continue
            P[i], S0[i], v = _oracle_update(groups[g], P[i], avg[i], S0[i], S1[i], step)
            if v is not None:
                S1[i] = v
        out.append([p.copy() for p in P])
    return out


def _run_ranks(world, mutation=None):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q, mutation)) for r in range(world)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(60)
    return procs, results


@pytest.mark.parametrize("mutation", ["sum", "no_gather"])
def test_dist_comparison_catches_a_planted_exchange_mistake(mutation):
    procs, results = _run_ranks(2, mutation)
    assert all(p.exitcode == 0 for p in procs)
    ref = _reference(2, results[0]["start"])
    same = all(np.array_equal(got, want)
               for r in range(2) for k, st in enumerate(results[r]["steps"])
               for got, want in zip(st["params"], ref[k]))
    assert not same, f"planted mistake {mutation!r} went unnoticed"


@pytest.mark.parametrize("world", [2, 3])
def test_dist_step_matches_single_process_oracle(world):
    procs, results = _run_ranks(world)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]

    start = results[0]["start"]
    for r in range(world):  # every rank starts from rank 0's parameters
        for a, b in zip(results[r]["start"], start):
            assert np.array_equal(a, b)
    ref = _reference(world, start)
    for r in range(world):
        for k, st in enumerate(results[r]["steps"]):
            assert st["grads_kept"] and st["views"]
            for i, (got, want) in enumerate(zip(st["params"], ref[k])):
                assert np.array_equal(got, want), f"rank {r} step {k + 1} tensor {i}"
    # each element of each tensor is updated by exactly one rank
    counts = [np.zeros(_numel(s), np.int32) for s, _, _ in TABLE]
    for r in range(world):
        for i, lo, hi in results[r]["pieces"]:
            counts[i][lo:hi] += 1
    assert all((c == 1).all() for c in counts)
    # sharded state: each rank holds state for its own segments only, so the
    # ranks' state buffers together are exactly one flat copy of the model
    descs = [_desc(s, role, g) for s, role, g in TABLE]
    _, buckets, total = ma.ma_shard_layout(descs, ma.group_table(_groups()), world, 2048)
    assert results[0]["nbuckets"] == len(buckets)
    assert sum(results[r]["state_elems"] for r in range(world)) == total


@pytest.fixture
def gloo_one_rank():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    try:
        yield
    finally:
        dist.destroy_process_group()


def test_dist_host_side_one_rank(gloo_one_rank):
    from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW

    params = [torch.full(s, float(i), dtype=torch.float32) for i, (s, _, _) in enumerate(TABLE)]
    opt = DistMuonAdamW([(p, role, g) for p, (_, role, g) in zip(params, TABLE)], _groups(), seg_cap=2048)
    # the parameters moved into the flat buffer, values kept, tensors now views of it
    for i, (p, (_, _, off)) in enumerate(zip(params, opt.slots)):
        assert bool((p == float(i)).all())
        if p.numel():
            assert p.data_ptr() == opt.flat_param[off:].data_ptr()
    # one rank updates everything: its pieces are whole tensors (empty ones have
    # none), its state is the flat buffer
    assert sorted(pc.index for pc in opt.pieces()) == [i for i, (s, _, _) in enumerate(TABLE) if _numel(s)]
    assert all(pc.lo == 0 and pc.hi == _numel(TABLE[pc.index][0]) for pc in opt.pieces())
    assert opt.state0.numel() == opt.flat_param.numel()
    assert opt.state_bytes == 4 * (opt.state0.numel() + opt.state1.numel())
    host = torch.zeros_like(opt.flat_grad)
    views = opt.host_views(host)
    assert [tuple(v.shape) for v in views] == [tuple(g.shape) for g in opt.grads]
    text = opt.describe()
    assert text.startswith("rank 0 of 1:") and text.count("bucket ") == len(opt.buckets)
    with pytest.raises(ValueError):
        opt.step_from_host(torch.zeros(3))
    with pytest.raises(ValueError):
        DistMuonAdamW([(torch.zeros(8, 8, dtype=torch.float16), H, 0)], _groups())
    with pytest.raises(ValueError):
        DistMuonAdamW([], _groups())
    with pytest.raises(ValueError):
        DistMuonAdamW([(torch.zeros(8, 8), H, 0)], _groups(), grad_dtype=torch.float16)


def test_dist_backward_accumulates_into_flat_buffer(gloo_one_rank):
    # with fp32 gradients the parameters' .grad are views of the flat buffer:
    # backward writes (and accumulates) there, and zero_grad keeps the views
    from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW

    torch.manual_seed(0)
    lin = torch.nn.Linear(32, 16, bias=True)
    opt = DistMuonAdamW([(lin.weight, H, 0), (lin.bias, H, 1)],
                        [("muon", ma.muon_hparams()), ("adamw", ma.adamw_hparams())])
    x = torch.randn(8, 32)
    lin(x).square().sum().backward()
    g1 = [lin.weight.grad.clone(), lin.bias.grad.clone()]
    assert lin.weight.grad.data_ptr() == opt.grads[0].data_ptr()
    assert torch.equal(opt.grads[0], g1[0]) and torch.equal(opt.grads[1], g1[1])
    lin(x).square().sum().backward()
    assert torch.allclose(opt.grads[0], 2 * g1[0]) and torch.allclose(opt.grads[1], 2 * g1[1])
    opt.zero_grad()
    assert float(opt.flat_grad.abs().sum()) == 0.0
    assert lin.weight.grad.data_ptr() == opt.grads[0].data_ptr()


def _resume_worker(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from adamw_hybrid_optimizer_muon_b200.dist import DistMuonAdamW

        class OracleDist(DistMuonAdamW):
            def _local_step(self, b):
                for pc in self.buckets[b].pieces:
                    grp = self.groups[pc.group]
                    s1 = None if pc.state1 is None else pc.state1.numpy()
                    W1, a, v = _oracle_update(grp, pc.param.numpy(), pc.grad.numpy(), pc.state0.numpy(), s1,
                                              grp.adamw.step)
                    pc.param.copy_(torch.from_numpy(W1))
                    pc.state0.copy_(torch.from_numpy(a))
                    if v is not None:
                        pc.state1.copy_(torch.from_numpy(v))

        def make(start):
            params = [torch.from_numpy(x.copy()) for x in start]
            return params, OracleDist([(p, role, g) for p, (_, role, g) in zip(params, TABLE)], _groups(),
                                      seg_cap=2048)

        init = np.random.default_rng(5)
        start = [np.asarray(init.standard_normal(s) * 0.02, dtype=np.float32) for s, _, _ in TABLE]
        steps = 3
        # uninterrupted
        pa, oa = make(start)
        for step in range(1, steps + 1):
            for g, v in zip(oa.grads, _grads(step, rank, world)):
                g.copy_(torch.from_numpy(v))
            oa.step()
            if step == 1:
                saved = {k: (v.clone() if torch.is_tensor(v) else v) for k, v in oa.state_dict().items()}
                mid = [p.numpy().copy() for p in pa]
        # resumed after step 1 from the saved parameters and state
        pb, ob = make(mid)
        ob.load_state_dict(saved)
        for step in range(2, steps + 1):
            for g, v in zip(ob.grads, _grads(step, rank, world)):
                g.copy_(torch.from_numpy(v))
            ob.step()
        same = all(torch.equal(a, b) for a, b in zip(pa, pb))
        refused = False
        try:
            ob.load_state_dict(dict(saved, layout="other"))
        except ValueError:
            refused = True
        q.put((rank, same and refused and ob.step_count == steps))
    finally:
        dist.destroy_process_group()


def test_dist_resume_from_state_dict():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    procs = [ctx.Process(target=_resume_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=300) for _ in range(2))
    for p in procs:
        p.join(60)
    assert all(p.exitcode == 0 for p in procs)
    assert results == {0: True, 1: True}

