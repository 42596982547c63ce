"""C-ABI boundary tests that need no GPU.

The library must load, export every function that include/muonadamw.h
declares, agree with the binding on struct layouts, partition bit-exactly
like the oracle, and reject bad arguments with the documented status code
before it touches any memory. With valid arguments and no usable device, the
call must fail loudly (MA_ERR_CUDA / MA_ERR_UNSUPPORTED), never fall back.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth
import adamw_hybrid_optimizer_muon_b200 as ma

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "muonadamw.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\**\s+\**([a-z_][a-z0-9_]*)\s*\(", src, flags=re.M)
    return sorted(set(names))


def test_header_symbols_exported():
    names = declared_functions()
    assert len(names) >= 15
    L = ma.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in muonadamw.h but not exported"


def test_debug_build_loads_and_exports_the_same_abi():
    # the debug library (guarded device indexing) is built beside the release
    # one; each reports which it is, and the debug one exports every symbol too
    assert ma.ma_debug_build() == (os.environ.get("MA_LIBRARY") == "debug")
    dbg = os.path.join(os.path.dirname(ma.LIB_PATH), "libmuonadamw_debug.so")
    D = ctypes.CDLL(dbg)
    for n in declared_functions():
        assert hasattr(D, n), f"{n} not exported by the debug build"
    D.ma_debug_build.restype = ctypes.c_int
    D.ma_status_string.restype = ctypes.c_char_p
    assert D.ma_debug_build() == 1
    assert D.ma_status_string(ma.MA_ERR_BOUNDS) == b"guarded device index out of bounds (debug build)"
    assert ma.lib().ma_status_string(ma.MA_ERR_BOUNDS) == b"guarded device index out of bounds (debug build)"


def test_binding_constants_match_header_macros():
    # the binding's copies of the header's size constants (the allocation-free
    # entry point's scratch size among them) must be the header's values
    src = open(HEADER).read()

    def macro(name):
        m = re.search(r"#define\s+" + name + r"\s+(.+)", src)
        assert m, name
        expr = re.sub(r"\((?:size_t|int64_t|int)\)", "", m.group(1).split("/*")[0])
        return int(eval(expr, {"__builtins__": {}}))  # plain integer arithmetic of the macro

    assert ma.STATIC_SCRATCH_BYTES == macro("MA_STATIC_SCRATCH_BYTES")
    assert ma.SHARD_ALIGN == macro("MA_SHARD_ALIGN")
    assert ma.MAX_NS_STEPS == macro("MA_MAX_NS_STEPS")
    assert ma.MAX_GROUPS == macro("MA_MAX_GROUPS")
    assert ma.MAX_BATCH == macro("MA_MAX_BATCH")
    assert len(ma.PROF_CLASSES) == macro("MA_PROF_CLASSES")


def test_struct_layouts_match():
    L = ma.lib()
    for which, cls in enumerate((ma.Tensor, ma.Group, ma.MuonHParams, ma.AdamWHParams)):
        assert L.ma_struct_size(which) == ctypes.sizeof(cls)
    assert L.ma_version() == 1
    assert L.ma_status_string(8) == b"device wait timed out"


def _desc(shape, role, group=0):
    t = ma.Tensor()
    t.ndim = len(shape)
    for d, s in enumerate(shape[:2]):
        t.shape[d] = s
    t.role = role
    t.group = group
    return t


@pytest.mark.parametrize("name", ["tiny", "d20", "7b", "aspect", "square"])
def test_partition_bit_exact_vs_oracle(name):
    wl = synth.WORKLOADS[name]()
    descs = [_desc(t.shape, t.role, t.group) for t in wl.tensors]
    assert ma.ma_partition(descs) == oracle.partition([(t.shape, t.role) for t in wl.tensors])


def test_partition_random_tables():
    r = np.random.default_rng(0)
    for _ in range(50):
        n = int(r.integers(1, 40))
        table = []
        for _ in range(n):
            nd = int(r.integers(0, 3))
            shape = tuple(int(x) for x in r.integers(0, 9, size=nd))
            table.append((shape, int(r.integers(0, 4))))
        got = ma.ma_partition([_desc(s, ro) for s, ro in table])
        assert got == oracle.partition(table)


def test_partition_rejects_rank3():
    with pytest.raises(ma.MAError) as e:
        ma.ma_partition([_desc((2, 3), 0), _desc((2, 3, 4), 0)])
    assert e.value.code == ma.MA_ERR_UNSUPPORTED


def _groups_for(wl):
    gs = []
    for g in wl.groups:
        G = ma.Group()
        G.kind = g.kind
        if g.kind == ma.MA_MUON:
            h = g.muon
            G.muon = ma.muon_hparams(h.lr, h.beta, h.weight_decay, h.eps, h.nesterov, h.ns_steps, h.coeffs,
                                     h.scale_mode, h.heads, h.precision)
        else:
            h = g.adamw
            G.adamw = ma.adamw_hparams(h.lr, h.beta1, h.beta2, h.eps, h.weight_decay, 1)
        gs.append(G)
    return gs


@pytest.mark.parametrize("name,world", [("7b", 1), ("7b", 2), ("7b", 8), ("d20", 3), ("aspect", 4), ("tiny", 2)])
def test_owner_assignment_exactly_once_and_balanced(name, world):
    wl = synth.WORKLOADS[name]()
    descs = [_desc(t.shape, t.role, t.group) for t in wl.tensors]
    owners = ma.ma_assign_owners(descs, _groups_for(wl), world)
    assert len(owners) == len(descs)
    assert all(0 <= o < world for o in owners)
    assert owners == ma.ma_assign_owners(descs, _groups_for(wl), world)  # deterministic
    # greedy bound: the heaviest rank exceeds the average by at most the largest item
    kinds = oracle.partition([(t.shape, t.role) for t in wl.tensors])
    for kind in (0, 1):
        items = [t.numel for t, k in zip(wl.tensors, kinds) if k == kind]
        if not items or kind == 0:
            continue
        load = [0] * world
        for t, k, o in zip(wl.tensors, kinds, owners):
            if k == kind:
                load[o] += t.numel
        assert max(load) <= sum(items) / world + max(items)


def test_validation_before_any_device_call():
    hp = ma.muon_hparams()
    L = ma.lib()
    fake = ctypes.c_void_p(0x1000)
    arr = (ctypes.c_void_p * 1)(0x100000)   # weights / AdamW params
    garr = (ctypes.c_void_p * 1)(0x200000)  # gradients
    marr = (ctypes.c_void_p * 1)(0x300000)  # momentum / exp_avg
    varr = (ctypes.c_void_p * 1)(0x400000)  # exp_avg_sq
    null = (ctypes.c_void_p * 1)(0)
    # C % 8 != 0
    rc = L.muon_step_batched(1, 16, 12, arr, garr, ma.MA_F32, marr, ctypes.byref(hp), fake, 1 << 30, None)
    assert rc == ma.MA_ERR_ALIGN
    # null pointer entry
    rc = L.muon_step_batched(1, 16, 16, null, garr, ma.MA_F32, marr, ctypes.byref(hp), fake, 1 << 30, None)
    assert rc == ma.MA_ERR_NULL
    # heads must divide R
    hp3 = ma.muon_hparams(heads=3)
    rc = L.muon_step_batched(1, 16, 16, arr, garr, ma.MA_F32, marr, ctypes.byref(hp3), fake, 1 << 30, None)
    assert rc == ma.MA_ERR_SHAPE
    # bad dtype, bad steps, bad coefficient count
    assert L.muon_step_batched(1, 16, 16, arr, garr, 7, marr, ctypes.byref(hp), fake, 1 << 30, None) == ma.MA_ERR_DTYPE
    bad = ma.muon_hparams(ns_steps=0)
    assert L.muon_step_batched(1, 16, 16, arr, garr, 0, marr, ctypes.byref(bad), fake, 1 << 30, None) == ma.MA_ERR_ARG
    bad = ma.muon_hparams(ns_steps=3, coeffs=((1.5, -0.5, 0), (1.5, -0.5, 0)))
    assert L.muon_step_batched(1, 16, 16, arr, garr, 0, marr, ctypes.byref(bad), fake, 1 << 30, None) == ma.MA_ERR_ARG
    # workspace too small / misaligned
    assert L.muon_step_batched(1, 16, 16, arr, garr, 0, marr, ctypes.byref(hp), fake, 16, None) == ma.MA_ERR_WORKSPACE
    assert L.muon_step_batched(1, 16, 16, arr, garr, 0, marr, ctypes.byref(hp), ctypes.c_void_p(0x1008), 1 << 30,
                               None) == ma.MA_ERR_WORKSPACE
    # empty batch is a no-op
    assert L.muon_step_batched(0, 16, 16, arr, garr, 0, marr, ctypes.byref(hp), None, 0, None) == ma.MA_OK
    # AdamW: bad step, bad betas
    ahp = ma.adamw_hparams(step=0)
    n1 = (ctypes.c_int64 * 1)(4)
    assert L.adamw_step_fused(1, arr, garr, 0, marr, varr, n1, ctypes.byref(ahp), None) == ma.MA_ERR_ARG
    ahp = ma.adamw_hparams(beta2=1.0)
    assert L.adamw_step_fused(1, arr, garr, 0, marr, varr, n1, ctypes.byref(ahp), None) == ma.MA_ERR_ARG
    ahp = ma.adamw_hparams()
    assert L.adamw_step_fused(1, null, garr, 0, marr, varr, n1, ctypes.byref(ahp), None) == ma.MA_ERR_NULL
    # buffers the call writes must be disjoint
    assert L.muon_step_batched(1, 16, 16, arr, garr, 0, arr, ctypes.byref(hp), fake, 1 << 30, None) == ma.MA_ERR_ARG
    two = (ctypes.c_void_p * 2)(0x100000, 0x100000 + 512)  # second matrix starts inside the first
    m2 = (ctypes.c_void_p * 2)(0x300000, 0x310000)
    g2 = (ctypes.c_void_p * 2)(0x200000, 0x210000)
    assert L.muon_step_batched(2, 16, 16, two, g2, 0, m2, ctypes.byref(hp), fake, 1 << 30, None) == ma.MA_ERR_ARG
    assert L.adamw_step_fused(1, arr, garr, 0, marr, marr, n1, ctypes.byref(ahp), None) == ma.MA_ERR_ARG


def test_valid_call_without_gpu_fails_loudly():
    try:
        import torch
        if torch.cuda.is_available():
            pytest.skip("a GPU is present")
    except ImportError:
        pass
    hp = ma.muon_hparams()
    L = ma.lib()
    w, g, m = ((ctypes.c_void_p * 1)(a) for a in (0x100000, 0x200000, 0x300000))
    rc = L.muon_step_batched(1, 16, 16, w, g, 0, m, ctypes.byref(hp), ctypes.c_void_p(0x10000), 1 << 30, None)
    assert rc in (ma.MA_ERR_CUDA, ma.MA_ERR_UNSUPPORTED)


def test_plan_sizing_on_host():
    wl = synth.llama7b()
    descs = []
    for i, t in enumerate(wl.tensors):
        d = _desc(t.shape, t.role, t.group)
        d.param, d.state0, d.state1, d.grad = (((4 * i + k + 1) << 32) for k in range(4))  # disjoint fake buffers
        d.grad_dtype = ma.MA_BF16
        descs.append(d)
    plan, ws = ma.ma_plan_create(descs, _groups_for(wl))
    hp = ma.muon_hparams()

    def sub(n, R, C):  # without a cap, sub-batches are halved to at most 4 GiB of workspace
        while ma.muon_workspace_bytes(n, R, C, hp) > 4 << 30 and n > 1:
            n //= 2
        return n
    assert (sub(128, 4096, 4096), sub(64, 4096, 11008), sub(32, 11008, 4096)) == (32, 16, 16)
    expect = max(ma.muon_workspace_bytes(32, 4096, 4096, hp), ma.muon_workspace_bytes(16, 4096, 11008, hp),
                 ma.muon_workspace_bytes(16, 11008, 4096, hp))
    # one workspace for the largest sub-batch, used by the sub-batches in turn
    assert ws == expect
    ma.ma_plan_destroy(plan)
    # a cap splits buckets into sub-batches that fit in it
    plan, ws2 = ma.ma_plan_create(descs, _groups_for(wl), ws_cap=1 << 30)
    assert 0 < ws2 <= 1 << 30
    ma.ma_plan_destroy(plan)
    with pytest.raises(ma.MAError) as e:
        ma.ma_plan_create(descs, _groups_for(wl), ws_cap=1 << 20)
    assert e.value.code == ma.MA_ERR_WORKSPACE
    # momentum overlap: ten Muon sub-batches get two halves, so that each
    # sub-batch's momentum pass can run under the chain of the one before it
    ma.ma_set_momentum_overlap(True)
    try:
        plan, ws = ma.ma_plan_create(descs, _groups_for(wl))
        assert ws == 2 * ((expect + 255) // 256 * 256)
        ma.ma_plan_destroy(plan)
        # a cap bounds the two halves together
        plan, ws2 = ma.ma_plan_create(descs, _groups_for(wl), ws_cap=4 << 30)
        assert 0 < ws2 <= 4 << 30
        ma.ma_plan_destroy(plan)
        plan, ws3 = ma.ma_plan_create(descs, _groups_for(wl), ws_cap=2 * ((expect + 255) // 256 * 256))
        assert ws3 == 2 * ((expect + 255) // 256 * 256)
        ma.ma_plan_destroy(plan)
        # a cap below two halves of the largest single matrix: one workspace
        one = max(ma.muon_workspace_bytes(1, 4096, 11008, hp), ma.muon_workspace_bytes(1, 11008, 4096, hp))
        plan, ws4 = ma.ma_plan_create(descs, _groups_for(wl), ws_cap=one + 4096)
        assert ws4 <= one + 4096
        ma.ma_plan_destroy(plan)
    finally:
        ma.ma_set_momentum_overlap(False)
    with pytest.raises(ma.MAError) as e:
        ma._check(ma.lib().ma_set_momentum_overlap(2), "ma_set_momentum_overlap")
    assert e.value.code == ma.MA_ERR_ARG


def _fake_descs(wl):
    descs = []
    for i, t in enumerate(wl.tensors):
        d = _desc(t.shape, t.role, t.group)
        d.param, d.state0, d.state1, d.grad = (((4 * i + k + 1) << 32) for k in range(4))
        d.grad_dtype = ma.MA_BF16
        descs.append(d)
    return descs


def test_plan_describe():
    wl = synth.llama7b()
    plan, ws = ma.ma_plan_create(_fake_descs(wl), _groups_for(wl))
    text = ma.ma_plan_describe(plan, _groups_for(wl))
    ma.ma_plan_destroy(plan)
    assert text.startswith(f"workspace {ws} bytes; AdamW: 67 tensors, ")
    assert "4096 x 4096, 128 matrices (bf16 grads), heads 1, sub-batches of 32, direct chain" in text
    assert "4096 x 11008, 64 matrices (bf16 grads), heads 1, sub-batches of 16, Gram-space chain" in text
    assert "11008 x 4096, 32 matrices (bf16 grads), heads 1, sub-batches of 16, Gram-space chain" in text
    segs = [ln for ln in text.splitlines() if ln.startswith("segment")]
    assert segs[0] == "segment 0: AdamW" and len(segs) == 1 + 4 + 4 + 2  # no sharing at this size
    ma.ma_set_momentum_overlap(True)
    try:
        plan, ws = ma.ma_plan_create(_fake_descs(wl), _groups_for(wl))
        text = ma.ma_plan_describe(plan, _groups_for(wl))
        ma.ma_plan_destroy(plan)
    finally:
        ma.ma_set_momentum_overlap(False)
    assert text.startswith(f"workspace {ws} bytes in two halves of {ws // 2} (momentum passes under the previous "
                           f"chain); AdamW: 67 tensors, ")
    # the d20 set: its three buckets share one chain of Newton-Schulz launches
    wl = synth.d20()
    plan, _ = ma.ma_plan_create(_fake_descs(wl), _groups_for(wl))
    text = ma.ma_plan_describe(plan, _groups_for(wl))
    ma.ma_plan_destroy(plan)
    segs = [ln for ln in text.splitlines() if ln.startswith("segment")]
    assert len(segs) == 2 and segs[1].count("[bucket") == 3, text


def test_plan_group_table_limits():
    """MA_MAX_GROUPS groups are accepted, one more is refused before anything is built."""
    def groups(k):
        out = []
        for i in range(k):
            G = ma.Group()
            G.kind = ma.MA_ADAMW if i % 2 else ma.MA_MUON
            if G.kind == ma.MA_MUON:
                G.muon = ma.muon_hparams(lr=0.01 * (i + 1))
            else:
                G.adamw = ma.adamw_hparams(lr=0.001 * (i + 1))
            out.append(G)
        return out
    descs = []
    for i in range(32):
        d = _desc((64, 128) if i % 2 == 0 else (128,), ma.ROLE_HIDDEN, i)
        d.param, d.state0, d.state1, d.grad = (((4 * i + k + 1) << 32) for k in range(4))
        d.grad_dtype = ma.MA_BF16
        descs.append(d)
    plan, ws = ma.ma_plan_create(descs, groups(32))
    text = ma.ma_plan_describe(plan, groups(32))
    ma.ma_plan_destroy(plan)
    lines = text.splitlines()
    assert sum(ln.startswith("bucket ") for ln in lines) == 16  # one 64 x 128 bucket per Muon group
    segs = [ln for ln in lines if ln.startswith("segment")]
    # the 16 small buckets share launches, eight jobs at most per launch
    assert len(segs) == 3 and segs[1].count("[bucket") == 8 and segs[2].count("[bucket") == 8
    with pytest.raises(ma.MAError) as e:
        ma.ma_plan_create(descs, groups(33))
    assert e.value.code == ma.MA_ERR_UNSUPPORTED


def test_plan_rejects_overlapping_written_buffers():
    wl = synth.tiny()

    def desc(shape, role, group, base):
        d = _desc(shape, role, group)
        d.param, d.state0, d.state1, d.grad = base, base + (1 << 30), base + (2 << 30), base + (3 << 30)
        return d
    a = desc((256, 512), ma.ROLE_HIDDEN, 0, 1 << 36)
    b = desc((512,), ma.ROLE_HIDDEN, 1, 2 << 36)
    plan, _ = ma.ma_plan_create([a, b], _groups_for(wl))  # disjoint: accepted
    ma.ma_plan_destroy(plan)
    c = desc((512,), ma.ROLE_HIDDEN, 1, 2 << 36)
    c.param = a.param + 256 * 512 * 4 - 4  # starts inside the last element of a's parameter
    with pytest.raises(ma.MAError) as e:
        ma.ma_plan_create([a, c], _groups_for(wl))
    assert e.value.code == ma.MA_ERR_ARG
    with pytest.raises(ma.MAError) as e:
        ma.ma_plan_create([a, a], _groups_for(wl))  # the same tensor twice
    assert e.value.code == ma.MA_ERR_ARG
    d = desc((512,), ma.ROLE_HIDDEN, 1, 3 << 36)
    d.state1 = d.state0  # exp_avg and exp_avg_sq in one buffer
    with pytest.raises(ma.MAError) as e:
        ma.ma_plan_create([a, d], _groups_for(wl))
    assert e.value.code == ma.MA_ERR_ARG


def test_plan_rejects_kind_mismatch():
    wl = synth.tiny()
    d0 = _desc((256, 512), ma.ROLE_HIDDEN, 1)  # a Muon matrix in the AdamW group
    d0.param = d0.state0 = d0.state1 = d0.grad = 0x100000
    with pytest.raises(ma.MAError) as e:
        ma.ma_plan_create([d0], _groups_for(wl))
    assert e.value.code == ma.MA_ERR_ARG


def test_muonadamw_state_dict_roundtrip_on_host():
    # the optimizer object and its state buffers can be built without a GPU
    # (the plan, and with it the library's device work, is made on the first step)
    import torch
    params = [torch.randn(16, 32), torch.randn(32), torch.randn(8, 16)]
    table = [(params[0], ma.ROLE_HIDDEN, 0), (params[1], ma.ROLE_HIDDEN, 1), (params[2], ma.ROLE_EMBED, 1)]
    groups = [("muon", ma.muon_hparams()), ("adamw", ma.adamw_hparams())]
    a = ma.MuonAdamW(table, groups)
    assert [s1 is None for _, s1 in a.state] == [True, False, False]
    for s0, s1 in a.state:
        s0.normal_()
        if s1 is not None:
            s1.uniform_()
    a.step_count = 7
    b = ma.MuonAdamW(table, groups)
    b.load_state_dict(a.state_dict())
    assert b.step_count == 7
    for (a0, a1), (b0, b1) in zip(a.state, b.state):
        assert torch.equal(a0, b0) and a0.data_ptr() != b0.data_ptr()
        assert (a1 is None and b1 is None) or torch.equal(a1, b1)
    c = ma.MuonAdamW(table[:2], groups)
    with pytest.raises(ValueError):
        c.load_state_dict(a.state_dict())


def test_plan_status_without_gpu_fails_loudly():
    assert ma.lib().ma_plan_status(None, None) == ma.MA_ERR_NULL
    wl = synth.tiny()
    plan, _ = ma.ma_plan_create(_fake_descs(wl), _groups_for(wl))
    try:
        assert ma.ma_plan_status(plan, 0) == ma.MA_ERR_CUDA  # no device: an error, never a fake OK
    finally:
        ma.ma_plan_destroy(plan)


@pytest.mark.parametrize("shape,heads,kw,gspace", [
    ((512, 1024), 1, {}, True),                      # m n = 2^19 exactly, n = 2 m
    ((1024, 512), 1, {}, True),                      # tall: the unit is its transpose
    ((512, 1016), 1, {}, False),                     # m n below 2^19
    ((672, 840), 1, {}, True),                       # 4 n = 5 m exactly (m n above 2^19)
    ((672, 832), 1, {}, False),                      # 4 n < 5 m
    ((1024, 1024), 1, {}, False),                    # square
    ((128, 4096), 1, {}, True),                      # m = 128
    ((120, 4400), 1, {}, False),                     # m < 128
    ((4096, 4096), 32, {}, True),                    # head slices of 128 x 4096
    ((512, 1024), 1, {"precision": 1}, False),       # fp32 mode keeps the direct chain
    ((512, 1024), 1, {"coeffs": ((2.0, -1.5, 0.5),)}, False),  # c != 0
])
def test_gram_space_selection(shape, heads, kw, gspace):
    # which units take the Gram-space chain: m >= 128, 4 n >= 5 m and
    # m n >= 2^19 (m the short side of a unit), bf16 operands, no c term
    d = _desc(shape, ma.ROLE_HIDDEN, 0)
    d.param, d.state0, d.state1, d.grad = (1 << 32), (2 << 32), (3 << 32), (4 << 32)
    d.grad_dtype = ma.MA_BF16
    G = ma.Group()
    G.kind = ma.MA_MUON
    G.muon = ma.muon_hparams(heads=heads, **kw)
    plan, _ = ma.ma_plan_create([d], [G])
    text = ma.ma_plan_describe(plan, [G])
    ma.ma_plan_destroy(plan)
    assert ("Gram-space chain" in text) == gspace, text
    assert ("direct chain" in text) == (not gspace), text
