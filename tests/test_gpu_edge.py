"""Edge cases of the whole step on the GPU, against the oracle or bit for bit.

* a mixed parameter table: bf16 and fp32 gradients of one shape (separate
  buckets), a per-head fp32-mode group, an embedding, a bias, a 0-D scalar in
  a group without weight decay, and empty tensors;
* a workspace cap that splits buckets into sub-batches, and a bucket of more
  than 256 matrices: results bit-identical to the unsplit plan;
* 1 and 16 Newton-Schulz iterations;
* resume: k steps, state copied into fresh buffers, more steps, bit for bit;
* fp32 mode on larger matrices (1e-5);
* shared Newton-Schulz launches (grouped buckets) against one call per bucket,
  bit for bit;
* a muon_step_batched call beyond 4 GiB of workspace (run as sub-batches)
  against two smaller calls, bit for bit;
* degenerate shapes: a single row, 8 x 8, very tall and very wide matrices.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import synth
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import (TOL_BF16, TOL_F32, bf16_round, check_muon, check_state, dev_f32, dev_grad, f32, host,
                         momentum_terms)

pytestmark = pytest.mark.gpu


def _mhp(**kw):
    base = dict(lr=0.02, beta=0.95, weight_decay=0.01, eps=1e-7, nesterov=True, ns_steps=5,
                coeffs=((1.5, -0.5, 0.0),), scale_mode=0, heads=1, precision=0)
    base.update(kw)
    return base


def _ahp(**kw):
    base = dict(lr=0.01, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01)
    base.update(kw)
    return base


def _as32(d):
    return {k: (f32(v) if isinstance(v, float) else v) for k, v in d.items()}


def test_mixed_table_two_steps():
    r = np.random.default_rng(200)
    H, E = ma.ROLE_HIDDEN, ma.ROLE_EMBED
    # (shape, role, group, grad dtype)
    table = [((256, 512), H, 0, "bf16"), ((256, 512), H, 0, "f32"), ((384, 128), H, 1, "bf16"),
             ((1000, 64), E, 2, "bf16"), ((37,), H, 2, "bf16"), ((), H, 3, "f32"), ((0,), H, 2, "bf16"),
             ((0, 16), H, 0, "bf16"), ((256, 512), H, 0, "bf16")]
    mg = [_mhp(), _mhp(heads=2, precision=1, nesterov=False, scale_mode=1)]
    ag = [_ahp(), _ahp(lr=0.003, weight_decay=0.0)]
    groups = [("muon", ma.muon_hparams(**mg[0])), ("muon", ma.muon_hparams(**mg[1])),
              ("adamw", ma.adamw_hparams(**ag[0])), ("adamw", ma.adamw_hparams(**ag[1]))]
    P0 = [(r.standard_normal(s) * 0.02).astype(np.float32) for s, *_ in table]
    params = [dev_f32(p) for p in P0]
    opt = ma.MuonAdamW([(p, role, g) for p, (s, role, g, _) in zip(params, table)], groups)
    og = [dict(kind=0, **_as32(mg[0])), dict(kind=0, **_as32(mg[1])), dict(kind=1, **_as32(ag[0])),
          dict(kind=1, **_as32(ag[1]))]
    for step in (1, 2):
        G = [bf16_round(r.standard_normal(s) * 1e-3) for s, *_ in table]
        Gd = [dev_grad(g, dt) for g, (_, _, _, dt) in zip(G, table)]
        before_p = [host(p) for p in params]
        before_s = [(host(a), None if b is None else host(b)) for a, b in opt.state]
        opt.step(Gd)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for i, ((shape, role, g, _), p) in enumerate(zip(table, params)):
            grp = og[g]
            if grp["kind"] == 0:
                if before_p[i].size == 0:
                    continue
                rw, rm = oracle.muon_update(before_p[i], G[i], before_s[i][0], grp["lr"], grp["beta"],
                                            grp["weight_decay"], grp["nesterov"], grp["ns_steps"], grp["coeffs"],
                                            grp["eps"], grp["scale_mode"], grp["heads"])
                check_muon(before_p[i], host(p), rw, grp["lr"], grp["weight_decay"],
                           TOL_F32 if grp["precision"] else TOL_BF16, what=f"tensor {i}")
                check_state(host(opt.state[i][0]), rm, momentum_terms(before_s[i][0], G[i], grp["beta"]))
            else:
                args = (step, grp["lr"], grp["beta1"], grp["beta2"], grp["eps"], grp["weight_decay"])
                rp, rm, rv = oracle.adamw_update(before_p[i], G[i], before_s[i][0], before_s[i][1], *args)
                tp, tm, tv = oracle.adamw_term_magnitudes(before_p[i], G[i], before_s[i][0], before_s[i][1], *args)
                check_state(host(p).reshape(-1), rp.reshape(-1), tp.reshape(-1), what=f"tensor {i}")
                check_state(host(opt.state[i][0]).reshape(-1), rm.reshape(-1), tm.reshape(-1))
                check_state(host(opt.state[i][1]).reshape(-1), rv.reshape(-1), tv.reshape(-1))


def _run_bucket(shapes_count, steps, ws_cap=0, seed=1):
    (R, C), n = shapes_count
    r = np.random.default_rng(seed)
    params = [dev_f32(r.standard_normal((R, C)) * 0.02) for _ in range(n)]
    opt = ma.MuonAdamW([(p, ma.ROLE_HIDDEN, 0) for p in params], [("muon", ma.muon_hparams())], ws_cap=ws_cap)
    for s in range(steps):
        gr = np.random.default_rng(seed * 100 + s)
        opt.step([dev_grad(bf16_round(gr.standard_normal((R, C)) * 1e-3), "bf16") for _ in range(n)])
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
    return params, opt


def test_workspace_cap_sub_batches_are_bit_identical():
    full, _ = _run_bucket(((256, 512), 7), 2)
    per2 = ma.muon_workspace_bytes(2, 256, 512, ma.muon_hparams())
    capped, opt = _run_bucket(((256, 512), 7), 2, ws_cap=per2)
    assert opt._plan.ws_bytes <= per2
    for a, b in zip(full, capped):
        assert torch.equal(a, b)


def test_bucket_of_more_than_256_matrices():
    params, _ = _run_bucket(((64, 128), 300), 1, seed=3)
    r = np.random.default_rng(3)
    W0 = [r.standard_normal((64, 128)) * 0.02 for _ in range(300)]
    gr = np.random.default_rng(300)
    G = [bf16_round(gr.standard_normal((64, 128)) * 1e-3) for _ in range(300)]
    hp = synth.MuonHP()
    for i in (0, 255, 256, 299):  # both sides of the 256-matrix launch split
        w0 = W0[i].astype(np.float32).astype(np.float64)
        rw, _ = oracle.muon_update(w0, G[i], np.zeros((64, 128)), f32(hp.lr), f32(hp.beta), f32(hp.weight_decay),
                                   eps=f32(hp.eps))
        check_muon(w0, host(params[i]), rw, f32(hp.lr), f32(hp.weight_decay), TOL_BF16, what=f"matrix {i}")


@pytest.mark.parametrize("steps", [1, 16])
def test_ns_step_counts(steps):
    R, C = 256, 512
    r = np.random.default_rng(10 + steps)
    W0 = (r.standard_normal((R, C)) * 0.02).astype(np.float32)
    g = bf16_round(r.standard_normal((R, C)) * 1e-3)
    hp = ma.muon_hparams(ns_steps=steps)
    Wd, Md = [dev_f32(W0)], [torch.zeros((R, C), device="cuda")]
    ws = torch.empty(ma.muon_workspace_bytes(1, R, C, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, [dev_grad(g, "bf16")], Md, hp, ws)
    torch.cuda.synchronize()
    rw, _ = oracle.muon_update(W0, g, np.zeros((R, C)), f32(0.02), f32(0.95), f32(0.01), steps=steps, eps=f32(1e-7))
    check_muon(W0, host(Wd[0]), rw, f32(0.02), f32(0.01), TOL_BF16)


def test_resume_from_copied_state_is_bit_identical():
    wl = synth.tiny()
    W0 = [synth.initial_weight(t, i) for i, t in enumerate(wl.tensors)]
    grads = [[torch.from_numpy(synth.gradient(wl, i, s)).cuda() for i in range(2)] for s in (1, 2, 3)]

    def make(params):
        gm, ga = wl.groups[0].muon, wl.groups[1].adamw
        return ma.MuonAdamW([(p, t.role, t.group) for p, t in zip(params, wl.tensors)],
                            [("muon", ma.muon_hparams()), ("adamw", ma.adamw_hparams(ga.lr, ga.beta1, ga.beta2,
                                                                                      ga.eps, ga.weight_decay))])
    pa = [torch.from_numpy(w).cuda() for w in W0]
    oa = make(pa)
    for g in grads:
        oa.step(g)
    pb = [torch.from_numpy(w).cuda() for w in W0]
    ob = make(pb)
    for g in grads[:2]:
        ob.step(g)
    torch.cuda.synchronize()
    # fresh buffers holding the copied parameters and state
    pc = [p.clone() for p in pb]
    oc = make(pc)
    for (s0, s1), (t0, t1) in zip(ob.state, oc.state):
        t0.copy_(s0)
        if s1 is not None:
            t1.copy_(s1)
    oc.step_count = ob.step_count
    oc.step(grads[2])
    torch.cuda.synchronize()
    for x, y in zip(pa, pc):
        assert torch.equal(x, y)
    for (s0, s1), (t0, t1) in zip(oa.state, oc.state):
        assert torch.equal(s0, t0) and (s1 is None or torch.equal(s1, t1))


@pytest.mark.parametrize("shape", [(4096, 11008), (11008, 4096)])
def test_fp32_mode_7b_mlp_shapes_exact_update(shape):
    """fp32 mode on the 7B-shaped set's MLP matrices (the longest K loops of the
    fp32 kernels; 11008 x 4096 takes the transpose path), at the 1e-5 bound
    with no allowance: from W = 0 the step writes W_new = -lr * scale * X_N,
    whose only rounding beyond the update itself is one fp32 product, so the
    fp32 storage of the weights puts no floor under the measured error."""
    r = np.random.default_rng(21)
    W0 = np.zeros(shape, np.float32)
    g = (r.standard_normal(shape) * 1e-3).astype(np.float32)
    hp = ma.muon_hparams(precision=1)
    Wd, Md = [dev_f32(W0)], [torch.zeros(shape, device="cuda")]
    ws = torch.empty(ma.muon_workspace_bytes(1, *shape, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, [dev_f32(g)], Md, hp, ws)
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
    rw, _ = oracle.muon_update(W0, g, np.zeros(shape), f32(0.02), f32(0.95), f32(0.01), eps=f32(1e-7))
    d_gpu, d_ref = host(Wd[0]), rw  # W_old = 0: the update is W_new itself
    err = np.linalg.norm(d_gpu - d_ref) / np.linalg.norm(d_ref)
    assert err <= TOL_F32, f"fp32-mode update relative error {err:.3e} > {TOL_F32}"


@pytest.mark.parametrize("shape", [(1024, 2048), (2048, 1024)])
def test_fp32_mode_larger(shape):
    r = np.random.default_rng(20)
    W0 = (r.standard_normal(shape) * 0.02).astype(np.float32)
    g = (r.standard_normal(shape) * 1e-3).astype(np.float32)
    hp = ma.muon_hparams(precision=1)
    Wd, Md = [dev_f32(W0)], [torch.zeros(shape, device="cuda")]
    ws = torch.empty(ma.muon_workspace_bytes(1, *shape, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, [dev_f32(g)], Md, hp, ws)
    torch.cuda.synchronize()
    rw, _ = oracle.muon_update(W0, g, np.zeros(shape), f32(0.02), f32(0.95), f32(0.01), eps=f32(1e-7))
    check_muon(W0, host(Wd[0]), rw, f32(0.02), f32(0.01), TOL_F32)


def test_grouped_newton_schulz_launches_match_per_bucket_calls():
    """A plan runs small Muon buckets through shared Newton-Schulz launches;
    every tile is computed as in a launch of its own bucket alone, so the
    result must equal one muon_step_batched call per bucket, bit for bit.
    Nine buckets (tall, wide, square, per-head; two cubic schedules) exceed
    the eight jobs one launch takes; two more with an A^2 term (c != 0) take
    a different kernel sequence and form a group of their own."""
    H = ma.ROLE_HIDDEN
    shapes = [(64, 128), (128, 64), (256, 512), (512, 256), (128, 128), (192, 64), (64, 320), (384, 128),
              (96, 96), (320, 64), (256, 256)]
    counts = [3, 2, 1, 2, 4, 1, 2, 1, 3, 2, 1]
    cubic2 = ((2.0, -1.25, 0.0), (1.7, -0.6, 0.0), (1.5, -0.5, 0.0), (1.5, -0.5, 0.0), (1.6, -0.55, 0.0))
    hps = [ma.muon_hparams(),
           ma.muon_hparams(coeffs=cubic2, lr=0.01, weight_decay=0.1, heads=2),
           ma.muon_hparams(coeffs=((3.4445, -4.7750, 2.0315),), scale_mode=1)]
    which = [0, 1, 0, 1, 0, 1, 0, 1, 0, 2, 2]
    r = np.random.default_rng(41)
    table, P0, G = [], [], []
    for bi, (shape, cnt) in enumerate(zip(shapes, counts)):
        for _ in range(cnt):
            table.append((shape, which[bi]))
            P0.append((r.standard_normal(shape) * 0.02).astype(np.float32))
            G.append(bf16_round(r.standard_normal(shape) * 1e-3))
    params = [dev_f32(p) for p in P0]
    opt = ma.MuonAdamW([(p, H, g) for p, (_, g) in zip(params, table)], [("muon", h) for h in hps])
    opt.step([dev_grad(g, "bf16") for g in G])
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
    grouped = opt.launches
    i = 0
    for bi, (shape, cnt) in enumerate(zip(shapes, counts)):
        hp = hps[which[bi]]
        Wd = [dev_f32(P0[i + k]) for k in range(cnt)]
        Md = [torch.zeros(shape, device="cuda") for _ in range(cnt)]
        ws = torch.empty(ma.muon_workspace_bytes(cnt, *shape, hp), dtype=torch.uint8, device="cuda")
        ma.muon_step_batched(Wd, [dev_grad(G[i + k], "bf16") for k in range(cnt)], Md, hp, ws)
        torch.cuda.synchronize()
        for k in range(cnt):
            assert torch.equal(Wd[k], params[i + k]), f"bucket {bi} matrix {k}"
            assert torch.equal(Md[k], opt.state[i + k][0]), f"bucket {bi} momentum {k}"
        i += cnt
    # Two launches of momentum and norm per bucket. Newton-Schulz: 8 cubic
    # buckets in one set, the ninth alone (2 kernels a step), the two quintic
    # buckets together (3 a step); a set with units of m <= 128 and of
    # m > 128 takes one kernel of each tile shape per kernel of the chain.
    def kinds(bis):
        small = [min(shapes[b][0] // hps[which[b]].heads, shapes[b][1]) <= 128 for b in bis]
        return int(any(small)) + int(not all(small))
    sets = [(range(0, 8), 2), (range(8, 9), 2), (range(9, 11), 3)]
    assert grouped == 2 * len(shapes) + sum(5 * per * kinds(b) for b, per in sets)


def test_batched_call_beyond_4gib_runs_in_sub_batches():
    """muon_step_batched on 48 matrices of 4096 x 4096 (4.6 GB of workspace)
    runs as two sub-batches of 24 inside the caller's workspace; the result
    must equal two calls of 24, bit for bit."""
    R = C = 4096
    n = 48
    hp = ma.muon_hparams()
    assert ma.muon_workspace_bytes(n, R, C, hp) > 4 << 30 >= ma.muon_workspace_bytes(n // 2, R, C, hp)
    gen = torch.Generator(device="cuda").manual_seed(5)
    W0 = torch.randn(n, R, C, device="cuda", generator=gen) * 0.02
    G = (torch.randn(n, R, C, device="cuda", generator=gen) * 1e-3).to(torch.bfloat16)
    Wa, Ma = W0.clone(), torch.zeros_like(W0)
    ws = torch.empty(ma.muon_workspace_bytes(n, R, C, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(list(Wa), list(G), list(Ma), hp, ws)
    Wb, Mb = W0.clone(), torch.zeros_like(W0)
    for s0 in (0, n // 2):
        sl = slice(s0, s0 + n // 2)
        ma.muon_step_batched(list(Wb[sl]), list(G[sl]), list(Mb[sl]), hp, ws)
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
    assert torch.equal(Wa, Wb) and torch.equal(Ma, Mb)
    assert not torch.equal(Wa, W0)


@pytest.mark.parametrize("shape", [(1, 64), (1, 4096), (8, 8), (4096, 8), (8, 4096), (200, 8), (3, 1000 * 8)])
def test_extreme_shapes(shape):
    """Degenerate Muon shapes: a single row (m = 1), an 8 x 8 matrix, very
    tall and very wide ones (m = 8 against n = 4096 or 8000), each through the
    single-CTA tensor-core path, against the oracle."""
    r = np.random.default_rng(sum(shape))
    W0 = (r.standard_normal(shape) * 0.02).astype(np.float32)
    g = bf16_round(r.standard_normal(shape) * 1e-3)
    hp = ma.muon_hparams()
    Wd, Md = [dev_f32(W0)], [torch.zeros(shape, device="cuda")]
    ws = torch.empty(ma.muon_workspace_bytes(1, *shape, hp), dtype=torch.uint8, device="cuda")
    ma.muon_step_batched(Wd, [dev_grad(g, "bf16")], Md, hp, ws)
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
    rw, _ = oracle.muon_update(W0, g, np.zeros(shape), f32(0.02), f32(0.95), f32(0.01), eps=f32(1e-7))
    check_muon(W0, host(Wd[0]), rw, f32(0.02), f32(0.01), TOL_BF16, what=str(shape))
