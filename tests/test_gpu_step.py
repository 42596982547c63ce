"""The whole MuonAdamW step through the plan (muonadamw_step) against the oracle.

* tiny: every element of every tensor, twelve steps (eager, fp32 mode, CUDA graph).
* d20 and the 7B-shaped set at full size, in the same launch configuration
  bench.py times. The oracle recomputes sampled matrices in full (one or two
  of each bucket; on the 7B set the first and the last, which lie in different
  sub-batches) and sampled elements of the AdamW tensors and of every momentum
  buffer, two steps from zero state.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import synth
import synth.device as sdev
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import TOL_BF16, TOL_F32, check_muon, check_state, host, hp32, momentum_terms

pytestmark = pytest.mark.gpu


def build_optimizer(wl, params, precision=0):
    groups = []
    for g in wl.groups:
        if g.kind == synth.KIND_MUON:
            h = g.muon
            groups.append(("muon", ma.muon_hparams(h.lr, h.beta, h.weight_decay, h.eps, h.nesterov, h.ns_steps,
                                                   h.coeffs, h.scale_mode, h.heads, precision)))
        else:
            h = g.adamw
            groups.append(("adamw", ma.adamw_hparams(h.lr, h.beta1, h.beta2, h.eps, h.weight_decay, 1)))
    return ma.MuonAdamW([(p, t.role, t.group) for p, t in zip(params, wl.tensors)], groups)


def oracle_groups(wl, precision=0):
    out = []
    for g in wl.groups:
        if g.kind == synth.KIND_MUON:
            h = hp32(g.muon)
            out.append(dict(kind=0, lr=h.lr, beta=h.beta, weight_decay=h.weight_decay, eps=h.eps,
                            nesterov=h.nesterov, ns_steps=h.ns_steps, coeffs=h.coeffs, scale_mode=h.scale_mode,
                            heads=h.heads))
        else:
            h = hp32(g.adamw)
            out.append(dict(kind=1, lr=h.lr, beta1=h.beta1, beta2=h.beta2, eps=h.eps,
                            weight_decay=h.weight_decay))
    return out


@pytest.mark.parametrize("precision,graph", [(0, False), (1, False), (0, True)])
def test_tiny_twelve_steps_every_element(precision, graph):
    """Twelve steps (the AdamW bias corrections and the momentum carry over),
    each checked element by element against one oracle step from the GPU's
    own pre-step values; eagerly, in fp32 mode, and replayed from a CUDA graph
    whose AdamW step counter is patched every step."""
    wl = synth.tiny()
    W0 = [synth.initial_weight(t, i) for i, t in enumerate(wl.tensors)]
    params = [torch.from_numpy(w).cuda() for w in W0]
    opt = build_optimizer(wl, params, precision)
    tensors = [dict(shape=t.shape, role=t.role, group=t.group) for t in wl.tensors]
    groups = oracle_groups(wl)
    state = [{} for _ in wl.tensors]
    ref = [w.astype(np.float64) for w in W0]
    gd = [torch.empty(t.shape, device="cuda") for t in wl.tensors]  # fixed buffers (one plan, one graph)
    for step in range(1, 13):
        G = [synth.gradient(wl, i, step) for i in range(len(wl.tensors))]
        for d, g in zip(gd, G):
            d.copy_(torch.from_numpy(g))  # fp32 gradients in this config
        before_p = [host(p) for p in params]
        before_s = [(host(s0), None if s1 is None else host(s1)) for s0, s1 in opt.state]
        opt.step(gd, graph=graph)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        # one oracle step from exactly the GPU's pre-step values
        st = [{"m": before_s[0][0]}, {"exp_avg": before_s[1][0], "exp_avg_sq": before_s[1][1]}]
        ref = oracle.muonadamw_step(tensors, groups, before_p, G, st, step)
        m = hp32(wl.groups[0].muon)
        check_muon(before_p[0], host(params[0]), ref[0], m.lr, m.weight_decay, TOL_F32 if precision else TOL_BF16)
        check_state(host(opt.state[0][0]), st[0]["m"], momentum_terms(before_s[0][0], G[0], m.beta), what="m")
        a = hp32(wl.groups[1].adamw)
        tp, tm, tv = oracle.adamw_term_magnitudes(before_p[1], G[1], before_s[1][0], before_s[1][1], step, a.lr,
                                                  a.beta1, a.beta2, a.eps, a.weight_decay)
        check_state(host(params[1]), ref[1], tp, what="gain")
        check_state(host(opt.state[1][0]), st[1]["exp_avg"], tm, what="exp_avg")
        check_state(host(opt.state[1][1]), st[1]["exp_avg_sq"], tv, what="exp_avg_sq")
    assert opt.launches == 1 + 2 + 2 * 5  # AdamW, momentum+norm, finalize, 5 x (Gram, apply)
    assert opt.graph_captures == (1 if graph else 0)


def _full_size_check(name, n_muon_samples=1, adamw_samples=200_000, seed=0):
    """n_muon_samples matrices of every bucket are recomputed in full: the
    bucket's first matrix and, for two or more, its last one (which the plan
    puts in the bucket's last sub-batch), then evenly spaced members."""
    wl = synth.WORKLOADS[name]()
    params = sdev.weights(wl)
    opt = build_optimizer(wl, params)
    kinds = oracle.partition([(t.shape, t.role) for t in wl.tensors])
    buckets = oracle.muon_buckets([(t.shape, t.role) for t in wl.tensors], [t.group for t in wl.tensors])

    def pick(members):
        k = min(n_muon_samples, len(members))
        pos = sorted({round(j * (len(members) - 1) / max(1, k - 1)) for j in range(k)}) if k > 1 else [0]
        return [members[p] for p in pos]

    sample_mats = [idx for b in buckets for idx in pick(b[3])]
    r = np.random.default_rng(seed)
    grads = None
    for step in (1, 2):
        grads = sdev.gradients(wl, step, out=grads)
        snap = {}
        for i in sample_mats:
            snap[i] = (host(params[i]), host(grads[i]), host(opt.state[i][0]))
        # sampled elements of everything else
        idx = {}
        for i, t in enumerate(wl.tensors):
            n = t.numel
            k = min(n, adamw_samples if kinds[i] == 1 else 4096)
            sel = torch.from_numpy(r.choice(n, size=k, replace=False) if k < n else np.arange(n)).cuda()
            flat = lambda x: x.reshape(-1)[sel]  # noqa: E731
            s0, s1 = opt.state[i]
            idx[i] = (sel, host(flat(params[i])), host(flat(grads[i])), host(flat(s0)),
                      None if s1 is None else host(flat(s1)))
        opt.step(grads)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for i in sample_mats:
            w0, g, m0 = snap[i]
            grp = hp32(wl.groups[wl.tensors[i].group].muon)
            rw, rm = oracle.muon_update(w0, g, m0, grp.lr, grp.beta, grp.weight_decay, grp.nesterov, grp.ns_steps,
                                        grp.coeffs, grp.eps, grp.scale_mode, grp.heads)
            check_muon(w0, host(params[i]), rw, grp.lr, grp.weight_decay, TOL_BF16, what=wl.tensors[i].name)
            check_state(host(opt.state[i][0]), rm, momentum_terms(m0, g, grp.beta), what="momentum")
        for i, t in enumerate(wl.tensors):
            sel, p0, g, s0, s1 = idx[i]
            flat = lambda x: x.reshape(-1)[sel]  # noqa: E731
            if kinds[i] == 1:
                a = hp32(wl.groups[t.group].adamw)
                rp, rm, rv = oracle.adamw_update(p0, g, s0, s1, step, a.lr, a.beta1, a.beta2, a.eps, a.weight_decay)
                tp, tm, tv = oracle.adamw_term_magnitudes(p0, g, s0, s1, step, a.lr, a.beta1, a.beta2, a.eps,
                                                          a.weight_decay)
                check_state(host(flat(params[i])), rp, tp, what=t.name)
                check_state(host(flat(opt.state[i][0])), rm, tm, what=t.name + ".exp_avg")
                check_state(host(flat(opt.state[i][1])), rv, tv, what=t.name + ".exp_avg_sq")
            else:
                grp = hp32(wl.groups[t.group].muon)
                rm, _ = oracle.momentum_update(s0, g, grp.beta, grp.nesterov)
                check_state(host(flat(opt.state[i][0])), rm, momentum_terms(s0, g, grp.beta),
                            what=t.name + ".m")
    return opt


def test_d20_full_size_sampled():
    _full_size_check("d20", n_muon_samples=2)


@pytest.mark.slow
def test_7b_full_size_sampled():
    # two matrices of each of the three buckets: the first and the last (which
    # lies in a later sub-batch: 32 matrices per sub-batch of the 4096^2 bucket,
    # 16 of the 4096x11008 and 11008x4096 buckets)
    _full_size_check("7b", n_muon_samples=2, adamw_samples=100_000)


@pytest.mark.slow
def test_aspect_full_size_sampled():
    # MLP 4096x14336 (wide) and 14336x4096 (transpose path), Q/K/V as 32 heads of
    # 128x4096, 10 % of units with rank-64 gradients
    _full_size_check("aspect", n_muon_samples=1)


@pytest.mark.slow
def test_square_full_size_sampled():
    # 64 matrices 4096^2, gradient scales spread over three decades
    _full_size_check("square", n_muon_samples=2)


@pytest.mark.parametrize("name", ["tiny", "d20"])
def test_step_from_host_equals_resident_step(name):
    # gradients copied from pinned host memory, overlapped with compute, give
    # bit-identical parameters and state to the step on resident gradients
    wl = synth.WORKLOADS[name]()
    pa = sdev.weights(wl)
    pb = [p.clone() for p in pa]
    opt_a, opt_b = build_optimizer(wl, pa), build_optimizer(wl, pb)
    dev_a = sdev.gradients(wl, 1)
    dev_b = [torch.zeros_like(g) for g in dev_a]
    for step in (1, 2):
        g = sdev.gradients(wl, step, out=dev_a)
        host_g = [x.cpu().pin_memory() for x in g]
        opt_a.step(dev_a)
        opt_b.step_from_host(host_g, dev_b)
        # once the copies have read the host buffers, the caller may reuse them
        # while the step still runs
        opt_b.host_copies_done.synchronize()
        for h in host_g:
            h.fill_(float("nan"))
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for x, y in zip(pa, pb):
            assert torch.equal(x, y)
        for (s0, s1), (t0, t1) in zip(opt_a.state, opt_b.state):
            assert torch.equal(s0, t0) and (s1 is None or torch.equal(s1, t1))
