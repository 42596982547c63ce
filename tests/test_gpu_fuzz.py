"""Seeded random parameter tables through the whole step, against the oracle.

Each table mixes Muon matrices of random shape (rows and columns from 8 to
600, columns a multiple of 8: tall, wide and square, short sides on both
sides of the 128-row single-CTA limit and of the 256-row tile edges), four
Muon groups (the cubic and a schedule with c != 0, each whole and split into
heads), bf16 and fp32 gradients, and a few AdamW tensors. The plan buckets,
sub-batches and groups them as it would any table. After each of two steps
every Muon matrix is checked against the oracle, and every AdamW tensor and
momentum buffer element by element.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import (TOL_BF16, bf16_round, check_muon, check_state, dev_f32, dev_grad, f32, host,
                         momentum_terms)

pytestmark = pytest.mark.gpu

CUBIC = ((1.5, -0.5, 0.0),)
QUINTIC = ((2.0, -1.5, 0.5), (1.5, -0.5, 0.0), (1.875, -1.25, 0.375), (1.5, -0.5, 0.0), (1.5, -0.5, 0.0))
MUON_GROUPS = [dict(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, coeffs=CUBIC, scale_mode=0, heads=1),
               dict(lr=0.01, beta=0.9, weight_decay=0.05, nesterov=False, coeffs=QUINTIC, scale_mode=1, heads=1),
               dict(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, coeffs=CUBIC, scale_mode=0, heads=2),
               dict(lr=0.01, beta=0.9, weight_decay=0.05, nesterov=False, coeffs=QUINTIC, scale_mode=1, heads=4)]
ADAMW = dict(lr=0.01, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01)
AG = len(MUON_GROUPS)  # index of the AdamW group


def _table(seed, n_muon=20):
    """(shape, role, group, grad dtype) rows."""
    r = np.random.default_rng(seed)
    table = []
    for _ in range(n_muon):
        g = int(r.integers(0, len(MUON_GROUPS)))
        h = MUON_GROUPS[g]["heads"]
        R = h * int(r.integers(max(1, 8 // h), 600 // h + 1))
        C = 8 * int(r.integers(1, 76))
        table.append(((R, C), ma.ROLE_HIDDEN, g, "bf16" if r.random() < 0.7 else "f32"))
    for _ in range(4):
        if r.random() < 0.6:
            table.append(((int(r.integers(1, 3000)),), ma.ROLE_HIDDEN, AG, "bf16"))
        else:
            table.append(((int(r.integers(2, 300)), 8 * int(r.integers(1, 20))), ma.ROLE_EMBED, AG, "bf16"))
    return table


@pytest.mark.parametrize("seed", [11, 12, 13])
def test_random_tables_two_steps(seed):
    table = _table(seed)
    r = np.random.default_rng(seed + 1000)
    P0 = [(r.standard_normal(s) * 0.02).astype(np.float32) for s, *_ in table]
    params = [dev_f32(p) for p in P0]
    groups = [("muon", ma.muon_hparams(**m)) for m in MUON_GROUPS] + [("adamw", ma.adamw_hparams(**ADAMW))]
    opt = ma.MuonAdamW([(p, role, g) for p, (_, role, g, _) in zip(params, table)], groups)
    a = {k: f32(v) for k, v in ADAMW.items()}
    for step in (1, 2):
        G = [bf16_round(r.standard_normal(s) * 1e-3) for s, *_ in table]
        before_p = [host(p) for p in params]
        before_s = [(host(x), None if y is None else host(y)) for x, y in opt.state]
        opt.step([dev_grad(g, dt) for g, (_, _, _, dt) in zip(G, table)])
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for i, ((shape, role, g, _), p) in enumerate(zip(table, params)):
            what = f"seed {seed} step {step} tensor {i} {shape} group {g}"
            if g < AG:
                m = MUON_GROUPS[g]
                coeffs = tuple(tuple(f32(x) for x in c) for c in m["coeffs"])
                rw, rm = oracle.muon_update(before_p[i], G[i], before_s[i][0], f32(m["lr"]), f32(m["beta"]),
                                            f32(m["weight_decay"]), m["nesterov"], 5, coeffs, f32(1e-7),
                                            m["scale_mode"], m["heads"])
                check_muon(before_p[i], host(p), rw, f32(m["lr"]), f32(m["weight_decay"]), TOL_BF16, what=what)
                check_state(host(opt.state[i][0]), rm, momentum_terms(before_s[i][0], G[i], f32(m["beta"])),
                            what=what)
            else:
                args = (step, a["lr"], a["beta1"], a["beta2"], a["eps"], a["weight_decay"])
                rp, rm, rv = oracle.adamw_update(before_p[i], G[i], before_s[i][0], before_s[i][1], *args)
                tp, tm, tv = oracle.adamw_term_magnitudes(before_p[i], G[i], before_s[i][0], before_s[i][1], *args)
                check_state(host(p).reshape(-1), rp.reshape(-1), tp.reshape(-1), what=what)
                check_state(host(opt.state[i][0]).reshape(-1), rm.reshape(-1), tm.reshape(-1), what=what)
                check_state(host(opt.state[i][1]).reshape(-1), rv.reshape(-1), tv.reshape(-1), what=what)
