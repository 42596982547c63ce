"""Short units (at most 128 rows) against the oracle.

Units with m <= 128 run on the single-CTA instance of the Newton-Schulz
kernels: the per-head slices of Q/K/V (128 x 4096, 128 x 1024) and small
matrices. The 128 x 4096 slices take the Gram-space chain (one Gram, 128 x 128
symmetric products, one final apply); the others the direct iteration.
Cases: ragged column counts, fewer than 128 rows, a single row, head
slices, and a per-iteration coefficient table, compared with the fp64 oracle
at the bf16 tolerance; two calls on the same inputs agree bit for bit.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import TOL_BF16, bf16_round, check_muon, check_state, dev_f32, dev_grad, f32, host, momentum_terms

pytestmark = pytest.mark.gpu

CASES = [
    # (R, C), heads, batch
    ((128, 4096), 1, 2),    # Gram space: 128 x 128 products
    ((4096, 4096), 32, 1),  # 32 head slices of 128 x 4096 (Gram space)
    ((64, 1024), 1, 3),     # 64 rows: the rest of the 128-row tile is zero
    ((96, 520), 1, 2),      # ragged rows and columns
    ((128, 256), 1, 1),     # one 128 x 256 tile
    ((1, 64), 1, 2),        # one row
    ((384, 1024), 3, 2),    # three head slices of 128 x 1024
]


def _hp(coeffs, heads=1):
    return ma.muon_hparams(coeffs=coeffs, ns_steps=len(coeffs) if len(coeffs) > 1 else 5, heads=heads)


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0][0]}x{c[0][1]}h{c[1]}b{c[2]}")
def test_short_units_match_oracle(case):
    (R, C), heads, batch = case
    hp = _hp(((1.5, -0.5, 0.0),), heads)
    r = np.random.default_rng(R * 7 + C)
    W0 = [(r.standard_normal((R, C)) * 0.02).astype(np.float32) for _ in range(batch)]
    Wd = [dev_f32(w) for w in W0]
    Md = [torch.zeros((R, C), device="cuda") for _ in range(batch)]
    ws = torch.empty(ma.muon_workspace_bytes(batch, R, C, hp), dtype=torch.uint8, device="cuda")
    for step in range(2):
        G = [bf16_round(r.standard_normal((R, C)) * 1e-3) for _ in range(batch)]
        before = [(host(w), host(m)) for w, m in zip(Wd, Md)]
        ma.muon_step_batched(Wd, [dev_grad(g, "bf16") for g in G], Md, hp, ws)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for (w0, m0), g, w, m in zip(before, G, Wd, Md):
            rw, rm = oracle.muon_update(w0, g, m0, f32(0.02), f32(0.95), f32(0.01), True, 5, ((1.5, -0.5, 0.0),),
                                        f32(1e-7), 0, heads)
            check_state(host(m), rm, momentum_terms(m0, g, f32(0.95)), what="momentum")
            check_muon(w0, host(w), rw, f32(0.02), f32(0.01), TOL_BF16, what=f"{R}x{C} heads {heads}")


def test_short_units_coefficient_table_and_repeatability():
    # a different (a, b) per iteration; the same inputs twice give the same bits
    R, C, heads = 512, 2048, 4
    co = ((2.0, -1.0, 0.0), (1.75, -0.75, 0.0), (1.5, -0.5, 0.0), (1.5, -0.5, 0.0))  # p(1) = 1 each
    hp = _hp(co, heads)
    r = np.random.default_rng(5)
    W0 = (r.standard_normal((R, C)) * 0.02).astype(np.float32)
    g = bf16_round(r.standard_normal((R, C)) * 1e-3)
    outs = []
    for _ in range(2):
        Wd, Md = [dev_f32(W0)], [torch.zeros((R, C), device="cuda")]
        ws = torch.empty(ma.muon_workspace_bytes(1, R, C, hp), dtype=torch.uint8, device="cuda")
        ma.muon_step_batched(Wd, [dev_grad(g, "bf16")], Md, hp, ws)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        outs.append(Wd[0].clone())
    assert torch.equal(outs[0], outs[1])
    rw, _ = oracle.muon_update(W0, g, np.zeros((R, C)), f32(0.02), f32(0.95), f32(0.01), True, len(co),
                               tuple(tuple(f32(x) for x in c) for c in co), f32(1e-7), 0, heads)
    check_muon(W0, host(outs[0]), rw, f32(0.02), f32(0.01), TOL_BF16, what="coefficient table")
