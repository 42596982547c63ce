"""The Gram-space Newton-Schulz chain against the oracle.

Wide units (n >= 1.25 m, m >= 128, m n >= 2^19; bf16 operands, no A^2 term) run
X_N = Q_N X_0 with Q and A updated by symmetric m x m products (upper tiles,
mirrored) instead of N Grams and N applies on X. The oracle runs the pages'
iteration itself, so these cases check the reformulation end to end: wide
and tall (transposed) matrices, ragged sizes on both sides, the 1.25 ratio
at its boundary, wide and tall head slices, one iteration, a per-iteration
coefficient table, cautious decay, two steps (momentum carried), and
repeatability.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle
import adamw_hybrid_optimizer_muon_b200 as ma
from gpu_helpers import TOL_BF16, bf16_round, check_muon, check_state, dev_f32, dev_grad, f32, host, momentum_terms

pytestmark = pytest.mark.gpu

CASES = [
    # (R, C), heads, coefficient table, cautious
    ((512, 1024), 1, ((1.5, -0.5, 0.0),), False),
    ((1024, 512), 1, ((1.5, -0.5, 0.0),), False),       # tall: X = u^T, written back transposed
    ((672, 840), 1, ((1.5, -0.5, 0.0),), False),        # n = 1.25 m exactly, m = 2.6 tiles
    ((520, 2056), 1, ((1.5, -0.5, 0.0),), True),        # ragged both ways, cautious decay
    ((1536, 4096), 3, ((1.5, -0.5, 0.0),), False),      # three head slices of 512 x 4096
    ((2048, 512), 2, ((1.5, -0.5, 0.0),), False),       # two tall head slices of 1024 x 512 (transposed)
    ((768, 2048), 1, ((2.0, -1.0, 0.0), (1.75, -0.75, 0.0), (1.5, -0.5, 0.0)), False),  # 3 iterations, a table
    ((512, 1536), 1, ((1.5, -0.5, 0.0),) * 1, False),   # steps = 1 below
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0][0]}x{c[0][1]}h{c[1]}n{len(c[2])}")
def test_gram_space_chain_matches_oracle(case):
    (R, C), heads, co, cautious = case
    steps = len(co) if len(co) > 1 else (1 if (R, C) == (512, 1536) else 5)
    co32 = tuple(tuple(f32(x) for x in c) for c in co)
    hp = ma.muon_hparams(coeffs=co, ns_steps=steps, heads=heads, cautious=cautious)
    r = np.random.default_rng(R + 3 * C)
    batch = 2
    W0 = [(r.standard_normal((R, C)) * 0.02).astype(np.float32) for _ in range(batch)]
    Wd = [dev_f32(w) for w in W0]
    Md = [torch.zeros((R, C), device="cuda") for _ in range(batch)]
    ws = torch.empty(ma.muon_workspace_bytes(batch, R, C, hp), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        G = [bf16_round(r.standard_normal((R, C)) * 1e-3) for _ in range(batch)]
        before = [(host(w), host(m)) for w, m in zip(Wd, Md)]
        ma.muon_step_batched(Wd, [dev_grad(g, "bf16") for g in G], Md, hp, ws)
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        for (w0, m0), g, w, m in zip(before, G, Wd, Md):
            rw, rm = oracle.muon_update(w0, g, m0, f32(0.02), f32(0.95), f32(0.01), True, steps, co32, f32(1e-7), 0,
                                        heads, cautious)
            check_state(host(m), rm, momentum_terms(m0, g, f32(0.95)), what="momentum")
            # (cautious: the decay mask is decided in floating point; where the two
            # sides decide differently, O * W is near zero and so is the difference)
            check_muon(w0, host(w), rw, f32(0.02), f32(0.01), TOL_BF16, what=f"{R}x{C} h{heads} n{steps}")


def test_gram_space_chain_is_taken_and_repeatable():
    # one 1024 x 2048 matrix: momentum pass, norm finalize, then the Gram, the
    # Q_1 kernel, 3N - 3 symmetric products and the final apply (N = 5: 15
    # chain launches against 10 for the direct iteration); same bits twice
    R, C = 1024, 2048
    r = np.random.default_rng(9)
    W0 = (r.standard_normal((R, C)) * 0.02).astype(np.float32)
    g = dev_grad(bf16_round(r.standard_normal((R, C)) * 1e-3), "bf16")
    outs = []
    for _ in range(2):
        p = dev_f32(W0)
        opt = ma.MuonAdamW([(p, ma.ROLE_HIDDEN, 0)], [("muon", ma.muon_hparams())])
        opt.step([g])
        torch.cuda.synchronize()
        assert ma.ma_device_status() == ma.MA_OK
        assert opt.launches == 2 + 1 + 1 + 12 + 1
        outs.append(p.clone())
    assert torch.equal(outs[0], outs[1])


@pytest.mark.parametrize("shape", [(2056, 2600), (2056, 2056)], ids=["gram_space", "direct"])
def test_deep_final_apply_ragged_matches_oracle(shape):
    # m = 2056 >= 2048 takes the deep final-apply variant (5-stage ring, X read
    # per lane) with a ragged last tile row (2056 = 8 x 256 + 8): on the
    # Gram-space chain (a = 0, no X term) and on the direct chain (a * X term)
    R, C = shape
    hp = ma.muon_hparams()
    r = np.random.default_rng(R + C)
    batch = 2
    W0 = [(r.standard_normal((R, C)) * 0.02).astype(np.float32) for _ in range(batch)]
    Wd = [dev_f32(w) for w in W0]
    Md = [torch.zeros((R, C), device="cuda") for _ in range(batch)]
    ws = torch.empty(ma.muon_workspace_bytes(batch, R, C, hp), dtype=torch.uint8, device="cuda")
    G = [bf16_round(r.standard_normal((R, C)) * 1e-3) for _ in range(batch)]
    ma.muon_step_batched(Wd, [dev_grad(g, "bf16") for g in G], Md, hp, ws)
    torch.cuda.synchronize()
    assert ma.ma_device_status() == ma.MA_OK
    co32 = ((f32(1.5), f32(-0.5), f32(0.0)),)
    for w0, g, w, m in zip(W0, G, Wd, Md):
        rw, rm = oracle.muon_update(w0, g, np.zeros_like(w0), f32(0.02), f32(0.95), f32(0.01), True, 5, co32,
                                    f32(1e-7), 0, 1, False)
        check_state(host(m), rm, momentum_terms(np.zeros_like(w0), g, f32(0.95)), what="momentum")
        check_muon(w0, host(w), rw, f32(0.02), f32(0.01), TOL_BF16, what=f"{R}x{C} deep final")
