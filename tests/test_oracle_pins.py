"""Pins for the fp64 CPU oracle, run without a GPU.

Each test checks the oracle against something outside itself: the constants
the pages print, an SVD closed form, a fixed point, a closed form after k
steps, an invariance, or a scalar special case. The set is chosen so that a
plausible slip fails at least one test: a dropped term, a wrong sign or
index, a transposed operand, a misplaced eps, or decay applied to the wrong
weight.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_constants.json")


def p_scalar(sigma, coeffs, steps):
    """The NS polynomial p(s) = a s + b s^3 + c s^5, applied to a scalar `steps` times."""
    sched = oracle.coeff_schedule(coeffs, steps)
    s = np.asarray(sigma, dtype=np.float64)
    for a, b, c in sched:
        s = a * s + b * s ** 3 + c * s ** 5
    return s


def svd_closed_form(X, coeffs, steps):
    U, S, Vt = np.linalg.svd(np.asarray(X, dtype=np.float64), full_matrices=False)
    return (U * p_scalar(S, coeffs, steps)) @ Vt


def rng(seed):
    return np.random.default_rng(seed)


# --------------------------------------------------------------------------- constants

def test_page_constants_match_golden():
    g = json.load(open(GOLDEN))
    assert oracle.CUBIC == (g["ns_cubic"]["value"]["a"], g["ns_cubic"]["value"]["b"],
                            g["ns_cubic"]["value"]["c"])
    assert oracle.DEFAULT_NS_STEPS == g["ns_steps"]["value"]
    assert oracle.DEFAULT_MOMENTUM == g["momentum_decay"]["value"]
    hp = synth.MuonHP()
    assert hp.coeffs[0] == oracle.CUBIC and hp.ns_steps == 5 and hp.beta == 0.95


def test_cubic_scalar_fixed_points():
    # p(1) = 1 (orthogonal matrices are fixed points) and p(0) = 0
    assert p_scalar(1.0, [oracle.CUBIC], 1) == 1.0
    assert p_scalar(0.0, [oracle.CUBIC], 1) == 0.0
    # a 1x1 matrix reduces to the scalar polynomial
    for x in (0.3, 0.9, 1.2):
        assert oracle.ns_iterate([[x]], [oracle.CUBIC], 1)[0, 0] == pytest.approx(1.5 * x - 0.5 * x ** 3,
                                                                                 abs=1e-15)


# --------------------------------------------------------------------------- Newton-Schulz

@pytest.mark.parametrize("shape,rank", [((8, 16), None), ((16, 8), None), ((32, 32), None),
                                        ((16, 32), 4), ((1, 7), None), ((7, 1), None)])
@pytest.mark.parametrize("coeffs,steps", [([oracle.CUBIC], 5), ([oracle.CUBIC], 1),
                                          ([(2.0, -1.5, 0.5)], 3),
                                          ([(1.5, -0.5, 0.0), (2.0, -1.5, 0.5), (1.2, -0.1, -0.05)], 3)])
def test_ns_matches_svd_closed_form(shape, rank, coeffs, steps):
    r = rng(1)
    m, n = shape
    if rank is None:
        X = r.standard_normal(shape)
    else:
        X = r.standard_normal((m, rank)) @ r.standard_normal((rank, n))
    X = X / np.linalg.norm(X, 2) * 0.9  # spectral norm 0.9, inside the cubic's basin
    got = oracle.ns_iterate(X, coeffs, steps)
    ref = svd_closed_form(X, coeffs, steps)
    assert np.linalg.norm(got - ref) <= 1e-12 * max(1.0, np.linalg.norm(ref))


def test_ns_literal_page_form():
    # the page's own orientation X (X^T X) gives the same result as the short-side Gram
    r = rng(2)
    X = r.standard_normal((6, 10)) * 0.1
    Y = X.copy()
    for _ in range(5):
        Y = 1.5 * Y - 0.5 * Y @ (Y.T @ Y)
    assert np.allclose(oracle.ns_iterate(X), Y, rtol=0, atol=1e-14)


@pytest.mark.parametrize("shape", [(16, 16), (8, 24), (24, 8)])
def test_orthogonal_is_fixed_point(shape):
    r = rng(3)
    m, n = shape
    Q, _ = np.linalg.qr(r.standard_normal((max(m, n), min(m, n))))
    Q = Q if m >= n else Q.T
    assert np.allclose(oracle.ns_iterate(Q), Q, rtol=0, atol=1e-13)


def test_normalised_orthogonal_is_not_fixed_point():
    # Frobenius normalisation maps every singular value of an m x m orthogonal Q to 1/sqrt(m)
    r = rng(4)
    m = 16
    Q, _ = np.linalg.qr(r.standard_normal((m, m)))
    out = oracle.orthogonalize(Q, eps=0.0)
    S = np.linalg.svd(out, compute_uv=False)
    assert np.allclose(S, p_scalar(1.0 / math.sqrt(m), [oracle.CUBIC], 5), rtol=1e-13)
    assert np.allclose(out, Q * p_scalar(1.0 / math.sqrt(m), [oracle.CUBIC], 5), atol=1e-14)


@pytest.mark.parametrize("shape", [(8, 20), (20, 8), (12, 12)])
def test_orthogonalize_svd_closed_form(shape):
    # normalisation + orientation + NS, pinned for tall and wide inputs alike
    r = rng(5)
    u = r.standard_normal(shape) * 1e-3
    eps = 1e-7
    U, S, Vt = np.linalg.svd(u, full_matrices=False)
    ref = (U * p_scalar(S / (np.linalg.norm(u) + eps), [oracle.CUBIC], 5)) @ Vt
    got = oracle.orthogonalize(u, eps=eps)
    assert np.linalg.norm(got - ref) <= 1e-12 * np.linalg.norm(ref)


def test_orthogonalize_invariances():
    r = rng(6)
    u = r.standard_normal((10, 26))
    base = oracle.orthogonalize(u, eps=0.0)
    assert np.allclose(oracle.orthogonalize(37.5 * u, eps=0.0), base, atol=1e-13)
    assert np.allclose(oracle.orthogonalize(u.T, eps=0.0), base.T, atol=1e-13)


def test_rank_one_is_not_destroyed():
    # The "Rank-1 Matrix Hazard" section says NS zeroes a rank-1 matrix. For the
    # cubic, a Frobenius-normalised rank-1 matrix has sigma = 1 = p(1): it is a fixed point.
    r = rng(7)
    x = r.standard_normal(128)
    y = r.standard_normal(1)
    u = np.outer(x, y)  # the [128, 1] head shape the page names
    out = oracle.orthogonalize(u, eps=0.0)
    ref = np.outer(x / np.linalg.norm(x), y / np.linalg.norm(y))
    assert np.allclose(out, ref, atol=1e-14)
    assert np.linalg.norm(out) == pytest.approx(1.0, rel=1e-14)


def test_rank_deficient_stays_rank_r():
    r = rng(8)
    u = r.standard_normal((32, 4)) @ r.standard_normal((4, 48))
    out = oracle.orthogonalize(u)
    S = np.linalg.svd(out, compute_uv=False)
    assert np.all(S[4:] < 1e-12) and np.all(S[:4] > 1e-3)


def test_zero_direction_gives_zero():
    out = oracle.orthogonalize(np.zeros((4, 6)))
    assert np.all(out == 0.0)


# --------------------------------------------------------------------------- momentum

@pytest.mark.parametrize("nesterov", [False, True])
def test_momentum_closed_form_constant_grad(nesterov):
    beta = 0.95
    g = rng(9).standard_normal((3, 5))
    m = np.zeros_like(g)
    for k in range(1, 9):
        m, u = oracle.momentum_update(m, g, beta, nesterov)
        assert np.allclose(m, (1 - beta ** k) * g, rtol=1e-14, atol=0)
        expect_u = (1 - beta ** (k + 1)) * g if nesterov else (1 - beta ** k) * g
        assert np.allclose(u, expect_u, rtol=1e-14, atol=0)


def test_nesterov_direction_equals_heavy_ball_direction():
    # EMA Nesterov u_k = (1 - beta) (g_k + beta b_k), where b_k = beta b_{k-1} + g_k (heavy ball)
    beta = 0.95
    r = rng(10)
    m = np.zeros((6, 9))
    b = np.zeros((6, 9))
    for _ in range(6):
        g = r.standard_normal((6, 9))
        m, u = oracle.momentum_update(m, g, beta, True)
        b = beta * b + g
        assert np.allclose(u, (1 - beta) * (g + beta * b), rtol=1e-12, atol=1e-15)
        assert np.allclose(oracle.orthogonalize(u, eps=0.0), oracle.orthogonalize(g + beta * b, eps=0.0),
                           atol=1e-12)


# --------------------------------------------------------------------------- AdamW

@pytest.mark.parametrize("wd", [0.0, 0.01, 0.3])
@pytest.mark.parametrize("gscale", [1e-3, 1e-9])
def test_adamw_closed_form_constant_grad(wd, gscale):
    lr, b1, b2, eps = 0.02, 0.9, 0.95, 1e-8
    r = rng(11)
    p0 = r.standard_normal(64) * 0.02
    g = r.standard_normal(64) * gscale
    p, m, v = p0.copy(), np.zeros(64), np.zeros(64)
    rho = 1.0 - lr * wd
    step_dir = g / (np.abs(g) + eps)  # bias-corrected m / (sqrt(v) + eps) for constant g
    for k in range(1, 8):
        p, m, v = oracle.adamw_update(p, g, m, v, k, lr, b1, b2, eps, wd)
        assert np.allclose(m, (1 - b1 ** k) * g, rtol=1e-13, atol=0)
        assert np.allclose(v, (1 - b2 ** k) * g * g, rtol=1e-13, atol=0)
        geo = k if wd == 0.0 else (1 - rho ** k) / (1 - rho)
        p_ref = rho ** k * p0 - lr * step_dir * geo
        assert np.allclose(p, p_ref, rtol=1e-12, atol=1e-14)  # terms are ~1e-2; cancellation near 0


def test_adamw_first_step_is_sign_like():
    g = np.array([3e-3, -2e-5, 0.0, 7.0])
    p, _, _ = oracle.adamw_update(np.ones(4), g, np.zeros(4), np.zeros(4), 1, 0.1, 0.9, 0.95, 1e-8, 0.0)
    assert np.allclose(p, 1 - 0.1 * g / (np.abs(g) + 1e-8), rtol=0, atol=1e-15)


# --------------------------------------------------------------------------- Muon step

@pytest.mark.parametrize("shape,heads,nesterov,mode", [((16, 40), 1, True, 0), ((40, 16), 1, True, 0),
                                                       ((40, 16), 1, False, 1), ((32, 24), 2, True, 0),
                                                       ((24, 24), 3, True, 2)])
def test_muon_one_step_closed_form(shape, heads, nesterov, mode):
    lr, beta, wd, eps = 0.02, 0.95, 0.01, 1e-7
    r = rng(12)
    W0 = r.standard_normal(shape) * 0.02
    g = r.standard_normal(shape) * 1e-3
    W1, m1 = oracle.muon_update(W0, g, np.zeros(shape), lr, beta, wd, nesterov, 5, [oracle.CUBIC], eps,
                                mode, heads)
    c = (1 - beta) * (1 + beta) if nesterov else (1 - beta)
    R, C = shape
    rh = R // heads
    O = np.zeros(shape)
    for h in range(heads):
        gs = g[h * rh:(h + 1) * rh]
        U, S, Vt = np.linalg.svd(gs, full_matrices=False)
        s = {0: math.sqrt(max(1.0, rh / C)), 1: math.sqrt(rh / C), 2: 1.0}[mode]
        O[h * rh:(h + 1) * rh] = s * (U * p_scalar(c * S / (c * np.linalg.norm(gs) + eps), [oracle.CUBIC], 5)) @ Vt
    assert np.allclose(m1, (1 - beta) * g, rtol=1e-14, atol=0)
    ref = (1 - lr * wd) * W0 - lr * O
    assert np.linalg.norm(W1 - ref) <= 1e-12 * np.linalg.norm(ref)


def test_shape_scale_values():
    assert oracle.shape_scale(11008, 4096, 0) == pytest.approx(math.sqrt(11008 / 4096))
    assert oracle.shape_scale(4096, 11008, 0) == 1.0
    assert oracle.shape_scale(4096, 11008, 1) == pytest.approx(math.sqrt(4096 / 11008))
    assert oracle.shape_scale(5, 3, 2) == 1.0


# --------------------------------------------------------------------------- partition

def test_partition_rules():
    H, E, U, F = oracle.ROLE_HIDDEN, oracle.ROLE_EMBED, oracle.ROLE_UNEMBED, oracle.ROLE_FORCE_ADAMW
    table = [((), H), ((7,), H), ((3, 4), H), ((3, 4), E), ((3, 4), U), ((3, 4), F), ((1, 1), H), ((0,), H)]
    assert oracle.partition(table) == [1, 1, 0, 1, 1, 1, 0, 1]
    with pytest.raises(oracle.UnsupportedTensor):
        oracle.partition([((2, 3, 4), H)])


@pytest.mark.parametrize("name,muon,adamw,buckets", [("7b", 224, 67, 3), ("d20", 120, 83, 3),
                                                     ("tiny", 1, 1, 1), ("aspect", 5, 0, 3)])
def test_partition_counts_and_exactly_once(name, muon, adamw, buckets):
    wl = synth.WORKLOADS[name]()
    sr = [(t.shape, t.role) for t in wl.tensors]
    kinds = oracle.partition(sr)
    assert kinds.count(0) == muon and kinds.count(1) == adamw
    bk = oracle.muon_buckets(sr, [t.group for t in wl.tensors])
    assert len(bk) == buckets
    flat = [i for b in bk for i in b[3]]
    assert sorted(flat) == [i for i, k in enumerate(kinds) if k == 0]  # every Muon tensor exactly once
    for grp, R, C, members in bk:
        assert all(wl.tensors[i].shape == (R, C) and wl.tensors[i].group == grp for i in members)
        assert members == sorted(members)  # first-appearance order


# --------------------------------------------------------------------------- whole step

def test_muonadamw_two_steps_closed_forms():
    wl = synth.tiny()
    tensors = [dict(shape=t.shape, role=t.role, group=t.group) for t in wl.tensors]
    gm, ga = wl.groups[0].muon, wl.groups[1].adamw
    groups = [dict(kind=0, lr=gm.lr, beta=gm.beta, weight_decay=gm.weight_decay, eps=gm.eps,
                   nesterov=gm.nesterov, ns_steps=gm.ns_steps, coeffs=gm.coeffs, scale_mode=gm.scale_mode,
                   heads=gm.heads),
              dict(kind=1, lr=ga.lr, beta1=ga.beta1, beta2=ga.beta2, eps=ga.eps, weight_decay=ga.weight_decay)]
    W0 = [synth.initial_weight(t, i).astype(np.float64) for i, t in enumerate(wl.tensors)]
    g = [synth.gradient(wl, i, 1).astype(np.float64) for i in range(2)]
    state = [{}, {}]
    P1 = oracle.muonadamw_step(tensors, groups, W0, g, state, 1)
    # AdamW closed form for step 1 from zero state
    rho = 1 - ga.lr * ga.weight_decay
    ref_gain = rho * W0[1] - ga.lr * g[1] / (np.abs(g[1]) + ga.eps)
    assert np.allclose(P1[1], ref_gain, rtol=1e-12, atol=1e-18)
    # Muon closed form for step 1 from zero momentum (256x512 is wide: no transpose, s = 1)
    c = (1 - gm.beta ** 2)
    U, S, Vt = np.linalg.svd(g[0].astype(np.float64), full_matrices=False)
    O = (U * p_scalar(c * S / (c * np.linalg.norm(g[0].astype(np.float64)) + gm.eps), [oracle.CUBIC], 5)) @ Vt
    ref_w = (1 - gm.lr * gm.weight_decay) * W0[0] - gm.lr * O
    assert np.linalg.norm(P1[0] - ref_w) <= 1e-12 * np.linalg.norm(ref_w)
    # a second step with the same gradient follows the momentum closed form
    P2 = oracle.muonadamw_step(tensors, groups, P1, g, state, 2)
    assert np.allclose(state[0]["m"], (1 - gm.beta ** 2) * g[0], rtol=1e-13)
    assert np.allclose(state[1]["exp_avg_sq"], (1 - ga.beta2 ** 2) * g[1].astype(np.float64) ** 2, rtol=1e-13)
    assert P2[0].shape == (256, 512)


def test_bf16_storage_roundtrip_is_exact():
    # gradients stored as bf16 are bf16-representable fp32 values; the oracle reads them exactly
    x = np.array([1.0, -2.5, 3.140625, 1e-3, 0.0], dtype=np.float32)
    b = synth.f32_to_bf16_bits(x)
    y = synth.bf16_bits_to_f32(b)
    assert y[0] == 1.0 and y[1] == -2.5 and y[2] == 3.140625 and y[4] == 0.0
    assert abs(y[3] - 1e-3) <= 1e-3 * 2 ** -8
    # ties go to even
    t = np.array([np.float32(1.0) + np.float32(2 ** -8)], dtype=np.float32)
    assert synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(t))[0] == 1.0


@pytest.mark.parametrize("shape", [(16, 40), (40, 16)])
def test_cautious_decay_closed_form(shape):
    # O from the SVD closed form; the decay mask follows the sign agreement of O and W
    lr, beta, wd, eps = 0.02, 0.95, 0.1, 1e-7
    r = rng(30)
    g = r.standard_normal(shape) * 1e-3
    U, S, Vt = np.linalg.svd(g, full_matrices=False)
    c = (1 - beta) * (1 + beta)
    R, C = shape
    O = math.sqrt(max(1.0, R / C)) * (U * p_scalar(c * S / (c * np.linalg.norm(g) + eps), [oracle.CUBIC], 5)) @ Vt
    mag = np.abs(r.standard_normal(shape)) * 0.02
    for W0, expect in ((np.sign(O) * mag, (1 - lr * wd) * np.sign(O) * mag - lr * O),     # all agree: full decay
                       (-np.sign(O) * mag, -np.sign(O) * mag - lr * O)):                    # none agree: no decay
        W1, _ = oracle.muon_update(W0, g, np.zeros(shape), lr, beta, wd, cautious=True)
        assert np.allclose(W1, expect, rtol=1e-12, atol=1e-15)
    W0 = r.standard_normal(shape) * 0.02   # mixed signs
    W1, _ = oracle.muon_update(W0, g, np.zeros(shape), lr, beta, wd, cautious=True)
    agree = O * W0 > 0
    assert 0 < agree.sum() < agree.size
    assert np.allclose(W1[agree], ((1 - lr * wd) * W0 - lr * O)[agree], rtol=1e-12, atol=1e-15)
    assert np.allclose(W1[~agree], (W0 - lr * O)[~agree], rtol=1e-12, atol=1e-15)
