"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in an oracle function (on the CPU, through
monkeypatching) and runs the pins of tests/test_oracle_pins.py that cover
that function. At least one pin must fail. A mutation that every pin accepts
would show a hole in the pins.
"""
import math

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

CUBIC = oracle.CUBIC


# ------------------------------------------------------------------ mutated oracle functions

def ns_b_sign(X, coeffs=(CUBIC,), steps=5):
    X = np.array(X, dtype=np.float64, copy=True)
    for a, b, c in oracle.coeff_schedule(coeffs, steps):
        A = X @ X.T
        X = a * X - b * (A @ X) + c * (A @ (A @ X))
    return X


def ns_drop_c_A(X, coeffs=(CUBIC,), steps=5):
    X = np.array(X, dtype=np.float64, copy=True)
    for a, b, c in oracle.coeff_schedule(coeffs, steps):
        A = X @ X.T
        X = a * X + b * (A @ X) + c * (A @ X)
    return X


def ns_transposed_operand(X, coeffs=(CUBIC,), steps=5):
    X = np.array(X, dtype=np.float64, copy=True)
    for a, b, c in oracle.coeff_schedule(coeffs, steps):
        A = X @ X.T
        X = a * X + b * (A @ X).T + c * (A @ (A @ X))  # (AX)^T in place of AX
    return X


def ns_first_coeff_only(X, coeffs=(CUBIC,), steps=5):
    X = np.array(X, dtype=np.float64, copy=True)
    a, b, c = oracle.coeff_schedule(coeffs, steps)[0]
    for _ in range(steps):
        A = X @ X.T
        X = a * X + b * (A @ X) + c * (A @ (A @ X))
    return X


def orth_no_norm(u, coeffs=(CUBIC,), steps=5, eps=1e-7):
    u = np.asarray(u, dtype=np.float64)
    R, C = u.shape
    X = u.T if R > C else u
    X = oracle.ns_iterate(X, coeffs, steps)
    return X.T if R > C else X


def orth_no_transpose_back(u, coeffs=(CUBIC,), steps=5, eps=1e-7):
    u = np.asarray(u, dtype=np.float64)
    R, C = u.shape
    X = u.T if R > C else u
    X = X / (np.linalg.norm(X) + eps)
    X = oracle.ns_iterate(X, coeffs, steps)
    return X.reshape(R, C) if R > C else X


def orth_eps_squared(u, coeffs=(CUBIC,), steps=5, eps=1e-7):
    u = np.asarray(u, dtype=np.float64)
    R, C = u.shape
    X = u.T if R > C else u
    X = X / math.sqrt(np.sum(X * X) + 1e-3)
    X = oracle.ns_iterate(X, coeffs, steps)
    return X.T if R > C else X


def mom_nesterov_old(m, g, beta, nesterov):
    m = np.asarray(m, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m_new = beta * m + (1.0 - beta) * g
    u = beta * m + (1.0 - beta) * g if nesterov else m_new
    return m_new, u


def mom_no_damping(m, g, beta, nesterov):
    m = np.asarray(m, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m_new = beta * m + g
    u = beta * m_new + g if nesterov else m_new
    return m_new, u


def adamw_no_bias_corr(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    p, g, m, v = (np.asarray(x, dtype=np.float64) for x in (p, g, m, v))
    m = beta1 * m + (1 - beta1) * g
    v = beta2 * v + (1 - beta2) * g * g
    return p * (1 - lr * weight_decay) - lr * m / (np.sqrt(v) + eps), m, v


def adamw_eps_inside(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    p, g, m, v = (np.asarray(x, dtype=np.float64) for x in (p, g, m, v))
    m = beta1 * m + (1 - beta1) * g
    v = beta2 * v + (1 - beta2) * g * g
    mh, vh = m / (1 - beta1 ** step), v / (1 - beta2 ** step)
    return p * (1 - lr * weight_decay) - lr * mh / np.sqrt(vh + eps), m, v


def adamw_decay_after(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    p, g, m, v = (np.asarray(x, dtype=np.float64) for x in (p, g, m, v))
    m = beta1 * m + (1 - beta1) * g
    v = beta2 * v + (1 - beta2) * g * g
    mh, vh = m / (1 - beta1 ** step), v / (1 - beta2 ** step)
    return (p - lr * mh / (np.sqrt(vh) + eps)) * (1 - lr * weight_decay), m, v


def adamw_beta1_for_v(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    return oracle_adamw(p, g, m, v, step, lr, beta1, beta1, eps, weight_decay)


def scale_inverted(R, C, mode=0):
    if mode == 0:
        return math.sqrt(max(1.0, C / R))
    return oracle_shape_scale(R, C, mode)


def muon_decay_no_lr(W, g, m, lr, beta, weight_decay, nesterov=True, steps=5, coeffs=(CUBIC,), eps=1e-7,
                     scale_mode=0, heads=1):
    Wn, mn = oracle_muon_update(W, g, m, lr, beta, weight_decay, nesterov, steps, coeffs, eps, scale_mode, heads)
    W = np.asarray(W, dtype=np.float64)
    return Wn + lr * weight_decay * W - weight_decay * W, mn


def muon_heads_by_columns(W, g, m, lr, beta, weight_decay, nesterov=True, steps=5, coeffs=(CUBIC,), eps=1e-7,
                          scale_mode=0, heads=1):
    if heads == 1:
        return oracle_muon_update(W, g, m, lr, beta, weight_decay, nesterov, steps, coeffs, eps, scale_mode, heads)
    W = np.asarray(W, dtype=np.float64)
    R, C = W.shape
    cw = C // heads
    m_new, u = oracle.momentum_update(m, g, beta, nesterov)
    O = np.empty_like(W)
    for h in range(heads):
        sl = slice(h * cw, (h + 1) * cw)
        O[:, sl] = oracle.shape_scale(R, cw, scale_mode) * oracle.orthogonalize(u[:, sl], coeffs, steps, eps)
    return W * (1 - lr * weight_decay) - lr * O, m_new


def muon_cautious_inverted(W, g, m, lr, beta, weight_decay, nesterov=True, steps=5, coeffs=(CUBIC,), eps=1e-7,
                           scale_mode=0, heads=1, cautious=False):
    if not cautious:
        return oracle_muon_update(W, g, m, lr, beta, weight_decay, nesterov, steps, coeffs, eps, scale_mode, heads)
    Wn, mn = oracle_muon_update(W, g, m, lr, beta, 0.0, nesterov, steps, coeffs, eps, scale_mode, heads)
    W = np.asarray(W, dtype=np.float64)
    O = (W - Wn) / lr  # the scaled update
    return W - lr * weight_decay * W * (O * W < 0) - lr * O, mn  # decays where the signs differ


def muon_cautious_ignored(W, g, m, lr, beta, weight_decay, nesterov=True, steps=5, coeffs=(CUBIC,), eps=1e-7,
                          scale_mode=0, heads=1, cautious=False):
    return oracle_muon_update(W, g, m, lr, beta, weight_decay, nesterov, steps, coeffs, eps, scale_mode, heads)


def kind_embed_to_muon(ndim, role):
    if ndim == 2 and role == oracle.ROLE_EMBED:
        return oracle.KIND_MUON
    return oracle_kind_of(ndim, role)


oracle_adamw = oracle.adamw_update
oracle_shape_scale = oracle.shape_scale
oracle_muon_update = oracle.muon_update
oracle_kind_of = oracle.kind_of


# ------------------------------------------------------------------ pins per function

NS_PINS = [
    (pins.test_ns_matches_svd_closed_form, dict(shape=(8, 16), rank=None, coeffs=[CUBIC], steps=5)),
    (pins.test_ns_matches_svd_closed_form, dict(shape=(16, 32), rank=4, coeffs=[(2.0, -1.5, 0.5)], steps=3)),
    (pins.test_ns_matches_svd_closed_form,
     dict(shape=(8, 16), rank=None, coeffs=[(1.5, -0.5, 0.0), (2.0, -1.5, 0.5), (1.2, -0.1, -0.05)], steps=3)),
    (pins.test_ns_matches_svd_closed_form, dict(shape=(32, 32), rank=None, coeffs=[CUBIC], steps=5)),
    (pins.test_ns_literal_page_form, {}),
    (pins.test_cubic_scalar_fixed_points, {}),
]
ORTH_PINS = [(pins.test_orthogonalize_svd_closed_form, dict(shape=s)) for s in [(8, 20), (20, 8)]] + [
    (pins.test_normalised_orthogonal_is_not_fixed_point, {})]
MOM_PINS = [(pins.test_momentum_closed_form_constant_grad, dict(nesterov=n)) for n in (False, True)] + [
    (pins.test_nesterov_direction_equals_heavy_ball_direction, {})]
ADAMW_PINS = [(pins.test_adamw_closed_form_constant_grad, dict(wd=wd, gscale=gs))
              for wd in (0.0, 0.3) for gs in (1e-3, 1e-9)] + [(pins.test_adamw_first_step_is_sign_like, {})]
MUON_PINS = [(pins.test_muon_one_step_closed_form, dict(shape=s, heads=h, nesterov=True, mode=0))
             for s, h in [((16, 40), 1), ((40, 16), 1), ((32, 24), 2)]] + [(pins.test_shape_scale_values, {})]
CAUTIOUS_PINS = [(pins.test_cautious_decay_closed_form, dict(shape=s)) for s in [(16, 40), (40, 16)]]
PART_PINS = [(pins.test_partition_rules, {}),
             (pins.test_partition_counts_and_exactly_once, dict(name="7b", muon=224, adamw=67, buckets=3))]

MUTATIONS = [
    ("ns_iterate", ns_b_sign, NS_PINS),
    ("ns_iterate", ns_drop_c_A, NS_PINS),
    ("ns_iterate", ns_transposed_operand, NS_PINS),
    ("ns_iterate", ns_first_coeff_only, NS_PINS),
    ("orthogonalize", orth_no_norm, ORTH_PINS),
    ("orthogonalize", orth_no_transpose_back, ORTH_PINS),
    ("orthogonalize", orth_eps_squared, ORTH_PINS),
    ("momentum_update", mom_nesterov_old, MOM_PINS),
    ("momentum_update", mom_no_damping, MOM_PINS),
    ("adamw_update", adamw_no_bias_corr, ADAMW_PINS),
    ("adamw_update", adamw_eps_inside, ADAMW_PINS),
    ("adamw_update", adamw_decay_after, ADAMW_PINS),
    ("adamw_update", adamw_beta1_for_v, ADAMW_PINS),
    ("shape_scale", scale_inverted, MUON_PINS),
    ("muon_update", muon_decay_no_lr, MUON_PINS),
    ("muon_update", muon_heads_by_columns, MUON_PINS),
    ("muon_update", muon_cautious_inverted, CAUTIOUS_PINS),
    ("muon_update", muon_cautious_ignored, CAUTIOUS_PINS),
    ("kind_of", kind_embed_to_muon, PART_PINS),
]


@pytest.mark.parametrize("name,fn,cases", MUTATIONS, ids=[f"{n}:{f.__name__}" for n, f, _ in MUTATIONS])
def test_planted_mistake_fails_a_pin(monkeypatch, name, fn, cases):
    monkeypatch.setattr(oracle, name, fn)
    caught = 0
    for pin, kw in cases:
        try:
            pin(**kw)
        except (AssertionError, ValueError, IndexError):
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake {fn.__name__} in oracle.{name}"


def test_unmutated_oracle_passes_the_same_pins():
    for _, _, cases in MUTATIONS:
        for pin, kw in cases:
            pin(**kw)
