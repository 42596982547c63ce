"""CPU oracle for the MuonAdamW optimizer step (fp64, NumPy).

TEST INFRASTRUCTURE ONLY. Only the test suite, the smoke check in
``__graft_entry__`` and the CPU-baseline / reference arms of ``bench.py`` may
import this package. The GPU library never calls it, and the two share no
code: no kernels, headers, helpers, tables or constants.

Everything is computed in float64 from the exact stored inputs. bf16 gradients
are upcast exactly and no bf16 rounding is emulated. The functions follow the
method as these pages describe it:

* "How nanochat Combines Muon and AdamW in a Single Optimizer" (instagit):
  "Parameter Grouping Strategy", "AdamW Step Implementation", "Muon Step
  Implementation", and the FAQ "Which parameters does Muon optimize versus
  AdamW in nanochat?".
* "MuonClip Optimizer" (wiki): "Newton-Schulz Orthogonalization" (the cubic
  iteration), "Momentum" (the EMA form with decay 0.95) and "Design Decisions"
  (5 iterations).
* "Guidelines for whether to use muon for parameters" (KellerJordan/Muon issue
  31): the hidden / non-hidden split, and the RMS-to-RMS rationale.
* "nemo_automodel.components.optim.muown_triton": the ``_finish`` contract.
  Its scale comes from the global matrix shape. lr and the bias corrections
  are runtime scalars. Weights are decayed in place.
* "Qwen Training Details: Full-Network Muon Optimizer and Residual Stream
  Design", "Confirmed": per-head orthogonalisation, and forcing AdamW on
  some projections.

Readings where the pages are silent:

* Frobenius normalisation ``X0 = u / (||u||_F + eps)`` with eps = 1e-7.
* Nesterov form ``u = beta*m_new + (1-beta)*g``.
* Shape scale ``s = sqrt(max(1, R/C))`` (mode 0), ``sqrt(R/C)`` (mode 1),
  or 1 (mode 2).
* Decoupled weight decay ``W*(1 - lr*wd)``, applied to the pre-update weight;
  the cautious option decays only where the update and the weight share a sign.
* AdamW eps is added after the bias-corrected square root.
* Head h of an R x C matrix split into H heads is rows [h*R/H, (h+1)*R/H).

Parity pins (tests/test_oracle_pins.py) tie each function to something
outside itself: an SVD closed form, fixed points, closed forms after k steps,
invariances, brute force, and the constants the pages print. The shape-scale
*choice*, the normalisation eps and the Nesterov *form* are readings the pages
do not fix. Their arithmetic is pinned, but whether the choice matches the
pages' own code is parity unpinned.
"""
from __future__ import annotations

import math

import numpy as np

KIND_MUON = 0
KIND_ADAMW = 1
ROLE_HIDDEN = 0
ROLE_EMBED = 1
ROLE_UNEMBED = 2
ROLE_FORCE_ADAMW = 3

# "MuonClip Optimizer", "Newton-Schulz Orthogonalization": X <- 1.5 X - 0.5 X (X^T X)
CUBIC = (1.5, -0.5, 0.0)
# "MuonClip Optimizer", "Design Decisions": 5 iterations, momentum decay 0.95
DEFAULT_NS_STEPS = 5
DEFAULT_MOMENTUM = 0.95


class UnsupportedTensor(ValueError):
    pass


# ---------------------------------------------------------------------------
# partition ("Parameter Grouping Strategy"; Muon issue 31; Qwen "Confirmed")

def kind_of(ndim: int, role: int) -> int:
    """Which optimizer a tensor gets.

    Tensors with fewer than two dimensions go to AdamW. 2-D matrices go to
    Muon ("Parameter Grouping Strategy"), except the embedding and unembedding
    (head) matrices. Their input or output is not RMS-normed, so they belong
    to the non-hidden set (issue 31). Tensors that the caller forces onto
    AdamW also go there (Qwen "Confirmed": router / GR projections). The
    method is defined for 2-D matrices only, so ndim >= 3 is rejected.
    """
    if ndim < 0:
        raise UnsupportedTensor("negative ndim")
    if ndim <= 1:
        return KIND_ADAMW
    if ndim >= 3:
        raise UnsupportedTensor("ndim >= 3 is not defined for this method")
    if role in (ROLE_EMBED, ROLE_UNEMBED, ROLE_FORCE_ADAMW):
        return KIND_ADAMW
    if role != ROLE_HIDDEN:
        raise UnsupportedTensor(f"unknown role {role}")
    return KIND_MUON


def partition(shapes_roles) -> list:
    """Kind (KIND_MUON / KIND_ADAMW) per tensor, in table order."""
    return [kind_of(len(tuple(shape)), role) for shape, role in shapes_roles]


def muon_buckets(shapes_roles, groups_of) -> list:
    """Same-shape, same-group Muon matrices, bucketed in first-appearance order.

    Stacking same-shape matrices so that they run as one batch follows "Muon
    Step Implementation" (gradients and parameters are stacked). Returns a
    list of (group, R, C, [tensor indices]).
    """
    kinds = partition(shapes_roles)
    order = []
    members = {}
    for i, ((shape, _role), kind) in enumerate(zip(shapes_roles, kinds)):
        if kind != KIND_MUON:
            continue
        key = (groups_of[i], int(shape[0]), int(shape[1]))
        if key not in members:
            members[key] = []
            order.append(key)
        members[key].append(i)
    return [(k[0], k[1], k[2], members[k]) for k in order]


# ---------------------------------------------------------------------------
# AdamW ("AdamW Step Implementation"; muown_triton ``_finish``: runtime BC1/BC2)

def adamw_update(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    """One AdamW step on one tensor. Returns new (p, m, v) as float64 arrays.

    ``step`` is the 1-based index of the step being taken. The bias
    corrections 1 - beta^step are runtime scalars.
    """
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    m_new = beta1 * m + (1.0 - beta1) * g
    v_new = beta2 * v + (1.0 - beta2) * g * g
    m_hat = m_new / (1.0 - beta1 ** step)
    v_hat = v_new / (1.0 - beta2 ** step)
    p_new = p * (1.0 - lr * weight_decay) - lr * m_hat / (np.sqrt(v_hat) + eps)
    return p_new, m_new, v_new


# ---------------------------------------------------------------------------
# Muon pieces

def momentum_update(m, g, beta, nesterov):
    """EMA momentum ("MuonClip Optimizer", "Momentum"), plus the Nesterov option.

    m_new = beta*m + (1-beta)*g. With Nesterov the direction is
    u = beta*m_new + (1-beta)*g, the same EMA applied once more to the fresh
    gradient. Without it, u = m_new.
    """
    m = np.asarray(m, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m_new = beta * m + (1.0 - beta) * g
    u = beta * m_new + (1.0 - beta) * g if nesterov else m_new
    return m_new, u


def coeff_schedule(coeffs, steps):
    """(a, b, c) for each of ``steps`` iterations. A single triple is reused."""
    coeffs = [tuple(float(x) for x in c) for c in coeffs]
    if len(coeffs) == 1:
        return coeffs * steps
    if len(coeffs) < steps:
        raise ValueError("fewer coefficient triples than iterations")
    return coeffs[:steps]


def ns_iterate(X, coeffs=(CUBIC,), steps=DEFAULT_NS_STEPS):
    """Newton-Schulz iteration, with no normalisation.

    The page prints the cubic X <- 1.5 X - 0.5 X (X^T X) ("MuonClip
    Optimizer", "Newton-Schulz Orthogonalization"). Its general odd-polynomial
    form is X <- a X + b X (X^T X) + c X (X^T X)^2. X (X^T X) equals
    (X X^T) X, so the Gram is formed on the short side. On a wide X
    (rows <= cols), A = X X^T is the smaller matrix.
    """
    X = np.array(X, dtype=np.float64, copy=True)
    for a, b, c in coeff_schedule(coeffs, steps):
        A = X @ X.T
        AX = A @ X
        Xn = a * X + b * AX
        if c != 0.0:
            Xn = Xn + c * (A @ AX)
        X = Xn
    return X


def orthogonalize(u, coeffs=(CUBIC,), steps=DEFAULT_NS_STEPS, eps=1e-7):
    """Frobenius-normalise u, make it wide, run Newton-Schulz, restore the orientation."""
    u = np.asarray(u, dtype=np.float64)
    R, C = u.shape
    transposed = R > C
    X = u.T if transposed else u
    X = X / (np.linalg.norm(X) + eps)
    X = ns_iterate(X, coeffs, steps)
    return X.T if transposed else X


def shape_scale(R, C, mode=0):
    """Update scale from the global matrix shape (muown_triton ``_finish``).

    The pages say only that the scale depends on the global shape. The
    RMS-to-RMS rationale (issue 31) suggests sqrt(fan_out / fan_in). Mode 0
    clips that at 1.
    """
    if mode == 0:
        return math.sqrt(max(1.0, R / C))
    if mode == 1:
        return math.sqrt(R / C)
    if mode == 2:
        return 1.0
    raise ValueError("scale mode")


def muon_update(W, g, m, lr, beta, weight_decay, nesterov=True, steps=DEFAULT_NS_STEPS,
                coeffs=(CUBIC,), eps=1e-7, scale_mode=0, heads=1, cautious=False):
    """One Muon step on one R x C matrix. Returns new (W, m) as float64.

    Steps, in the order of "Muon Step Implementation": momentum (plus
    Nesterov), then orthogonalisation, then decoupled decay and the write
    back. With ``heads > 1`` each block of R/heads rows is orthogonalised on
    its own (Qwen "Confirmed": per-head orthogonalisation), and the scale uses
    the slice shape.

    ``cautious``: the same page names "cautious weight decay" without defining
    it. The reading taken: decay only the elements where the orthogonalised
    update O and the pre-update weight W have the same sign (O*W > 0). Parity
    of this reading is unpinned by the pages.
    """
    W = np.asarray(W, dtype=np.float64)
    R, C = W.shape
    if heads < 1 or R % heads != 0:
        raise UnsupportedTensor("rows must split evenly into heads")
    m_new, u = momentum_update(m, g, beta, nesterov)
    rh = R // heads
    O = np.empty_like(W)
    for h in range(heads):
        sl = slice(h * rh, (h + 1) * rh)
        O[sl] = shape_scale(rh, C, scale_mode) * orthogonalize(u[sl], coeffs, steps, eps)
    if cautious:
        W_new = W - lr * weight_decay * W * (O * W > 0) - lr * O
    else:
        W_new = W * (1.0 - lr * weight_decay) - lr * O
    return W_new, m_new


# ---------------------------------------------------------------------------
# whole step over a parameter table ("The MuonAdamW Class Architecture")

def muonadamw_step(tensors, groups, params, grads, state, step):
    """One MuonAdamW step over every tensor in the table.

    tensors: list of dicts with "shape", "role", "group".
    groups:  list of dicts with "kind" and its hyperparameters (MuonHP/AdamWHP fields).
    params / grads: lists of arrays. state: list of dicts that this function
    fills ("m" for Muon; "exp_avg", "exp_avg_sq" for AdamW). Missing state
    starts at zero, as it is created on the first step.
    Returns the list of new parameters (float64). ``state`` is updated in place.
    """
    kinds = partition([(t["shape"], t["role"]) for t in tensors])
    out = []
    for i, t in enumerate(tensors):
        grp = groups[t["group"]]
        if grp["kind"] != kinds[i]:
            raise UnsupportedTensor(f"tensor {i} is in a group of the wrong kind")
        p = np.asarray(params[i], dtype=np.float64)
        g = np.asarray(grads[i], dtype=np.float64)
        st = state[i]
        if kinds[i] == KIND_ADAMW:
            m = st.get("exp_avg", np.zeros_like(p))
            v = st.get("exp_avg_sq", np.zeros_like(p))
            p, st["exp_avg"], st["exp_avg_sq"] = adamw_update(
                p, g, m, v, step, grp["lr"], grp["beta1"], grp["beta2"], grp["eps"],
                grp["weight_decay"])
        else:
            m = st.get("m", np.zeros_like(p))
            p, st["m"] = muon_update(
                p, g, m, grp["lr"], grp["beta"], grp["weight_decay"], grp["nesterov"],
                grp["ns_steps"], grp["coeffs"], grp["eps"], grp["scale_mode"], grp["heads"],
                grp.get("cautious", False))
        out.append(p)
    return out


# ---------------------------------------------------------------------------
# tolerance helpers used by the parity tests

def rel_frobenius(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    num = np.linalg.norm(x - ref)
    return num / den if den > 0 else num


def adamw_term_magnitudes(p, g, m, v, step, lr, beta1, beta2, eps, weight_decay):
    """Per-element sum of |addends| in each updated quantity, for the cancellation-safe bound.

    The step term lr * m_hat / (sqrt(v_hat) + eps) contains the sum
    beta1*m + (1-beta1)*g, which can cancel. Its addends enter in absolute
    value, so the bound follows the magnitudes that the computation handles
    (forward error propagation), not just the magnitude of the final result.
    """
    p = np.asarray(p, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    v_new = beta2 * v + (1.0 - beta2) * g * g
    v_hat = v_new / (1.0 - beta2 ** step)
    t_m = np.abs(beta1 * m) + np.abs((1.0 - beta1) * g)
    t_v = np.abs(beta2 * v) + np.abs((1.0 - beta2) * g * g)
    t_p = np.abs(p * (1.0 - lr * weight_decay)) + lr * (t_m / (1.0 - beta1 ** step)) / (np.sqrt(v_hat) + eps)
    return t_p, t_m, t_v
