"""Shared helpers for the GPU parity tests (not collected as tests).

Tolerances come from the method's target precision and are stated here:

* AdamW and momentum state: per element |x - ref| <= 1e-6 * (sum of |addends|),
  with the addends taken from the oracle's own update (guards cancellation).
* Muon update ``dW = W_new - (1 - lr*wd) * W_old``: relative Frobenius error
  <= 2e-2 with bf16 Newton-Schulz operands and <= 1e-5 in fp32 mode, plus the
  fp32 storage rounding of W_new itself (2^-23 * ||W_new||_F), which the
  update cannot be more precise than.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
import synth

TOL_BF16 = 2e-2
TOL_F32 = 1e-5
TOL_STATE = 1e-6


def f32(x: float) -> float:
    """A hyperparameter as the library receives it: rounded to fp32, then exact in fp64."""
    return float(np.float32(x))


def hp32(hp):
    """Copy of a synth MuonHP / AdamWHP with every float field rounded to fp32."""
    import dataclasses
    kw = {}
    for f in dataclasses.fields(hp):
        v = getattr(hp, f.name)
        if isinstance(v, float):
            v = f32(v)
        elif f.name == "coeffs":
            v = tuple(tuple(f32(x) for x in c) for c in v)
        kw[f.name] = v
    return type(hp)(**kw)


def dev_f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()


def dev_grad(g: np.ndarray, dtype: str) -> torch.Tensor:
    """Upload fp32 values that are bf16-representable as a bf16 tensor (or fp32)."""
    if dtype == "bf16":
        bits = synth.f32_to_bf16_bits(g).view(np.int16)
        return torch.from_numpy(np.ascontiguousarray(bits)).cuda().view(torch.bfloat16)
    return dev_f32(g)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.detach().cpu().numpy().astype(np.float64)


def bf16_round(a: np.ndarray) -> np.ndarray:
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(a, np.float32))).reshape(np.shape(a))


def check_state(got, ref, terms, tol=TOL_STATE, what="state"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    bound = tol * np.asarray(terms, np.float64) + 1e-30
    bad = np.abs(got - ref) > bound
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements exceed the bound; worst "
                           f"{np.max(np.abs(got - ref) / bound):.3g}x")


def muon_update_error(W_old, W_new_gpu, W_new_ref, lr, wd):
    rho = 1.0 - lr * wd
    d_gpu = np.asarray(W_new_gpu, np.float64) - rho * np.asarray(W_old, np.float64)
    d_ref = np.asarray(W_new_ref, np.float64) - rho * np.asarray(W_old, np.float64)
    num = np.linalg.norm(d_gpu - d_ref)
    den = np.linalg.norm(d_ref)
    storage = 2.0 ** -23 * np.linalg.norm(W_new_ref)
    return num, den, storage


def check_muon(W_old, W_new_gpu, W_new_ref, lr, wd, tol, what="muon"):
    num, den, storage = muon_update_error(W_old, W_new_gpu, W_new_ref, lr, wd)
    assert num <= tol * den + storage, f"{what}: relative update error {num / max(den, 1e-300):.3e} > {tol}"
    return num / max(den, 1e-300)


def oracle_muon(W, g, m, hp: synth.MuonHP):
    return oracle.muon_update(W, g, m, hp.lr, hp.beta, hp.weight_decay, hp.nesterov, hp.ns_steps, hp.coeffs,
                              hp.eps, hp.scale_mode, hp.heads, hp.cautious)


def momentum_terms(m_old, g, beta):
    return np.abs(beta * np.asarray(m_old, np.float64)) + np.abs((1 - beta) * np.asarray(g, np.float64))
