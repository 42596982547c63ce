"""Device-side draws for workloads too large for host memory.

Same recipe as the host draws in ``synth`` (weights N(0, 0.02^2) fp32; gradients
N(0, std^2) in the spec's dtype, with the square sweep's per-matrix scale and
the aspect sweep's rank-64 units). Each tensor uses its own CUDA generator,
seeded from the (base, tensor, step, stream) tuple. Only torch random draws and
dtype conversion happen here: none of the optimizer's arithmetic.
"""
from __future__ import annotations

import math

import torch

from . import (DTYPE_BF16, STREAM_GRAD, STREAM_LOWRANK, STREAM_WEIGHT, KIND_MUON, Workload, grad_scale,
               lowrank_units, torch_seed)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def weights(wl: Workload, device="cuda", base: int = 0) -> list:
    out = []
    for i, spec in enumerate(wl.tensors):
        g = _gen(device, torch_seed(i, 0, STREAM_WEIGHT, base))
        out.append(torch.randn(spec.shape, generator=g, device=device, dtype=torch.float32).mul_(0.02))
    return out


def gradients(wl: Workload, step: int, device="cuda", base: int = 0, out: list | None = None) -> list:
    """Gradients for ``step``; writes into ``out`` (same shapes and dtypes) when given."""
    lowrank = lowrank_units(wl, base=base) if any(t.lowrank_rank for t in wl.tensors) else set()
    res = []
    for i, spec in enumerate(wl.tensors):
        std = grad_scale(spec, i, base)
        g = _gen(device, torch_seed(i, step, STREAM_GRAD, base))
        x = torch.randn(spec.shape, generator=g, device=device, dtype=torch.float32).mul_(std)
        if spec.lowrank_rank > 0 and len(spec.shape) == 2:
            grp = wl.groups[spec.group]
            heads = grp.muon.heads if grp.kind == KIND_MUON else 1
            R, C = spec.shape
            rh, r = R // heads, spec.lowrank_rank
            lg = _gen(device, torch_seed(i, step, STREAM_LOWRANK, base))
            for h in range(heads):
                if (i, h) in lowrank:
                    P = torch.randn((rh, r), generator=lg, device=device)
                    Q = torch.randn((r, C), generator=lg, device=device)
                    x[h * rh:(h + 1) * rh] = (P @ Q) * (std / math.sqrt(r))
        dt = torch.bfloat16 if spec.grad_dtype == DTYPE_BF16 else torch.float32
        if out is not None:
            out[i].copy_(x.to(dt))
            res.append(out[i])
        else:
            res.append(x.to(dt))
        del x
    return res
