"""Seeded synthetic inputs for the MuonAdamW optimizer step.

This module is shared by the tests, the benchmark and the CPU oracle's callers.
It holds no arithmetic of the optimizer itself: it only describes parameter
sets (shapes, roles, groups, hyperparameters) and draws seeded random weights
and gradients for them.

Recipe (every draw is reproducible from its seed tuple):

* Host draws use ``numpy.random.Generator(PCG64(SeedSequence([0, t, step, stream])))``
  where ``t`` is the tensor's index in the table, ``step`` the optimizer step the
  gradient belongs to (1-based; 0 for initial weights) and ``stream`` one of the
  ``STREAM_*`` constants below.
* Initial weights are N(0, 0.02^2) in fp32.
* Gradients are N(0, std^2) with the config's std, drawn in fp32 and, where the
  config stores bf16 gradients, rounded to bf16 with round-to-nearest-even.
* Device draws (for workloads too large for host memory) use a CUDA
  ``torch.Generator`` seeded with :func:`torch_seed` of the same tuple; they are
  a different random stream than the host draws but follow the same recipe.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Iterable

import numpy as np

# tensor roles (who gets Muon and who gets AdamW is decided elsewhere)
ROLE_HIDDEN = 0
ROLE_EMBED = 1
ROLE_UNEMBED = 2
ROLE_FORCE_ADAMW = 3

KIND_MUON = 0
KIND_ADAMW = 1

STREAM_GRAD = 0
STREAM_WEIGHT = 1
STREAM_LOWRANK = 2
STREAM_SCALE = 3
STREAM_SELECT = 4

DTYPE_F32 = "f32"
DTYPE_BF16 = "bf16"


@dataclasses.dataclass
class MuonHP:
    lr: float = 0.02
    beta: float = 0.95
    weight_decay: float = 0.01
    eps: float = 1e-7
    nesterov: bool = True
    ns_steps: int = 5
    coeffs: tuple = ((1.5, -0.5, 0.0),)  # one (a, b, c) reused, or one per iteration
    scale_mode: int = 0  # 0: sqrt(max(1,R/C)), 1: sqrt(R/C), 2: 1
    heads: int = 1
    precision: int = 0  # 0: bf16 operands, 1: fp32 compute
    cautious: bool = False  # decay only where update and weight share a sign


@dataclasses.dataclass
class AdamWHP:
    lr: float = 0.02
    beta1: float = 0.9
    beta2: float = 0.95
    eps: float = 1e-8
    weight_decay: float = 0.01


@dataclasses.dataclass
class Group:
    kind: int  # KIND_MUON or KIND_ADAMW
    muon: MuonHP = dataclasses.field(default_factory=MuonHP)
    adamw: AdamWHP = dataclasses.field(default_factory=AdamWHP)


@dataclasses.dataclass
class TensorSpec:
    name: str
    shape: tuple
    role: int
    group: int
    grad_dtype: str = DTYPE_BF16
    grad_std: float = 1e-3
    # square sweep: per-matrix gradient scale drawn log-uniform in [10^lo, 10^hi]
    grad_scale_log10: tuple | None = None
    # aspect sweep: rows of the gradient per low-rank block (one block per head
    # slice or per whole matrix) and which blocks are low-rank
    lowrank_rank: int = 0

    @property
    def numel(self) -> int:
        n = 1
        for s in self.shape:
            n *= int(s)
        return n


@dataclasses.dataclass
class Workload:
    name: str
    tensors: list
    groups: list
    description: str = ""

    @property
    def numel(self) -> int:
        return sum(t.numel for t in self.tensors)


# ---------------------------------------------------------------------------
# bf16 helpers (storage format of the inputs, not part of the optimizer)

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the 16-bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    nan = np.isnan(x)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# parameter sets

def _muon_group(**kw) -> Group:
    return Group(kind=KIND_MUON, muon=MuonHP(**kw))


def _adamw_group(**kw) -> Group:
    return Group(kind=KIND_ADAMW, adamw=AdamWHP(**kw))


def tiny() -> Workload:
    """One 256x512 fp32 weight on Muon plus a 512-element fp32 gain on AdamW."""
    groups = [
        _muon_group(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, ns_steps=5),
        _adamw_group(lr=0.02, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01),
    ]
    tensors = [
        TensorSpec("w", (256, 512), ROLE_HIDDEN, 0, DTYPE_F32, 1e-3),
        TensorSpec("gain", (512,), ROLE_HIDDEN, 1, DTYPE_F32, 1e-3),
    ]
    return Workload("tiny", tensors, groups,
                    "one 256x512 fp32 Muon weight + one 512 fp32 AdamW gain, fp32 grads N(0,1e-3^2)")


def _lm(name: str, layers: int, d: int, mlp_shapes: list, vocab: int, n_scalars_per_layer: int,
        desc: str) -> Workload:
    groups = [
        _muon_group(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, ns_steps=5),
        _adamw_group(lr=0.02, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01),
    ]
    t: list = []
    t.append(TensorSpec("embed", (vocab, d), ROLE_EMBED, 1))
    for layer in range(layers):
        for nm in ("q", "k", "v", "o"):
            t.append(TensorSpec(f"l{layer}.{nm}", (d, d), ROLE_HIDDEN, 0))
        for i, shp in enumerate(mlp_shapes):
            t.append(TensorSpec(f"l{layer}.mlp{i}", shp, ROLE_HIDDEN, 0))
        t.append(TensorSpec(f"l{layer}.norm_attn", (d,), ROLE_HIDDEN, 1))
        t.append(TensorSpec(f"l{layer}.norm_mlp", (d,), ROLE_HIDDEN, 1))
        for j in range(n_scalars_per_layer):
            t.append(TensorSpec(f"l{layer}.scalar{j}", (), ROLE_HIDDEN, 1))
    t.append(TensorSpec("norm_final", (d,), ROLE_HIDDEN, 1))
    t.append(TensorSpec("unembed", (vocab, d), ROLE_UNEMBED, 1))
    return Workload(name, t, groups, desc)


def d20() -> Workload:
    """nanochat-like depth-20 parameter set (d_model 1280)."""
    return _lm("d20", 20, 1280, [(1280, 5120), (5120, 1280)], 65536, 2,
               "20 layers d1280: Q/K/V/O 1280x1280, MLP 1280x5120 + 5120x1280 on Muon; "
               "embed/unembed 65536x1280, 41 gains, 40 0-D scalars on AdamW; fp32 W/state, bf16 grads")


def llama7b() -> Workload:
    """7B-shaped parameter set (32 layers, d 4096, MLP 11008)."""
    return _lm("7b", 32, 4096, [(4096, 11008), (4096, 11008), (11008, 4096)], 32000, 0,
               "32 layers d4096: Q/K/V/O 4096x4096, MLP 2x(4096x11008) + 11008x4096 on Muon; "
               "embed/unembed 32000x4096 and 65 RMSNorm gains on AdamW; fp32 W/state, bf16 grads")


def square(batch: int = 64, n: int = 4096) -> Workload:
    """Batch of square matrices with per-matrix gradient scales log-uniform in [1e-4, 1e-1]."""
    groups = [_muon_group(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, ns_steps=5)]
    t = [TensorSpec(f"sq{i}", (n, n), ROLE_HIDDEN, 0, DTYPE_BF16, 1.0, grad_scale_log10=(-4.0, -1.0))
         for i in range(batch)]
    return Workload(f"square{batch}x{n}", t, groups,
                    f"{batch} matrices {n}x{n}, bf16 grads N(0,1) x per-matrix 10^U[-4,-1]")


def aspect(d: int = 4096, ff: int = 14336, heads: int = 32) -> Workload:
    """Wide/tall MLP matrices (transpose path) plus per-head Q/K/V orthogonalisation."""
    groups = [
        _muon_group(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, ns_steps=5),
        _muon_group(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, ns_steps=5, heads=heads),
    ]
    t = [TensorSpec("mlp_up", (d, ff), ROLE_HIDDEN, 0, lowrank_rank=64),
         TensorSpec("mlp_down", (ff, d), ROLE_HIDDEN, 0, lowrank_rank=64)]
    for nm in ("q", "k", "v"):
        t.append(TensorSpec(nm, (d, d), ROLE_HIDDEN, 1, lowrank_rank=64))
    return Workload(f"aspect{d}x{ff}h{heads}", t, groups,
                    f"MLP {d}x{ff} and {ff}x{d}; Q/K/V {d}x{d} as {heads} heads of {d // heads}x{d}; "
                    "bf16 grads N(0,1e-3^2), 10% of units rank-64")


def rect(batch: int = 8, R: int = 4096, C: int = 11008) -> Workload:
    """Batch of the 7B-shaped set's MLP matrices (4096 x 11008 by default; 11008 x 4096 is the tall
    one), grads N(0, 1e-3^2) in bf16."""
    groups = [_muon_group(lr=0.02, beta=0.95, weight_decay=0.01, nesterov=True, ns_steps=5)]
    t = [TensorSpec(f"mlp{i}", (R, C), ROLE_HIDDEN, 0) for i in range(batch)]
    return Workload(f"rect{batch}x{R}x{C}", t, groups, f"{batch} matrices {R}x{C}, bf16 grads N(0,1e-3^2)")


WORKLOADS = {"tiny": tiny, "d20": d20, "square": square, "aspect": aspect, "7b": llama7b,
             # few-GB cases for profiler captures: 8 square 4096x4096 matrices, 8 of
             # the 7B set's 4096x11008 MLP matrices, and 8 of its 11008x4096 ones
             "square8": lambda: square(8), "rect8": lambda: rect(8), "tall8": lambda: rect(8, 11008, 4096)}


# ---------------------------------------------------------------------------
# host draws

def rng(tensor_index: int, step: int, stream: int, base: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([base, tensor_index, step, stream])))


def torch_seed(tensor_index: int, step: int, stream: int, base: int = 0) -> int:
    """A 63-bit seed for a torch generator derived from the same tuple."""
    ss = np.random.SeedSequence([base, tensor_index, step, stream])
    return int(ss.generate_state(1, dtype=np.uint64)[0] & np.uint64((1 << 63) - 1))


def initial_weight(spec: TensorSpec, tensor_index: int, base: int = 0) -> np.ndarray:
    g = rng(tensor_index, 0, STREAM_WEIGHT, base)
    return (g.standard_normal(spec.shape, dtype=np.float32) * np.float32(0.02)).astype(np.float32)


def grad_scale(spec: TensorSpec, tensor_index: int, base: int = 0) -> float:
    if spec.grad_scale_log10 is None:
        return spec.grad_std
    lo, hi = spec.grad_scale_log10
    e = rng(tensor_index, 0, STREAM_SCALE, base).uniform(lo, hi)
    return spec.grad_std * float(10.0 ** e)


def lowrank_units(wl: Workload, fraction: float = 0.1, base: int = 0) -> set:
    """Seeded choice of the (tensor_index, head) units whose gradients are low-rank."""
    units = []
    for ti, spec in enumerate(wl.tensors):
        if spec.lowrank_rank <= 0 or len(spec.shape) != 2:
            continue
        heads = wl.groups[spec.group].muon.heads if wl.groups[spec.group].kind == KIND_MUON else 1
        for h in range(heads):
            units.append((ti, h))
    if not units:
        return set()
    k = max(1, int(round(fraction * len(units))))
    sel = rng(0, 0, STREAM_SELECT, base).choice(len(units), size=k, replace=False)
    return {units[i] for i in sorted(sel.tolist())}


def gradient(wl: Workload, tensor_index: int, step: int, base: int = 0,
             lowrank: set | None = None) -> np.ndarray:
    """fp32 gradient values (already bf16-representable when the spec stores bf16)."""
    spec = wl.tensors[tensor_index]
    std = grad_scale(spec, tensor_index, base)
    g = rng(tensor_index, step, STREAM_GRAD, base).standard_normal(spec.shape, dtype=np.float32)
    g *= np.float32(std)
    if spec.lowrank_rank > 0 and len(spec.shape) == 2:
        if lowrank is None:
            lowrank = lowrank_units(wl, base=base)
        grp = wl.groups[spec.group]
        heads = grp.muon.heads if grp.kind == KIND_MUON else 1
        R, C = spec.shape
        rh = R // heads
        r = spec.lowrank_rank
        lr_rng = rng(tensor_index, step, STREAM_LOWRANK, base)
        for h in range(heads):
            if (tensor_index, h) in lowrank:
                P = lr_rng.standard_normal((rh, r), dtype=np.float32)
                Q = lr_rng.standard_normal((r, C), dtype=np.float32)
                g[h * rh:(h + 1) * rh] = (P @ Q) * np.float32(std / math.sqrt(r))
    if spec.grad_dtype == DTYPE_BF16:
        g = bf16_bits_to_f32(f32_to_bf16_bits(g)).reshape(spec.shape)
    return g.astype(np.float32)


def grad_storage(spec: TensorSpec, g: np.ndarray) -> np.ndarray:
    """The gradient in its stored dtype: fp32 array, or uint16 bf16 bit patterns."""
    if spec.grad_dtype == DTYPE_BF16:
        return f32_to_bf16_bits(g).reshape(spec.shape)
    return np.ascontiguousarray(g, dtype=np.float32)


def iter_units(wl: Workload) -> Iterable:
    for ti, spec in enumerate(wl.tensors):
        yield ti, spec
