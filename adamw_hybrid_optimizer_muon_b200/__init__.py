"""Python binding of the B200 MuonAdamW library (ctypes over ``lib/libmuonadamw.so``).

Argument marshalling only: every step of the optimizer runs in the library's
CUDA kernels. PyTorch supplies device memory and streams. The functions keep
the C names (``ma_partition``, ``muon_step_batched``, ``adamw_step_fused``,
``muonadamw_step``, ...). A missing or unloadable library raises
``LibraryMissing``. There is no fallback of any kind.
"""
from __future__ import annotations

import ctypes
import os
from typing import Sequence

__all__ = [
    "LibraryMissing", "MAError", "lib", "MuonHParams", "AdamWHParams", "Group", "Tensor",
    "MA_OK", "MA_F32", "MA_BF16", "MA_MUON", "MA_ADAMW", "ROLE_HIDDEN", "ROLE_EMBED", "ROLE_UNEMBED",
    "ROLE_FORCE_ADAMW", "ShardSlot", "ShardBucket", "SHARD_ALIGN", "ma_partition", "ma_assign_owners",
    "ma_shard_layout", "muon_workspace_bytes", "muon_step_batched",
    "muon_step_batched_noalloc", "STATIC_SCRATCH_BYTES", "ns_iterate_workspace_bytes", "ns_iterate_bf16",
    "adamw_step_fused", "ma_plan_create", "muonadamw_step", "muonadamw_step_graph", "muonadamw_step_from_host",
    "ma_plan_describe", "ma_plan_destroy", "ma_plan_status", "ma_device_status", "ma_device_status_async",
    "ma_set_wait_limit_ns", "ma_set_momentum_overlap", "ma_debug_build", "MA_ERR_BOUNDS",
    "ma_selftest_wait_timeout", "ma_profile_enable", "ma_profile_collect", "PROF_CLASSES", "group_table", "Plan",
    "MuonAdamW", "muon_hparams", "adamw_hparams",
]

HERE = os.path.dirname(os.path.abspath(__file__))
# The release library, or (MA_LIBRARY=debug) the build with guarded device
# indexing, lib/libmuonadamw_debug.so; both are compiled by build.py.
LIB_PATH = os.path.join(HERE, "lib", "libmuonadamw_debug.so" if os.environ.get("MA_LIBRARY") == "debug"
                        else "libmuonadamw.so")

MA_OK, MA_ERR_NULL, MA_ERR_SHAPE, MA_ERR_DTYPE, MA_ERR_ALIGN, MA_ERR_WORKSPACE = 0, 1, 2, 3, 4, 5
MA_ERR_UNSUPPORTED, MA_ERR_CUDA, MA_ERR_TIMEOUT, MA_ERR_ARG, MA_ERR_BOUNDS = 6, 7, 8, 9, 10
MA_F32, MA_BF16 = 0, 1
MA_MUON, MA_ADAMW = 0, 1
ROLE_HIDDEN, ROLE_EMBED, ROLE_UNEMBED, ROLE_FORCE_ADAMW = 0, 1, 2, 3
MAX_NS_STEPS = 16
MAX_GROUPS = 32
MAX_BATCH = 256


class LibraryMissing(RuntimeError):
    """The compiled library is absent or cannot be loaded (there is no CPU fallback)."""


class MAError(RuntimeError):
    """A C entry point returned a nonzero status; ``code`` holds it."""
    def __init__(self, code: int, what: str = ""):
        self.code = int(code)
        msg = _lib_status_string(code)
        super().__init__(f"{what}: {msg} (status {code})" if what else f"{msg} (status {code})")


# ---------------------------------------------------------------------------- structs (mirror muonadamw.h)

class MuonHParams(ctypes.Structure):
    """ma_muon_hparams_t: Muon hyperparameters (lr, beta, weight decay, eps, Nesterov,
    Newton-Schulz schedule, scale mode, heads, precision, cautious decay)."""
    _fields_ = [("lr", ctypes.c_float), ("beta", ctypes.c_float), ("weight_decay", ctypes.c_float),
                ("eps", ctypes.c_float), ("nesterov", ctypes.c_int32), ("ns_steps", ctypes.c_int32),
                ("n_coeffs", ctypes.c_int32), ("coeffs", (ctypes.c_float * 3) * MAX_NS_STEPS),
                ("scale_mode", ctypes.c_int32), ("heads", ctypes.c_int32), ("precision", ctypes.c_int32),
                ("cautious", ctypes.c_int32)]


class AdamWHParams(ctypes.Structure):
    """ma_adamw_hparams_t: AdamW hyperparameters and the 1-based step being taken."""
    _fields_ = [("lr", ctypes.c_float), ("beta1", ctypes.c_float), ("beta2", ctypes.c_float),
                ("eps", ctypes.c_float), ("weight_decay", ctypes.c_float), ("step", ctypes.c_int64)]


class Group(ctypes.Structure):
    """ma_group_t: one parameter group, Muon or AdamW by ``kind``."""
    _fields_ = [("kind", ctypes.c_int32), ("muon", MuonHParams), ("adamw", AdamWHParams)]


class Tensor(ctypes.Structure):
    """ma_tensor_t: one tensor of the table (device pointers, gradient dtype, shape, role, group)."""
    _fields_ = [("param", ctypes.c_void_p), ("grad", ctypes.c_void_p), ("grad_dtype", ctypes.c_int32),
                ("state0", ctypes.c_void_p), ("state1", ctypes.c_void_p), ("ndim", ctypes.c_int32),
                ("shape", ctypes.c_int64 * 2), ("role", ctypes.c_int32), ("group", ctypes.c_int32)]


class ShardSlot(ctypes.Structure):
    """ma_shard_slot_t: where a tensor sits in the flat buffers of a sharded step."""
    _fields_ = [("bucket", ctypes.c_int32), ("owner", ctypes.c_int32), ("offset", ctypes.c_int64)]


class ShardBucket(ctypes.Structure):
    """ma_shard_bucket_t: one bucket of a sharded step (kind, tensors, start, per-rank segment)."""
    _fields_ = [("kind", ctypes.c_int32), ("count", ctypes.c_int32), ("start", ctypes.c_int64),
                ("seg", ctypes.c_int64)]


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded library. Raises LibraryMissing when it has not been built."""
    global _LIB
    if _LIB is not None:
        return _LIB
    if not os.path.exists(LIB_PATH):
        raise LibraryMissing(f"{LIB_PATH} is missing: build it with `python -m adamw_hybrid_optimizer_muon_b200.build`")
    try:
        L = ctypes.CDLL(LIB_PATH)
    except OSError as e:
        raise LibraryMissing(f"cannot load {LIB_PATH}: {e}") from e
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    pp = ctypes.POINTER(ctypes.c_void_p)
    sig = {
        "ma_status_string": (ctypes.c_char_p, [i32]),
        "ma_version": (i32, []),
        "ma_struct_size": (sz, [i32]),
        "ma_partition": (i32, [ctypes.POINTER(Tensor), i32, ctypes.POINTER(ctypes.c_int32)]),
        "ma_assign_owners": (i32, [ctypes.POINTER(Tensor), i32, ctypes.POINTER(Group), i32, i32,
                                   ctypes.POINTER(ctypes.c_int32)]),
        "ma_shard_layout": (i32, [ctypes.POINTER(Tensor), i32, ctypes.POINTER(Group), i32, i32, i64,
                                  ctypes.POINTER(ShardSlot), ctypes.POINTER(ShardBucket), ctypes.POINTER(i32),
                                  ctypes.POINTER(i64)]),
        "muon_workspace_bytes": (sz, [i32, i64, i64, ctypes.POINTER(MuonHParams)]),
        "muon_step_batched": (i32, [i32, i64, i64, pp, pp, i32, pp, ctypes.POINTER(MuonHParams), vp, sz, vp]),
        "ns_iterate_workspace_bytes": (sz, [i32, i64, i64]),
        "ns_iterate_bf16": (i32, [i32, i64, i64, vp, vp, ctypes.POINTER(ctypes.c_float), i32, i32, vp, sz, vp]),
        "adamw_step_fused": (i32, [i32, pp, pp, i32, pp, pp, ctypes.POINTER(ctypes.c_int64),
                                   ctypes.POINTER(AdamWHParams), vp]),
        "ma_plan_create": (i32, [ctypes.POINTER(Tensor), i32, ctypes.POINTER(Group), i32, ctypes.POINTER(vp),
                                 ctypes.POINTER(sz)]),
        "muonadamw_step": (i32, [vp, ctypes.POINTER(Group), vp, sz, vp]),
        "muonadamw_step_from_host": (i32, [vp, ctypes.POINTER(Group), pp, vp, sz, vp, vp]),
        "ma_plan_last_launches": (i32, [vp]),
        "muonadamw_step_graph": (i32, [vp, ctypes.POINTER(Group), vp, sz, vp]),
        "ma_plan_graph_captures": (i32, [vp]),
        "ma_plan_describe": (i32, [vp, ctypes.POINTER(Group), ctypes.c_char_p, sz]),
        "ma_plan_destroy": (None, [vp]),
        "ma_device_status": (i32, [vp, i32]),
        "ma_device_status_async": (i32, [vp, vp]),
        "ma_plan_status": (i32, [vp, vp]),
        "ma_set_wait_limit_ns": (i32, [i64]),
        "ma_set_momentum_overlap": (i32, [i32]),
        "ma_debug_build": (i32, []),
        "ma_selftest_wait_timeout": (i32, [i64, vp]),
        "muon_step_batched_noalloc": (i32, [i32, i64, i64, pp, pp, i32, pp, ctypes.POINTER(MuonHParams), vp]),
        "ma_profile_enable": (i32, [i32]),
        "ma_profile_collect": (i32, [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_int64),
                                     ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    for which, cls in enumerate((Tensor, Group, MuonHParams, AdamWHParams, ShardSlot, ShardBucket)):
        if L.ma_struct_size(which) != ctypes.sizeof(cls):
            raise LibraryMissing(f"ABI mismatch for {cls.__name__}: C {L.ma_struct_size(which)} "
                                 f"vs Python {ctypes.sizeof(cls)}")
    _LIB = L
    return L


def _lib_status_string(code: int) -> str:
    try:
        return lib().ma_status_string(int(code)).decode()
    except LibraryMissing:
        return "status"


def _check(code: int, what: str) -> None:
    if code != MA_OK:
        raise MAError(code, what)


# ---------------------------------------------------------------------------- marshalling helpers

def _ptr(x) -> int:
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _ptr_array(xs) -> ctypes.Array:
    arr = (ctypes.c_void_p * max(1, len(xs)))()
    for i, x in enumerate(xs):
        arr[i] = _ptr(x)
    return arr


def _stream(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(stream, int):
        return stream
    return int(stream.cuda_stream)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return MA_BF16
    if t.dtype == torch.float32:
        return MA_F32
    raise MAError(MA_ERR_DTYPE, f"unsupported gradient dtype {t.dtype}")


def muon_hparams(lr=0.02, beta=0.95, weight_decay=0.01, eps=1e-7, nesterov=True, ns_steps=5,
                 coeffs=((1.5, -0.5, 0.0),), scale_mode=0, heads=1, precision=0, cautious=False) -> MuonHParams:
    """Build Muon hyperparameters; ``coeffs`` is one (a, b, c) triple for every iteration or one per iteration."""
    hp = MuonHParams()
    hp.lr, hp.beta, hp.weight_decay, hp.eps = lr, beta, weight_decay, eps
    hp.nesterov, hp.ns_steps, hp.n_coeffs = int(bool(nesterov)), int(ns_steps), len(coeffs)
    if len(coeffs) > MAX_NS_STEPS:
        raise MAError(MA_ERR_ARG, "too many coefficient triples")
    for k, (a, b, c) in enumerate(coeffs):
        hp.coeffs[k][0], hp.coeffs[k][1], hp.coeffs[k][2] = a, b, c
    hp.scale_mode, hp.heads, hp.precision = int(scale_mode), int(heads), int(precision)
    hp.cautious = int(bool(cautious))
    return hp


def adamw_hparams(lr=0.02, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.01, step=1) -> AdamWHParams:
    """Build AdamW hyperparameters."""
    hp = AdamWHParams()
    hp.lr, hp.beta1, hp.beta2, hp.eps, hp.weight_decay, hp.step = lr, beta1, beta2, eps, weight_decay, int(step)
    return hp


# ---------------------------------------------------------------------------- entry points

def ma_partition(tensors: Sequence[Tensor]) -> list:
    """Kind (MA_MUON or MA_ADAMW) of each tensor descriptor, by rank and role (host-only)."""
    n = len(tensors)
    arr = (Tensor * max(1, n))(*tensors)
    out = (ctypes.c_int32 * max(1, n))()
    _check(lib().ma_partition(arr, n, out), "ma_partition")
    return [int(out[i]) for i in range(n)]


def ma_assign_owners(tensors: Sequence[Tensor], groups: Sequence[Group], world_size: int) -> list:
    """Owner rank of each tensor for a sharded data-parallel step over ``world_size`` ranks (host-only)."""
    n = len(tensors)
    arr = (Tensor * max(1, n))(*tensors)
    garr = (Group * max(1, len(groups)))(*groups)
    out = (ctypes.c_int32 * max(1, n))()
    _check(lib().ma_assign_owners(arr, n, garr, len(groups), int(world_size), out), "ma_assign_owners")
    return [int(out[i]) for i in range(n)]


SHARD_ALIGN = 64  # MA_SHARD_ALIGN


def ma_shard_layout(tensors: Sequence[Tensor], groups: Sequence[Group], world_size: int, seg_cap: int):
    """Flat-buffer layout of a sharded data-parallel step (host-only).

    Returns (slots, buckets, total): per tensor a (bucket, owner, offset) tuple
    (owner -1 for AdamW tensors, which are split by element range), per bucket
    a (kind, count, start, seg) tuple, and the flat buffers' length in elements.
    """
    n = len(tensors)
    arr = (Tensor * max(1, n))(*tensors)
    garr = (Group * max(1, len(groups)))(*groups)
    slots = (ShardSlot * max(1, n))()
    buckets = (ShardBucket * max(1, n))()
    nb, total = ctypes.c_int(0), ctypes.c_int64(0)
    _check(lib().ma_shard_layout(arr, n, garr, len(groups), int(world_size), int(seg_cap), slots, buckets,
                                 ctypes.byref(nb), ctypes.byref(total)), "ma_shard_layout")
    return ([(int(s.bucket), int(s.owner), int(s.offset)) for s in slots[:n]],
            [(int(b.kind), int(b.count), int(b.start), int(b.seg)) for b in buckets[:nb.value]],
            int(total.value))


def muon_workspace_bytes(batch: int, R: int, C: int, hp: MuonHParams) -> int:
    """Workspace bytes muon_step_batched needs for ``batch`` R x C matrices."""
    v = lib().muon_workspace_bytes(int(batch), int(R), int(C), ctypes.byref(hp))
    if v == ctypes.c_size_t(-1).value:
        raise MAError(MA_ERR_ARG, "muon_workspace_bytes")
    return int(v)


def muon_step_batched(W, G, M, hp: MuonHParams, ws, ws_bytes: int | None = None, stream=None,
                      gdt: int | None = None, shape=None) -> None:
    """One Muon step on same-shape matrices. W, G, M: sequences of torch tensors (or device pointers)."""
    batch = len(W)
    if shape is None:
        R, C = (int(W[0].shape[0]), int(W[0].shape[1])) if batch else (0, 0)
    else:
        R, C = int(shape[0]), int(shape[1])
    if gdt is None:
        gdt = _dtype_code(G[0]) if batch else MA_F32
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size() if ws is not None else 0
    _check(lib().muon_step_batched(batch, R, C, _ptr_array(W), _ptr_array(G), int(gdt), _ptr_array(M),
                                   ctypes.byref(hp), _ptr(ws), int(ws_bytes), _stream(stream)),
           "muon_step_batched")


STATIC_SCRATCH_BYTES = 64 << 20  # MA_STATIC_SCRATCH_BYTES


def muon_step_batched_noalloc(W, G, M, hp: MuonHParams, stream=None, gdt: int | None = None, shape=None) -> None:
    """muon_step_batched without a workspace argument: for callers that cannot
    allocate device memory. Its scratch is the library's fixed device array of
    STATIC_SCRATCH_BYTES per GPU, shared by every call: calls that overlap on
    the GPU race. The first call on a device looks up the array's address and
    should come before any stream capture. Raises MAError(MA_ERR_WORKSPACE)
    when the step needs more scratch than the array holds."""
    batch = len(W)
    if shape is None:
        R, C = (int(W[0].shape[0]), int(W[0].shape[1])) if batch else (0, 0)
    else:
        R, C = int(shape[0]), int(shape[1])
    if gdt is None:
        gdt = _dtype_code(G[0]) if batch else MA_F32
    _check(lib().muon_step_batched_noalloc(batch, R, C, _ptr_array(W), _ptr_array(G), int(gdt), _ptr_array(M),
                                           ctypes.byref(hp), _stream(stream)), "muon_step_batched_noalloc")


def ns_iterate_workspace_bytes(batch: int, m: int, n: int) -> int:
    """Workspace bytes ns_iterate_bf16 needs for ``batch`` m x n matrices."""
    return int(lib().ns_iterate_workspace_bytes(int(batch), int(m), int(n)))


def ns_iterate_bf16(X_in, X_out, coeffs, steps: int, ws, ws_bytes: int | None = None, stream=None) -> None:
    """Newton-Schulz iterations (no normalisation) on a [batch, m, n] bf16 tensor with m <= n."""
    batch, m, n = (int(s) for s in X_in.shape)
    flat = [float(x) for c in coeffs for x in c]
    carr = (ctypes.c_float * len(flat))(*flat)
    if ws_bytes is None:
        ws_bytes = ws.numel() * ws.element_size()
    _check(lib().ns_iterate_bf16(batch, m, n, _ptr(X_in), _ptr(X_out), carr, len(coeffs), int(steps), _ptr(ws),
                                 int(ws_bytes), _stream(stream)), "ns_iterate_bf16")


def adamw_step_fused(P, G, M, V, hp: AdamWHParams, stream=None, gdt: int | None = None, numel=None) -> None:
    """One multi-tensor AdamW step over parallel lists of fp32 params, gradients, exp_avg and exp_avg_sq."""
    n = len(P)
    if gdt is None:
        gdt = _dtype_code(G[0]) if n else MA_F32
    if numel is None:
        numel = [int(p.numel()) for p in P]
    nar = (ctypes.c_int64 * max(1, n))(*numel)
    _check(lib().adamw_step_fused(n, _ptr_array(P), _ptr_array(G), int(gdt), _ptr_array(M), _ptr_array(V), nar,
                                  ctypes.byref(hp), _stream(stream)), "adamw_step_fused")


def ma_plan_create(tensors: Sequence[Tensor], groups: Sequence[Group], ws_cap: int = 0):
    """Plan a parameter table; returns (plan handle, workspace bytes the step needs)."""
    n = len(tensors)
    arr = (Tensor * max(1, n))(*tensors)
    garr = (Group * max(1, len(groups)))(*groups)
    plan = ctypes.c_void_p()
    ws = ctypes.c_size_t(int(ws_cap))
    _check(lib().ma_plan_create(arr, n, garr, len(groups), ctypes.byref(plan), ctypes.byref(ws)), "ma_plan_create")
    return plan, int(ws.value)


def muonadamw_step(plan, groups: Sequence[Group], ws, ws_bytes: int, stream=None) -> None:
    """One MuonAdamW step over the planned table, gradients already on the device."""
    garr = (Group * max(1, len(groups)))(*groups)
    _check(lib().muonadamw_step(plan, garr, _ptr(ws), int(ws_bytes), _stream(stream)), "muonadamw_step")


def ma_plan_describe(plan, groups: Sequence[Group]) -> str:
    """Text description of the plan's buckets, sub-batches and launch segments (host-only)."""
    garr = (Group * max(1, len(groups)))(*groups)
    size = 1 << 14
    while True:
        buf = ctypes.create_string_buffer(size)
        rc = lib().ma_plan_describe(plan, garr, buf, size)
        if rc != MA_ERR_SHAPE or size >= 1 << 24:
            _check(rc, "ma_plan_describe")
            return buf.value.decode()
        size *= 4


def muonadamw_step_graph(plan, groups: Sequence[Group], ws, ws_bytes: int, stream=None) -> None:
    """muonadamw_step replayed from a CUDA graph the plan captures and keeps."""
    garr = (Group * max(1, len(groups)))(*groups)
    _check(lib().muonadamw_step_graph(plan, garr, _ptr(ws), int(ws_bytes), _stream(stream)), "muonadamw_step_graph")


def muonadamw_step_from_host(plan, groups: Sequence[Group], host_grads, ws, ws_bytes: int, stream=None,
                             copy_stream=None) -> None:
    """One step whose gradients are copied from host memory (pinned tensors or host pointers) on copy_stream,
    overlapped with the compute on stream."""
    garr = (Group * max(1, len(groups)))(*groups)
    _check(lib().muonadamw_step_from_host(plan, garr, _ptr_array(host_grads), _ptr(ws), int(ws_bytes),
                                          _stream(stream), _stream(copy_stream) if copy_stream is not None
                                          else _stream(stream)), "muonadamw_step_from_host")


def ma_plan_destroy(plan) -> None:
    """Free a plan (and its CUDA graph, if one was captured)."""
    lib().ma_plan_destroy(plan)


def ma_device_status(stream=None, reset: bool = True) -> int:
    """Wait for ``stream``, then read (and by default reset) this device's status word."""
    return int(lib().ma_device_status(_stream(stream), int(bool(reset))))


def ma_plan_status(plan, stream=None) -> int:
    """Wait for ``stream``, then read and clear the status word of the device the plan's steps ran on."""
    return int(lib().ma_plan_status(plan, _stream(stream)))


def ma_device_status_async(host_dst, stream=None) -> None:
    """Enqueue a copy of the device status word into host_dst (a pinned int32 tensor element or address)."""
    _check(lib().ma_device_status_async(_ptr(host_dst), _stream(stream)), "ma_device_status_async")


def ma_set_wait_limit_ns(limit_ns: int) -> None:
    """Time limit of the kernels' bounded waits, in nanoseconds (default 2 s)."""
    _check(lib().ma_set_wait_limit_ns(int(limit_ns)), "ma_set_wait_limit_ns")


def ma_debug_build() -> bool:
    """Whether the loaded library is the build with guarded device indexing."""
    return bool(lib().ma_debug_build())


def ma_set_momentum_overlap(on: bool) -> None:
    """Momentum passes under the previous sub-batch's chain, on a side stream, for plans created
    after the call (default off: slower on a B200, see the header)."""
    _check(lib().ma_set_momentum_overlap(1 if on else 0), "ma_set_momentum_overlap")


def ma_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch a block whose wait can only time out; the status word must then read MA_ERR_TIMEOUT."""
    _check(lib().ma_selftest_wait_timeout(int(limit_ns), _stream(stream)), "ma_selftest_wait_timeout")


PROF_CLASSES = ("adamw", "momentum", "finalize", "ns_gram", "ns_apply", "ns_gramsq", "ns_final", "momentum_side",
                "ns_q1")


def ma_profile_enable(on: bool) -> None:
    """Bracket every later launch of this thread with CUDA events (ma_profile_collect reads them)."""
    _check(lib().ma_profile_enable(int(bool(on))), "ma_profile_enable")


def ma_profile_collect() -> dict:
    """Per kernel class: {"ms", "launches", "flops", "bytes"} summed since the last collect."""
    k = len(PROF_CLASSES)
    ms, cnt = (ctypes.c_double * k)(), (ctypes.c_int64 * k)()
    fl, by = (ctypes.c_double * k)(), (ctypes.c_double * k)()
    _check(lib().ma_profile_collect(ms, cnt, fl, by), "ma_profile_collect")
    return {name: {"ms": ms[i], "launches": int(cnt[i]), "flops": fl[i], "bytes": by[i]}
            for i, name in enumerate(PROF_CLASSES)}


# ---------------------------------------------------------------------------- user-level wrappers

def group_table(groups) -> list:
    """ma_group_t entries from ("muon", MuonHParams) / ("adamw", AdamWHParams) pairs."""
    table = []
    for kind, hp in groups:
        g = Group()
        g.kind = MA_MUON if kind == "muon" else MA_ADAMW
        if g.kind == MA_MUON:
            g.muon = hp
        else:
            g.adamw = hp
        table.append(g)
    return table


class Plan:
    """Owns an ma_plan_t and its device workspace (a torch uint8 buffer)."""

    def __init__(self, tensors: Sequence[Tensor], groups: Sequence[Group], ws_cap: int = 0, device=None):
        import torch
        self.tensors = list(tensors)
        self.groups = list(groups)
        self.handle, self.ws_bytes = ma_plan_create(self.tensors, self.groups, ws_cap)
        self.ws = torch.empty(max(self.ws_bytes, 256), dtype=torch.uint8, device=device or "cuda")

    def step(self, groups: Sequence[Group] | None = None, stream=None, graph: bool = False) -> None:
        fn = muonadamw_step_graph if graph else muonadamw_step
        fn(self.handle, groups if groups is not None else self.groups, self.ws, self.ws.numel(), stream)

    def step_from_host(self, host_grads, groups: Sequence[Group] | None = None, stream=None,
                       copy_stream=None) -> None:
        muonadamw_step_from_host(self.handle, groups if groups is not None else self.groups, host_grads, self.ws,
                                 self.ws.numel(), stream, copy_stream)

    @property
    def launches(self) -> int:
        return int(lib().ma_plan_last_launches(self.handle))

    @property
    def graph_captures(self) -> int:
        return int(lib().ma_plan_graph_captures(self.handle))

    def status(self, stream=None) -> int:
        """Wait for ``stream``; MA_OK or the first device-side error of the steps since the last read."""
        return ma_plan_status(self.handle, stream)

    def describe(self, groups: Sequence[Group] | None = None) -> str:
        """What a step runs: workspace, buckets, sub-batches and shared launches."""
        return ma_plan_describe(self.handle, groups if groups is not None else self.groups)

    def close(self) -> None:
        if self.handle is not None and self.handle.value:
            ma_plan_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class MuonAdamW:
    """Torch-facing optimizer over (param, role, group) entries.

    ``params``: list of (tensor, role, group_index). The fp32 params live on the
    GPU. Gradients are read from ``param.grad`` (fp32 or bf16), or from the
    ``grads`` list given to :meth:`step`. ``groups``: list of
    ("muon", MuonHParams) or ("adamw", AdamWHParams). State buffers are
    allocated here, zero-initialised, and owned by this object. The AdamW
    step counter advances on every call.
    """

    def __init__(self, params, groups, ws_cap: int = 0):
        import torch
        self.entries = list(params)
        self.groups = group_table(groups)
        self.state = []
        self.step_count = 0
        self._ws_cap = ws_cap
        self._plan = None
        self._grad_ptrs = None
        kinds = ma_partition([self._desc(p, role, grp, None) for p, role, grp in self.entries])
        for (p, role, grp), kind in zip(self.entries, kinds):
            s0 = torch.zeros_like(p)
            s1 = torch.zeros_like(p) if kind == MA_ADAMW else None
            self.state.append((s0, s1))

    @staticmethod
    def _desc(p, role, grp, g, s0=None, s1=None) -> Tensor:
        t = Tensor()
        t.param = _ptr(p)
        t.grad = _ptr(g)
        t.grad_dtype = _dtype_code(g) if g is not None else MA_F32
        t.state0 = _ptr(s0)
        t.state1 = _ptr(s1)
        t.ndim = p.dim()
        for d in range(min(2, p.dim())):
            t.shape[d] = int(p.shape[d])
        t.role = int(role)
        t.group = int(grp)
        return t

    def _ensure_plan(self, grads):
        ptrs = tuple(_ptr(g) for g in grads)
        if self._plan is not None and ptrs == self._grad_ptrs:
            return
        if self._plan is not None:
            self._plan.close()
        descs = [self._desc(p, role, grp, g, s0, s1)
                 for (p, role, grp), g, (s0, s1) in zip(self.entries, grads, self.state)]
        self._plan = Plan(descs, self.groups, self._ws_cap, device=self.entries[0][0].device)
        self._grad_ptrs = ptrs

    def _advance(self):
        self.step_count += 1
        for g in self.groups:
            if g.kind == MA_ADAMW:
                g.adamw.step = self.step_count

    def step(self, grads=None, stream=None, graph: bool = False) -> None:
        """One step. graph=True replays the step from a CUDA graph that the plan
        captures on first use (same results; one launch instead of one per kernel).
        A plan, and with it the graph, belongs to one set of gradient buffers:
        keep them at fixed addresses (as persistent ``.grad`` tensors are)."""
        if grads is None:
            grads = [p.grad for p, _, _ in self.entries]
        self._ensure_plan(grads)
        self._advance()
        self._plan.step(self.groups, stream, graph)

    def step_from_host(self, host_grads, device_grads, stream=None, copy_stream=None) -> None:
        """One step whose gradients arrive from host memory.

        host_grads: pinned CPU tensors (or host pointers), one per entry.
        device_grads: the device buffers that receive them (same shapes and
        dtypes); the library copies each group of gradients on copy_stream
        (default: a stream owned by this optimizer) and overlaps the copies
        with the compute on stream.

        The call returns before the copies have read host_grads: do not write
        to them until ``host_copies_done`` (a CUDA event recorded on the copy
        stream after the last copy) has completed, e.g.
        ``opt.host_copies_done.synchronize()``.
        """
        import torch
        self._ensure_plan(device_grads)
        if copy_stream is None:
            if getattr(self, "_copy_stream", None) is None:
                self._copy_stream = torch.cuda.Stream(device=self.entries[0][0].device)
            copy_stream = self._copy_stream
        self._advance()
        self._plan.step_from_host(host_grads, self.groups, stream, copy_stream)
        cs = copy_stream if isinstance(copy_stream, torch.cuda.Stream) else torch.cuda.ExternalStream(int(copy_stream))
        self.host_copies_done = torch.cuda.Event()
        self.host_copies_done.record(cs)

    def state_dict(self) -> dict:
        """The step count and the state buffers (the tensors themselves, not
        copies): per entry (momentum, None) for Muon, (exp_avg, exp_avg_sq)
        for AdamW."""
        return {"step": self.step_count, "state": list(self.state)}

    def load_state_dict(self, sd: dict) -> None:
        """Copy a state_dict of an optimizer over the same table into this one."""
        if len(sd["state"]) != len(self.state):
            raise ValueError("state of another parameter table")
        for (a0, a1), (b0, b1) in zip(self.state, sd["state"]):
            if a0.shape != b0.shape or (a1 is None) != (b1 is None):
                raise ValueError("state of another parameter table")
            a0.copy_(b0)
            if a1 is not None:
                a1.copy_(b1)
        self.step_count = int(sd["step"])

    @property
    def launches(self) -> int:
        return self._plan.launches if self._plan is not None else 0

    @property
    def graph_captures(self) -> int:
        """How many times the plan captured its CUDA graph (graph steps only)."""
        return self._plan.graph_captures if self._plan is not None else 0

    def describe(self) -> str:
        """What a step runs (buckets, sub-batches, shared launches); needs one step first."""
        if self._plan is None:
            raise RuntimeError("no plan yet: the plan is built on the first step")
        return self._plan.describe(self.groups)
