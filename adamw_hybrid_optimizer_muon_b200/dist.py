"""Sharded data-parallel MuonAdamW step over a ``torch.distributed`` process group.

The distributed variant of the optimizer in "How nanochat Combines Muon and
AdamW in a Single Optimizer" ("Distributed Training Support") keeps the same
two update rules and adds communication around them: gradients are reduced
across the data-parallel ranks, each rank updates a share of the parameters,
and the updated parameters reach every rank again, with the reductions
overlapping the compute. Here the three phases are:

1. reduce-scatter (average) of each bucket's gradients, so that each rank
   receives the averaged gradients of its own segment of the bucket; every
   bucket's reduction is queued at once;
2. as each bucket's reduction completes, the library's MuonAdamW step on
   that rank's segment: the Muon matrices it owns whole (Newton-Schulz mixes
   all rows of a matrix, and "nemo_automodel.components.optim.muown_triton"
   treats batched matrices as independent and wants the input axis complete
   on the rank), and its element range of the bucket's AdamW tensors (AdamW
   is elementwise);
3. all-gather of each bucket's updated segments into every rank's replica,
   queued right after that bucket's step, so it overlaps the next bucket's.

Layout: every rank holds the whole model's parameters in one flat fp32 buffer
and its gradients in one flat buffer with the same element offsets, both laid
out by ``ma_shard_layout`` (buckets, each cut into one equal segment per
rank). The model's parameter tensors become views into the flat parameter
buffer, and ``grads[i]`` views into the flat gradient buffer (also set as
``.grad`` when the gradient dtype is the parameter's). Optimizer state exists
only for this rank's segments: 1/world_size of the single-GPU state.

The collectives are NCCL's (or gloo's, for CPU ranks); every update runs in
the library's kernels. Tests on CPU ranks replace ``_local_step``.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import torch
import torch.distributed as dist

from . import (MA_ADAMW, MA_MUON, ROLE_HIDDEN, Tensor, _dtype_code, _ptr, group_table, lib, ma_partition,
               ma_plan_create, ma_plan_destroy, ma_shard_layout, muonadamw_step)

__all__ = ["DistMuonAdamW", "Piece", "ShardBucketView"]


@dataclass
class Piece:
    """One part of the model that this rank updates: a whole Muon matrix or a
    range of an AdamW tensor. ``lo``/``hi`` index the tensor's flattened
    elements; the views cover exactly that range."""
    index: int          # tensor index in the parameter table
    kind: int           # MA_MUON or MA_ADAMW
    group: int
    lo: int
    hi: int
    param: torch.Tensor     # view into the flat parameter buffer
    grad: torch.Tensor      # view into this rank's reduced-gradient shard
    state0: torch.Tensor    # momentum (Muon) or exp_avg (AdamW)
    state1: torch.Tensor | None  # exp_avg_sq (AdamW)


@dataclass
class ShardBucketView:
    """A bucket of the layout with this rank's views of it."""
    kind: int
    start: int
    seg: int
    grad_bucket: torch.Tensor      # world_size * seg gradients (reduce-scatter input)
    grad_shard: torch.Tensor       # seg reduced gradients (reduce-scatter output)
    param_bucket: torch.Tensor     # world_size * seg parameters (all-gather output)
    param_seg: torch.Tensor        # this rank's seg parameters (all-gather input)
    s0: int = 0                    # offset of the segment in the rank's shard buffers
    s1: int = 0                    # offset in the exp_avg_sq buffer (AdamW buckets)
    pieces: list = field(default_factory=list)


class DistMuonAdamW:
    """MuonAdamW over data-parallel ranks with sharded optimizer state.

    ``params``: list of (tensor, role, group_index), identical on every rank
    (same shapes, roles and groups in the same order). ``groups``: list of
    ("muon", MuonHParams) or ("adamw", AdamWHParams). ``grad_dtype``: dtype of
    the flat gradient buffer (default: fp32). ``seg_cap``: the largest segment
    one rank gets per bucket, in elements (smaller buckets overlap more, larger
    ones launch fewer, bigger kernels). ``broadcast_from``: rank whose initial
    parameters every rank starts from (None: keep each rank's own).

    After construction the parameters live in ``flat_param``; fill
    ``grads[i]`` (or ``param.grad``, when the dtypes match) and call
    :meth:`step`. The step runs on the current CUDA stream; it leaves the
    gradient buffer as it found it.
    """

    def __init__(self, params, groups, process_group=None, grad_dtype=None, seg_cap: int = 1 << 27,
                 broadcast_from: int | None = 0):
        self.pg = process_group
        self.world = dist.get_world_size(process_group)
        self.rank = dist.get_rank(process_group)
        self.entries = list(params)
        self.groups = group_table(groups)
        self.step_count = 0
        if not self.entries:
            raise ValueError("no parameters")
        device = self.entries[0][0].device
        gdt = grad_dtype or torch.float32
        if gdt not in (torch.float32, torch.bfloat16):
            raise ValueError("gradients must be fp32 or bf16")
        descs = []
        for p, role, grp in self.entries:
            if p.dtype != torch.float32 or p.device != device:
                raise ValueError("parameters must be fp32 and on one device")
            t = Tensor()
            t.ndim = p.dim()
            for d in range(min(2, p.dim())):
                t.shape[d] = int(p.shape[d])
            t.role, t.group = int(role), int(grp)
            descs.append(t)
        self.kinds = ma_partition(descs)
        slots, buckets, total = ma_shard_layout(descs, self.groups, self.world, seg_cap)
        self.slots = slots
        self._layout_key = hashlib.sha256(repr((slots, buckets, total, str(gdt))).encode()).hexdigest()
        self.flat_param = torch.zeros(total, dtype=torch.float32, device=device)
        self.flat_grad = torch.zeros(total, dtype=gdt, device=device)
        self.grads = []
        for (p, _, _), (_, _, off) in zip(self.entries, slots):
            n = p.numel()
            view = self.flat_param[off:off + n].view(p.shape)
            view.copy_(p.detach())
            p.data = view
            g = self.flat_grad[off:off + n].view(p.shape)
            self.grads.append(g)
            if gdt == p.dtype:
                p.grad = g
        if broadcast_from is not None and self.world > 1:
            dist.broadcast(self.flat_param, src=broadcast_from, group=process_group)

        seg_total = sum(seg for _, _, _, seg in buckets)
        adamw_total = sum(seg for kind, _, _, seg in buckets if kind == MA_ADAMW)
        self.grad_shard = torch.zeros(seg_total, dtype=gdt, device=device)
        self.state0 = torch.zeros(seg_total, dtype=torch.float32, device=device)
        self.state1 = torch.zeros(adamw_total, dtype=torch.float32, device=device)
        self.buckets = []
        soff = s1off = 0
        for kind, _, start, seg in buckets:
            mine = start + self.rank * seg
            bv = ShardBucketView(kind, start, seg,
                                 self.flat_grad[start:start + self.world * seg], self.grad_shard[soff:soff + seg],
                                 self.flat_param[start:start + self.world * seg], self.flat_param[mine:mine + seg],
                                 soff, s1off)
            self.buckets.append(bv)
            soff += seg
            if kind == MA_ADAMW:
                s1off += seg
        for i, ((p, _, grp), (b, owner, off)) in enumerate(zip(self.entries, slots)):
            bv = self.buckets[b]
            mine = bv.start + self.rank * bv.seg
            n = p.numel()
            if bv.kind == MA_MUON:
                if owner != self.rank:
                    continue
                lo, hi = off, off + n
            else:
                lo, hi = max(off, mine), min(off + n, mine + bv.seg)
            if hi <= lo:
                continue
            r0, r1 = bv.s0 + lo - mine, bv.s0 + hi - mine
            shape = tuple(p.shape) if bv.kind == MA_MUON else (hi - lo,)
            s1 = None
            if bv.kind == MA_ADAMW:
                a0 = bv.s1 + lo - mine
                s1 = self.state1[a0:a0 + hi - lo]
            bv.pieces.append(Piece(i, bv.kind, int(grp), lo - off, hi - off, self.flat_param[lo:hi].view(shape),
                                   self.grad_shard[r0:r1].view(shape), self.state0[r0:r1].view(shape), s1))
        self._plans = None
        self._ws = None
        self._side = None   # stream the reductions are issued from (CUDA only)

    # ------------------------------------------------------------------ step

    def _advance(self):
        self.step_count += 1
        for g in self.groups:
            if g.kind == MA_ADAMW:
                g.adamw.step = self.step_count

    def _build_plans(self):
        self._plans = []
        need = 0
        for bv in self.buckets:
            if not bv.pieces:
                self._plans.append(None)
                continue
            descs = []
            for pc in bv.pieces:
                t = Tensor()
                t.param, t.grad, t.grad_dtype = _ptr(pc.param), _ptr(pc.grad), _dtype_code(pc.grad)
                t.state0, t.state1 = _ptr(pc.state0), _ptr(pc.state1)
                t.ndim = pc.param.dim()
                for d in range(pc.param.dim()):
                    t.shape[d] = int(pc.param.shape[d])
                t.role = int(self.entries[pc.index][1]) if pc.kind == MA_MUON else ROLE_HIDDEN
                t.group = pc.group
                descs.append(t)
            handle, ws = ma_plan_create(descs, self.groups)
            self._plans.append(handle)
            need = max(need, ws)
        self._ws = torch.empty(max(need, 256), dtype=torch.uint8, device=self.flat_param.device)

    def _local_step(self, b: int) -> None:
        """Update this rank's pieces of bucket ``b`` (reduced gradients in place)."""
        if self._plans is None:
            self._build_plans()
        plan = self._plans[b]
        if plan is not None:
            muonadamw_step(plan, self.groups, self._ws, self._ws.numel())

    def step(self) -> None:
        """One data-parallel step: reduce-scatter, local update, all-gather (all asynchronous on the device)."""
        self._run(None)

    def step_from_host(self, host_flat: torch.Tensor) -> None:
        """One step whose gradients come from ``host_flat``, a pinned CPU tensor
        shaped and typed like ``flat_grad`` (``host_views`` gives its per-tensor
        views). Each bucket's gradients are copied on a side stream and that
        bucket's reduce-scatter starts as soon as its copy lands, so the copies
        overlap the reductions and the updates of the buckets before it.

        The call returns before the copies have read ``host_flat``: do not
        write to it until ``host_copies_done`` (a CUDA event recorded after the
        last copy) has completed, e.g. ``opt.host_copies_done.synchronize()``,
        or the step may read the new values for some buckets."""
        if host_flat.shape != self.flat_grad.shape or host_flat.dtype != self.flat_grad.dtype:
            raise ValueError("host_flat must match flat_grad in shape and dtype")
        self._run(host_flat)

    def host_views(self, host_flat: torch.Tensor) -> list:
        """Per-tensor views of a flat host gradient buffer (same offsets as ``grads``)."""
        return [host_flat[off:off + g.numel()].view(g.shape) for g, (_, _, off) in zip(self.grads, self.slots)]

    def _run(self, host_flat) -> None:
        self._advance()
        cuda = self.flat_grad.is_cuda
        if not cuda and host_flat is not None:
            self.flat_grad.copy_(host_flat)
            host_flat = None
        side = None
        if cuda:
            # the reductions are issued from a side stream, which first waits
            # for everything queued so far (the gradients' producers, the last
            # step's reads of flat_grad); NCCL then waits on the side stream
            # only, so a copy or reduction never waits for an update
            if self._side is None:
                self._side = torch.cuda.Stream(device=self.flat_grad.device)
            side = self._side
            side.wait_stream(torch.cuda.current_stream(self.flat_grad.device))
        reduces = []
        for bv in self.buckets:
            if not bv.seg:
                reduces.append(None)
                continue
            if side is None:
                reduces.append(dist.reduce_scatter_tensor(bv.grad_shard, bv.grad_bucket, op=dist.ReduceOp.AVG,
                                                          group=self.pg, async_op=True))
                continue
            with torch.cuda.stream(side):
                if host_flat is not None:
                    n = self.world * bv.seg
                    bv.grad_bucket.copy_(host_flat[bv.start:bv.start + n], non_blocking=True)
                reduces.append(dist.reduce_scatter_tensor(bv.grad_shard, bv.grad_bucket, op=dist.ReduceOp.AVG,
                                                          group=self.pg, async_op=True))
        if side is not None and host_flat is not None:
            # every copy from host_flat is queued on `side` before this event
            self.host_copies_done = torch.cuda.Event()
            self.host_copies_done.record(side)
        gathers = []
        for b, bv in enumerate(self.buckets):
            if reduces[b] is not None:
                reduces[b].wait()
            self._local_step(b)
            if bv.seg:
                gathers.append(dist.all_gather_into_tensor(bv.param_bucket, bv.param_seg, group=self.pg,
                                                           async_op=True))
        for w in gathers:
            w.wait()

    def state_dict(self) -> dict:
        """This rank's optimizer state: the step count, its state buffers (the
        tensors themselves, not copies) and a key of the layout they belong to.
        Each rank saves its own; a resumed run needs the same table, world size
        and segment cap."""
        return {"step": self.step_count, "world": self.world, "rank": self.rank, "layout": self._layout_key,
                "state0": self.state0, "state1": self.state1}

    def load_state_dict(self, sd: dict) -> None:
        """Restore what :meth:`state_dict` returned on this rank of an identical setup."""
        if (sd["world"], sd["rank"], sd["layout"]) != (self.world, self.rank, self._layout_key):
            raise ValueError("optimizer state of another layout, world size or rank")
        self.state0.copy_(sd["state0"])
        self.state1.copy_(sd["state1"])
        self.step_count = int(sd["step"])

    def zero_grad(self) -> None:
        """Zero the flat gradient buffer. The ``.grad`` views stay in place, so
        that backward keeps accumulating into the buffer (setting ``.grad`` to
        None instead would detach the parameters from it)."""
        self.flat_grad.zero_()

    # ------------------------------------------------------------------ introspection

    @property
    def launches(self) -> int:
        """Kernel launches of this rank's last step (all buckets)."""
        return sum(int(lib().ma_plan_last_launches(h)) for h in (self._plans or []) if h is not None)

    @property
    def state_bytes(self) -> int:
        """Optimizer-state bytes this rank holds."""
        return 4 * (self.state0.numel() + self.state1.numel())

    def pieces(self) -> list:
        """Every piece this rank updates, bucket by bucket."""
        return [pc for bv in self.buckets for pc in bv.pieces]

    def describe(self) -> str:
        lines = [f"rank {self.rank} of {self.world}: {len(self.buckets)} buckets, flat {self.flat_param.numel()} "
                 f"elements, state {self.state_bytes} bytes"]
        for b, bv in enumerate(self.buckets):
            kind = "muon" if bv.kind == MA_MUON else "adamw"
            lines.append(f"  bucket {b} {kind}: start {bv.start}, segment {bv.seg}, "
                         f"{len(bv.pieces)} pieces here ({sum(pc.hi - pc.lo for pc in bv.pieces)} elements)")
        return "\n".join(lines)

    def close(self) -> None:
        if self._plans:
            for h in self._plans:
                if h is not None:
                    ma_plan_destroy(h)
        self._plans = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
