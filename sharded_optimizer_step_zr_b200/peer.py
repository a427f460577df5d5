"""PeerZero: one rank of a ZeRO-1/2 job across GPUs, one process per GPU.

The fused step reads this rank's owned slice of every replica's gradient
buffer through peer loads (the reduce-scatter) and stores each updated bf16
parameter into every rank's parameter buffer through peer stores (the
all-gather) -- over NVLink / NVSwitch on a multi-GPU node.  Buffers are
shared between the processes with CUDA IPC; torch.distributed carries the
handles, the barriers around the step and, with clipping, the exchange of
the per-rank sums of squares.

Every replica keeps its full gradient in the plan's owner-major layout
(``grad_view(t)`` is tensor t's slice of it, for the backward pass to write
into) -- or, for the stage-3 layer loop with grad_slot_elems, only two
rotating gradient slots of one layer each (``grad_slots``; every replica's
slot j at byte address ``grad_slot_bases[w][j]``), which the caller lays
out and steps layer by layer with zr_step_bucket on a grouped plan.
Stages 1 and 2: ``param_buffer`` holds the full bf16 parameters in the
global layout, written by every rank's step.  Stage 3: each rank keeps
only ``param_shard``, its bf16 parameters in owned order, and ``gather``
assembles whole tensors (one layer, ahead of its use) from every rank's
shard through the same peer mappings.
"""
from __future__ import annotations

from . import (ZR_PARAMS_OWNED, ZR_PARTITION_FLAT, zr_gather_params, zr_ipc_close, zr_ipc_export, zr_ipc_open,
               zr_plan_owner_offsets, zr_plan_set_gather_targets, zr_step)
from .plan import ZrPlan


class PeerFailure(RuntimeError):
    """A peer did not reach a phase boundary of the step (it exited, hung or
    lost its connection) within the process group's timeout.  Raised on the
    host before this rank launches anything that would read or write that
    peer's memory."""


def sync_point(dist, group, phase, step):
    """Every rank's arrival at `phase` of `step`.  The process group's own
    timeout bounds the wait; a failure becomes a PeerFailure naming the phase
    and step, so a caller can stop (or rebuild the group) between steps."""
    try:
        dist.barrier(group)
    except Exception as e:      # gloo and NCCL report a lost peer differently
        raise PeerFailure(f"step {step}, {phase}: a peer did not arrive ({type(e).__name__}: {e})") from e


class PeerZero:
    """One rank of a ZeRO job across processes (one per GPU) over CUDA IPC:
    the shared gradient buffer (owner-major), and either every rank's full
    parameter buffer (stages 1, 2: the step's stores are the all-gather) or
    this rank's parameter shard (stage 3: gather() assembles layers).
    Every rank constructs it, steps and closes it together."""

    def __init__(self, group, shapes, mode=ZR_PARTITION_FLAT, bucket_cap_bytes=25 << 20, lr=3e-4,
                 beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, max_grad_norm=0.0, device=None,
                 stage=2, groups=None, grad_slot_elems=0):
        import torch
        import torch.distributed as dist
        if stage not in (1, 2, 3):
            raise ValueError("stage is 1, 2 or 3")
        if grad_slot_elems and stage != 3:
            raise ValueError("gradient slots are the stage-3 layer loop's")
        self.dist, self.group, self.stage = dist, group, stage
        self.world_size = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        self.device = device
        self.plan = ZrPlan(shapes, self.world_size, self.rank, mode, bucket_cap_bytes, lr, beta1, beta2,
                           eps, weight_decay, max_grad_norm, device=device, groups=groups)
        self.offsets = zr_plan_owner_offsets(self.plan.handle, self.world_size)
        P = self.plan.padded_numel
        # One allocation holds both shared buffers, so each peer maps one
        # IPC handle per rank: the gradient buffer -- or, with
        # grad_slot_elems, two rotating gradient slots of that many elements
        # (one layer's gradients at a time) -- then (256-byte aligned) the
        # full parameter buffer (stages 1, 2) or this rank's parameter shard
        # (stage 3).  The gradient part has the same size on every rank, so
        # the second part starts at the same offset everywhere.
        round128 = lambda x: max(128, (x + 127) // 128 * 128)
        slot = round128(grad_slot_elems) if grad_slot_elems else 0
        half = 2 * slot if grad_slot_elems else round128(max(P, self.offsets[-1]))
        second = round128(self.plan.owned_numel) if stage == 3 else half
        self._shared = torch.zeros(half + second, dtype=torch.bfloat16, device=device)
        self.grad_buffer = None if grad_slot_elems else self._shared[:half]
        self.grad_slots = [self._shared[:slot], self._shared[slot:2 * slot]] if grad_slot_elems else None
        everyone = [None] * self.world_size
        dist.all_gather_object(everyone, zr_ipc_export(self._shared), group=group)
        self._opened = []
        error = None
        try:
            grad_bases, second_bases = [], []
            for w, handle in enumerate(everyone):
                base = self._shared.data_ptr() if w == self.rank else zr_ipc_open(handle)
                if w != self.rank:
                    self._opened.append(base)
                grad_bases.append(base)
                second_bases.append(base + 2 * half)
            start = 2 * self.offsets[self.rank]                 # bytes: bf16 elements
            self.grad_ptrs = None if grad_slot_elems else [b + start for b in grad_bases]
            # with slots: every replica's slot j starts at byte grad_slot_bases[w][j]
            self.grad_slot_bases = [[b, b + 2 * slot] for b in grad_bases] if grad_slot_elems else None
            if stage == 3:
                self.param_shard = self._shared[half:half + self.plan.owned_numel]
                self.shard_ptrs = second_bases
                self.plan.set_param_layout(ZR_PARAMS_OWNED)
            else:
                self.param_buffer = self._shared[half:]
                zr_plan_set_gather_targets(self.plan.handle, second_bases)
            self._segments = self.plan.segments()
        except Exception as e:      # e.g. a peer's buffer that cannot be mapped
            error = e
        self._agree_set_up(error)

    def _agree_set_up(self, error):
        """Every rank learns whether every rank mapped its peers' buffers (one
        all-reduce in place of the set-up's closing barrier).  If any rank
        failed, every rank unmaps what it opened and raises PeerFailure, so
        no rank is left waiting for another and none steps."""
        import torch
        dist, group = self.dist, self.group
        dev = self.device if dist.get_backend(group) == "nccl" else torch.device("cpu")
        flag = torch.tensor([0 if error is None else 1], dtype=torch.int32, device=dev)
        try:
            dist.all_reduce(flag, op=dist.ReduceOp.MAX, group=group)
        except Exception as e:
            raise PeerFailure(f"set-up: a peer did not arrive ({type(e).__name__}: {e})") from e
        if int(flag.item()) == 0:
            return
        for addr in self._opened:
            zr_ipc_close(addr)
        self._opened = []
        self.plan.close()
        where = f"this rank ({type(error).__name__}: {error})" if error is not None else "another rank"
        raise PeerFailure(f"set-up: {where} could not map the peers' buffers") from error

    def grad_pieces(self, tensor_index):
        """[(offset in the tensor, view of the owner-major buffer)] of tensor
        `tensor_index`'s gradient, one piece per owner."""
        pieces = sorted((s["offset_in_tensor"], s["owner"], s["owned_offset"], s["length"])
                        for s in self._segments if s["tensor"] == tensor_index)
        return [(off, self.grad_buffer[self.offsets[r] + o: self.offsets[r] + o + n])
                for off, r, o, n in pieces]

    def grad_view(self, tensor_index, shape=None):
        """Tensor `tensor_index`'s gradient as one view of the owner-major
        buffer: always possible for whole-tensor ownership, and for flat
        partitions whose chunk is a multiple of 8 elements."""
        pieces = self.grad_pieces(tensor_index)
        start = pieces[0][1].data_ptr()
        n = 0
        for _, view in pieces:
            if view.data_ptr() != start + 2 * n:
                raise ValueError("tensor is split across rank regions; use grad_pieces()")
            n += view.numel()
        v = self.grad_buffer[(start - self.grad_buffer.data_ptr()) // 2:][:n]
        return v.view(shape) if shape is not None else v

    def _exchange_sumsq(self):
        self.plan.grad_sumsq(self.grad_ptrs, self.plan.partials[self.rank:self.rank + 1])
        self.all_gather_partials()

    def all_gather_partials(self):
        """Every rank's entry of the clip's partials array (each rank's own
        S_r written there already) to every rank: the scalar exchange of the
        global-norm clip."""
        import torch
        dist = self.dist
        part = self.plan.partials
        backend = dist.get_backend(self.group)
        mine = part[self.rank:self.rank + 1].clone()
        if backend != "nccl":
            mine = mine.cpu()
        gathered = [torch.empty_like(mine) for _ in range(self.world_size)]
        dist.all_gather(gathered, mine, group=self.group)
        part.copy_(torch.cat(gathered).to(part.device))

    def step(self, master, m, v, step):
        """One optimizer step of this rank (every rank calls it together).
        Raises PeerFailure, before launching, if a peer is missing."""
        import torch
        torch.cuda.current_stream().synchronize()      # this replica's gradients are written
        sync_point(self.dist, self.group, "gradients ready", step)   # ... and every other replica's
        if self.plan.max_grad_norm > 0:
            self._exchange_sumsq()
        out = self.param_shard if self.stage == 3 else None
        zr_step(self.plan.handle, self.grad_ptrs, master, m, v, out, step)
        torch.cuda.current_stream().synchronize()
        sync_point(self.dist, self.group, "parameters written", step)   # every slice / shard is written

    def gather(self, first_tensor, n_tensors, dst, stream=None, max_ctas=0):
        """Stage 3: tensors [first_tensor, first_tensor + n_tensors) whole,
        in the global layout, into dst (bf16, on this GPU), read from every
        rank's shard through the peer mappings.  Valid after a step (whose
        last phase boundary every rank has passed); asynchronous on
        `stream`, so it can run a layer ahead of use (prefetch)."""
        if self.stage != 3:
            raise ValueError("gather is the stage-3 parameter all-gather")
        zr_gather_params(self.plan.handle, first_tensor, n_tensors, self.shard_ptrs, dst, stream, max_ctas)

    def bound_gather(self, first_tensor, n_tensors, dst, stream=None, max_ctas=0):
        """gather() with its arguments marshalled once: a callable for a
        per-layer prefetch loop (see ZrPlan.bound_gather)."""
        if self.stage != 3:
            raise ValueError("gather is the stage-3 parameter all-gather")
        return self.plan.bound_gather(first_tensor, n_tensors, self.shard_ptrs, dst, stream, max_ctas)

    def close(self):
        """Unmaps the peers' buffers (after a barrier: no rank still reads
        them) and destroys the plan."""
        if self._opened:
            self.dist.barrier(self.group)
            for addr in self._opened:
                zr_ipc_close(addr)
            self._opened = []
        self.plan.close()
