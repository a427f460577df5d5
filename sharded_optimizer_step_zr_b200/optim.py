"""ZeroAdamW: the sharded step behind a torch-optimizer-style interface.

    opt = ZeroAdamW(model.parameters(), group=None, lr=3e-4)     # or a process group
    loss.backward(); opt.step(); opt.zero_grad()

The model's bf16 parameters become views of the full bf16 parameter buffer
that every rank's step writes (the all-gather), and their .grad tensors
views of the replica's gradient buffer in the plan's owner-major layout, so
autograd accumulates straight into it ("DDP -> ZeRO" blog, section 2.1:
gradients are written into flat buckets as the backward pass produces
them).  Each rank holds only its owned slice of the fp32 master weights and
Adam moments (ZeRO stage 1/2).  With one rank the plan's own buffers are
used; with a process group of several ranks the buffers are shared between
the processes over CUDA IPC (PeerZero), and the step reads the other
replicas' gradients and writes every rank's parameters through peer memory;
every rank's model must then start from the same parameters (each rank's
fp32 master slice is taken from its own copy).

Only the buffer plumbing lives here: the step itself runs in libzr.so.
"""
from __future__ import annotations

from . import ZR_PARTITION_FLAT, ZR_PARTITION_WHOLE_TENSOR


class ZeroAdamW:
    """ZeRO stage 1/2 AdamW with a torch-optimizer interface (see the module
    docstring): step(), zero_grad(), set_lr(), save() / load(), close().

    overlap=True steps each bucket as soon as the backward pass has filled
    it ("Scaling training to thousands of GPUs", 03:41 DP: a bucket's
    collective starts as soon as backward has produced its gradients): a
    hook after every parameter's gradient accumulation counts the bucket's
    tensors, and the last one enqueues zr_step_bucket for the bucket on a
    side stream that waits for the backward's work so far (across
    processes, after a barrier: every replica's part of the bucket is
    written).  A bucket's tensors are not read again by the rest of the
    backward, so their update can run beside it.  step() then steps buckets
    that got no gradient, finishes the clip when there is one, and joins the
    side stream.  One backward per step in this mode."""

    def __init__(self, params, group=None, lr=3e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.1,
                 max_grad_norm=0.0, partition="flat", bucket_cap_mb=25, overlap=False):
        import torch
        self.params = [p for p in params]
        if not self.params:
            raise ValueError("no parameters")
        dev = self.params[0].device
        for p in self.params:
            if p.dtype != torch.bfloat16 or p.device != dev or dev.type != "cuda":
                raise ValueError("parameters must be bf16 tensors on one CUDA device")
        if partition not in ("flat", "whole"):
            raise ValueError("partition is 'flat' or 'whole'")
        mode = {"flat": ZR_PARTITION_FLAT, "whole": ZR_PARTITION_WHOLE_TENSOR}[partition]
        shapes = [tuple(p.shape) for p in self.params]
        self.hp = dict(lr=lr, beta1=betas[0], beta2=betas[1], eps=eps, weight_decay=weight_decay,
                       max_grad_norm=max_grad_norm)
        hp = tuple(self.hp.values())
        cap = int(bucket_cap_mb * (1 << 20))
        world = 1
        if group is not None:
            import torch.distributed as dist
            world = dist.get_world_size(group)
        if world > 1:
            from .peer import PeerZero
            self.peer = PeerZero(group, shapes, mode, cap, *hp, device=dev)
            self.plan = self.peer.plan
            self.grad_buffer = self.peer.grad_buffer
            self.param_buffer = self.peer.param_buffer
            self.offsets = self.peer.offsets
        else:
            from .plan import ZrPlan
            self.peer = None
            self.plan = ZrPlan(shapes, 1, 0, mode, cap, *hp, device=dev)
            self.offsets = [0, self.plan.padded_numel]
            self.grad_buffer = torch.zeros(max(self.plan.padded_numel, 8), dtype=torch.bfloat16, device=dev)
            self.param_buffer = torch.zeros(max(self.plan.padded_numel, 8), dtype=torch.bfloat16, device=dev)
        segs = self.plan.segments()
        goff = [0]
        for p in self.params:
            goff.append(goff[-1] + p.numel())
        # parameters: views of the full bf16 buffer (global layout), current values kept
        with torch.no_grad():
            for t, p in enumerate(self.params):
                view = self.param_buffer[goff[t]:goff[t + 1]].view(p.shape)
                view.copy_(p)
                p.data = view
        # gradients: views of the owner-major buffer where a tensor is one run there
        self._copy_in = []
        self._bound = []
        for t, p in enumerate(self.params):
            pieces = sorted((s["offset_in_tensor"], s["owner"], s["owned_offset"], s["length"])
                            for s in segs if s["tensor"] == t)
            starts = [self.offsets[r] + o for _, r, o, _ in pieces]
            contiguous = all(starts[i] + pieces[i][3] == starts[i + 1] for i in range(len(pieces) - 1))
            if pieces and contiguous:
                p.grad = self.grad_buffer[starts[0]:starts[0] + p.numel()].view(p.shape)
                self._bound.append((p, starts[0]))
            else:
                p.grad = torch.zeros_like(p)
                self._copy_in.append((p, [(off, self.offsets[r] + o, n) for off, r, o, n in pieces]))
        # this rank's fp32 master weights (from the bf16 parameters), moments at zero
        rank = self.plan.rank
        n = self.plan.owned_numel
        self.master = torch.zeros(max(n, 8), dtype=torch.float32, device=dev)
        flat = self.param_buffer
        for owned, glob, length in self.plan.runs():
            self.master[owned:owned + length] = flat[glob:glob + length].float()
        self.m = torch.zeros_like(self.master)
        self.v = torch.zeros_like(self.master)
        self.rank, self.step_count = rank, 0
        self._grads = [self.grad_buffer[self.offsets[rank]:]]
        self.overlap = bool(overlap)
        self._hooks = []
        if self.overlap:
            # each tensor's bucket; hooks count a bucket's tensors as autograd fills them
            bucket_of = {}
            for s_ in segs:
                if s_["tensor"] >= 0:
                    bucket_of[int(s_["tensor"])] = int(s_["bucket"])
            self._bucket_tensors = {}
            for t in range(len(self.params)):
                if t in bucket_of:
                    self._bucket_tensors.setdefault(bucket_of[t], []).append(t)
            self._side = torch.cuda.Stream(device=dev)
            self._seen = {b: set() for b in self._bucket_tensors}
            self._stepped = set()
            for b, ts in self._bucket_tensors.items():
                for t in ts:
                    self._hooks.append(self.params[t].register_post_accumulate_grad_hook(self._make_hook(b, t)))

    def _make_hook(self, b, t):
        def hook(p):
            if b in self._stepped:
                raise RuntimeError("overlap: a second backward before step(); "
                                   "gradients cannot be accumulated over several passes in this mode")
            self._seen[b].add(t)
            if len(self._seen[b]) == len(self._bucket_tensors[b]):
                self._step_bucket(b)
        return hook

    def _bind_and_copy_in(self, tensors=None):
        """Autograd accumulates into a bound .grad in place; should anything
        have replaced it with a new tensor, copy that in and bind again; the
        .grad of a tensor split across rank regions is copied in."""
        flat_grad = self.grad_buffer.view(-1)
        for p, start in self._bound:
            if tensors is not None and id(p) not in tensors:
                continue
            view = flat_grad[start:start + p.numel()]
            if p.grad is None or p.grad.data_ptr() != view.data_ptr():
                if p.grad is not None:
                    view.copy_(p.grad.reshape(-1))
                else:
                    view.zero_()
                p.grad = view.view(p.shape)
        for p, pieces in self._copy_in:
            if tensors is not None and id(p) not in tensors:
                continue
            g = p.grad.reshape(-1)
            for off, start, n in pieces:
                flat_grad[start:start + n].copy_(g[off:off + n])

    def _step_bucket(self, b):
        """Bucket b's gradients are complete on this replica: step the
        bucket (across processes once every replica's are) on the side
        stream."""
        import torch
        from . import zr_step_bucket
        from .peer import sync_point
        t = self.step_count + 1
        cur = torch.cuda.current_stream()
        self._bind_and_copy_in({id(self.params[i]) for i in self._bucket_tensors[b]})
        if self.peer is not None:
            cur.synchronize()
            sync_point(self.peer.dist, self.peer.group, f"bucket {b} gradients ready", t)
            grads = self.peer.grad_ptrs
        else:
            grads = self._grads
        self._side.wait_stream(cur)
        zr_step_bucket(self.plan.handle, b, grads, self.master, self.m, self.v,
                       None if self.peer is not None else self.param_buffer, t, self._side)
        self._stepped.add(b)

    def zero_grad(self, set_to_none=False):
        """Zeroes the gradient buffer; the .grad views stay bound (set_to_none
        is ignored: releasing them would detach autograd from the buffer)."""
        self.grad_buffer.zero_()
        for p, _ in self._copy_in:
            p.grad.zero_()

    def set_lr(self, lr):
        """The learning rate for the following steps (a schedule)."""
        self.hp["lr"] = lr
        self.plan.set_adamw(*self.hp.values())

    def step(self):
        """One optimizer step: this rank's slice of the averaged gradient,
        AdamW on its fp32 state, the bf16 result into every rank's
        parameters.  With several ranks, every rank calls it together."""
        if self.overlap:
            return self._finish_overlapped()
        self._bind_and_copy_in()
        self.step_count += 1
        if self.peer is not None:
            self.peer.step(self.master, self.m, self.v, self.step_count)
        else:
            self.plan.step(self._grads, self.master, self.m, self.v, self.param_buffer, self.step_count)
        return None

    def _finish_overlapped(self):
        import torch
        from . import zr_step_finish
        from .peer import sync_point
        for b in sorted(self._bucket_tensors):
            if b not in self._stepped:
                if self._seen[b]:
                    raise RuntimeError(f"overlap: bucket {b} received gradients for only some of its tensors")
                self._step_bucket(b)
        t = self.step_count + 1
        cur = torch.cuda.current_stream()
        cur.wait_stream(self._side)
        if self.plan.max_grad_norm > 0:
            if self.peer is not None:
                me = self.plan.rank
                self.plan.bucket_sumsq(self.plan.partials[me:me + 1])
                self.peer.all_gather_partials()
                # (the finish reads the gradients again only when W <= 4; they are all still there)
                zr_step_finish(self.plan.handle, self.peer.grad_ptrs, self.master, self.m, self.v, None, t, cur)
            else:
                zr_step_finish(self.plan.handle, self._grads, self.master, self.m, self.v, self.param_buffer,
                               t, cur)
        if self.peer is not None:
            cur.synchronize()
            sync_point(self.peer.dist, self.peer.group, "parameters written", t)
        self.step_count = t
        self._seen = {b: set() for b in self._bucket_tensors}
        self._stepped = set()
        return None

    def save(self, path):
        """This rank's fp32 master / m / v and the step count to `path` (one
        file per rank; zr_state_export_params turns a complete set into a
        whole-model file)."""
        from . import zr_state_save
        zr_state_save(self.plan.handle, path, self.master, self.m, self.v, self.step_count)

    def load(self, path):
        """Restores this rank's state and step count from `path` (a shard of
        the same partition and rank) and writes the restored master weights,
        rounded to bf16, into this rank's parameters."""
        from . import zr_state_load
        self.step_count = zr_state_load(self.plan.handle, path, self.master, self.m, self.v)
        for owned, glob, length in self.plan.runs():
            self.param_buffer[glob:glob + length] = self.master[owned:owned + length].to(self.param_buffer.dtype)

    def close(self):
        for h in self._hooks:
            h.remove()
        self._hooks = []
        if self.peer is not None:
            self.peer.close()
        else:
            self.plan.close()


def unit_grad_layout(segments, first, count, last_unit, world_size):
    """Where one unit's (tensors first .. first + count - 1) gradients sit in
    a gradient slot.  Each owner's elements of the unit are one run in its
    owned order; the slot holds those runs owner by owner, each starting at
    its owned offset's phase mod 8, so that for every rank r there is an
    offset d_r with replica w's slot + d_r serving as r's grad_ptrs[w] for
    the unit's tiles (slot element d_r + owned offset, 16-byte aligned).  The
    last unit's run also covers the flat zero pad (its bucket holds it).

    Returns (pieces of each tensor as (offset in tensor, slot offset,
    length), d_r per rank, slot elements used).  A tensor whose pieces are
    contiguous in the slot can be one .grad view of it; with a flat chunk
    that is a multiple of 8 elements (or one rank) every tensor is."""
    segs = [s for s in segments
            if first <= s["tensor"] < first + count or (last_unit and s["tensor"] == -1)]
    pieces = {t: [] for t in range(first, first + count)}
    ptr_off = [0] * world_size
    cursor = 0
    for r in range(world_size):
        mine = sorted((s["owned_offset"], s["tensor"], s["offset_in_tensor"], s["length"])
                      for s in segs if s["owner"] == r)
        if not mine:
            continue
        lo = mine[0][0]
        hi = mine[-1][0] + mine[-1][3]
        base = (cursor + 7) // 8 * 8 + lo % 8
        for o, t, off, n in mine:
            if t >= 0:
                pieces[t].append((off, base + (o - lo), n))
        ptr_off[r] = base - lo
        cursor = base + (hi - lo)
    for t in pieces:
        pieces[t].sort()
    return pieces, ptr_off, cursor


def contiguous_in_slot(pieces):
    """Slot offset of a tensor whose pieces (sorted by offset in the tensor)
    follow each other in the slot from its first element, else None."""
    if not pieces:
        return 0
    if pieces[0][0] != 0:
        return None
    for (off, pos, n), (off2, pos2, _) in zip(pieces, pieces[1:]):
        if off2 != off + n or pos2 != pos + n:
            return None
    return pieces[0][1]


class Zero3:
    """ZeRO stage 3 for a torch module ("Scaling training to thousands of
    GPUs", talk summary, section 11:24 ZeRO; "CS336 lecture 8", section
    "ZeRO levels"): each rank keeps only its bf16 shard of the parameters
    (owned order) and its fp32 master / m / v slice; a module's parameters
    are gathered from all shards just before its forward and again just
    before its backward -- in both passes the next module's ahead of time,
    on a side stream (backward_prefetch=False keeps the backward's in line).

    Every module that owns parameters directly gets one of two rotating
    gather slots (module i: slot i mod 2), and its parameters stay views of
    that slot, so only two modules' parameters are ever whole.  Autograd's
    saved weights are those views: the slot is refilled with the module's
    parameters before its backward reads them.  Gradients are bound to the
    replica's gradient buffer as in ZeroAdamW.  The rotation assumes the
    units run as a chain: forward in the order of module.parameters(), each
    once, and backward in reverse (a sequential stack of layers); a
    parameter used by a module other than its owner (tied weights) is not
    supported, since that module would read whatever the slot holds.  With
    a process group, every rank's module must start from the same
    parameters (each rank's shard is cut from its own copy).

        z = Zero3(model, group=None, lr=3e-4)
        loss = model(x).sum(); loss.backward(); z.step(); z.zero_grad()

    reduce_in_backward=True is the gradient side of stage 3: no replica
    keeps its whole gradient.  The plan's buckets are the units (one per
    module), gradients accumulate into two rotating gradient slots (module
    i: slot i mod 2, laid out so every owner's part is one run), and as
    soon as a module's gradients are complete the fused step reduces that
    module's slice from every replica's slot (through peer memory across
    processes) and updates it -- zr_step_bucket on the module's bucket --
    after which the slot is cleared for module i - 2.  z.step() then only
    steps modules that received no gradient and advances the count.  With
    clipping the backward's per-module calls are the reduce and the sums of
    squares, keeping the rank's fp32 averaged gradient (ZeRO-2's sharded
    gradient); z.step() exchanges the ranks' sums of squares
    (zr_bucket_sumsq) and applies the clipped update (zr_step_finish).  One
    backward per step (no accumulation over several), and every parameter
    of a module receiving a gradient.
    """

    def __init__(self, module, group=None, lr=3e-4, betas=(0.9, 0.999), eps=1e-8, weight_decay=0.1,
                 max_grad_norm=0.0, partition="flat", bucket_cap_mb=25, backward_prefetch=True,
                 reduce_in_backward=False):
        import torch
        from . import ZR_PARAMS_OWNED
        self.module = module
        params = list(module.parameters())
        if not params:
            raise ValueError("no parameters")
        dev = params[0].device
        for p in params:
            if p.dtype != torch.bfloat16 or p.device != dev or dev.type != "cuda":
                raise ValueError("parameters must be bf16 tensors on one CUDA device")
        if partition not in ("flat", "whole"):
            raise ValueError("partition is 'flat' or 'whole'")
        # the units: modules owning parameters directly, each a run of consecutive tensors
        index = {id(p): i for i, p in enumerate(params)}
        self.units = []
        for mod in module.modules():
            own = list(mod.parameters(recurse=False))
            if not own:
                continue
            ids = [index[id(p)] for p in own]
            if ids != list(range(ids[0], ids[0] + len(ids))):
                raise ValueError("a module's parameters must be consecutive in module.parameters()")
            self.units.append((mod, ids[0], len(ids)))
        self.units.sort(key=lambda u: u[1])
        mode = {"flat": ZR_PARTITION_FLAT, "whole": ZR_PARTITION_WHOLE_TENSOR}[partition]
        shapes = [tuple(p.shape) for p in params]
        self.hp = dict(lr=lr, beta1=betas[0], beta2=betas[1], eps=eps, weight_decay=weight_decay,
                       max_grad_norm=max_grad_norm)
        hp = tuple(self.hp.values())
        cap = int(bucket_cap_mb * (1 << 20))
        world = 1
        if group is not None:
            import torch.distributed as dist
            world = dist.get_world_size(group)
        self.reduce_in_backward = bool(reduce_in_backward)
        groups = None
        slot_elems = 0
        if self.reduce_in_backward:
            groups = [0] * len(params)
            for u, (_, a, k) in enumerate(self.units):
                for t in range(a, a + k):
                    groups[t] = u
            # the units' gradient layouts, from the host-only plan (same tables on every rank)
            from .plan import ZrPlan
            probe = ZrPlan(shapes, world, 0, mode, cap, *hp, bind=False, groups=groups)
            segs = probe.segments()
            probe.close()
            self._unit_layouts = [unit_grad_layout(segs, a, k, a + k == len(params), world)
                                  for _, a, k in self.units]
            self._unit_bucket = []
            for _, a, k in self.units:
                bs = {s["bucket"] for s in segs if a <= s["tensor"] < a + k}
                self._unit_bucket.append(bs.pop() if bs else None)
            slot_elems = max(8, max(L[2] for L in self._unit_layouts))
        if world > 1:
            from .peer import PeerZero
            self.peer = PeerZero(group, shapes, mode, cap, *hp, device=dev, stage=3, groups=groups,
                                 grad_slot_elems=slot_elems)
            self.plan = self.peer.plan
            self.grad_buffer = self.peer.grad_buffer
            self.offsets = self.peer.offsets
            self.shard = self.peer.param_shard
            shard_ptrs = self.peer.shard_ptrs
            if self.reduce_in_backward:
                self.grad_slots = self.peer.grad_slots
                self._slot_bases = self.peer.grad_slot_bases            # [w][slot] byte addresses
        else:
            from .plan import ZrPlan
            self.peer = None
            self.plan = ZrPlan(shapes, 1, 0, mode, cap, *hp, device=dev, groups=groups)
            self.plan.set_param_layout(ZR_PARAMS_OWNED)
            self.offsets = [0, self.plan.padded_numel]
            if self.reduce_in_backward:
                self.grad_buffer = None
                self.grad_slots = [torch.zeros(slot_elems, dtype=torch.bfloat16, device=dev) for _ in range(2)]
                self._slot_bases = [[g.data_ptr() for g in self.grad_slots]]
            else:
                self.grad_buffer = torch.zeros(max(self.plan.padded_numel, 8), dtype=torch.bfloat16, device=dev)
            self.shard = torch.zeros(max(self.plan.owned_numel, 8), dtype=torch.bfloat16, device=dev)
            shard_ptrs = [self.shard]
        # this rank's shard and fp32 state from the current (whole) parameters
        goff = [0]
        for p in params:
            goff.append(goff[-1] + p.numel())
        whole = torch.cat([p.detach().reshape(-1) for p in params])
        n = self.plan.owned_numel
        self.master = torch.zeros(max(n, 8), dtype=torch.float32, device=dev)
        for owned, glob, length in self.plan.runs():
            if glob < whole.numel():
                k = min(length, whole.numel() - glob)
                self.shard[owned:owned + k] = whole[glob:glob + k]
        self.master[:n] = self.shard[:n].float()
        self.m = torch.zeros_like(self.master)
        self.v = torch.zeros_like(self.master)
        del whole
        # two slots; each unit's parameters become views of its slot
        biggest = max(goff[a + k] - goff[a] for _, a, k in self.units)
        self.slots = [torch.zeros(max(biggest, 8), dtype=torch.bfloat16, device=dev) for _ in range(2)]
        self.side = torch.cuda.Stream(device=dev)
        self.ready = [torch.cuda.Event() for _ in self.units]
        self._hooks = []
        for u, (mod, a, k) in enumerate(self.units):
            slot = self.slots[u % 2]
            with torch.no_grad():
                for t in range(a, a + k):
                    p = params[t]
                    p.data = slot[goff[t] - goff[a]:goff[t + 1] - goff[a]].view(p.shape)
            self._hooks.append(mod.register_forward_pre_hook(self._make_forward_hook(u)))
            self._hooks.append(mod.register_full_backward_pre_hook(self._make_backward_hook(u)))
        self._shard_ptrs, self._slot_of = shard_ptrs, [self.slots[u % 2] for u in range(len(self.units))]
        self._bound_gathers = {}
        self._prefetched = [False] * len(self.units)
        self.back_ready = [torch.cuda.Event() for _ in self.units]
        self._back_prefetched = [False] * len(self.units)
        self.backward_prefetch = backward_prefetch
        self.params = params
        self._bound, self._copy_in = [], []
        if self.reduce_in_backward:
            self._bind_grad_slots()
            self.step_count = 0
            return
        # gradients: as ZeroAdamW
        segs = self.plan.segments()
        for t, p in enumerate(params):
            pieces = sorted((s["offset_in_tensor"], s["owner"], s["owned_offset"], s["length"])
                            for s in segs if s["tensor"] == t)
            starts = [self.offsets[r] + o for _, r, o, _ in pieces]
            contiguous = all(starts[i] + pieces[i][3] == starts[i + 1] for i in range(len(pieces) - 1))
            if pieces and contiguous:
                p.grad = self.grad_buffer[starts[0]:starts[0] + p.numel()].view(p.shape)
                self._bound.append((p, starts[0]))
            else:
                p.grad = torch.zeros_like(p)
                self._copy_in.append((p, [(off, self.offsets[r] + o, n_) for off, r, o, n_ in pieces]))
        self.step_count = 0

    def _bind_grad_slots(self):
        """reduce_in_backward: every parameter's .grad a view of its unit's
        slot; hooks that fire once a unit's gradients are all accumulated."""
        import torch
        W, me = self.plan.world_size, self.plan.rank
        self._unit_grad_ptrs = []
        self._unit_grad_views = []
        for u, (_, a, k) in enumerate(self.units):
            pieces, ptr_off, used = self._unit_layouts[u]
            slot = self.grad_slots[u % 2]
            views = []
            for t in range(a, a + k):
                p = self.params[t]
                at = contiguous_in_slot(pieces[t])
                if at is not None:
                    v = slot[at:at + p.numel()].view(p.shape)
                    p.grad = v
                    views.append((p, v, None))
                else:
                    # split across two owners' runs that do not meet: its own .grad, copied in
                    p.grad = torch.zeros_like(p)
                    views.append((p, None, [(off, slot[pos:pos + n]) for off, pos, n in pieces[t]]))
            self._unit_grad_views.append(views)
            self._unit_grad_ptrs.append([self._slot_bases[w][u % 2] + 2 * ptr_off[me] for w in range(W)])
            for p in [self.params[t] for t in range(a, a + k)]:
                self._hooks.append(p.register_post_accumulate_grad_hook(self._make_grad_hook(u, p)))
        self._unit_seen = [set() for _ in self.units]
        self._unit_done = [False] * len(self.units)

    def _make_grad_hook(self, u, param):
        def hook(p):
            if self._unit_done[u]:
                raise RuntimeError("reduce_in_backward: a second backward before step(); "
                                   "gradients cannot be accumulated over several passes in this mode")
            self._unit_seen[u].add(id(param))
            if len(self._unit_seen[u]) == len(self._unit_grad_views[u]):
                self._reduce_unit(u)
        return hook

    def _reduce_unit(self, u):
        """Unit u's gradients are complete on this replica: (every replica's,
        across processes) reduce its slice and update it, then clear the slot."""
        import torch
        from . import zr_step_bucket
        from .peer import sync_point
        cur = torch.cuda.current_stream()
        t = self.step_count + 1
        for p, v, split in self._unit_grad_views[u]:
            if split is not None:
                g = p.grad.reshape(-1) if p.grad is not None else None
                for off, dst in split:
                    if g is None:
                        dst.zero_()
                    else:
                        dst.copy_(g[off:off + dst.numel()])
                if p.grad is not None:
                    p.grad.zero_()
                continue
            if p.grad is None:
                v.zero_()
            elif p.grad.data_ptr() != v.data_ptr():        # autograd replaced the view: copy in
                v.copy_(p.grad)
            p.grad = v
        if self.peer is not None:
            cur.synchronize()                              # this replica's gradients are written
            sync_point(self.peer.dist, self.peer.group, f"layer {u} gradients ready", t)
        if self._unit_bucket[u] is not None:
            zr_step_bucket(self.plan.handle, self._unit_bucket[u], self._unit_grad_ptrs[u], self.master, self.m,
                           self.v, self.shard, t, cur)
        if self.peer is not None:
            cur.synchronize()
            sync_point(self.peer.dist, self.peer.group, f"layer {u} reduced", t)   # no rank reads the slot now
        self.grad_slots[u % 2][:self._unit_layouts[u][2]].zero_()
        self._unit_done[u] = True

    def _gather(self, u, stream):
        # one bound call per (unit, stream): the arguments are marshalled once
        key = (u, stream.cuda_stream)
        fn = self._bound_gathers.get(key)
        if fn is None:
            _, a, k = self.units[u]
            fn = self._bound_gathers[key] = self.plan.bound_gather(a, k, self._shard_ptrs, self._slot_of[u], stream)
        fn()

    def _make_forward_hook(self, u):
        def hook(module, inputs):
            import torch
            cur = torch.cuda.current_stream()
            if self._prefetched[u]:
                cur.wait_event(self.ready[u])             # gathered on the side stream
                self._prefetched[u] = False
            else:
                self._gather(u, cur)
            if u + 1 < len(self.units):
                # the next unit's slot was the previous unit's: its forward is queued before this point
                self.side.wait_stream(cur)
                self._gather(u + 1, self.side)
                self.ready[u + 1].record(self.side)
                self._prefetched[u + 1] = True
        return hook

    def _make_backward_hook(self, u):
        def hook(module, grad_output):
            import torch
            cur = torch.cuda.current_stream()
            # the slot held later units since this unit's forward: refill it
            # (prefetched during the next unit's backward, or now)
            if self._back_prefetched[u]:
                cur.wait_event(self.back_ready[u])
                self._back_prefetched[u] = False
            else:
                self._gather(u, cur)
            if self.backward_prefetch and u >= 1:
                # unit u - 1's slot last held unit u + 1, whose backward is queued before this point
                self.side.wait_stream(cur)
                self._gather(u - 1, self.side)
                self.back_ready[u - 1].record(self.side)
                self._back_prefetched[u - 1] = True
        return hook

    def zero_grad(self, set_to_none=False):
        """Zeroes the gradient buffer (the .grad views stay bound); with
        reduce_in_backward the slots are already clear after each unit."""
        if self.reduce_in_backward:
            return
        self.grad_buffer.zero_()
        for p, _ in self._copy_in:
            p.grad.zero_()

    def set_lr(self, lr):
        """The learning rate for the following steps (a schedule)."""
        self.hp["lr"] = lr
        self.plan.set_adamw(*self.hp.values())

    def step(self):
        """One optimizer step (every rank together): the rank's slice of the
        averaged gradient, AdamW, the bf16 result into the rank's shard.
        With reduce_in_backward the backward has stepped every unit that got
        gradients: the rest are stepped here (zero gradient)."""
        from . import zr_step
        if self.reduce_in_backward:
            import torch
            from . import zr_step_finish
            from .peer import sync_point
            for u in range(len(self.units)):
                if self._unit_done[u]:
                    continue
                if self._unit_seen[u]:
                    raise RuntimeError(f"reduce_in_backward: module {u} received gradients for only some "
                                       "of its parameters")
                self._reduce_unit(u)
            if self.plan.max_grad_norm > 0:
                # the per-module calls were the reduce and the sums of squares:
                # the global norm, then the clipped update from the fp32 gradient
                t = self.step_count + 1
                cur = torch.cuda.current_stream()
                if self.peer is not None:
                    me = self.plan.rank
                    self.plan.bucket_sumsq(self.plan.partials[me:me + 1])
                    self.peer.all_gather_partials()
                zr_step_finish(self.plan.handle, None, self.master, self.m, self.v, self.shard, t, cur)
                if self.peer is not None:
                    cur.synchronize()
                    sync_point(self.peer.dist, self.peer.group, "parameters written", t)
            self.step_count += 1
            self._unit_seen = [set() for _ in self.units]
            self._unit_done = [False] * len(self.units)
            self._prefetched = [False] * len(self.units)
            self._back_prefetched = [False] * len(self.units)
            return
        flat_grad = self.grad_buffer.view(-1)
        for p, start in self._bound:
            view = flat_grad[start:start + p.numel()]
            if p.grad is None or p.grad.data_ptr() != view.data_ptr():
                if p.grad is not None:
                    view.copy_(p.grad.reshape(-1))
                else:
                    view.zero_()
                p.grad = view.view(p.shape)
        for p, pieces in self._copy_in:
            g = p.grad.reshape(-1)
            for off, start, n in pieces:
                flat_grad[start:start + n].copy_(g[off:off + n])
        self.step_count += 1
        if self.peer is not None:
            self.peer.step(self.master, self.m, self.v, self.step_count)
        else:
            self.plan.step([self.grad_buffer], self.master, self.m, self.v, self.shard, self.step_count)
        self._prefetched = [False] * len(self.units)
        self._back_prefetched = [False] * len(self.units)

    def save(self, path):
        """This rank's fp32 master / m / v and the step count to `path`."""
        from . import zr_state_save
        zr_state_save(self.plan.handle, path, self.master, self.m, self.v, self.step_count)

    def load(self, path):
        """Restores this rank's state and step count; its bf16 shard becomes
        the restored master weights rounded to bf16 (what the step writes)."""
        from . import zr_state_load
        self.step_count = zr_state_load(self.plan.handle, path, self.master, self.m, self.v)
        n = self.plan.owned_numel
        self.shard[:n] = self.master[:n].to(self.shard.dtype)
        self._prefetched = [False] * len(self.units)
        self._back_prefetched = [False] * len(self.units)

    def gather_all(self, out):
        """The whole model, in the global layout, into `out` (bf16)."""
        self.plan.gather_params(0, len(self.params), self._shard_ptrs, out)

    def close(self):
        """Removes the hooks (the module keeps the parameters last gathered
        into its slots) and releases the plan."""
        for h in self._hooks:
            h.remove()
        self._hooks = []
        if self.peer is not None:
            self.peer.close()
        else:
            self.plan.close()
