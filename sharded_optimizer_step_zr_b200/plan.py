"""ZrPlan: a plan plus its torch-allocated device workspace.

PyTorch only provides device memory and the stream; the step itself runs in
libzr.so's kernels through the C ABI.
"""
from __future__ import annotations

from . import (ZR_PARAMS_GLOBAL, ZR_PARAMS_OWNED, ZR_PARTITION_FLAT, zr_debug_reduce, zr_gather_params,
               zr_grad_sumsq, zr_plan_check_result, zr_plan_create, zr_plan_destroy, zr_plan_query,
               zr_plan_segments, zr_plan_set_adamw, zr_plan_set_checked, zr_plan_set_param_layout,
               zr_plan_set_sumsq_partials,
               zr_plan_set_workspace, zr_plan_verify, zr_plan_workspace_bytes, zr_step, zr_step_bucket,
               zr_step_finish, zr_step_host)


def _require_all(specs, device):
    """Checks buffer arguments before their addresses reach the library,
    which cannot see sizes.  specs: (buffer, name, dtype, min elements,
    host?).  Each must be a contiguous torch tensor of that dtype with at
    least that many elements (all checked first), then on `device` -- or in
    host memory for host buffers.  A plain integer is a raw address and None
    an absent buffer: both are left to the library's own checks."""
    import torch
    tensors = []
    for x, what, dtype, numel, host in specs:
        if x is None or isinstance(x, int):
            continue
        if not isinstance(x, torch.Tensor):
            raise TypeError(f"{what}: expected a torch tensor or an address, got {type(x).__name__}")
        if x.dtype != dtype:
            raise ValueError(f"{what}: dtype {x.dtype}, expected {dtype}")
        if not x.is_contiguous():
            raise ValueError(f"{what}: not contiguous")
        if x.numel() < numel:
            raise ValueError(f"{what}: {x.numel()} elements, the plan needs at least {numel}")
        tensors.append((x, what, host))
    for x, what, host in tensors:
        if host:
            if x.device.type != "cpu":
                raise ValueError(f"{what}: must be in host memory, is on {x.device}")
        elif x.device.type != "cuda" or (device is not None and x.device != device):
            raise ValueError(f"{what}: must be on {device if device is not None else 'a CUDA device'}, "
                             f"is on {x.device}")


class ZrPlan:
    """One rank's plan (zr_plan_create) with a torch-allocated device
    workspace (bound at construction unless bind=False) and, with clipping,
    the W-entry partials array.  Tensor arguments of the step calls are
    checked against the plan before their addresses reach the library;
    plain integers pass through as raw addresses."""

    def __init__(self, shapes, world_size, rank, mode=ZR_PARTITION_FLAT, bucket_cap_bytes=25 << 20,
                 lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, max_grad_norm=0.0,
                 device=None, stream=None, bind=True, groups=None):
        self.handle = zr_plan_create(shapes, world_size, rank, mode, bucket_cap_bytes, lr, beta1,
                                     beta2, eps, weight_decay, max_grad_norm, groups=groups)
        self.world_size = world_size
        self.rank = rank
        self.mode = mode
        self.max_grad_norm = max_grad_norm
        info = zr_plan_query(self.handle)
        self.total_numel = info["total_numel"]
        self.padded_numel = info["padded_numel"]
        self.owned_numel = info["owned_numel"]
        self.n_buckets = info["n_buckets"]
        self.workspace_bytes = zr_plan_workspace_bytes(self.handle)
        self.device = None
        self.param_layout = ZR_PARAMS_GLOBAL
        self.workspace = None
        self.partials = None
        if bind:
            self.bind(device, stream)

    def bind(self, device=None, stream=None):
        """Allocates the workspace on `device` and binds it (tables uploaded
        on `stream`); with clipping, also the partials array."""
        import torch
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        device = torch.device(device)
        if device.index is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.device = device
        # torch's caching allocator returns 512-byte aligned blocks
        self.workspace = torch.empty(max(256, self.workspace_bytes), dtype=torch.uint8, device=device)
        zr_plan_set_workspace(self.handle, self.workspace, self.workspace.numel(), stream)
        if self.max_grad_norm > 0:
            self.partials = torch.zeros(self.world_size, dtype=torch.float64, device=device)
            zr_plan_set_sumsq_partials(self.handle, self.partials)

    def segments(self):
        """All ranks' segments as dictionaries (zr_plan_segments)."""
        return zr_plan_segments(self.handle)

    def runs(self):
        """(owned_offset, global_offset, length) of this rank, by owned offset."""
        runs = [(s["owned_offset"], s["global_offset"], s["length"]) for s in self.segments()
                if s["owner"] == self.rank]
        return sorted(runs)

    def check_step_buffers(self, grads, master, m, v, param_out):
        """The step's buffers against the plan: W bf16 gradient buffers and
        fp32 master / m / v of owned_numel elements, a bf16 parameter buffer
        of padded_numel, all on the plan's device.  Raw addresses (ints) and
        None pass through to the library's own checks."""
        _require_all(self._step_specs(grads, master, m, v, param_out), self.device)

    def _step_specs(self, grads, master, m, v, param_out):
        import torch
        if self.owned_numel == 0:
            return []
        specs = []
        if grads is not None:      # None: a call that reads no gradients (zr_step_finish from scratch)
            if len(grads) != self.world_size:
                raise ValueError(f"grads: {len(grads)} buffers, the plan has W = {self.world_size}")
            specs += [(g, f"grads[{w}]", torch.bfloat16, self.owned_numel, False) for w, g in enumerate(grads)]
        specs += [(x, name, torch.float32, self.owned_numel, False) for x, name in ((master, "master"), (m, "m"),
                                                                                      (v, "v"))]
        specs.append((param_out, "param_out", torch.bfloat16, self.param_out_numel, False))
        return specs

    @property
    def param_out_numel(self):
        """Elements of the buffer the step writes bf16 parameters into: the
        full all-gather buffer, or this rank's shard (ZR_PARAMS_OWNED)."""
        return self.owned_numel if self.param_layout == ZR_PARAMS_OWNED else self.padded_numel

    def set_param_layout(self, layout, stream=None):
        """ZR_PARAMS_GLOBAL (param_out: the full buffer) or ZR_PARAMS_OWNED
        (param_out: this rank's shard, owned order)."""
        zr_plan_set_param_layout(self.handle, layout, stream)
        self.param_layout = layout

    def bound_gather(self, first_tensor, n_tensors, shards, dst, stream=None, max_ctas=0):
        """A callable f() that runs zr_gather_params on fixed arguments,
        marshalled once: a per-layer prefetch loop then pays one C call per
        gather, not the Python argument handling."""
        from . import _addr, _check, _lib, _ptr_array, _stream
        arr = _ptr_array(shards)
        args = (self.handle, int(first_tensor), int(n_tensors), arr, _addr(dst), int(max_ctas), _stream(stream))
        fn = _lib.zr_gather_params

        def gather_fn():
            st = fn(*args)
            if st:
                _check(st, "zr_gather_params")
        gather_fn._keepalive = (arr, shards, dst)
        return gather_fn

    def gather_params(self, first_tensor, n_tensors, shards, dst, stream=None, max_ctas=0):
        """Tensors [first_tensor, first_tensor + n_tensors) whole, in the
        global layout, into dst, from every rank's bf16 shard (owned order);
        max_ctas > 0 caps the grid (a prefetch beside compute)."""
        zr_gather_params(self.handle, first_tensor, n_tensors, shards, dst, stream, max_ctas)

    def step(self, grads, master, m, v, param_out, step, stream=None):
        """zr_step: the whole step for this rank, asynchronous on `stream`."""
        self.check_step_buffers(grads, master, m, v, param_out)
        zr_step(self.handle, grads, master, m, v, param_out, step, stream)

    def step_bucket(self, bucket, grads, master, m, v, param_out, step, stream=None):
        """zr_step_bucket: this rank's part of one bucket."""
        self.check_step_buffers(grads, master, m, v, param_out)
        zr_step_bucket(self.handle, bucket, grads, master, m, v, param_out, step, stream)

    def step_finish(self, grads, master, m, v, param_out, step, stream=None):
        """zr_step_finish: the clip's second half after every bucket."""
        self.check_step_buffers(grads, master, m, v, param_out)
        zr_step_finish(self.handle, grads, master, m, v, param_out, step, stream)

    def bound_step(self, grads, master, m, v, param_out, stream=None):
        """A callable f(step) that runs zr_step on fixed buffers with the
        arguments marshalled (and checked) once (for tight loops)."""
        from . import _addr, _check, _lib, _ptr_array, _stream
        self.check_step_buffers(grads, master, m, v, param_out)
        arr = _ptr_array(grads)
        args = (self.handle, arr, _addr(master), _addr(m), _addr(v), _addr(param_out))
        s = _stream(stream)
        fn = _lib.zr_step

        def step_fn(step):
            st = fn(*args, step, s)
            if st:
                _check(st, "zr_step")
        step_fn._keepalive = (arr, grads, master, m, v, param_out)
        return step_fn

    def step_host(self, host_grads, dev_grads, master, m, v, param_out, host_param_out, step,
                  stream=None):
        """zr_step_host: gradients from host memory, the result copied back."""
        import torch
        specs = self._step_specs(dev_grads, master, m, v, param_out)
        if self.owned_numel > 0:
            if len(host_grads) != self.world_size:
                raise ValueError(f"host_grads: {len(host_grads)} buffers, the plan has W = {self.world_size}")
            specs += [(g, f"host_grads[{w}]", torch.bfloat16, self.owned_numel, True)
                      for w, g in enumerate(host_grads)]
            specs.append((host_param_out, "host_param_out", torch.bfloat16, self.param_out_numel, True))
        _require_all(specs, self.device)
        zr_step_host(self.handle, host_grads, dev_grads, master, m, v, param_out, host_param_out,
                     step, stream)

    def grad_sumsq(self, grads, out, stream=None):
        """zr_grad_sumsq: this rank's sum of squares into out[0] (fp64)."""
        import torch
        specs = [(g, f"grads[{w}]", torch.bfloat16, self.owned_numel, False) for w, g in enumerate(grads)]
        _require_all(specs + [(out, "out", torch.float64, 1, False)], self.device)
        zr_grad_sumsq(self.handle, grads, out, stream)

    def bucket_sumsq(self, out, stream=None):
        """zr_bucket_sumsq: this rank's sum of squares after a bucket-by-bucket
        pass, into out[0] (fp64), without reading gradients."""
        import torch
        from . import zr_bucket_sumsq
        _require_all([(out, "out", torch.float64, 1, False)], self.device)
        zr_bucket_sumsq(self.handle, out, stream)

    def debug_reduce(self, grads, g_out, stream=None):
        """zr_debug_reduce: the averaged fp32 gradient, owned order."""
        import torch
        specs = [(g, f"grads[{w}]", torch.bfloat16, self.owned_numel, False) for w, g in enumerate(grads)]
        _require_all(specs + [(g_out, "g_out", torch.float32, self.owned_numel, False)], self.device)
        zr_debug_reduce(self.handle, grads, g_out, stream)

    def set_adamw(self, lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, max_grad_norm=0.0):
        """Hyperparameters for the following steps (e.g. this step's lr)."""
        zr_plan_set_adamw(self.handle, lr, beta1, beta2, eps, weight_decay, max_grad_norm)
        self.max_grad_norm = max_grad_norm

    def set_checked(self, enable=True):
        """Checked mode: verify the device tables before every launch."""
        zr_plan_set_checked(self.handle, enable)

    def verify(self, stream=None):
        """zr_plan_verify: one verification of the device tables now."""
        zr_plan_verify(self.handle, stream)

    def check_result(self, stream=None):
        """zr_plan_check_result: the checked-mode status (synchronises)."""
        return zr_plan_check_result(self.handle, stream)

    def close(self):
        """Destroys the plan (the workspace tensor is freed with this object)."""
        if self.handle:
            zr_plan_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
