"""ZrPlan: a plan plus its torch-allocated device workspace.

PyTorch only provides device memory and the stream; the step itself runs in
libzr.so's kernels through the C ABI.
"""
from __future__ import annotations

from . import (ZR_PARTITION_FLAT, zr_debug_reduce, zr_grad_sumsq, zr_plan_check_result, zr_plan_create,
               zr_plan_destroy, zr_plan_query, zr_plan_segments, zr_plan_set_checked, zr_plan_set_sumsq_partials,
               zr_plan_set_workspace, zr_plan_verify, zr_plan_workspace_bytes, zr_step, zr_step_bucket,
               zr_step_finish, zr_step_host)


class ZrPlan:
    def __init__(self, shapes, world_size, rank, mode=ZR_PARTITION_FLAT, bucket_cap_bytes=25 << 20,
                 lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1, max_grad_norm=0.0,
                 device=None, stream=None, bind=True):
        self.handle = zr_plan_create(shapes, world_size, rank, mode, bucket_cap_bytes, lr, beta1,
                                     beta2, eps, weight_decay, max_grad_norm)
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
        self.workspace = None
        self.partials = None
        if bind:
            self.bind(device, stream)

    def bind(self, device=None, stream=None):
        import torch
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        # torch's caching allocator returns 512-byte aligned blocks
        self.workspace = torch.empty(max(256, self.workspace_bytes), dtype=torch.uint8, device=device)
        zr_plan_set_workspace(self.handle, self.workspace, self.workspace.numel(), stream)
        if self.max_grad_norm > 0:
            self.partials = torch.zeros(self.world_size, dtype=torch.float64, device=device)
            zr_plan_set_sumsq_partials(self.handle, self.partials)

    def segments(self):
        return zr_plan_segments(self.handle)

    def runs(self):
        """(owned_offset, global_offset, length) of this rank, by owned offset."""
        runs = [(s["owned_offset"], s["global_offset"], s["length"]) for s in self.segments()
                if s["owner"] == self.rank]
        return sorted(runs)

    def step(self, grads, master, m, v, param_out, step, stream=None):
        zr_step(self.handle, grads, master, m, v, param_out, step, stream)

    def step_bucket(self, bucket, grads, master, m, v, param_out, step, stream=None):
        zr_step_bucket(self.handle, bucket, grads, master, m, v, param_out, step, stream)

    def step_finish(self, grads, master, m, v, param_out, step, stream=None):
        zr_step_finish(self.handle, grads, master, m, v, param_out, step, stream)

    def bound_step(self, grads, master, m, v, param_out, stream=None):
        """A callable f(step) that runs zr_step on fixed buffers with the
        arguments marshalled once (for tight loops)."""
        from . import _addr, _check, _lib, _ptr_array, _stream
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
        zr_step_host(self.handle, host_grads, dev_grads, master, m, v, param_out, host_param_out,
                     step, stream)

    def grad_sumsq(self, grads, out, stream=None):
        zr_grad_sumsq(self.handle, grads, out, stream)

    def debug_reduce(self, grads, g_out, stream=None):
        zr_debug_reduce(self.handle, grads, g_out, stream)

    def set_checked(self, enable=True):
        zr_plan_set_checked(self.handle, enable)

    def verify(self, stream=None):
        zr_plan_verify(self.handle, stream)

    def check_result(self, stream=None):
        return zr_plan_check_result(self.handle, stream)

    def close(self):
        if self.handle:
            zr_plan_destroy(self.handle)
            self.handle = 0

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
