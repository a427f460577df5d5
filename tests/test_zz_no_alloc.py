"""zr_step_no_alloc: the step for callers that cannot allocate device memory
(a plug-in whose host framework's allocator owns the GPU's memory, or a loop
that must not call cudaMalloc because it can synchronise the device).

It keeps its scratch in the library's fixed 4 MiB device array instead of a
caller-provided workspace, and runs zr_step's own kernels, so its results
must equal zr_step's bit for bit.  The GPU tests call it through the C ABI
on consecutive steps and compare master, m, v, the bf16 parameters and
this rank's sum of squares with zr_step's on the same inputs; they cover a
plan near the array's limit, the owned (ZeRO-3 shard) parameter layout,
plans that take turns on the array, and a steady-state loop that must not
copy its tile table again.  This file is collected last so that a failure
here cannot stop the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import sharded_optimizer_step_zr_b200 as zr
from sharded_optimizer_step_zr_b200.plan import ZrPlan

DEV = "cuda:0"


def _same_bits(got, want, what):
    g = got.detach().contiguous().view(torch.int32 if got.element_size() == 4 else torch.int16)
    w = want.detach().contiguous().view(torch.int32 if want.element_size() == 4 else torch.int16)
    assert torch.equal(g, w), f"{what}: {(g != w).sum().item()} elements differ"


class Pair:
    """One plan stepped twice on the same inputs: through zr_step (arm a,
    the plan's workspace) and through zr_step_no_alloc (arm b)."""

    def __init__(self, shapes, W, rank, mode, max_norm, cap=1 << 20, layout=zr.ZR_PARAMS_GLOBAL, seed=11):
        self.plan = ZrPlan(shapes, W, rank, mode, cap, 3e-4, 0.9, 0.999, 1e-8, 0.1, max_norm, device=DEV)
        if layout != zr.ZR_PARAMS_GLOBAL:
            self.plan.set_param_layout(layout)
        self.W, self.rank, self.seed, self.clip = W, rank, seed, max_norm > 0
        n = self.plan.owned_numel
        self.runs = self.plan.runs()
        self.grads = [torch.empty(max(n, 8), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
        master = torch.empty(max(n, 8), dtype=torch.float32, device=DEV)
        synth.fill_owned_master(master, self.runs, seed, n_valid=self.plan.total_numel)
        self.a = [master.clone(), torch.zeros_like(master), torch.zeros_like(master)]
        self.b = [master.clone(), torch.zeros_like(master), torch.zeros_like(master)]
        out_n = n if layout == zr.ZR_PARAMS_OWNED else self.plan.padded_numel
        self.out_a = torch.zeros(max(out_n, 8), dtype=torch.bfloat16, device=DEV)
        self.out_b = torch.zeros(max(out_n, 8), dtype=torch.bfloat16, device=DEV)
        self.partials_b = torch.zeros(W, dtype=torch.float64, device=DEV)

    def fill(self, step):
        for w in range(self.W):
            synth.fill_owned_grad(self.grads[w], self.runs, self.seed, step, w, 1e-2, 0.01,
                                  n_valid=self.plan.total_numel)
        if self.clip:
            # other ranks' sums of squares: fixed values, the same for both arms
            others = torch.tensor([0.25 * (w + 1) for w in range(self.W)], dtype=torch.float64, device=DEV)
            self.plan.partials.copy_(others)
            self.partials_b.copy_(others)

    def step_a(self, step):
        self.plan.step(self.grads, *self.a, self.out_a, step)

    def step_b(self, step):
        grad_arr = (ctypes.c_void_p * self.W)(*[g.data_ptr() for g in self.grads])
        status = zr.raw_call("zr_step_no_alloc", self.plan.handle, grad_arr, self.b[0].data_ptr(),
                             self.b[1].data_ptr(), self.b[2].data_ptr(), self.out_b.data_ptr(),
                             self.partials_b.data_ptr() if self.clip else None, step,
                             torch.cuda.current_stream().cuda_stream)
        assert status == zr.ZR_OK, zr.zr_status_string(status)

    def check(self, step):
        torch.cuda.synchronize()
        for x, y, what in zip(self.b, self.a, ("master", "m", "v")):
            _same_bits(x, y, f"{what} step {step}")
        _same_bits(self.out_b, self.out_a, f"bf16 parameters step {step}")
        if self.clip:
            assert self.partials_b[self.rank].item() == self.plan.partials[self.rank].item()

    def close(self):
        self.plan.close()


@pytest.mark.gpu
@pytest.mark.parametrize("shapes, W, rank, mode, max_norm, layout", [
    (synth.gpt2_small_shapes()[:20], 8, 0, 0, 0.0, zr.ZR_PARAMS_GLOBAL),         # flat, no clip
    ([(3000, 7), (5001,), (64, 64), (129,)], 8, 3, 0, 0.05, zr.ZR_PARAMS_GLOBAL),  # flat, clip, W > 4
    ([(10,), (4, 5), (7,), (3, 3), (4100,)], 3, 2, 1, 0.05, zr.ZR_PARAMS_GLOBAL),  # whole-tensor, clip, ragged
    ([(3000, 7), (5001,), (64, 64), (129,)], 4, 1, 0, 0.05, zr.ZR_PARAMS_OWNED),   # ZeRO-3 shard, clip, W <= 4
    (synth.gpt2_small_shapes()[:26], 8, 5, 1, 0.0, zr.ZR_PARAMS_OWNED),           # ZeRO-3 shard, whole-tensor
])
def test_no_alloc_matches_zr_step_on_consecutive_calls(shapes, W, rank, mode, max_norm, layout):
    p = Pair(shapes, W, rank, mode, max_norm, layout=layout)
    for step in (1, 2, 3):
        p.fill(step)
        p.step_a(step)
        p.step_b(step)
        p.check(step)
    p.close()


@pytest.mark.gpu
def test_no_alloc_near_the_scratch_limit():
    """The 1.3B set's whole-tensor rank-3 shard at W = 8 with clipping
    (163.7 M owned elements, about 80,000 tiles: 3.2 MB of the 4 MiB
    array), two consecutive steps, bit for bit against zr_step."""
    wl = synth.WORKLOADS["gpt_1p3b_w8_whole_clip"]
    p = Pair(wl.shapes, wl.world_size, wl.ranks[0], wl.mode, wl.max_grad_norm, cap=wl.bucket_cap_bytes)
    n_tiles = sum((length + 2047) // 2048 for _, _, length in p.runs)
    assert 32 * n_tiles + 8 * n_tiles > 3 << 20          # the table and partials fill most of the array
    for step in (1, 2):
        p.fill(step)
        p.step_a(step)
        p.step_b(step)
        p.check(step)
    p.close()


@pytest.mark.gpu
def test_no_alloc_plans_taking_turns_and_a_layout_change():
    """The array holds one plan's tile table at a time: plans that take
    turns (A, B, A) and a plan whose tables are rebuilt (a switch to the
    owned layout) each get their own table, so every call still equals
    zr_step bit for bit."""
    a = Pair([(3000, 7), (5001,), (129,)], 4, 1, 0, 0.0, seed=3)
    b = Pair([(777,), (64, 64), (40000,)], 2, 0, 1, 0.05, seed=5)
    for step, pair in ((1, a), (1, b), (2, a), (2, b), (3, a)):
        pair.fill(step)
        pair.step_a(step)
        pair.step_b(step)
        pair.check(step)
    # the same plan, its tile tables rebuilt for the owned layout
    c = Pair([(3000, 7), (5001,), (129,)], 4, 1, 0, 0.0, seed=7)
    c.fill(1)
    c.step_a(1)
    c.step_b(1)
    c.check(1)
    c.plan.set_param_layout(zr.ZR_PARAMS_OWNED)
    n = c.plan.owned_numel
    c.out_a = torch.zeros(n, dtype=torch.bfloat16, device=DEV)
    c.out_b = torch.zeros(n, dtype=torch.bfloat16, device=DEV)
    c.fill(2)
    c.step_a(2)
    c.step_b(2)
    c.check(2)
    for pair in (a, b, c):
        pair.close()


@pytest.mark.gpu
def test_no_alloc_steady_state_copies_nothing_from_the_host():
    """After the first call of a plan, later calls of the same plan enqueue
    only kernels (and, with clipping, a device-side memset of the clip's
    counters): no host-to-device copy of the tile table, so the call never
    waits on pageable host memory."""
    from torch.profiler import ProfilerActivity, profile
    p = Pair([(3000, 7), (5001,), (64, 64), (129,)], 8, 3, 0, 0.05)
    p.fill(1)
    p.step_b(1)                        # first call: the table is uploaded
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for step in (2, 3):
            p.step_b(step)
        torch.cuda.synchronize()
    names = [e.name for e in prof.events()]
    kernels = [x for x in names if "zr_tile_kernel" in x]
    if not kernels:
        pytest.skip("the profiler recorded no CUDA activity on this machine")
    assert len(kernels) == 4          # two passes per clipped step
    assert not any("HtoD" in x for x in names), [x for x in names if "emcpy" in x]
    p.close()


def test_no_alloc_rejects_plans_beyond_the_scratch():
    """A shard needing more tiles than the 4 MiB array holds is refused before
    any CUDA call (so this runs without a GPU too)."""
    h = zr.zr_plan_create([(1 << 30,)], 1, 0, 0, 1 << 20)
    try:
        grads = (ctypes.c_void_p * 1)(1 << 20)
        st = zr.raw_call("zr_step_no_alloc", h, grads, 1 << 20, 1 << 21, 1 << 22, 1 << 23, None, 1, None)
        assert st == zr.ZR_ERR_UNSUPPORTED
        with pytest.raises(zr.ZrError, match="static scratch"):
            zr.zr_step_no_alloc(h, [1 << 20], 1 << 20, 1 << 21, 1 << 22, 1 << 23, None, 1, stream=0)
    finally:
        zr.zr_plan_destroy(h)
