"""zr_step_no_alloc: the step for callers that cannot allocate device memory
(a plug-in whose host framework's allocator owns the GPU's memory, or a loop
that must not call cudaMalloc because it can synchronise the device).

It keeps its scratch in the library's fixed 4 MiB device array instead of a
caller-provided workspace.  The GPU test calls it through the C ABI on two
steps in a row and compares its outputs with zr_step's on the same inputs,
within the tolerances the other parity tests use.  This file is collected
last so that a failure here cannot stop the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
import sharded_optimizer_step_zr_b200 as zr
from sharded_optimizer_step_zr_b200.plan import ZrPlan

DEV = "cuda:0"


def _u16(t):
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)


def _close(got, want, what):
    got = got.detach().cpu().numpy().astype(np.float64)
    want = want.detach().cpu().numpy().astype(np.float64)
    ok = (np.abs(got - want) <= 1e-9 + 2e-6 * np.abs(want)) | (got == want)
    assert ok.all(), f"{what}: {(~ok).sum()} elements outside 1e-9 + 2e-6 |y|"


@pytest.mark.gpu
@pytest.mark.parametrize("shapes, W, rank, mode, max_norm", [
    (synth.gpt2_small_shapes()[:20], 8, 0, 0, 0.0),        # flat, no clip
    ([(3000, 7), (5001,), (64, 64), (129,)], 8, 3, 0, 0.05),  # flat, clip, W > 4
    ([(10,), (4, 5), (7,), (3, 3), (4100,)], 3, 2, 1, 0.05),  # whole-tensor, clip, ragged
])
def test_no_alloc_matches_zr_step_on_two_calls(shapes, W, rank, mode, max_norm):
    plan = ZrPlan(shapes, W, rank, mode, 1 << 20, 3e-4, 0.9, 0.999, 1e-8, 0.1, max_norm, device=DEV)
    n = plan.owned_numel
    runs = plan.runs()
    grads = [torch.empty(n, dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    master = torch.empty(n, dtype=torch.float32, device=DEV)
    synth.fill_owned_master(master, runs, 11, n_valid=plan.total_numel)
    state_a = [master.clone(), torch.zeros_like(master), torch.zeros_like(master)]
    state_b = [master.clone(), torch.zeros_like(master), torch.zeros_like(master)]
    out_a = torch.zeros(plan.padded_numel, dtype=torch.bfloat16, device=DEV)
    out_b = torch.zeros(plan.padded_numel, dtype=torch.bfloat16, device=DEV)
    partials_b = torch.zeros(W, dtype=torch.float64, device=DEV)
    for step in (1, 2):
        for w in range(W):
            synth.fill_owned_grad(grads[w], runs, 11, step, w, 1e-2, 0.01, n_valid=plan.total_numel)
        if max_norm > 0:
            # other ranks' sums of squares: fixed values, the same for both calls
            others = torch.tensor([0.25 * (w + 1) for w in range(W)], dtype=torch.float64, device=DEV)
            plan.partials.copy_(others)
            partials_b.copy_(others)
        plan.step(grads, *state_a, out_a, step)
        grad_arr = (ctypes.c_void_p * W)(*[g.data_ptr() for g in grads])
        status = zr.raw_call("zr_step_no_alloc", plan.handle, grad_arr, state_b[0].data_ptr(),
                             state_b[1].data_ptr(), state_b[2].data_ptr(), out_b.data_ptr(),
                             partials_b.data_ptr() if max_norm > 0 else None, step,
                             torch.cuda.current_stream().cuda_stream)
        assert status == zr.ZR_OK, zr.zr_status_string(status)
        torch.cuda.synchronize()
        for a, b, what in zip(state_a, state_b, ("master", "m", "v")):
            _close(b, a, f"{what} step {step}")
        ua, ub = _u16(out_a).astype(np.int64), _u16(out_b).astype(np.int64)
        assert np.abs(ua - ub).max() <= 1
        if max_norm > 0:
            assert partials_b[rank].item() == plan.partials[rank].item()
    plan.close()


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
