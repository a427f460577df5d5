"""The step inside a CUDA graph: zr_step_device_count captured once and
replayed three times gives what zr_step gives at steps 1, 2, 3 (the step
count and the AdamW scalars advance on the device at each replay)."""
import numpy as np
import pytest
import torch

import synth
from gpu_harness import DEV, GpuRank, assert_state_close, bits32

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("max_norm", [0.0, 0.05])
def test_captured_step_replays_as_successive_steps(max_norm):
    import sharded_optimizer_step_zr_b200 as zr
    shapes = synth.gpt2_small_shapes()[:20]
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, max_norm)
    eager = GpuRank(shapes, 8, 2, 0, 1 << 20, hp, seed=41)
    graphed = GpuRank(shapes, 8, 2, 0, 1 << 20, hp, seed=41)
    P = eager.plan.padded_numel
    out_e = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_g = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    d_step = torch.zeros(1, dtype=torch.int64, device=DEV)
    others = torch.full((8,), 0.3, dtype=torch.float64, device=DEV)
    if max_norm > 0:
        eager.plan.partials.copy_(others)
        graphed.plan.partials.copy_(others)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            zr.zr_step_device_count(graphed.plan.handle, graphed.grads, graphed.master, graphed.m,
                                    graphed.v, out_g, d_step)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    assert int(d_step.item()) == 0          # capturing ran nothing
    for t in (1, 2, 3):
        eager.fill_grads(t, 1e-2, 0.01)
        graphed.fill_grads(t, 1e-2, 0.01)
        eager.step(out_e, t)
        graph.replay()
        torch.cuda.synchronize()
        assert int(d_step.item()) == t
        for a, b, what in zip(eager.state(), graphed.state(), ("master", "m", "v")):
            assert_state_close(b, a, f"{what} step {t}")
            assert np.array_equal(bits32(a), bits32(b)), f"{what} step {t} not bit-identical"
        assert torch.equal(out_e.view(torch.int16), out_g.view(torch.int16))


def test_device_count_advances_on_a_rank_that_owns_nothing():
    """Whole-tensor ownership with more ranks than tensors: rank 5 owns
    nothing, yet its device step count advances with every call."""
    import sharded_optimizer_step_zr_b200 as zr
    g = GpuRank([(64,), (32,)], 8, 5, 1, 1 << 20, (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0), seed=3)
    assert g.plan.owned_numel == 0
    d_step = torch.zeros(1, dtype=torch.int64, device=DEV)
    out = torch.zeros(96 + 8, dtype=torch.bfloat16, device=DEV)
    for t in (1, 2, 3):
        zr.zr_step_device_count(g.plan.handle, g.grads, g.master, g.m, g.v, out, d_step)
    torch.cuda.synchronize()
    assert int(d_step.item()) == 3


def test_captured_step_follows_a_device_learning_rate():
    """zr_plan_set_device_lr: the graph captured once reads the lr from
    device memory at every replay; written on the device before each replay
    (a warmup schedule), the replays equal eager steps with that lr set
    through zr_plan_set_adamw, bit for bit."""
    import sharded_optimizer_step_zr_b200 as zr
    shapes = synth.gpt2_small_shapes()[:12]
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)
    eager = GpuRank(shapes, 4, 1, 0, 1 << 20, hp, seed=17)
    graphed = GpuRank(shapes, 4, 1, 0, 1 << 20, hp, seed=17)
    P = eager.plan.padded_numel
    out_e = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_g = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    d_step = torch.zeros(1, dtype=torch.int64, device=DEV)
    d_lr = torch.zeros(1, dtype=torch.float32, device=DEV)
    zr.zr_plan_set_device_lr(graphed.plan.handle, d_lr)
    graph = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            zr.zr_step_device_count(graphed.plan.handle, graphed.grads, graphed.master, graphed.m,
                                    graphed.v, out_g, d_step)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    for t in (1, 2, 3, 4):
        lr = 1e-3 * t / 4
        eager.fill_grads(t, 1e-2, 0.01)
        graphed.fill_grads(t, 1e-2, 0.01)
        eager.plan.set_adamw(lr, *hp[1:])
        eager.step(out_e, t)
        d_lr.fill_(lr)                       # the schedule, on the device
        graph.replay()
        torch.cuda.synchronize()
        for a, b, what in zip(eager.state(), graphed.state(), ("master", "m", "v")):
            assert np.array_equal(bits32(a), bits32(b)), f"{what} step {t}"
        assert torch.equal(out_e.view(torch.int16), out_g.view(torch.int16))
    zr.zr_plan_set_device_lr(graphed.plan.handle, None)
