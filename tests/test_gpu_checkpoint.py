"""Sharded checkpoints on the GPU: save -> load -> resume equals the
uninterrupted run bit for bit, and a resume on another partition (elastic:
W = 4 flat -> W = 3 whole-tensor) continues exactly as the unsharded oracle."""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import sharded_optimizer_step_zr_b200 as zr
from gpu_harness import DEV, GpuRank, bits32

pytestmark = pytest.mark.gpu

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)
SHAPES = [(300, 7), (1001,), (64, 64), (4099,), (5, 5, 5)]


def test_save_load_resume_is_exact(tmp_path):
    a = GpuRank(SHAPES, 4, 2, 0, 4096, HP, seed=8)
    out = torch.zeros(a.plan.padded_numel, dtype=torch.bfloat16, device=DEV)
    for t in (1, 2):
        a.fill_grads(t, 1e-2, 0.01)
        a.step(out, t)
    path = os.path.join(str(tmp_path), "r2.zrs")
    zr.zr_state_save(a.plan.handle, path, a.master, a.m, a.v, 2)
    b = GpuRank(SHAPES, 4, 2, 0, 4096, HP, seed=8)          # same gradient stream
    for t_ in (b.master, b.m, b.v):                           # state scrambled before the load
        t_.uniform_(-1.0, 1.0)
    assert zr.zr_state_load(b.plan.handle, path, b.master, b.m, b.v) == 2
    for g in (a, b):
        g.fill_grads(3, 1e-2, 0.01)
        g.step(out, 3)
    torch.cuda.synchronize()
    for x, y in zip(a.state(), b.state()):
        assert np.array_equal(bits32(x), bits32(y))
    # another rank's plan refuses the file
    c = GpuRank(SHAPES, 4, 1, 0, 4096, HP, seed=8)
    with pytest.raises(zr.ZrError) as e:
        zr.zr_state_load(c.plan.handle, path, c.master, c.m, c.v)
    assert e.value.status == zr.ZR_ERR_MISMATCH


def test_elastic_resume_on_another_partition(tmp_path):
    seed, steps = 12, 2
    src = [GpuRank(SHAPES, 4, r, 0, 4096, HP, seed) for r in range(4)]
    P = src[0].plan.padded_numel
    out = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    for t in range(1, steps + 1):
        for g in src:
            g.fill_grads(t, 1e-2, 0.01)
            g.step(out, t)
    paths = []
    for r, g in enumerate(src):
        p = os.path.join(str(tmp_path), f"w4_r{r}.zrs")
        zr.zr_state_save(g.plan.handle, p, g.master, g.m, g.v, steps)
        paths.append(p)
    # gather to a whole model on save: the bf16 export of the shard set is
    # the all-gather buffer the step wrote, bit for bit
    full = os.path.join(str(tmp_path), "model_bf16.bin")
    N = zr.zr_state_export_params(src[0].plan.handle, paths, zr.ZR_EXPORT_BF16, full)
    torch.cuda.synchronize()
    assert np.array_equal(np.fromfile(full, dtype="<u2"),
                          out[:N].cpu().view(torch.int16).numpy().view(np.uint16))
    # resume on W = 3, whole-tensor ownership
    dst = []
    for r in range(3):
        g = GpuRank(SHAPES, 3, r, 1, 4096, HP, seed)   # its initial state is replaced by the load
        p = os.path.join(str(tmp_path), f"w3_r{r}.zrs")
        zr.zr_state_reshard(g.plan.handle, paths, p)
        assert zr.zr_state_load(g.plan.handle, p, g.master, g.m, g.v) == steps
        dst.append(g)
    out3 = torch.zeros(dst[0].plan.padded_numel, dtype=torch.bfloat16, device=DEV)
    for g in dst:
        g.fill_grads(steps + 1, 1e-2, 0.01)
        g.step(out3, steps + 1)
    torch.cuda.synchronize()
    # the oracle's unsharded run of the same steps (4 replicas, then 3)
    oplan = oracle.Plan(SHAPES, 1, oracle.FLAT, 1 << 30)
    N = oplan.total_numel
    idx = torch.arange(N, dtype=torch.int64)
    master = synth.master_f32(seed, idx).numpy().copy()
    m, v = np.zeros(N, np.float32), np.zeros(N, np.float32)
    po = np.zeros(N, np.uint16)
    for t, W in ((1, 4), (2, 4), (3, 3)):
        reps = [synth.grad_bf16(seed, t, w, idx, 1e-2, 0.01).view(torch.int16).numpy()
                .view(np.uint16).copy() for w in range(W)]
        oracle.ddp_step(reps, master, m, v, po, HP, t)
    plan3 = oracle.Plan(SHAPES, 3, 1, 4096)
    for r, g in enumerate(dst):
        gi = plan3.owned_global_index(r)
        for got, want in zip(g.state(), (master, m, v)):
            assert np.array_equal(bits32(got), bits32(want[gi]))
    assert np.array_equal(out3.cpu().view(torch.int16).numpy().view(np.uint16), po)
