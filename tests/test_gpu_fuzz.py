"""Randomised parity: seeded random tensor sets, W (1..70), partition, rank,
bucket cap and clipping, each stepped twice on the GPU -- by zr_step, or
bucket by bucket in a random order -- and compared with the oracle."""
import numpy as np
import pytest
import torch

import oracle
from gpu_harness import DEV, GpuRank, OracleRank, assert_state_close, bf16_ulp_distance, bits32, u16

pytestmark = pytest.mark.gpu


def random_case(seed):
    rng = np.random.default_rng(seed)
    shapes = []
    for _ in range(int(rng.integers(1, 9))):
        nd = int(rng.integers(0, 3))
        shapes.append(tuple(int(x) for x in rng.integers(1, 90, size=nd)) if nd else ())
        if rng.random() < 0.3:
            shapes[-1] = (int(rng.integers(1, 9000)),)
    W = int(rng.choice([1, 2, 3, 4, 5, 8, 13, 16, 17, 32, 64, 70]))
    mode = int(rng.integers(0, 2))
    rank = int(rng.integers(0, W))
    cap = int(rng.integers(16, 40000))
    clip = float(rng.choice([0.0, 0.0, 0.02, 5.0]))
    per_bucket = bool(rng.random() < 0.5)
    return shapes, W, mode, rank, cap, clip, per_bucket, rng


@pytest.mark.parametrize("seed", range(40))
def test_random_case(seed):
    shapes, W, mode, rank, cap, clip, per_bucket, rng = random_case(seed)
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, clip)
    gpu = GpuRank(shapes, W, rank, mode, cap, hp, seed=1000 + seed)
    oplan = oracle.Plan(shapes, W, mode, cap)
    orc = OracleRank(oplan, rank, seed=1000 + seed)
    P = max(oplan.padded_numel, 8)
    out_g = torch.full((P,), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    out_o = np.full(P, 0xFFFF, dtype=np.uint16)
    others = rng.random(W) * 3.0
    for t in (1, 2):
        gpu.fill_grads(t, 1e-2, 0.01)
        orc.make_grads(t, 1e-2, 0.01)
        c = None
        if clip > 0:
            S_own = oracle.sumsq(oracle.reduce(orc.grads)) if oplan.owned_numel[rank] else 0.0
            S = 0.0
            for w in range(W):
                S += S_own if w == rank else float(others[w])
            c = oracle.clip_coef(S, clip)
            gpu.plan.partials.copy_(torch.from_numpy(others))
        if per_bucket:
            for b in rng.permutation(gpu.plan.n_buckets):
                gpu.plan.step_bucket(int(b), gpu.grads, gpu.master, gpu.m, gpu.v, out_g, t)
            gpu.plan.step_finish(gpu.grads, gpu.master, gpu.m, gpu.v, out_g, t)
        else:
            gpu.step(out_g, t)
        if oplan.owned_numel[rank]:
            orc.step(out_o, hp, t, clip=c)
        torch.cuda.synchronize()
        for got, want, what in zip(gpu.state(), (orc.master, orc.m, orc.v), ("master", "m", "v")):
            assert_state_close(got, want, f"{what} step {t}")
            if clip == 0:
                assert np.array_equal(bits32(got), bits32(want)), f"{what} step {t}"
        assert bf16_ulp_distance(u16(out_g)[:oplan.padded_numel], out_o[:oplan.padded_numel]).max() <= 1
