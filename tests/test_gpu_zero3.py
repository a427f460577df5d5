"""ZeRO-3 on the GPU: the step writing each rank's bf16 shard in owned order
(ZR_PARAMS_OWNED), and zr_gather_params assembling whole tensors from all
ranks' shards ("Scaling training to thousands of GPUs", talk summary,
section 11:24 ZeRO: stage 3 gathers a layer's parameters before use).

Every rank of a partition runs on one GPU, each with its own buffers; the
gather reads all of them (local memory standing in for peer mappings).  The
shards must equal the global-layout step at the rank's positions bit for
bit, and a gather must equal the oracle's unsharded bf16 parameters."""
import numpy as np
import pytest
import torch

import oracle
import sharded_optimizer_step_zr_b200 as zr
from gpu_harness import DEV, GpuRank, OracleRank, bf16_ulp_distance, bits32, u16

pytestmark = pytest.mark.gpu

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)

LAYOUTS = [
    ([(3, 5), (7,), (2, 2, 2), (4096 + 8,), (0,), (300, 7)], 3, 0, 4096),       # flat, pad, ragged, empty tensor
    ([(1000, 3), (8191,), (9, 9), (2048,), (17,)], 4, 1, 4096),                  # whole-tensor, odd sizes
    ([(40000,), (64, 65), (5001,), (2048 * 3,)], 8, 0, 1 << 20),                 # flat W = 8, many pieces
    ([(4097,), (33, 31), (5000,), (3,), (8, 8, 8)], 2, 1, 9000),                 # whole-tensor, misaligned
]


def step_all_ranks(shapes, W, mode, cap, layout, steps=2, seed=41):
    ranks = []
    for r in range(W):
        g = GpuRank(shapes, W, r, mode, cap, HP, seed)
        g.plan.set_param_layout(layout)
        n = g.plan.param_out_numel
        g.out = torch.full((max(n, 8),), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
        ranks.append(g)
    for t in range(1, steps + 1):
        for g in ranks:
            g.fill_grads(t, 1e-2, 0.01)
            g.step(g.out, t)
    torch.cuda.synchronize()
    return ranks


def oracle_params(shapes, W, mode, cap, steps=2, seed=41):
    oplan = oracle.Plan(shapes, W, mode, cap)
    out = np.zeros(max(oplan.padded_numel, 8), np.uint16)
    for r in range(W):
        o = OracleRank(oplan, r, seed)
        for t in range(1, steps + 1):
            o.make_grads(t, 1e-2, 0.01)
            o.step(out, HP, t)
    return oplan, out


@pytest.mark.parametrize("shapes, W, mode, cap", LAYOUTS)
def test_owned_layout_shards_equal_the_global_step(shapes, W, mode, cap):
    shard_ranks = step_all_ranks(shapes, W, mode, cap, zr.ZR_PARAMS_OWNED)
    global_ranks = step_all_ranks(shapes, W, mode, cap, zr.ZR_PARAMS_GLOBAL)
    oplan, want = oracle_params(shapes, W, mode, cap)
    for r, (s, g) in enumerate(zip(shard_ranks, global_ranks)):
        idx = oplan.owned_global_index(r)
        shard = u16(s.out)[: idx.size]
        assert np.array_equal(shard, u16(g.out)[idx]), r
        assert bf16_ulp_distance(shard, want[idx]).max(initial=0) <= 1
        for a, b in zip(s.state(), g.state()):
            assert np.array_equal(bits32(a), bits32(b))


@pytest.mark.parametrize("shapes, W, mode, cap", LAYOUTS)
def test_gather_assembles_whole_tensors(shapes, W, mode, cap):
    ranks = step_all_ranks(shapes, W, mode, cap, zr.ZR_PARAMS_OWNED)
    oplan, want = oracle_params(shapes, W, mode, cap)
    shards = [g.out for g in ranks]
    numels = [int(np.prod(s)) for s in shapes]
    goff = np.concatenate([[0], np.cumsum(numels)])
    # what the shards hold, placed at their global positions (exact copy semantics)
    placed = np.zeros(max(oplan.padded_numel, 8), np.uint16)
    for r, g in enumerate(ranks):
        idx = oplan.owned_global_index(r)
        placed[idx] = u16(g.out)[: idx.size]
    plan = ranks[0].plan
    ranges = [(0, len(shapes)), (1, 2), (len(shapes) - 1, 1), (0, 0)] + [(t, 1) for t in range(len(shapes))]
    for first, count in ranges:
        lo, hi = int(goff[first]), int(goff[first + count])
        dst = torch.full((max(hi - lo, 8),), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
        plan.gather_params(first, count, shards, dst)
        torch.cuda.synchronize()
        got = u16(dst)[: hi - lo]
        assert np.array_equal(got, placed[lo:hi]), (first, count)
        assert bf16_ulp_distance(got, want[lo:hi]).max(initial=0) <= 1
        assert np.all(u16(dst)[hi - lo:] == 0xFFFF)     # nothing written past the range


def test_layout_switches_and_refusals():
    shapes, W = [(4096,), (100,)], 2
    g = GpuRank(shapes, W, 1, 0, 1 << 20, HP, seed=3)
    ref = GpuRank(shapes, W, 1, 0, 1 << 20, HP, seed=3)
    g.plan.set_param_layout(zr.ZR_PARAMS_OWNED)
    g.plan.set_param_layout(zr.ZR_PARAMS_GLOBAL)       # back: the planned tables again
    out_g, out_r = (torch.zeros(g.plan.padded_numel, dtype=torch.bfloat16, device=DEV) for _ in range(2))
    for x, o in ((g, out_g), (ref, out_r)):
        x.fill_grads(1, 1e-2, 0.0)
        x.step(o, 1)
    torch.cuda.synchronize()
    assert torch.equal(out_g.view(torch.int16), out_r.view(torch.int16))
    with pytest.raises(zr.ZrError) as e:
        zr.zr_plan_set_param_layout(g.plan.handle, 2)
    assert e.value.status == zr.ZR_ERR_INVALID_ARG
    zr.zr_plan_set_gather_targets(g.plan.handle, [out_g, out_r])
    with pytest.raises(zr.ZrError) as e:
        zr.zr_plan_set_param_layout(g.plan.handle, zr.ZR_PARAMS_OWNED)
    assert e.value.status == zr.ZR_ERR_UNSUPPORTED
    zr.zr_plan_set_gather_targets(g.plan.handle, None)
    g.plan.set_param_layout(zr.ZR_PARAMS_OWNED)
    with pytest.raises(zr.ZrError) as e:
        zr.zr_plan_set_gather_targets(g.plan.handle, [out_g, out_r])
    assert e.value.status == zr.ZR_ERR_UNSUPPORTED
    with pytest.raises(zr.ZrError) as e:
        g.plan.gather_params(1, 2, [out_g, out_r], out_g)          # past the last tensor
    assert e.value.status == zr.ZR_ERR_INVALID_ARG


def test_owned_layout_through_buckets_and_host_copies():
    """Bucket-by-bucket steps and zr_step_host in the owned layout: the same
    shard as zr_step (the host copy in owned order)."""
    shapes, W, mode, cap = [(3000, 7), (5001,), (64, 64), (129,)], 4, 0, 8192
    a = GpuRank(shapes, W, 2, mode, cap, HP, seed=8)
    b = GpuRank(shapes, W, 2, mode, cap, HP, seed=8)
    c = GpuRank(shapes, W, 2, mode, cap, HP, seed=8)
    for x in (a, b, c):
        x.plan.set_param_layout(zr.ZR_PARAMS_OWNED)
    n = a.plan.owned_numel
    outs = [torch.zeros(n, dtype=torch.bfloat16, device=DEV) for _ in range(3)]
    host_out = torch.zeros(n, dtype=torch.bfloat16).pin_memory()
    for t in (1, 2):
        for x in (a, b, c):
            x.fill_grads(t, 1e-2, 0.01)
        a.step(outs[0], t)
        for bk in range(b.plan.n_buckets):
            b.plan.step_bucket(bk, b.grads, b.master, b.m, b.v, outs[1], t)
        b.plan.step_finish(b.grads, b.master, b.m, b.v, outs[1], t)
        host_grads = [x.cpu().pin_memory() for x in c.grads]
        c.plan.step_host(host_grads, c.grads, c.master, c.m, c.v, outs[2], host_out, t)
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    assert torch.equal(host_out.view(torch.int16), outs[0].cpu().view(torch.int16))


@pytest.mark.parametrize("seed", range(30))
def test_gather_random_sets(seed):
    """Random tensor sets (zero-element and odd sizes included), W 1..70,
    both partitions, random tensor ranges and grid caps: the gather equals
    the shards placed at their global positions by the oracle's owned ->
    global map, and writes nothing outside its range."""
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    rng = np.random.default_rng(seed)
    shapes = []
    for _ in range(int(rng.integers(1, 12))):
        k = rng.random()
        shapes.append(() if k < 0.1 else (0,) if k < 0.2 else
                      (int(rng.integers(1, 40000)),) if k < 0.6 else tuple(int(x) for x in rng.integers(1, 200, 2)))
    W = int(rng.choice([1, 2, 3, 5, 8, 13, 64, 70]))
    mode = int(rng.integers(0, 2))
    oplan = oracle.Plan(shapes, W, mode, 1 << 20)
    plan = ZrPlan(shapes, W, 0, mode, 1 << 20, *HP, device=DEV)
    owned = [int(x) for x in oplan.owned_numel]
    shards = [torch.randint(-32768, 32767, (max(n, 8),), dtype=torch.int16, device=DEV) for n in owned]
    placed = np.zeros(max(oplan.padded_numel, 8), np.uint16)
    for r in range(W):
        idx = oplan.owned_global_index(r)
        placed[idx] = shards[r][: idx.size].cpu().numpy().view(np.uint16)
    numels = [int(np.prod(s)) for s in shapes]
    goff = np.concatenate([[0], np.cumsum(numels)])
    for _ in range(4):
        first = int(rng.integers(0, len(shapes)))
        count = int(rng.integers(0, len(shapes) - first + 1))
        cap = int(rng.choice([0, 0, 1, 7, 64]))
        lo, hi = int(goff[first]), int(goff[first + count])
        dst = torch.full((hi - lo + 16,), -1, dtype=torch.int16, device=DEV)
        plan.gather_params(first, count, [s.view(torch.bfloat16) for s in shards], dst.view(torch.bfloat16),
                           max_ctas=cap)
        torch.cuda.synchronize()
        got = dst.cpu().numpy().view(np.uint16)
        assert np.array_equal(got[: hi - lo], placed[lo:hi]), (seed, first, count, cap)
        assert np.all(got[hi - lo:] == 0xFFFF)
    plan.close()
