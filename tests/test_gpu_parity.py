"""GPU parity: libzr.so's kernels against the oracle on the same seeded inputs.

Bars (element by element):
  * averaged fp32 gradient (zr_debug_reduce): bit-exact (fixed rank-order
    fold);
  * master / m / v after the steps: |x - y| <= 1e-9 + 2e-6 |y|;
  * bf16 parameters: within 1 ulp;
  * and, since the kernels evaluate the definition's fp32 operations in the
    same order with round-to-nearest intrinsics, bit-exactness is checked too.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import (DEV, GpuRank, OracleRank, assert_state_close, bf16_ulp_distance, bits32, u16)

pytestmark = pytest.mark.gpu

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)


def run_all_ranks(shapes, W, mode, cap, steps, sigma, outlier, seed=2024, hp=HP, ranks=None,
                  exact=True):
    """Step every rank (or `ranks`) on the GPU and in the oracle, writing into
    one parameter buffer each (the emulated all-gather), and compare."""
    oplan = oracle.Plan(shapes, W, mode, cap)
    ranks = list(range(W)) if ranks is None else ranks
    gpu = {r: GpuRank(shapes, W, r, mode, cap, hp, seed) for r in ranks}
    orc = {r: OracleRank(oplan, r, seed) for r in ranks}
    P = max(oplan.padded_numel, 8)
    out_gpu = torch.full((P,), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    out_orc = np.full(P, 0xFFFF, dtype=np.uint16)
    for t in range(1, steps + 1):
        for r in ranks:
            gpu[r].fill_grads(t, sigma, outlier)
            orc[r].make_grads(t, sigma, outlier)
            # inputs agree bit for bit
            n = oplan.owned_numel[r]
            for w in range(W):
                assert np.array_equal(u16(gpu[r].grads[w][:n]), orc[r].grads[w])
            g = gpu[r].reduce()
            torch.cuda.synchronize()
            assert np.array_equal(bits32(g), bits32(oracle.reduce(orc[r].grads))), f"reduce rank {r} step {t}"
            gpu[r].step(out_gpu, t)
            orc[r].step(out_orc, hp, t)
        torch.cuda.synchronize()
        for r in ranks:
            gm, gmm, gv = gpu[r].state()
            assert_state_close(gm, orc[r].master, f"master rank {r} step {t}")
            assert_state_close(gmm, orc[r].m, f"m rank {r} step {t}")
            assert_state_close(gv, orc[r].v, f"v rank {r} step {t}")
            if exact:
                assert np.array_equal(bits32(gm), bits32(orc[r].master))
                assert np.array_equal(bits32(gmm), bits32(orc[r].m))
                assert np.array_equal(bits32(gv), bits32(orc[r].v))
        got = u16(out_gpu)
        assert bf16_ulp_distance(got, out_orc).max() <= 1
        if exact:
            assert np.array_equal(got, out_orc)
    return gpu, orc, oplan


def test_generator_identical_on_cpu_and_gpu():
    idx = torch.arange(0, 1 << 20, dtype=torch.int64)
    for sigma, out in ((1e-2, 0.0), (1e-3, 0.01)):
        a = synth.grad_bf16(5, 2, 3, idx, sigma, out)
        b = synth.grad_bf16(5, 2, 3, idx.to(DEV), sigma, out).cpu()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    a = synth.master_f32(5, idx)
    b = synth.master_f32(5, idx.to(DEV)).cpu()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_tiny_both_ranks_three_steps():
    """The tiny workload: 4 tensors, W = 2, both ranks, flat, 1 MB buckets,
    N(0, 1e-2) gradients, 3 steps; both ranks fill one parameter buffer."""
    wl = synth.WORKLOADS["tiny"]
    _, _, oplan = run_all_ranks(wl.shapes, 2, 0, wl.bucket_cap_bytes, 3, 1e-2, 0.0, seed=wl.seed,
                                hp=wl.hp)
    assert oplan.total_numel == 1_441_792


@pytest.mark.parametrize("shapes, W, mode, cap", [
    ([(3, 5), (7,), (2, 2, 2)], 4, 0, 16),                 # pad > 0, tiny segments
    ([(4096 * 3 + 5,), (17,), (1,)], 1, 0, 1 << 20),       # W = 1, ragged tail, length 1
    ([(1000, 3), (8191,), (9, 9)], 3, 0, 4096),            # W = 3 (non power of two), pad 2
    ([(12345,), (8,), (777,), (64, 65)], 5, 0, 20000),     # W = 5
    ([(10,), (4, 5), (7,), (3, 3), (20,)], 3, 1, 40),      # whole-tensor, odd sizes
    ([(4097,), (33, 31), (5000,), (3,), (8, 8, 8)], 2, 1, 9000),  # whole-tensor, misaligned stores
    ([(16384,), (2048,), (4099,)], 8, 0, 1 << 20),         # W = 8, multi-tile
    ([(7, 1024), (100,)], 16, 0, 1 << 20),                 # W = 16
    ([(5000,), (300,)], 33, 0, 1 << 20),                   # W = 33: a partial second load group
    ([(4096,), (512,)], 64, 1, 1 << 20),                   # W = 64, whole-tensor, empty ranks
    ([(0,), (100,), (3, 0), (2050,)], 2, 0, 4096),         # zero-element tensors among the rest
    ([(0,), (100,), (3, 0), (2050,)], 3, 1, 4096),         # same, whole-tensor: rank 2 owns nothing
])
def test_edge_shapes(shapes, W, mode, cap):
    run_all_ranks(shapes, W, mode, cap, 2, 1e-3, 0.01)


@pytest.mark.parametrize("shapes", [[], [(0,)], [(0,), (3, 0)]])
@pytest.mark.parametrize("clip", [0.0, 1.0])
def test_sets_without_parameters(shapes, clip):
    """No parameters at all (no tensors, or only zero-element ones): every
    step call succeeds without touching memory, and a device step count
    still advances."""
    import sharded_optimizer_step_zr_b200 as zr
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    plan = ZrPlan(shapes, 2, 1, 0, 4096, *HP[:5], max_grad_norm=clip, device=DEV)
    assert (plan.total_numel, plan.padded_numel, plan.owned_numel) == (0, 0, 0)
    e16 = torch.empty(0, dtype=torch.bfloat16, device=DEV)
    e32 = torch.empty(0, dtype=torch.float32, device=DEV)
    plan.step([e16, e16], e32, e32, e32, e16, 1)
    for b in range(plan.n_buckets):
        plan.step_bucket(b, [e16, e16], e32, e32, e32, e16, 1)
    plan.step_finish([e16, e16], e32, e32, e32, e16, 1)
    d_step = torch.zeros(1, dtype=torch.int64, device=DEV)
    for _ in range(3):
        zr.zr_step_device_count(plan.handle, [e16, e16], e32, e32, e32, e16, d_step)
    torch.cuda.synchronize()
    assert d_step.item() == 3
    plan.close()


@pytest.mark.parametrize("t0", [1000, 10 ** 6, 2 ** 33 + 5])
def test_large_step_numbers(t0):
    """Three steps from step number t0 (bias corrections near or exactly 1;
    2**33 + 5 needs the 64-bit step), eager zr_step and the device-resident
    count (preset to t0 - 1) each against the oracle, bit for bit."""
    import sharded_optimizer_step_zr_b200 as zr
    shapes = [(4096 * 2 + 13,), (300, 3)]
    W = 4
    oplan = oracle.Plan(shapes, W, 0, 1 << 20)
    P = oplan.padded_numel
    for r in (0, W - 1):
        eager = GpuRank(shapes, W, r, 0, 1 << 20, HP, seed=77)
        counted = GpuRank(shapes, W, r, 0, 1 << 20, HP, seed=77)
        orc = OracleRank(oplan, r, seed=77)
        out_e = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
        out_c = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
        out_o = np.zeros(P, np.uint16)
        d_step = torch.full((1,), t0 - 1, dtype=torch.int64, device=DEV)
        for k in range(3):
            # gradients from generator steps 1..3; optimizer step numbers t0..t0+2
            eager.fill_grads(k + 1, 1e-3, 0.01)
            counted.fill_grads(k + 1, 1e-3, 0.01)
            orc.make_grads(k + 1, 1e-3, 0.01)
            eager.step(out_e, t0 + k)
            zr.zr_step_device_count(counted.plan.handle, counted.grads, counted.master, counted.m, counted.v,
                                    out_c, d_step)
            orc.step(out_o, HP, t0 + k)
        torch.cuda.synchronize()
        assert d_step.item() == t0 + 2
        for g in (eager, counted):
            for got, want in zip(g.state(), (orc.master, orc.m, orc.v)):
                assert np.array_equal(bits32(got), bits32(want)), (t0, r)
        mine = oplan.owned_global_index(r)
        mine = mine[mine < oplan.total_numel]
        for out in (out_e, out_c):
            assert np.array_equal(u16(out)[mine], out_o[mine])


def test_thirty_steps_stay_bit_exact():
    """30 consecutive steps (fresh gradients each step, flat W = 4, ragged
    tail): fp32 state and the bf16 buffer equal the oracle's bit for bit
    after every step -- no drift builds up."""
    shapes = [(50_000,), (3, 1001), (4096 + 3,)]
    W, cap = 4, 1 << 16
    oplan = oracle.Plan(shapes, W, 0, cap)
    P = oplan.padded_numel
    for r in (0, W - 1):
        gpu = GpuRank(shapes, W, r, 0, cap, HP, seed=31)
        orc = OracleRank(oplan, r, seed=31)
        out_g = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
        out_o = np.zeros(P, np.uint16)
        for t in range(1, 31):
            gpu.fill_grads(t, 1e-3, 0.01)
            orc.make_grads(t, 1e-3, 0.01)
            gpu.step(out_g, t)
            orc.step(out_o, HP, t)
            torch.cuda.synchronize()
            for got, want in zip(gpu.state(), (orc.master, orc.m, orc.v)):
                assert np.array_equal(bits32(got), bits32(want)), (r, t)
        mine = oplan.owned_global_index(r)
        assert np.array_equal(u16(out_g)[mine], out_o[mine])


@pytest.mark.parametrize("clip", [0.0, 1.0])
def test_learning_rate_schedule(clip):
    """zr_plan_set_adamw between steps: a warmup-then-cosine lr over five
    steps (and, with clipping, a changing max_grad_norm), both ranks of a
    flat W = 2 partition, against the oracle stepping with the same
    per-step hyperparameters."""
    import math
    shapes = [(4096 * 3 + 5,), (300,)]
    W = 2
    oplan = oracle.Plan(shapes, W, 0, 1 << 20)
    P = oplan.padded_numel
    ranks = [GpuRank(shapes, W, r, 0, 1 << 20, HP, seed=13, max_grad_norm=clip) for r in range(W)]
    orcs = [OracleRank(oplan, r, seed=13) for r in range(W)]
    out_g = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_o = np.zeros(P, np.uint16)
    for t in range(1, 6):
        lr = 1e-3 * min(1.0, t / 2) * 0.5 * (1 + math.cos(math.pi * t / 6))
        mgn = clip * (1.0 + 0.5 * t) if clip > 0 else 0.0
        hp = (lr, 0.9, 0.999, 1e-8, 0.1, mgn)
        S_parts = []
        for g, o in zip(ranks, orcs):
            g.fill_grads(t, 1e-2, 0.01)
            o.make_grads(t, 1e-2, 0.01)
            S_parts.append(oracle.sumsq(oracle.reduce(o.grads)))
        c = None
        if clip > 0:
            S = 0.0
            for x in S_parts:
                S += x
            c = oracle.clip_coef(S, mgn)
            for g in ranks:
                g.plan.partials.copy_(torch.tensor(S_parts, dtype=torch.float64))
        for g, o in zip(ranks, orcs):
            g.plan.set_adamw(*hp)
            g.step(out_g, t)
            o.step(out_o, hp, t, clip=c)
        torch.cuda.synchronize()
        for g, o in zip(ranks, orcs):
            for got, want in zip(g.state(), (o.master, o.m, o.v)):
                if clip == 0:
                    assert np.array_equal(bits32(got), bits32(want)), t
                else:
                    assert_state_close(got, want, f"step {t}")
        assert bf16_ulp_distance(u16(out_g), out_o).max() <= 1


def test_max_world_size():
    """W = 512, the ABI's maximum (the pointer array's largest instantiation):
    first, middle and last rank."""
    run_all_ranks([(512 * 40 + 3,), (100,)], 512, 0, 1 << 20, 2, 1e-3, 0.01, ranks=[0, 255, 511])


def test_special_values():
    """±0, subnormals, huge values, inf and NaN in the replicas."""
    shapes = [(4096 + 24,)]
    W = 4
    rng = np.random.default_rng(0)
    n = 4096 + 24
    vals = (rng.standard_normal((W, n)) * 1e-3).astype(np.float32)
    vals[:, 0] = -0.0                           # all -0: the fold keeps the sign
    vals[0, 1], vals[1:, 1] = 0.0, -0.0
    vals[:, 2] = 1e-39                           # bf16 subnormals
    vals[:, 3] = np.float32(-3e38)               # fp32 overflow to -inf in the fold
    vals[0, 4] = np.inf
    vals[1, 5] = np.nan
    vals[:, 6] = np.float32(1e30) * np.array([1, -1, 1, -1])   # exact cancellation
    vals[:, 7] = np.float32(2.0 ** -130)
    vals[:, 8:16] = np.float32(1e-3) * np.arange(8)
    grads = [oracle.f32_to_bf16_array(vals[w]) for w in range(W)]
    oplan = oracle.Plan(shapes, W, 0, 1 << 20)
    P = oplan.padded_numel
    out_gpu = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_orc = np.zeros(P, dtype=np.uint16)
    for r in range(W):
        gr = GpuRank(shapes, W, r, 0, 1 << 20, HP, seed=1)
        orr = OracleRank(oplan, r, seed=1)
        idx = oplan.owned_global_index(r)
        sl = [g[idx] for g in grads]
        gr.set_grads(sl)
        orr.grads = sl
        g = gr.reduce()
        torch.cuda.synchronize()
        ref = oracle.reduce(sl)
        same = (bits32(g) == bits32(ref)) | (np.isnan(g.cpu().numpy()) & np.isnan(ref))
        assert same.all()
        gr.step(out_gpu, 1)
        orr.step(out_orc, HP, 1)
        torch.cuda.synchronize()
        for got, want, what in zip(gr.state(), (orr.master, orr.m, orr.v), ("master", "m", "v")):
            assert_state_close(got, want, what)
    assert bf16_ulp_distance(u16(out_gpu), out_orc).max() <= 1


@pytest.mark.parametrize("W, mode", [(8, 0), (3, 0), (8, 1), (4, 1)])
def test_clip_all_ranks(W, mode):
    """Global-norm clip (max_norm small enough to bite): other ranks' sums of
    squares come from zr_grad_sumsq, this rank's from zr_step itself."""
    shapes = [(3000, 7), (5001,), (64, 64), (129,), (17, 5)]
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.05)
    seed = 99
    oplan = oracle.Plan(shapes, W, mode, 8192)
    gpu = [GpuRank(shapes, W, r, mode, 8192, hp, seed) for r in range(W)]
    orc = [OracleRank(oplan, r, seed) for r in range(W)]
    partials = torch.zeros(W, dtype=torch.float64, device=DEV)
    P = oplan.padded_numel
    out_gpu = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_orc = np.zeros(P, dtype=np.uint16)
    for t in (1, 2):
        for r in range(W):
            gpu[r].fill_grads(t, 1e-2, 0.01)
            orc[r].make_grads(t, 1e-2, 0.01)
        # the oracle's global S in rank order of per-rank partials
        S_parts = [oracle.sumsq(oracle.reduce(o.grads)) for o in orc]
        S = 0.0
        for x in S_parts:
            S += x
        c = oracle.clip_coef(S, hp[5])
        assert c < 1.0
        for r in range(W):
            gpu[r].plan.grad_sumsq(gpu[r].grads, partials[r:r + 1])
        torch.cuda.synchronize()
        got_parts = partials.cpu().numpy()
        for r in range(W):
            assert abs(got_parts[r] - S_parts[r]) <= 1e-12 * S_parts[r]
        for r in range(W):
            gpu[r].plan.partials.copy_(partials)
            before = partials[r].item()
            gpu[r].step(out_gpu, t)
            torch.cuda.synchronize()
            # zr_step's own pass reproduces zr_grad_sumsq's value bit for bit
            assert gpu[r].plan.partials[r].item() == before
            orc[r].step(out_orc, hp, t, clip=c)
        torch.cuda.synchronize()
        for r in range(W):
            for got, want, what in zip(gpu[r].state(), (orc[r].master, orc[r].m, orc[r].v),
                                       ("master", "m", "v")):
                assert_state_close(got, want, f"{what} rank {r} step {t}")
        assert bf16_ulp_distance(u16(out_gpu), out_orc).max() <= 1


def test_average_matches_ieee_division_for_every_input():
    """Stage 1's averaging (s / W: a multiply by 1/W for powers of two, a
    division otherwise) gives the bits of IEEE division for every one of the
    2^32 fp32 values s -- subnormal quotients included -- and every W the
    library accepts."""
    from sharded_optimizer_step_zr_b200 import ZR_MAX_WORLD_SIZE, zr_debug_average_check
    bad = torch.full((ZR_MAX_WORLD_SIZE,), -1, dtype=torch.int64, device=DEV)
    zr_debug_average_check(1, ZR_MAX_WORLD_SIZE, bad)
    torch.cuda.synchronize()
    bad = bad.cpu().numpy()
    assert (bad == 0).all(), {w + 1: int(b) for w, b in enumerate(bad) if b}


def test_clip_combine_paths_agree():
    """S_r of a plan of at most 8 groups of 1024 tiles (summed by one CTA) and
    of a plan of more groups (a grid of CTAs) follow the same fixed order:
    the same gradients, followed in tile order by 3907 tiles of zeros whose
    partials are +0.0, give the same bits.  W = 1, flat; the extra tensor is
    declared first, so it is packed last, in a bucket of its own."""
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, 1.0)
    own = [(4_000_000,), (3_200_000,), (3_000_000,)]      # one 20.4 MB bucket: about 4980 tiles
    extra = 3907 * 2048                                     # a multiple of the tile: same cuts after it
    small = ZrPlan(own, 1, 0, 0, 25 << 20, *hp, device=DEV)
    grid = ZrPlan([(extra,)] + own, 1, 0, 0, 25 << 20, *hp, device=DEV)
    assert (small.n_buckets, grid.n_buckets) == (1, 2)
    n = small.owned_numel
    gen = torch.Generator(device=DEV).manual_seed(7)
    g = (torch.randn(n, generator=gen, device=DEV) * 1e-2).to(torch.bfloat16)
    g_grid = torch.cat([torch.zeros(extra, dtype=torch.bfloat16, device=DEV), g])
    s_small = torch.zeros(1, dtype=torch.float64, device=DEV)
    s_grid = torch.zeros(1, dtype=torch.float64, device=DEV)
    small.grad_sumsq([g], s_small)
    grid.grad_sumsq([g_grid], s_grid)
    torch.cuda.synchronize()
    assert s_small.item() == s_grid.item()
    want = oracle.sumsq(oracle.reduce([u16(g)]))
    assert abs(s_small.item() - want) <= 1e-12 * want
    small.close()
    grid.close()


def test_unwritten_positions_untouched():
    """A rank writes exactly its own positions of the parameter buffer."""
    shapes = [(1000,), (333,), (4100,)]
    for mode in (0, 1):
        oplan = oracle.Plan(shapes, 3, mode, 2048)
        for r in range(3):
            gr = GpuRank(shapes, 3, r, mode, 2048, HP, seed=4)
            gr.fill_grads(1, 1e-3, 0.0)
            out = torch.full((oplan.padded_numel,), 0x7FC1, dtype=torch.int16, device=DEV)
            gr.step(out.view(torch.bfloat16), 1)
            torch.cuda.synchronize()
            got = out.cpu().numpy().view(np.uint16)
            mine = np.zeros(oplan.padded_numel, dtype=bool)
            mine[oplan.owned_global_index(r)] = True
            assert np.all(got[~mine] == 0x7FC1)
            assert not np.any(got[mine] == 0x7FC1)


def test_bad_alignment_rejected_on_device():
    import sharded_optimizer_step_zr_b200 as zr
    gr = GpuRank([(4096,)], 2, 0, 0, 1 << 20, HP, seed=1)
    out = torch.zeros(4096 + 8, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(zr.ZrError) as e:
        zr.zr_step(gr.plan.handle, [gr.grads[0].data_ptr() + 2, gr.grads[1]], gr.master, gr.m, gr.v,
                   out, 1)
    assert e.value.status == zr.ZR_ERR_ALIGNMENT
    with pytest.raises(zr.ZrError) as e:
        zr.zr_step(gr.plan.handle, gr.grads, gr.master.data_ptr() + 4, gr.m, gr.v, out, 1)
    assert e.value.status == zr.ZR_ERR_ALIGNMENT


@pytest.mark.parametrize("shapes, W, rank, mode, max_norm", [
    (synth.gpt2_small_shapes()[:30], 8, 1, 0, 0.0),               # flat, many chunks
    ([(4096 * 3 + 5,), (17,), (1,), (300, 7)], 3, 2, 0, 0.0),     # ragged tiles, pad
    ([(1000, 3), (8191,), (9, 9), (2048,)], 4, 1, 1, 0.05),       # whole-tensor, clip, re-read
    ([(3000, 7), (5001,), (64, 64), (129,)], 8, 3, 0, 0.05),      # clip with g scratch
])
def test_step_host_matches_step(shapes, W, rank, mode, max_norm):
    """zr_step_host (gradients from pinned host memory, chunked copy-in /
    step / copy-out pipeline) gives zr_step's results bit for bit."""
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, max_norm)
    ref = GpuRank(shapes, W, rank, mode, 4096, hp, seed=31)
    pipe = GpuRank(shapes, W, rank, mode, 4096, hp, seed=31)
    n = ref.plan.owned_numel
    P = ref.plan.padded_numel
    out_ref = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_dev = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    host_out = torch.full((P,), -1, dtype=torch.int16).pin_memory()
    dev_grads = [torch.zeros(max(n, 8), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    others = torch.tensor([0.5] * W, dtype=torch.float64, device=DEV)
    for t in (1, 2):
        ref.fill_grads(t, 1e-2, 0.01)
        host_grads = [g.cpu().pin_memory() for g in ref.grads]
        if max_norm > 0:
            ref.plan.partials.copy_(others)
            pipe.plan.partials.copy_(others)
        ref.step(out_ref, t)
        pipe.plan.step_host(host_grads, dev_grads, pipe.master, pipe.m, pipe.v, out_dev,
                            host_out.view(torch.bfloat16), t)
        torch.cuda.synchronize()
        for a, b, what in zip(ref.state(), pipe.state(), ("master", "m", "v")):
            assert np.array_equal(bits32(a), bits32(b)), f"{what} step {t}"
        for w in range(W):
            assert torch.equal(dev_grads[w][:n].view(torch.int16), ref.grads[w][:n].view(torch.int16))
        assert torch.equal(out_ref.view(torch.int16), out_dev.view(torch.int16))
        oplan = oracle.Plan(shapes, W, mode, 4096)
        mine = oplan.owned_global_index(rank)
        assert np.array_equal(host_out.numpy()[mine], out_ref.view(torch.int16).cpu().numpy()[mine])
        rest = np.ones(P, dtype=bool)
        rest[mine] = False
        assert np.all(host_out.numpy()[rest] == -1)
