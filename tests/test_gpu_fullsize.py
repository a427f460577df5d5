"""Parity at the workloads' full sizes, in the launch configuration the
benchmark times (zr_step through ZrPlan on one rank's whole shard), after
three steps for configs 2-4 and the 25 MB sweep points, after one for the
other 32 points of the sweep.

The oracle cannot step every element of these shards quickly, but the
step is elementwise once the clip coefficient is known, so it is checked on
sampled owned elements (random ones plus both ends of every segment), each
recomputed by the oracle from its own host-generated inputs.  For the
clipped workload the coefficient needs the global sum of squares over all
1.3 B parameters: the host computes it with the oracle's reduce and sumsq
over every rank's shard (inputs from the C twin of the generator).
"""
import concurrent.futures as cf
import dataclasses
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import DEV, assert_state_close, bf16_ulp_distance, bits32, u16
from sharded_optimizer_step_zr_b200.plan import ZrPlan

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def sample_owned(plan_runs, n_owned, k=20000, seed=0):
    rng = np.random.default_rng(seed)
    idx = set(rng.integers(0, n_owned, size=k).tolist())
    for owned, _, length in plan_runs:
        idx.update([owned, owned + length - 1, min(owned + 7, owned + length - 1)])
    idx.update([0, n_owned - 1])
    return np.array(sorted(i for i in idx if 0 <= i < n_owned), dtype=np.int64)


def owned_to_global(runs, owned_idx):
    starts = np.array([r[0] for r in runs], dtype=np.int64)
    globs = np.array([r[1] for r in runs], dtype=np.int64)
    j = np.searchsorted(starts, owned_idx, side="right") - 1
    return globs[j] + (owned_idx - starts[j])


def host_global_sumsq(oplan, wl, step, threads):
    """S = sum over ranks in rank order of the oracle's S_r (owned order,
    chunked), from host-generated replicas."""
    chunk = 1 << 24

    def rank_sumsq(r):
        total = 0.0
        for owned, glob, length in oplan.runs(r):
            for c0 in range(0, length, chunk):
                n = min(chunk, length - c0)
                reps = [synth.grad_bf16_range_c(wl.seed, step, w, glob + c0, n, wl.grad_sigma,
                                                wl.outlier_frac, n_valid=oplan.total_numel)
                        for w in range(wl.world_size)]
                total += oracle.sumsq(oracle.reduce(reps))
        return total

    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        parts = list(ex.map(rank_sumsq, range(wl.world_size)))
    S = 0.0
    for x in parts:
        S += x
    return S, parts


SWEEP = {wl.name: wl for wl in synth.sweep_workloads()}
# The Llama set at W = 2: rank 1 owns 3.37 G elements, so owned offsets pass
# 2**31 (and byte offsets of the fp32 state 2**34); about 81 GB on the device.
# Replica counts that are not powers of two (a true division by W; three
# full groups of 8 replicas, and one partial group), on the 1.3B set.
LARGE = {"llama_7b_w2": dataclasses.replace(synth.WORKLOADS["llama_7b_w64"], name="llama_7b_w2",
                                            world_size=2, ranks=(1,)),
         "sweep_1p3b_flat_w24_cap25": dataclasses.replace(SWEEP["sweep_1p3b_flat_w32_cap25"],
                                                          name="sweep_1p3b_flat_w24_cap25", world_size=24,
                                                          ranks=(13,)),
         "sweep_1p3b_whole_w6_cap25": dataclasses.replace(SWEEP["sweep_1p3b_whole_w8_cap25"],
                                                          name="sweep_1p3b_whole_w6_cap25", world_size=6,
                                                          ranks=(2,)),
         # the widest replica counts (up to the library's limit), last rank
         "sweep_1p3b_flat_w512_cap25": dataclasses.replace(SWEEP["sweep_1p3b_flat_w64_cap25"],
                                                           name="sweep_1p3b_flat_w512_cap25", world_size=512,
                                                           ranks=(511,)),
         "sweep_1p3b_flat_w96_cap25": dataclasses.replace(SWEEP["sweep_1p3b_flat_w64_cap25"],
                                                          name="sweep_1p3b_flat_w96_cap25", world_size=96,
                                                          ranks=(50,))}

# Configs 2-4 (and the last rank of config 4, whose offsets pass 2**32; and
# a shard of more than 2**31 elements), and
# the 1.3B sweep at the 25 MB cap: three steps, each with fresh gradients,
# so the checked m and v carry state from the earlier steps.
THREE_STEP = ([("gpt2_124m_w8", None), ("llama_7b_w64", None), ("llama_7b_w64", 63),
               ("gpt_1p3b_w8_whole_clip", None), ("llama_7b_w2", None),
               ("sweep_1p3b_flat_w24_cap25", None), ("sweep_1p3b_whole_w6_cap25", None),
               ("sweep_1p3b_flat_w512_cap25", None), ("sweep_1p3b_flat_w96_cap25", None)] +
              [(f"sweep_1p3b_{m}_w{w}_cap25", None) for m in ("flat", "whole") for w in (2, 8, 32, 64)])
# The rest of the sweep (caps 1, 5, 100 and 400 MB): one step each.
ONE_STEP = [(f"sweep_1p3b_{m}_w{w}_cap{c}", None) for m in ("flat", "whole") for w in (2, 8, 32, 64)
            for c in (1, 5, 100, 400)]


@pytest.mark.parametrize("name, rank, steps", [(n, r, 3) for n, r in THREE_STEP] +
                         [(n, r, 1) for n, r in ONE_STEP])
def test_full_size_sampled(name, rank, steps):
    wl = synth.WORKLOADS.get(name) or SWEEP.get(name) or LARGE[name]
    rank = wl.ranks[0] if rank is None else rank
    W = wl.world_size
    clip = wl.max_grad_norm > 0
    plan = ZrPlan(wl.shapes, W, rank, wl.mode, wl.bucket_cap_bytes, *wl.hp, device=DEV)
    n = plan.owned_numel
    runs = plan.runs()
    grads = [torch.empty(n, dtype=torch.bfloat16, device=DEV) for _ in range(W)]
    master = torch.empty(n, dtype=torch.float32, device=DEV)
    synth.fill_owned_master(master, runs, wl.seed, n_valid=plan.total_numel)
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    sentinel = -16447   # 0xBFC1 as int16: a value the step never writes by chance here
    param_out = torch.full((plan.padded_numel,), sentinel, dtype=torch.int16, device=DEV)
    g_gpu = torch.empty(n, dtype=torch.float32, device=DEV)

    oplan = oracle.Plan(wl.shapes, W, wl.mode, wl.bucket_cap_bytes)
    own = sample_owned(runs, n)
    glob = owned_to_global(runs, own)
    assert np.array_equal(glob, owned_to_global(sorted(oplan.runs(rank)), own))
    tg = torch.from_numpy(glob)
    own_t = torch.from_numpy(own).to(DEV)
    p_ref = synth.master_f32(wl.seed, tg, n_valid=oplan.total_numel).numpy().copy()
    m_ref = np.zeros_like(p_ref)
    v_ref = np.zeros_like(p_ref)

    for step in range(1, steps + 1):
        for w in range(W):
            synth.fill_owned_grad(grads[w], runs, wl.seed, step, w, wl.grad_sigma, wl.outlier_frac,
                                  n_valid=plan.total_numel)
        c = None
        if clip:
            # other ranks' S_w for this step on the GPU (zr_grad_sumsq on their own shards)
            parts_gpu = torch.zeros(W, dtype=torch.float64, device=DEV)
            for r in range(W):
                if r == rank:
                    continue
                pr = ZrPlan(wl.shapes, W, r, wl.mode, wl.bucket_cap_bytes, *wl.hp, device=DEV)
                rr = pr.runs()
                gr = [torch.empty(max(pr.owned_numel, 8), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
                for w in range(W):
                    synth.fill_owned_grad(gr[w], rr, wl.seed, step, w, wl.grad_sigma, wl.outlier_frac,
                                          n_valid=pr.total_numel)
                pr.grad_sumsq(gr, parts_gpu[r:r + 1])
                torch.cuda.synchronize()
                del gr
                pr.close()
                torch.cuda.empty_cache()
            plan.partials.copy_(parts_gpu)
            S, parts_host = host_global_sumsq(oplan, wl, step, threads=min(32, os.cpu_count() or 1))
            c = oracle.clip_coef(S, wl.max_grad_norm)

        plan.debug_reduce(grads, g_gpu)
        plan.step(grads, master, m, v, param_out.view(torch.bfloat16), step)
        torch.cuda.synchronize()

        if clip:
            got_parts = plan.partials.cpu().numpy()
            for r in range(W):
                assert abs(got_parts[r] - parts_host[r]) <= 1e-12 * parts_host[r], (step, r)

        # the oracle steps the sampled elements from their own host-generated gradients
        reps = [u16(synth.grad_bf16(wl.seed, step, w, tg, wl.grad_sigma, wl.outlier_frac,
                                    n_valid=oplan.total_numel)) for w in range(W)]
        g_ref = oracle.reduce(reps)
        assert np.array_equal(bits32(g_gpu[own_t]), bits32(g_ref)), f"reduced gradient, step {step}"
        if clip:
            oracle.scale(g_ref, c)
        oracle.adamw(wl.hp, step, g_ref, p_ref, m_ref, v_ref)

    assert_state_close(master[own_t].cpu().numpy(), p_ref, f"master after {steps} steps")
    assert_state_close(m[own_t].cpu().numpy(), m_ref, f"m after {steps} steps")
    assert_state_close(v[own_t].cpu().numpy(), v_ref, f"v after {steps} steps")
    out_ref = oracle.f32_to_bf16_array(p_ref)
    got = param_out[tg.to(DEV)].cpu().numpy().view(np.uint16)
    assert bf16_ulp_distance(got, out_ref).max() <= 1
    # positions this rank does not own stay untouched
    rng = np.random.default_rng(1)
    probe = rng.integers(0, plan.padded_numel, size=20000)
    mine = np.zeros(probe.size, dtype=bool)
    for owned, g0, length in runs:
        mine |= (probe >= g0) & (probe < g0 + length)
    vals = param_out[torch.from_numpy(probe[~mine]).to(DEV)].cpu().numpy()
    assert np.all(vals == sentinel)
    plan.close()
    del grads, master, m, v, param_out, g_gpu
    torch.cuda.empty_cache()
