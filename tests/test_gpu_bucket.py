"""Bucket-by-bucket stepping (zr_step_bucket / zr_step_finish).

"Scaling training to thousands of GPUs", 03:41 DP: a bucket's collective is
launched as soon as backward has produced its gradients; "CS336 lecture 8",
ZeRO level 2: a gradient is released as soon as it is reduced.  Calling the
per-bucket entry once per bucket, in any order (then zr_step_finish when
clipping), must give zr_step's result bit for bit, and zr_step's result is
checked against the oracle elsewhere; here it is also checked directly.
With clipping and W > 4, each bucket's gradients are overwritten right after
its call (released), and the finish must not read them.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from gpu_harness import DEV, GpuRank, OracleRank, assert_state_close, bf16_ulp_distance, bits32, u16

pytestmark = pytest.mark.gpu


def bucket_owned_ranges(plan, bucket):
    return [(s["owned_offset"], s["length"]) for s in plan.segments()
            if s["owner"] == plan.rank and s["bucket"] == bucket]


GPT2_BLOCKS = [0, 0] + [1 + i // 12 for i in range(24)]      # the first 26 tensors: embeddings, 2 blocks


@pytest.mark.parametrize("shapes, W, rank, mode, cap, max_norm, groups", [
    (synth.gpt2_small_shapes()[:26], 8, 0, 0, 1 << 20, 0.0, None),          # flat, many buckets
    ([(4096 * 3 + 5,), (17,), (1,), (300, 7)], 3, 1, 0, 9000, 0.0, None),    # ragged tiles, pad
    ([(1000, 3), (8191,), (9, 9), (2048,)], 4, 2, 1, 4096, 0.0, None),       # whole-tensor
    ([(3000, 7), (5001,), (64, 64), (129,)], 8, 3, 0, 8192, 0.05, None),    # clip, W > 4 (scratch)
    ([(3000, 7), (5001,), (64, 64), (129,)], 8, 5, 1, 8192, 0.05, None),    # clip, whole-tensor
    ([(3000, 7), (5001,), (64, 64), (129,)], 3, 1, 0, 8192, 0.05, None),    # clip, W <= 4 (re-read)
    # buckets by tensor group (one per GPT-2 block): the per-layer reduce of ZeRO-3
    (synth.gpt2_small_shapes()[:26], 8, 3, 0, 0, 0.0, GPT2_BLOCKS),
    (synth.gpt2_small_shapes()[:26], 3, 1, 1, 0, 0.05, GPT2_BLOCKS),
])
def test_buckets_equal_full_step(shapes, W, rank, mode, cap, max_norm, groups):
    hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, max_norm)
    full = GpuRank(shapes, W, rank, mode, cap, hp, seed=21, groups=groups)
    byb = GpuRank(shapes, W, rank, mode, cap, hp, seed=21, groups=groups)
    oplan = oracle.Plan(shapes, W, mode, cap, groups=groups)
    if groups is not None:
        assert byb.plan.n_buckets == len(set(groups))
    orc = OracleRank(oplan, rank, seed=21)
    P = oplan.padded_numel
    out_full = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_byb = torch.zeros(P, dtype=torch.bfloat16, device=DEV)
    out_orc = np.zeros(P, dtype=np.uint16)
    others = torch.tensor([0.125 * (w + 1) for w in range(W)], dtype=torch.float64, device=DEV)
    rng = np.random.default_rng(rank)
    nb = byb.plan.n_buckets
    for t in (1, 2, 3):
        full.fill_grads(t, 1e-2, 0.01)
        byb.fill_grads(t, 1e-2, 0.01)
        orc.make_grads(t, 1e-2, 0.01)
        if max_norm > 0:
            full.plan.partials.copy_(others)
            byb.plan.partials.copy_(others)
        full.step(out_full, t)
        # with clipping and W > 4 (or a grouped plan) pass 1 keeps the fp32
        # averaged gradient, so each bucket's gradients may go right away
        release = max_norm > 0 and (W > 4 or groups is not None)
        if max_norm > 0:
            want_sumsq = torch.zeros(1, dtype=torch.float64, device=DEV)
            byb.plan.grad_sumsq(byb.grads, want_sumsq)
        for b in rng.permutation(nb):
            byb.plan.step_bucket(int(b), byb.grads, byb.master, byb.m, byb.v, out_byb, t)
            if release:
                # the bucket's gradients are released: overwrite them
                for owned, length in bucket_owned_ranges(byb.plan, int(b)):
                    for g in byb.grads:
                        g[owned: owned + length] = float("nan")
        if max_norm > 0:
            # this rank's S_r from the per-bucket pass, without the gradients
            got_sumsq = torch.zeros(1, dtype=torch.float64, device=DEV)
            byb.plan.bucket_sumsq(got_sumsq)
            torch.cuda.synchronize()
            assert got_sumsq.item() == want_sumsq.item()
        byb.plan.step_finish(None if release else byb.grads, byb.master, byb.m, byb.v, out_byb, t)
        c = None
        if max_norm > 0:
            S = 0.0
            for w in range(W):
                S += oracle.sumsq(oracle.reduce(orc.grads)) if w == rank else float(others[w])
            c = oracle.clip_coef(S, max_norm)
        orc.step(out_orc, hp, t, clip=c)
        torch.cuda.synchronize()
        for a, b_, what in zip(full.state(), byb.state(), ("master", "m", "v")):
            assert np.array_equal(bits32(a), bits32(b_)), f"{what} step {t}"
        assert torch.equal(out_full.view(torch.int16), out_byb.view(torch.int16))
        if max_norm > 0:
            assert byb.plan.partials[rank].item() == full.plan.partials[rank].item()
        for got, want, what in zip(byb.state(), (orc.master, orc.m, orc.v), ("master", "m", "v")):
            assert_state_close(got, want, f"{what} vs oracle step {t}")
        assert bf16_ulp_distance(u16(out_byb), out_orc).max() <= 1


def test_bucket_argument_checks():
    import sharded_optimizer_step_zr_b200 as zr
    gr = GpuRank([(4096,), (100,)], 2, 0, 0, 1024, (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0), seed=1)
    out = torch.zeros(4196 + 8, dtype=torch.bfloat16, device=DEV)
    for bad in (-1, gr.plan.n_buckets):
        with pytest.raises(zr.ZrError) as e:
            gr.plan.step_bucket(bad, gr.grads, gr.master, gr.m, gr.v, out, 1)
        assert e.value.status == zr.ZR_ERR_INVALID_ARG
    # finish on a plan without clipping does nothing
    gr.plan.step_finish(None, gr.master, gr.m, gr.v, out, 1)
