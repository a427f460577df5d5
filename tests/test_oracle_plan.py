"""Pins for the oracle's partition / bucket / segment planner.

Pages: "Scaling training to thousands of GPUs", 11:24 ZeRO (flatten then shard
into W equal pieces, FSDP1; whole tensors for Muon / FSDP2) and 03:41 DP
(bucket_cap_mb buckets launched as backward produces them); "DDP -> ZeRO" blog
section 2.1 (25 MB default bucket); "CS336 lecture 8" ZeRO-1 sketch (each rank
owns params[my_slice]).
"""
import itertools

import numpy as np
import pytest

import oracle
import synth
from golden_plans import all_golden_plans

FIELDS = ("bucket", "tensor", "owner", "offset_in_tensor", "length", "global_offset",
          "owned_offset")


def seg_tuples(plan):
    return [tuple(int(s[f]) for f in FIELDS) for s in plan.segments]


@pytest.mark.parametrize("g", all_golden_plans(), ids=lambda g: g["name"])
def test_hand_derived_tables(g):
    plan = oracle.Plan(g["shapes"], g["world_size"], g["mode"], g["cap_bytes"], groups=g["groups"])
    assert (plan.total_numel, plan.padded_numel, plan.chunk, plan.n_buckets) == \
        (g["N"], g["padded"], g["C"], g["n_buckets"])
    assert seg_tuples(plan) == g["segments"]
    if g["owned_numel"] is not None:
        assert plan.owned_numel.tolist() == g["owned_numel"]


def check_invariants(plan):
    shapes, W = plan.shapes, plan.world_size
    numels = [synth.numel(s) for s in shapes]
    N = sum(numels)
    goff = np.concatenate([[0], np.cumsum(numels)]).astype(np.int64)
    assert plan.total_numel == N
    segs = plan.segments
    def tiles_exactly(intervals, end):
        """Intervals (start, length) cover [0, end) exactly once."""
        at = 0
        for start, length in sorted(intervals):
            assert length > 0 and start == at, (start, at)
            at = start + length
        assert at == end

    # exact cover of [0, padded): every element in exactly one segment
    tiles_exactly([(int(s["global_offset"]), int(s["length"])) for s in segs], plan.padded_numel)
    # per rank: owned offsets tile [0, owned_numel) exactly
    for r in range(W):
        tiles_exactly([(int(s["owned_offset"]), int(s["length"])) for s in segs[segs["owner"] == r]],
                      int(plan.owned_numel[r]))
    assert plan.owned_numel.sum() == plan.padded_numel
    # tensor pieces concatenate back to [0, numel) and sit at the declared offset
    for t, n in enumerate(numels):
        pieces = sorted((int(s["offset_in_tensor"]), int(s["length"]), int(s["global_offset"]))
                        for s in segs if s["tensor"] == t)
        pos = 0
        for off, ln, go in pieces:
            assert off == pos and go == goff[t] + off
            pos += ln
        assert pos == n
        assert len({int(s["bucket"]) for s in segs if s["tensor"] == t}) <= 1
    # buckets: reverse declaration order, cap respected unless a single tensor
    if len(numels) and plan.groups is not None:
        # one bucket per group, the last group first
        bt = plan.tensor_bucket
        distinct = sorted(set(plan.groups), reverse=True)
        assert plan.n_buckets == len(distinct)
        assert [distinct.index(g) for g in plan.groups] == bt.tolist()
    elif len(numels):
        bt = plan.tensor_bucket
        assert bt[-1] == 0 and all(bt[i] >= bt[i + 1] for i in range(len(bt) - 1))
        for b in range(plan.n_buckets):
            members = [t for t in range(len(numels)) if bt[t] == b]
            assert members, "empty bucket"
            nbytes = sum(2 * numels[t] for t in members)
            assert nbytes <= plan.bucket_cap_bytes or len(members) == 1
            # the next tensor in backward order would not have fit
            if b + 1 < plan.n_buckets:
                nxt = max(t for t in range(len(numels)) if bt[t] == b + 1)
                assert nbytes + 2 * numels[nxt] > plan.bucket_cap_bytes
    # segment order: bucket, then backward tensor order, then offset (pad last)
    keys = [(int(s["bucket"]), -(int(s["tensor"]) if s["tensor"] >= 0 else -10**9),
             int(s["offset_in_tensor"])) for s in segs]
    assert keys == sorted(keys)
    if plan.mode == oracle.FLAT:
        C = plan.chunk
        assert C == -(-N // W) and plan.padded_numel == W * C
        assert plan.padded_numel - N < max(W, 1)
        for s in segs:
            owner, goff_s, length = int(s["owner"]), int(s["global_offset"]), int(s["length"])
            assert owner == goff_s // C
            assert int(s["owned_offset"]) == goff_s - owner * C
            assert (goff_s + length - 1) // C == owner
            if s["tensor"] == -1:
                assert s["bucket"] == 0 and goff_s >= N
    else:
        assert plan.padded_numel == N
        for t in range(len(numels)):
            owners = {int(s["owner"]) for s in segs if s["tensor"] == t}
            assert len(owners) <= 1


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_workload_plans_invariants(name):
    wl = synth.WORKLOADS[name]
    plan = oracle.Plan(wl.shapes, wl.world_size, wl.mode, wl.bucket_cap_bytes)
    check_invariants(plan)


def test_random_plans_invariants():
    rng = np.random.default_rng(4)
    for trial in range(300):
        nt = int(rng.integers(0, 9))
        shapes = [tuple(int(x) for x in rng.integers(0, 40, size=int(rng.integers(0, 3))))
                  for _ in range(nt)]
        W = int(rng.integers(1, 9))
        mode = int(rng.integers(0, 2))
        cap = int(rng.integers(1, 400))
        plan = oracle.Plan(shapes, W, mode, cap)
        check_invariants(plan)


def test_random_grouped_plans_invariants():
    """Buckets given by tensor groups: one bucket per group, in reverse
    order; owners, global and owned offsets are those of the same set
    under the cap rule (buckets change only bucket ids and segment order)."""
    rng = np.random.default_rng(12)
    for trial in range(300):
        nt = int(rng.integers(0, 10))
        shapes = [tuple(int(x) for x in rng.integers(0, 40, size=int(rng.integers(0, 3))))
                  for _ in range(nt)]
        groups = np.cumsum(rng.integers(0, 2, size=nt)).tolist()
        W = int(rng.integers(1, 9))
        mode = int(rng.integers(0, 2))
        plan = oracle.Plan(shapes, W, mode, 0, groups=groups)
        check_invariants(plan)
        ref = oracle.Plan(shapes, W, mode, 1 << 20)
        key = lambda seg: (int(seg["tensor"]), int(seg["offset_in_tensor"]))
        rest = lambda segs: sorted((key(x), int(x["owner"]), int(x["length"]), int(x["global_offset"]),
                                    int(x["owned_offset"])) for x in segs)
        assert rest(plan.segments) == rest(ref.segments)
        assert plan.owned_numel.tolist() == ref.owned_numel.tolist()


def test_grouped_plans_reject_decreasing_groups():
    with pytest.raises(ValueError):
        oracle.Plan([(4,), (5,), (6,)], 2, oracle.FLAT, 0, groups=[0, 1, 0])
    # one group: a single bucket holding everything (and the flat pad)
    plan = oracle.Plan([(4,), (5,), (6,)], 2, oracle.FLAT, 0, groups=[3, 3, 3])
    assert plan.n_buckets == 1 and set(plan.segments["bucket"].tolist()) == {0}


def test_parameter_counts_of_the_sets():
    """The sets are shaped like the workloads: GPT-2 small has 124,439,808
    parameters in 148 tensors; Llama-7B has 6,738,415,616 (about 6.7B), and
    its W = 64 flat shard is 105,287,744 (about 105M)."""
    counts = {k: (len(f()), sum(synth.numel(s) for s in f())) for k, f in synth.PARAM_SETS.items()}
    assert counts["gpt2_124m"] == (148, 124_439_808)
    assert counts["gpt_1p3b"] == (292, 1_315_819_520)
    assert counts["llama_7b"] == (291, 6_738_415_616)
    assert counts["tiny"] == (4, 1_441_792)
    plan = oracle.Plan(synth.llama_7b_shapes(), 64, oracle.FLAT, 25 << 20)
    assert plan.chunk == 105_287_744 and plan.padded_numel == plan.total_numel
    plan = oracle.Plan(synth.gpt2_small_shapes(), 8, oracle.FLAT, 25 << 20)
    assert plan.chunk == 15_554_976


def brute_force_makespan(numels, W):
    best = None
    for assign in itertools.product(range(W), repeat=len(numels)):
        loads = [0] * W
        for n, r in zip(numels, assign):
            loads[r] += n
        best = max(loads) if best is None else min(best, max(loads))
    return best


def test_lpt_within_grahams_bound_of_optimal():
    """Graham (1969): LPT's makespan <= (4/3 - 1/(3W)) * optimal."""
    rng = np.random.default_rng(6)
    for trial in range(150):
        nt = int(rng.integers(1, 9))
        W = int(rng.integers(1, 4))
        numels = [int(x) for x in rng.integers(1, 100, size=nt)]
        plan = oracle.Plan([(n,) for n in numels], W, oracle.WHOLE_TENSOR, 1 << 30)
        opt = brute_force_makespan(numels, W)
        assert plan.owned_numel.max() * 3 * W <= (4 * W - 1) * opt
        assert plan.owned_numel.max() >= opt


def test_lpt_loads_do_not_depend_on_declaration_order():
    """With distinct sizes, the multiset of rank loads is a function of the
    sizes alone."""
    rng = np.random.default_rng(8)
    numels = [int(x) for x in rng.choice(np.arange(1, 10_000), size=12, replace=False)]
    ref = sorted(oracle.Plan([(n,) for n in numels], 5, oracle.WHOLE_TENSOR, 1 << 30).owned_numel)
    for _ in range(5):
        perm = rng.permutation(numels)
        got = sorted(oracle.Plan([(int(n),) for n in perm], 5, oracle.WHOLE_TENSOR, 1 << 30).owned_numel)
        assert got == ref


def test_bad_arguments_rejected():
    with pytest.raises(ValueError):
        oracle.Plan([(4,)], 0, oracle.FLAT, 16)
    with pytest.raises(ValueError):
        oracle.Plan([(4,)], 2, 7, 16)
    with pytest.raises(ValueError):
        oracle.Plan([(-1, 4)], 2, oracle.FLAT, 16)
