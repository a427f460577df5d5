"""The gradient slots of Zero3(reduce_in_backward=True), on the host: for
random module stacks, both partitions and several world sizes, every
element a rank's fused step reads for a unit -- replica slot + the rank's
offset + the element's owned offset, segment by segment, the flat pad
included -- lies inside the slot's used part and is the element where that
tensor position's gradient is placed; every rank's offset keeps 16-byte
alignment; tensors do not overlap; and each unit is one bucket.  With a
flat chunk that is a multiple of 8 (or one rank) every tensor is one view
of the slot."""
import numpy as np
import pytest

import synth
from sharded_optimizer_step_zr_b200 import ZR_PARTITION_FLAT, ZR_PARTITION_WHOLE_TENSOR
from sharded_optimizer_step_zr_b200.optim import contiguous_in_slot, unit_grad_layout
from sharded_optimizer_step_zr_b200.plan import ZrPlan


def check_stack(shapes, unit_sizes, W, mode):
    groups = [u for u, k in enumerate(unit_sizes) for _ in range(k)]
    numels = [synth.numel(s) for s in shapes]
    n_views = n_split = 0
    for rank in range(W):
        plan = ZrPlan(shapes, W, rank, mode, 0, bind=False, groups=groups)
        segs = plan.segments()
        chunk = plan.padded_numel // W if mode == ZR_PARTITION_FLAT else 0
        assert plan.n_buckets == len(unit_sizes)
        a = 0
        for u, k in enumerate(unit_sizes):
            last = a + k == len(shapes)
            pieces, ptr_off, used = unit_grad_layout(segs, a, k, last, W)
            mine = [s for s in segs if (a <= s["tensor"] < a + k) or (s["tensor"] == -1 and last)]
            assert len({s["bucket"] for s in mine}) <= 1
            assert ptr_off[rank] % 8 == 0
            where = {}
            for t in range(a, a + k):
                for off, pos, n in pieces[t]:
                    where[(t, off)] = (pos, n)
            for s in mine:
                if s["owner"] != rank:
                    continue
                lo = ptr_off[rank] + s["owned_offset"]
                assert 0 <= lo and lo + s["length"] <= used
                if s["tensor"] >= 0:
                    assert where[(s["tensor"], s["offset_in_tensor"])] == (lo, s["length"])
            spans = sorted((pos, pos + n) for t in range(a, a + k) for _, pos, n in pieces[t])
            assert all(x[1] <= y[0] for x, y in zip(spans, spans[1:]))
            for t in range(a, a + k):
                assert sum(n for _, _, n in pieces[t]) == numels[t]
                at = contiguous_in_slot(pieces[t])
                n_views += at is not None
                n_split += at is None
                if mode == ZR_PARTITION_WHOLE_TENSOR or W == 1 or chunk % 8 == 0:
                    assert at is not None
            a += k
        plan.close()
    return n_views, n_split


@pytest.mark.parametrize("mode", [ZR_PARTITION_FLAT, ZR_PARTITION_WHOLE_TENSOR])
def test_unit_gradient_slots_cover_each_ranks_reads(mode):
    rng = np.random.default_rng(31)
    views = split = 0
    for _ in range(120):
        n_units = int(rng.integers(1, 6))
        unit_sizes = [int(rng.integers(1, 4)) for _ in range(n_units)]
        shapes = [tuple(int(x) for x in rng.integers(0, 50, size=int(rng.integers(1, 3))))
                  for _ in range(sum(unit_sizes))]
        for W in (1, 2, 3, 4):
            v, sp = check_stack(shapes, unit_sizes, W, mode)
            views, split = views + v, split + sp
    assert views > 1000
    assert (split > 0) == (mode == ZR_PARTITION_FLAT)     # flat chunks not a multiple of 8 occur


def test_gpt2_blocks_as_units():
    shapes = synth.gpt2_small_shapes()
    unit_sizes = [2] + [12] * 12 + [2]
    for mode in (ZR_PARTITION_FLAT, ZR_PARTITION_WHOLE_TENSOR):
        views, split = check_stack(shapes, unit_sizes, 8, mode)
        assert split == 0
