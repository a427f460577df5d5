"""Owner-major layout used by the peer-memory step (host logic, CPU): rank r's
owned elements sit at [offsets[r], offsets[r+1]) of every replica's full
gradient buffer, and every tensor is one contiguous piece of it."""
import numpy as np
import pytest

import oracle
import synth
import sharded_optimizer_step_zr_b200 as zr


@pytest.mark.parametrize("shapes, W, mode", [
    (synth.gpt2_small_shapes(), 8, 0), (synth.gpt_1p3b_shapes(), 8, 1),
    ([(3, 5), (7,), (2, 2, 2)], 4, 0), ([(10,), (4, 5), (7,), (3, 3), (20,)], 3, 1),
])
def test_owner_offsets(shapes, W, mode):
    op = oracle.Plan(shapes, W, mode, 1 << 20)
    h = zr.zr_plan_create(shapes, W, 0, mode, 1 << 20)
    try:
        off = zr.zr_plan_owner_offsets(h, W)
        segs = zr.zr_plan_segments(h)
    finally:
        zr.zr_plan_destroy(h)
    rounded = [(int(n) + 7) // 8 * 8 for n in op.owned_numel]
    assert off == [0] + list(np.cumsum(rounded))
    assert all(o % 8 == 0 for o in off)
    if mode == 0 and op.chunk % 8 == 0:
        assert off == [r * op.chunk for r in range(W + 1)]      # the global layout itself
    if mode == 0 and op.chunk % 8:
        return
    # every tensor is contiguous in the owner-major layout
    for t in range(len(shapes)):
        pieces = sorted((s["offset_in_tensor"], off[s["owner"]] + s["owned_offset"], s["length"])
                        for s in segs if s["tensor"] == t)
        for (o1, p1, l1), (o2, p2, _) in zip(pieces, pieces[1:]):
            assert o2 == o1 + l1 and p2 == p1 + l1
