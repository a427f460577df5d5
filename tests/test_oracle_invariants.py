"""Invariants the pages fix, checked on the oracle.

* "CS336 lecture 8", ZeRO-1 sketch and its notes: updating each rank's slice
  and then all-gathering gives the same model as updating everything
  (each rank needs only its own slice's gradient and moments), so the
  concatenation of all W ranks' sharded updates equals the unsharded
  data-parallel AdamW step on the averaged gradient -- bit for bit.
* "Scaling training to thousands of GPUs", 11:24 ZeRO: flatten, pad and shard;
  unpad(pad(x)) must give x back exactly.
"""
import numpy as np
import pytest

import oracle
import synth

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)


def full_replicas(plan, seed, step, W, sigma, outlier):
    idx = np.arange(plan.padded_numel, dtype=np.int64)
    import torch
    t = torch.from_numpy(idx)
    return [synth.grad_bf16(seed, step, w, t, sigma, outlier, n_valid=plan.total_numel)
            .view(torch.int16).numpy().view(np.uint16).copy() for w in range(W)]


def initial_master(plan, seed):
    import torch
    idx = torch.arange(plan.padded_numel, dtype=torch.int64)
    return synth.master_f32(seed, idx, n_valid=plan.total_numel).numpy().copy()


@pytest.mark.parametrize("shapes, W, mode, cap, clip", [
    (synth.tiny_shapes(), 2, oracle.FLAT, 1 << 20, None),
    ([(3, 5), (7,), (2, 2, 2)], 4, oracle.FLAT, 16, None),
    ([(33, 7), (129,), (5, 5, 5), (64,), (1,)], 3, oracle.FLAT, 300, 0.05),
    ([(10,), (4, 5), (7,), (3, 3), (20,)], 3, oracle.WHOLE_TENSOR, 40, None),
    ([(300, 7), (1001,), (64, 64), (17,)], 5, oracle.WHOLE_TENSOR, 2048, 0.05),
])
def test_sharded_equals_unsharded_bitwise(shapes, W, mode, cap, clip):
    plan = oracle.Plan(shapes, W, mode, cap)
    P = plan.padded_numel
    seed = 77
    # unsharded comparator: every element, full replica buffers
    master_d = initial_master(plan, seed)
    m_d, v_d = np.zeros(P, np.float32), np.zeros(P, np.float32)
    out_d = np.zeros(P, np.uint16)
    # sharded: per-rank fp32 state in owned order
    idx = [plan.owned_global_index(r) for r in range(W)]
    master_s = [master_d[i].copy() for i in idx]
    m_s = [np.zeros(i.size, np.float32) for i in idx]
    v_s = [np.zeros(i.size, np.float32) for i in idx]
    out_s = np.full(P, 0xFFFF, np.uint16)
    for t in (1, 2, 3):
        full = full_replicas(plan, seed, t, W, 1e-2, 0.01)
        c = None
        if clip is not None:
            g_all = oracle.reduce([f[: plan.total_numel] for f in full])
            c = oracle.clip_coef(oracle.sumsq(g_all), clip)
        oracle.ddp_step(full, master_d, m_d, v_d, out_d, HP, t, clip=c)
        for r in range(W):
            oracle.rank_step(plan, r, [f[idx[r]] for f in full], master_s[r], m_s[r], v_s[r],
                             out_s, HP, t, clip=c)
    for r in range(W):
        assert np.array_equal(master_s[r].view(np.uint32), master_d[idx[r]].view(np.uint32))
        assert np.array_equal(m_s[r].view(np.uint32), m_d[idx[r]].view(np.uint32))
        assert np.array_equal(v_s[r].view(np.uint32), v_d[idx[r]].view(np.uint32))
    assert np.array_equal(out_s, out_d)
    # the flat zero pad stays zero through every step
    assert np.all(out_d[plan.total_numel:] == 0)
    assert np.all(master_d[plan.total_numel:] == 0)


def test_pad_unpad_round_trip():
    rng = np.random.default_rng(12)
    for _ in range(50):
        shapes = [tuple(int(x) for x in rng.integers(0, 9, size=int(rng.integers(0, 3))))
                  for _ in range(int(rng.integers(0, 6)))]
        W = int(rng.integers(1, 7))
        plan = oracle.Plan(shapes, W, oracle.FLAT, 64)
        tensors = [rng.integers(0, 1 << 16, size=synth.numel(s), dtype=np.uint64).astype(np.uint16)
                   for s in shapes]
        flat = oracle.pad(tensors, plan.padded_numel)
        assert flat.size == plan.padded_numel
        assert np.all(flat[plan.total_numel:] == 0)
        back = oracle.unpad(flat, [t.size for t in tensors])
        for a, b in zip(tensors, back):
            assert np.array_equal(a, b)
        # pad(unpad(y)) == y when y's pad is zero
        y = rng.integers(0, 1 << 16, size=plan.padded_numel, dtype=np.uint64).astype(np.uint16)
        y[plan.total_numel:] = 0
        assert np.array_equal(oracle.pad(oracle.unpad(y, [t.size for t in tensors]),
                                         plan.padded_numel), y)
