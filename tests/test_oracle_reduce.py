"""Pins for the oracle's reduce: the local stand-in for the gradient
reduce-scatter.

Pages: "CS336 lecture 8", ZeRO-1 code sketch (reduce-scatter with SUM, each
rank keeps its slice); "Scaling training to thousands of GPUs", 03:41 DP
(replicas' gradients are summed and averaged) and 11:24 ZeRO (AllReduce =
reduce-scatter + all-gather).  Reading: fp32 left fold in rank order starting
from replica 0, then one IEEE division by W.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from fp_exact import bf16_bits_to_fraction, round_to_f32


def bf16(x) -> np.ndarray:
    """bf16 bit patterns of exactly representable values."""
    a = np.asarray(x, dtype=np.float32)
    bits = a.view(np.uint32)
    assert np.all((bits & 0xFFFF) == 0), "value not representable in bf16"
    return (bits >> 16).astype(np.uint16)


def exact_fold(replica_bits, W):
    """Left fold with one correctly rounded fp32 addition per step, then a
    correctly rounded division, all in exact rational arithmetic."""
    s = bf16_bits_to_fraction(int(replica_bits[0]))
    for w in range(1, W):
        s = Fraction(float(round_to_f32(s + bf16_bits_to_fraction(int(replica_bits[w])))))
    s = Fraction(float(round_to_f32(s)))
    return round_to_f32(s / W)


def test_single_replica_is_identity():
    rng = np.random.default_rng(0)
    g = oracle.f32_to_bf16_array(rng.standard_normal(1000).astype(np.float32))
    assert np.array_equal(oracle.reduce([g]).view(np.uint32),
                          oracle.bf16_bits_to_f32(g).view(np.uint32))


def test_two_replicas_equal_correctly_rounded_sum_over_two():
    """bf16 + bf16 is exact in fp64, so one fp32 rounding of that sum is the
    fp32 addition; W = 2 then halves it exactly (normal range)."""
    rng = np.random.default_rng(1)
    a = oracle.f32_to_bf16_array((rng.standard_normal(5000) * 10.0 ** rng.integers(-8, 8, 5000)).astype(np.float32))
    b = oracle.f32_to_bf16_array((rng.standard_normal(5000) * 10.0 ** rng.integers(-8, 8, 5000)).astype(np.float32))
    exact = oracle.bf16_bits_to_f32(a).astype(np.float64) + oracle.bf16_bits_to_f32(b).astype(np.float64)
    want = exact.astype(np.float32) / np.float32(2)
    assert np.array_equal(oracle.reduce([a, b]).view(np.uint32), want.view(np.uint32))


def test_no_replica_dropped_powers_of_two():
    """Replica w holds 2**w: the sum is 2**W - 1 exactly, so any dropped or
    repeated replica changes the result."""
    for W in (2, 3, 5, 8, 16):
        grads = [bf16([2.0 ** w] * 4) for w in range(W)]
        want = np.float32((2.0 ** W - 1) / W)
        assert np.all(oracle.reduce(grads) == want), W


def test_left_fold_order_is_rank_order():
    """1 + 2^-24 is a tie that rounds back to 1 (even), so the left fold
    1, 2^-24, 2^-24 stays 1 while any other order gives 1 + 2^-23."""
    grads = [bf16([1.0]), bf16([2.0 ** -24]), bf16([2.0 ** -24])]
    assert oracle.reduce(grads)[0] == np.float32(1.0) / np.float32(3.0)
    grads = [bf16([2.0 ** -24]), bf16([2.0 ** -24]), bf16([1.0])]
    assert oracle.reduce(grads)[0] == np.float32(1.0 + 2.0 ** -23) / np.float32(3.0)


def test_sign_of_zero_follows_replica_zero():
    """The fold starts at g_0 (not at +0): all -0 replicas give -0."""
    g = oracle.reduce([bf16([-0.0]), bf16([-0.0]), bf16([-0.0])])
    assert np.signbit(g[0]) and g[0] == 0


def test_non_power_of_two_division_is_ieee():
    """W = 3, 5, 7: the division by W is one correctly rounded fp32 division."""
    for W in (3, 5, 7):
        grads = [bf16([1.0, 3.0, -2.5])] + [bf16([0.0, 0.0, 0.0])] * (W - 1)
        got = oracle.reduce(grads)
        for j, x in enumerate([1.0, 3.0, -2.5]):
            assert got[j] == round_to_f32(Fraction(x) / W)


@pytest.mark.parametrize("W", [2, 3, 4, 7, 8, 13, 32, 64])
def test_brute_force_exact_arithmetic(W):
    """Tiny inputs, every W: the fold equals the same sequence of roundings
    carried out in exact rational arithmetic."""
    rng = np.random.default_rng(100 + W)
    n = 24
    mags = 10.0 ** rng.integers(-30, 30, size=(W, n))
    vals = (rng.standard_normal((W, n)) * mags).astype(np.float32)
    vals[:, :2] = 0.0
    vals[0, 2] = -0.0
    grads = [oracle.f32_to_bf16_array(vals[w]) for w in range(W)]
    got = oracle.reduce(grads)
    for i in range(n):
        want = exact_fold([grads[w][i] for w in range(W)], W)
        assert got[i] == want or (got[i] == 0 and want == 0), (i, got[i], want)


def test_reduce_scatter_then_gather_equals_all_reduce():
    """Per-rank folds over the owned chunks, concatenated in global order, are
    bit-identical to the fold over the full replica buffers."""
    rng = np.random.default_rng(3)
    W, shapes = 4, [(33, 7), (129,), (5, 5, 5), (64,)]
    plan = oracle.Plan(shapes, W, oracle.FLAT, 256)
    full = [oracle.f32_to_bf16_array(rng.standard_normal(plan.padded_numel).astype(np.float32))
            for _ in range(W)]
    for w in range(W):
        full[w][plan.total_numel:] = 0
    all_reduce = oracle.reduce(full)
    gathered = np.empty(plan.padded_numel, dtype=np.float32)
    for r in range(W):
        idx = plan.owned_global_index(r)
        gathered[idx] = oracle.reduce([f[idx] for f in full])
    assert np.array_equal(gathered.view(np.uint32), all_reduce.view(np.uint32))
