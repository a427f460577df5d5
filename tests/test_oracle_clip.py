"""Pins for the optional global gradient-norm clip.

The pages do not describe clipping; the workload with clip at 1.0 uses the
common global-norm convention: S = sum of squares of the averaged gradient
over all N parameters (all ranks), c = min(1, max_norm / (sqrt(S) + 1e-6)),
g <- g * c before the moments.  Pins: closed forms and
torch.nn.utils.clip_grad_norm_ in fp64.
"""
import math

import numpy as np
import torch

import oracle


def test_all_ones_closed_form():
    """Every replica 1.0 over N params: g = 1, S = N exactly,
    c = min(1, max_norm / (sqrt(N) + 1e-6))."""
    N, W = 4096, 4
    ones = np.full(N, 0x3F80, dtype=np.uint16)
    g = oracle.reduce([ones] * W)
    assert np.all(g == 1.0)
    S = oracle.sumsq(g)
    assert S == float(N)
    assert oracle.clip_coef(S, 1.0) == np.float32(1.0 / (math.sqrt(N) + 1e-6))
    assert oracle.clip_coef(S, 1e6) == 1.0


def test_norm_two_gives_half():
    g = np.array([2.0, 0.0, 0.0], np.float32)
    assert oracle.clip_coef(oracle.sumsq(g), 1.0) == np.float32(1.0 / (2.0 + 1e-6))


def test_small_norm_is_untouched():
    g = np.array([0.1, -0.2, 0.3], np.float32)
    c = oracle.clip_coef(oracle.sumsq(g), 1.0)
    assert c == 1.0
    h = g.copy()
    oracle.scale(h, 1.0)
    assert np.array_equal(h, g)


def test_against_torch_clip_grad_norm_fp64():
    rng = np.random.default_rng(5)
    g = (rng.standard_normal(100_000) * 0.01).astype(np.float32)
    S = oracle.sumsq(g)
    t = torch.nn.Parameter(torch.zeros(g.size, dtype=torch.float64))
    t.grad = torch.from_numpy(g.astype(np.float64))
    norm = torch.nn.utils.clip_grad_norm_([t], max_norm=1.0)
    assert abs(math.sqrt(S) - float(norm)) <= 1e-12 * float(norm)
    c = oracle.clip_coef(S, 1.0)
    ref_scaled = t.grad.numpy()
    ours = g.copy()
    oracle.scale(ours, c)
    assert np.all(np.abs(ours - ref_scaled) <= 1.2e-7 * np.abs(ref_scaled) + 1e-30)


def test_squares_are_exact_in_fp64():
    """sumsq of one element is the exact square (24-bit significand squared
    fits in 53 bits)."""
    x = np.float32(1.0 + 2.0 ** -23)
    assert oracle.sumsq(np.array([x], np.float32)) == (1.0 + 2.0 ** -23) ** 2


def test_sumsq_is_accurate_over_many_terms():
    """1 followed by 2**20 copies of 2**-27: the exact sum of squares is
    1 + 2**20 * 2**-54 = 1 + 2**-34.  A plain running sum drops every
    2**-54 against the 1 and returns 1.0; the oracle must not."""
    g = np.full(1 + (1 << 20), 2.0 ** -27, np.float32)
    g[0] = 1.0
    assert oracle.sumsq(g) == 1.0 + 2.0 ** -34
    # and a long random sum agrees with an exactly rounded reference
    import math
    rng = np.random.default_rng(13)
    h = (rng.standard_normal(200_000) * 10.0 ** rng.integers(-6, 3, 200_000)).astype(np.float32)
    exact = math.fsum(float(x) * float(x) for x in h.astype(np.float64))
    assert abs(oracle.sumsq(h) - exact) <= 4 * 2.0 ** -53 * exact


def test_rank_partials_sum_to_global():
    """Per-rank S_r (owned order) summed in rank order equal the global S
    (global order) within 1e-12 relative."""
    rng = np.random.default_rng(9)
    shapes = [(300, 7), (1001,), (64, 64)]
    for mode in (oracle.FLAT, oracle.WHOLE_TENSOR):
        plan = oracle.Plan(shapes, 4, mode, 4096)
        g_glob = (rng.standard_normal(plan.padded_numel) * 0.01).astype(np.float32)
        g_glob[plan.total_numel:] = 0
        S = oracle.sumsq(g_glob[: plan.total_numel])
        parts = 0.0
        for r in range(4):
            parts += oracle.sumsq(g_glob[plan.owned_global_index(r)])
        assert abs(parts - S) <= 1e-12 * S
