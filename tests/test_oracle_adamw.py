"""Pins for the oracle's AdamW on the owned slice.

Pages: "CS336 lecture 8", ZeRO-1 code sketch (the slice's fp32 moments m1, m2
are updated and the slice's parameters step by lr * update) and the 16
bytes/param ledger (fp32 master, m, v); "DDP -> ZeRO" blog section 1.1 (AdamW
keeps fp32 master, m, v) and 3.3 (lr 3e-4).  The pages do not print the rule;
it is Adam with bias correction (Kingma & Ba 2015) and decoupled weight decay
(Loshchilov & Hutter 2019).  Pins: the constant-gradient closed form, the zero
gradient, and torch.optim.AdamW evaluated in fp64.
"""
import numpy as np
import pytest
import torch

import oracle

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)


def test_constant_gradient_closed_form():
    """With g fixed over steps, m_t / (1 - b1^t) = g and v_t / (1 - b2^t) = g^2
    in real arithmetic, so each step is p <- p (1 - lr wd) - lr g / (|g| + eps)."""
    rng = np.random.default_rng(0)
    n = 2000
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    g = (rng.standard_normal(n) * 10.0 ** rng.integers(-4, 1, n)).astype(np.float32)
    p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    lr, wd, eps = 3e-4, 0.1, 1e-8
    want = p0.astype(np.float64)
    gd = g.astype(np.float64)
    for t in (1, 2, 3):
        oracle.adamw(HP, t, g, p, m, v)
        want = want * (1.0 - lr * wd) - lr * gd / (np.abs(gd) + eps)
        err = np.abs(p.astype(np.float64) - want)
        assert np.all(err <= 1e-6 * np.maximum(np.abs(want), lr)), (t, err.max())


def test_zero_gradient_only_decays():
    rng = np.random.default_rng(1)
    p0 = (rng.standard_normal(100) * 0.02).astype(np.float32)
    p, m, v = p0.copy(), np.zeros(100, np.float32), np.zeros(100, np.float32)
    oracle.adamw(HP, 1, np.zeros(100, np.float32), p, m, v)
    assert np.all(m == 0) and np.all(v == 0)
    want = p0.astype(np.float64) * (1.0 - 3e-4 * 0.1)
    # two fp32 roundings: the decay factor and the product
    assert np.all(np.abs(p - want) <= 1.2e-7 * np.abs(want))


def test_step_direction_opposes_gradient():
    p = np.zeros(4, np.float32)
    m, v = np.zeros(4, np.float32), np.zeros(4, np.float32)
    oracle.adamw(HP, 1, np.array([1.0, -1.0, 1e-3, -1e-3], np.float32), p, m, v)
    assert p[0] < 0 < p[1] and p[2] < 0 < p[3]
    # first step of Adam is lr * sign(g) (|g| >> eps)
    assert np.allclose(np.abs(p), 3e-4, rtol=1e-5)


@pytest.mark.parametrize("hp", [HP, (1e-3, 0.8, 0.95, 1e-6, 0.01, 0.0), (5e-2, 0.5, 0.9, 1e-4, 0.0, 0.0)])
def test_against_torch_adamw_fp64(hp):
    """Library special case: torch.optim.AdamW in fp64 on the same fp32
    inputs, over 3 steps with fresh gradients."""
    lr, b1, b2, eps, wd, _ = hp
    rng = np.random.default_rng(2)
    n = 5000
    p0 = (rng.standard_normal(n) * 0.02).astype(np.float32)
    grads = [(rng.standard_normal(n) * 10.0 ** rng.integers(-5, 0, n)).astype(np.float32)
             for _ in range(3)]
    p, m, v = p0.copy(), np.zeros(n, np.float32), np.zeros(n, np.float32)
    tp = torch.nn.Parameter(torch.from_numpy(p0.astype(np.float64)))
    f32 = lambda x: float(np.float32(x))      # the oracle takes fp32 hyperparameters
    opt = torch.optim.AdamW([tp], lr=f32(lr), betas=(f32(b1), f32(b2)), eps=f32(eps),
                            weight_decay=f32(wd), foreach=False, fused=False)
    # sum of |terms| of m: the yardstick for rounding error under cancellation
    m_scale = np.zeros(n)
    for t, g in enumerate(grads, start=1):
        m_scale = f32(b1) * m_scale + (1 - f32(b1)) * np.abs(g.astype(np.float64))
        oracle.adamw(hp, t, g, p, m, v)
        tp.grad = torch.from_numpy(g.astype(np.float64))
        opt.step()
    st = opt.state[tp]
    ref_p = tp.detach().numpy()
    ref_m = st["exp_avg"].numpy()
    ref_v = st["exp_avg_sq"].numpy()
    scale = np.maximum(np.abs(ref_p), lr)
    assert np.all(np.abs(p - ref_p) <= 2e-6 * scale), np.max(np.abs(p - ref_p) / scale)
    assert np.all(np.abs(m - ref_m) <= 1e-6 * m_scale + 1e-30)
    assert np.all(np.abs(v - ref_v) <= 1e-6 * np.abs(ref_v) + 1e-30)


def test_scalars_follow_their_definitions():
    s = oracle.adamw_scalars(HP, 2)
    assert s["step_size"] == np.float32(3e-4 / (1 - 0.9 ** 2)) or \
        abs(s["step_size"] - 3e-4 / (1 - np.float64(np.float32(0.9)) ** 2)) < 1e-10
    assert abs(s["bc2_sqrt"] - np.sqrt(1 - np.float64(np.float32(0.999)) ** 2)) < 1e-7
    assert abs(s["decay"] - (1 - 3e-4 * 0.1)) < 1e-7


@pytest.mark.parametrize("t", [10 ** 6, 2 ** 33 + 5])
def test_bias_corrections_vanish_at_large_steps(t):
    """At these step numbers β1^t and β2^t (β2 = 0.999: below e^-999) are
    below the smallest fp64 subnormal, so both bias corrections are exactly
    1: step_size is fp32(lr) and sqrt(1 - β2^t) is 1.  The step number is a
    64-bit integer: 2**33 + 5 cut to 32 bits would be step 5, whose
    corrections are far from 1."""
    s = oracle.adamw_scalars(HP, t)
    assert s["step_size"] == np.float32(3e-4)
    assert s["bc2_sqrt"] == 1.0
    # the element step is then AdamW without bias correction
    g = np.array([1e-3, -2e-2, 0.0], np.float32)
    p = np.array([0.5, -0.25, 1.0], np.float32)
    m = np.array([2e-4, -1e-3, 0.0], np.float32)
    v = np.array([3e-7, 4e-4, 0.0], np.float32)
    p64, m64, v64 = p.astype(np.float64), m.astype(np.float64), v.astype(np.float64)
    b1, b2 = np.float64(np.float32(0.9)), np.float64(np.float32(0.999))
    m_new = b1 * m64 + (1 - b1) * g
    v_new = b2 * v64 + (1 - b2) * g.astype(np.float64) ** 2
    want = p64 * (1 - 3e-4 * 0.1) - 3e-4 * m_new / (np.sqrt(v_new) + 1e-8)
    oracle.adamw(HP, t, g, p, m, v)
    assert np.allclose(p, want, rtol=2e-6, atol=1e-9)
    assert np.allclose(m, m_new, rtol=2e-6, atol=1e-12) and np.allclose(v, v_new, rtol=2e-6, atol=1e-15)
