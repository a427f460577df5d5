"""Shared set-up for the GPU parity tests: the same seeded inputs on the GPU
(for libzr.so) and on the host (for the oracle)."""
import numpy as np
import torch

import oracle
import synth
from sharded_optimizer_step_zr_b200.plan import ZrPlan

DEV = "cuda:0"


def u16(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 bit patterns (host copy)."""
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16).copy()


def bits32(a) -> np.ndarray:
    if isinstance(a, torch.Tensor):
        a = a.detach().cpu().numpy()
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


class GpuRank:
    """One rank's plan and device buffers."""

    def __init__(self, shapes, W, rank, mode, cap, hp, seed, max_grad_norm=None, groups=None):
        lr, b1, b2, eps, wd, mgn = hp
        if max_grad_norm is not None:
            mgn = max_grad_norm
        self.plan = ZrPlan(shapes, W, rank, mode, cap, lr, b1, b2, eps, wd, mgn, device=DEV, groups=groups)
        self.W, self.rank, self.seed = W, rank, seed
        n = self.plan.owned_numel
        self.runs = self.plan.runs()
        self.grads = [torch.empty(max(n, 8), dtype=torch.bfloat16, device=DEV) for _ in range(W)]
        self.master = torch.empty(max(n, 8), dtype=torch.float32, device=DEV)
        synth.fill_owned_master(self.master, self.runs, seed, n_valid=self.plan.total_numel)
        self.m = torch.zeros_like(self.master)
        self.v = torch.zeros_like(self.master)

    def fill_grads(self, step, sigma, outlier):
        for w in range(self.W):
            synth.fill_owned_grad(self.grads[w], self.runs, self.seed, step, w, sigma, outlier,
                                  n_valid=self.plan.total_numel)

    def set_grads(self, arrays_u16):
        for w in range(self.W):
            self.grads[w][: len(arrays_u16[w])].copy_(
                torch.from_numpy(arrays_u16[w].view(np.int16)).view(torch.bfloat16))

    def reduce(self):
        g = torch.empty(max(self.plan.owned_numel, 8), dtype=torch.float32, device=DEV)
        self.plan.debug_reduce(self.grads, g)
        return g[: self.plan.owned_numel]

    def step(self, param_out, t):
        self.plan.step(self.grads, self.master, self.m, self.v, param_out, t)

    def state(self):
        n = self.plan.owned_numel
        return (self.master[:n].cpu().numpy(), self.m[:n].cpu().numpy(), self.v[:n].cpu().numpy())


class OracleRank:
    """The same rank on the host, stepped by the oracle."""

    def __init__(self, oplan, rank, seed):
        self.p, self.rank, self.seed = oplan, rank, seed
        self.idx = oplan.owned_global_index(rank)
        t = torch.from_numpy(self.idx)
        self.master = synth.master_f32(seed, t, n_valid=oplan.total_numel).numpy().copy()
        self.m = np.zeros_like(self.master)
        self.v = np.zeros_like(self.master)
        self.grads = None

    def make_grads(self, step, sigma, outlier):
        t = torch.from_numpy(self.idx)
        self.grads = [u16(synth.grad_bf16(self.seed, step, w, t, sigma, outlier,
                                          n_valid=self.p.total_numel))
                      for w in range(self.p.world_size)]
        return self.grads

    def step(self, param_out, hp, t, clip=None):
        oracle.rank_step(self.p, self.rank, self.grads, self.master, self.m, self.v, param_out, hp, t,
                         clip=clip)


def assert_state_close(got, want, what):
    """Tolerance of the step: |x - y| <= 1e-9 + 2e-6 |y| (NaN matches NaN)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    both_nan = np.isnan(got) & np.isnan(want)
    with np.errstate(invalid="ignore"):           # inf - inf: decided by got == want
        ok = both_nan | (np.abs(got - want) <= 1e-9 + 2e-6 * np.abs(want)) | (got == want)
    if not ok.all():
        bad = np.flatnonzero(~ok)[:5]
        raise AssertionError(f"{what}: {(~ok).sum()} mismatches, e.g. at {bad}: got {got[bad]} want {want[bad]}")


def bf16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    """Distance in bf16 units in the last place between bit patterns (NaN
    pairs count as 0; sign-magnitude mapped to a monotone integer line)."""
    def line(x):
        x = x.astype(np.int64)
        return np.where(x & 0x8000, -(x & 0x7FFF), x & 0x7FFF)
    nan_a = ((a & 0x7F80) == 0x7F80) & ((a & 0x7F) != 0)
    nan_b = ((b & 0x7F80) == 0x7F80) & ((b & 0x7F) != 0)
    d = np.abs(line(a) - line(b))
    d[nan_a & nan_b] = 0
    d[nan_a ^ nan_b] = 1 << 20
    return d
