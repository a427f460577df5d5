"""Seeded synthetic inputs for the sharded optimizer step.

This module is shared by the tests, the benchmark and the oracle checks.  It
holds none of the optimizer step's arithmetic: it only describes the
parameter-set shapes of the workloads and draws, from a counter-based
generator, the W gradient replicas and the initial fp32 master weights.

Generator (identical bits on the CPU and on a CUDA device)
----------------------------------------------------------
Every value is a pure function of ``(seed, kind, step, replica, index)``.
``index`` is the element's position in the *global* flat layout
(declaration order), so every rank, the unsharded comparator and the GPU see
the same gradient for the same parameter element.

* ``mix64`` is the splitmix64 output function (Steele, Lea & Flood,
  "Fast splittable pseudorandom number generators", OOPSLA 2014; the
  finaliser constants are Stafford's "Mix13").
* A stream key is built by chaining ``mix64`` over the seed, the kind tag,
  the step, the replica and a lane number; element ``i`` of a lane is
  ``mix64(key + (i + 1) * GAMMA)``, i.e. the ``i``-th splitmix64 output of
  the stream.
* Normal deviates use the classic "sum of twelve uniforms" construction:
  lanes 0..2 give 3 x 64 bits = twelve 16-bit uniforms ``U_k`` in
  ``[0, 65535]``; ``sum(U_k) - 393210`` is an exact integer with variance
  ``65536**2 - 1``, so ``x = (sum - 393210) * float32(sigma / 65536)`` is a
  deviate of standard deviation ``sigma`` (one fp32 rounding; tails end at
  +-6 sigma).
* Outliers: lane 3 gives an independent Bernoulli(frac) draw per element and
  replica (``top 32 bits < round(frac * 2**32)``); a selected value is
  multiplied by ``outlier_scale`` in fp32 before the bf16 rounding.
* Gradients are rounded to bf16 with round-to-nearest-even; master weights
  stay fp32.  Elements at ``index >= N`` (the flat-partition zero pad) are 0.

Only integer operations, one exact int->fp32 conversion, one fp32 multiply
(two with an outlier) and the RNE bf16 conversion are involved, so torch on
the CPU, torch on CUDA and the C routine in ``csynth.c`` agree bit for bit
(a test checks it).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field

import numpy as np
import torch

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX_C1 = 0xBF58476D1CE4E5B9
MIX_C2 = 0x94D049BB133111EB

KIND_GRAD = 1
KIND_MASTER = 2

SUM12_MEAN = 393210          # 12 * 65535 / 2
OUTLIER_FRAC_DEFAULT = 0.01
OUTLIER_SCALE_DEFAULT = 100.0


def _s64(x: int) -> int:
    """Unsigned 64-bit integer -> the signed int64 with the same bits."""
    x &= M64
    return x - (1 << 64) if x >> 63 else x


def mix64(x: int) -> int:
    """splitmix64 output function on a Python int (exact, unsigned 64-bit)."""
    x &= M64
    x = ((x ^ (x >> 30)) * MIX_C1) & M64
    x = ((x ^ (x >> 27)) * MIX_C2) & M64
    return x ^ (x >> 31)


def stream_key(seed: int, kind: int, step: int, replica: int, lane: int) -> int:
    k = mix64(seed)
    for part in (kind, step, replica, lane):
        k = mix64(k + (part + 1) * GAMMA)
    return k


def _mix64_t(z: torch.Tensor) -> torch.Tensor:
    """splitmix64 output function on an int64 tensor (two's-complement wrap;
    logical right shifts emulated with a mask)."""
    z = (z ^ ((z >> 30) & ((1 << 34) - 1))) * _s64(MIX_C1)
    z = (z ^ ((z >> 27) & ((1 << 37) - 1))) * _s64(MIX_C2)
    return z ^ ((z >> 31) & ((1 << 33) - 1))


def _lane_t(key: int, idx: torch.Tensor) -> torch.Tensor:
    return _mix64_t((idx + 1) * _s64(GAMMA) + _s64(key))


def sigma_scale(sigma: float) -> float:
    """The fp32 multiplier applied to the centred sum of twelve uniforms."""
    return float(np.float32(sigma / 65536.0))


def outlier_threshold(frac: float) -> int:
    return int(round(frac * 4294967296.0))


def normal_f32(seed: int, kind: int, step: int, replica: int, idx: torch.Tensor,
               sigma: float) -> torch.Tensor:
    """fp32 N(0, sigma) deviates (sum of twelve uniforms) for int64 ``idx``."""
    total = None
    for lane in range(3):
        u = _lane_t(stream_key(seed, kind, step, replica, lane), idx)
        for sh in (0, 16, 32, 48):
            f = (u >> sh) & 0xFFFF
            total = f if total is None else total + f
    centred = (total - SUM12_MEAN).to(torch.float32)          # exact: |c| < 2**24
    return centred * torch.tensor(sigma_scale(sigma), dtype=torch.float32, device=idx.device)


def grad_bf16(seed: int, step: int, replica: int, idx: torch.Tensor, sigma: float,
              outlier_frac: float = 0.0, outlier_scale: float = OUTLIER_SCALE_DEFAULT,
              n_valid: int | None = None) -> torch.Tensor:
    """bf16 gradient values of replica ``replica`` at global indices ``idx``."""
    x = normal_f32(seed, KIND_GRAD, step, replica, idx, sigma)
    if outlier_frac > 0.0:
        u = _lane_t(stream_key(seed, KIND_GRAD, step, replica, 3), idx)
        hit = ((u >> 32) & 0xFFFFFFFF) < outlier_threshold(outlier_frac)
        x = torch.where(hit, x * torch.tensor(outlier_scale, dtype=torch.float32,
                                              device=idx.device), x)
    if n_valid is not None:
        x = torch.where(idx < n_valid, x, torch.zeros_like(x))
    return x.to(torch.bfloat16)


def master_f32(seed: int, idx: torch.Tensor, sigma: float = 0.02,
               n_valid: int | None = None) -> torch.Tensor:
    """Initial fp32 master weights at global indices ``idx``."""
    x = normal_f32(seed, KIND_MASTER, 0, 0, idx, sigma)
    if n_valid is not None:
        x = torch.where(idx < n_valid, x, torch.zeros_like(x))
    return x


# ----------------------------------------------------------------------------
# Parameter sets shaped like the workloads (declaration order).
# ----------------------------------------------------------------------------

def tiny_shapes():
    return [(512, 512), (512, 1024), (1024, 512), (131072,)]


def gpt2_small_shapes():
    """GPT-2 small (124M): tied head; wte, wpe, 12 blocks, final LayerNorm."""
    d, v, ctx, L = 768, 50257, 1024, 12
    shapes = [(v, d), (ctx, d)]
    for _ in range(L):
        shapes += [(d,), (d,),                      # ln_1 weight, bias
                   (d, 3 * d), (3 * d,),            # attn qkv weight, bias
                   (d, d), (d,),                    # attn proj weight, bias
                   (d,), (d,),                      # ln_2 weight, bias
                   (d, 4 * d), (4 * d,),            # mlp fc weight, bias
                   (4 * d, d), (d,)]                # mlp proj weight, bias
    shapes += [(d,), (d,)]                          # ln_f
    return shapes


def gpt_1p3b_shapes(L=24):
    """GPT-style 1.3B: d=2048, 24 blocks, MLP 8192, vocab 50304, 2048 learned
    positions, biases and LayerNorm weight/bias, tied head.  L < 24 keeps the
    first L blocks (a smaller case of the same shapes)."""
    d, v, ctx, f = 2048, 50304, 2048, 8192
    shapes = [(v, d), (ctx, d)]
    for _ in range(L):
        shapes += [(d,), (d,), (d, 3 * d), (3 * d,), (d, d), (d,),
                   (d,), (d,), (d, f), (f,), (f, d), (d,)]
    shapes += [(d,), (d,)]
    return shapes


def llama_7b_shapes(L=32):
    """Llama-7B: untied embedding and head, RMSNorm weights, no biases;
    each block declares attn_norm, q, k, v, o, mlp_norm, gate, up, down.
    L < 32 keeps the first L blocks (a smaller case of the same shapes)."""
    d, v, f = 4096, 32000, 11008
    shapes = [(v, d)]
    for _ in range(L):
        shapes += [(d,), (d, d), (d, d), (d, d), (d, d), (d,), (f, d), (f, d), (d, f)]
    shapes += [(d,), (v, d)]
    return shapes


PARAM_SETS = {
    "tiny": tiny_shapes,
    "gpt2_124m": gpt2_small_shapes,
    "gpt_1p3b": gpt_1p3b_shapes,
    "llama_7b": llama_7b_shapes,
    # smaller cases of the same shapes, for profiler captures of a few GB
    "llama_7b_4blk": lambda: llama_7b_shapes(4),
    "gpt_1p3b_6blk": lambda: gpt_1p3b_shapes(6),
}

MB = 1 << 20


@dataclass(frozen=True)
class Workload:
    """One configuration of the step: parameter set, replicas, partition."""
    name: str
    param_set: str
    world_size: int
    ranks: tuple
    mode: int                    # 0 = flat, 1 = whole-tensor
    bucket_cap_mb: float
    grad_sigma: float
    outlier_frac: float
    max_grad_norm: float = 0.0   # <= 0: no clipping
    steps: int = 3
    lr: float = 3e-4
    beta1: float = 0.9
    beta2: float = 0.999
    eps: float = 1e-8
    weight_decay: float = 0.1
    seed: int = 1234
    extra: dict = field(default_factory=dict)

    @property
    def shapes(self):
        return PARAM_SETS[self.param_set]()

    @property
    def bucket_cap_bytes(self) -> int:
        return int(self.bucket_cap_mb * MB)

    @property
    def hp(self):
        return (self.lr, self.beta1, self.beta2, self.eps, self.weight_decay,
                self.max_grad_norm)


WORKLOADS = {
    # 4 tensors, W=2, both ranks, flat, 1 MB buckets, N(0, 1e-2) grads, 3 steps.
    "tiny": Workload("tiny", "tiny", 2, (0, 1), 0, 1, 1e-2, 0.0),
    # GPT-2 small, W=8, rank 0, flat, 25 MB buckets, N(0, 1e-3) + 1 % x100.
    "gpt2_124m_w8": Workload("gpt2_124m_w8", "gpt2_124m", 8, (0,), 0, 25, 1e-3, 0.01),
    # 1.3B GPT, W=8, rank 3, whole-tensor (LPT), 25 MB buckets, clip at 1.0.
    "gpt_1p3b_w8_whole_clip": Workload("gpt_1p3b_w8_whole_clip", "gpt_1p3b", 8, (3,), 1, 25,
                                       1e-3, 0.01, max_grad_norm=1.0),
    # Llama-7B, W=64, rank 0, flat, 25 MB buckets, N(0, 1e-3).
    "llama_7b_w64": Workload("llama_7b_w64", "llama_7b", 64, (0,), 0, 25, 1e-3, 0.0),
    # Small cases of the same kernels, for profiler captures of a few hundred MB:
    # the W = 64 flat step and the whole-tensor clip step on the GPT-2 set.
    "gpt2_124m_w64": Workload("gpt2_124m_w64", "gpt2_124m", 64, (0,), 0, 25, 1e-3, 0.0),
    "gpt2_124m_w8_whole_clip": Workload("gpt2_124m_w8_whole_clip", "gpt2_124m", 8, (3,), 1, 25,
                                        1e-3, 0.01, max_grad_norm=1.0),
    # The same kernels as the Llama-7B W = 64 and the 1.3B clipped workloads on
    # the first blocks of those sets (about 4.5 and 2.5 GB on the device): the
    # DRAM counters taken on them are scaled to the full workloads by owned params.
    "llama_7b_4blk_w64": Workload("llama_7b_4blk_w64", "llama_7b_4blk", 64, (0,), 0, 25, 1e-3, 0.0),
    "gpt_1p3b_6blk_w8_whole_clip": Workload("gpt_1p3b_6blk_w8_whole_clip", "gpt_1p3b_6blk", 8, (3,), 1, 25,
                                            1e-3, 0.01, max_grad_norm=1.0),
}


def sweep_workloads():
    """1.3B set: bucket cap {1,5,25,100,400} MB x W {2,8,32,64} x {flat, whole}."""
    out = []
    for mode in (0, 1):
        for w in (2, 8, 32, 64):
            for cap in (1, 5, 25, 100, 400):
                name = f"sweep_1p3b_{'flat' if mode == 0 else 'whole'}_w{w}_cap{cap}"
                out.append(Workload(name, "gpt_1p3b", w, (0,), mode, cap, 1e-3, 0.01))
    return out


def numel(shape) -> int:
    n = 1
    for d in shape:
        n *= int(d)
    return n


# ----------------------------------------------------------------------------
# Filling owned-order buffers from a plan's segment list.
# ----------------------------------------------------------------------------

def rank_runs(segments, rank):
    """(owned_offset, global_offset, length) of ``rank``'s segments, by owned offset.

    ``segments`` is any sequence of records with fields ``owner``,
    ``owned_offset``, ``global_offset`` and ``length``."""
    runs = [(int(s["owned_offset"]), int(s["global_offset"]), int(s["length"]))
            for s in segments if int(s["owner"]) == rank]
    runs.sort()
    return runs


def fill_owned_grad(out: torch.Tensor, runs, seed, step, replica, sigma, outlier_frac,
                    n_valid, chunk=1 << 24):
    """Write replica ``replica``'s bf16 gradient for the owned elements ``runs``
    into the 1-D owned-order tensor ``out`` (any device), chunk by chunk."""
    dev = out.device
    for owned, glob, length in runs:
        for c0 in range(0, length, chunk):
            n = min(chunk, length - c0)
            idx = torch.arange(glob + c0, glob + c0 + n, dtype=torch.int64, device=dev)
            out[owned + c0: owned + c0 + n] = grad_bf16(seed, step, replica, idx, sigma,
                                                        outlier_frac, n_valid=n_valid)


def fill_owned_master(out: torch.Tensor, runs, seed, n_valid, sigma=0.02, chunk=1 << 24):
    dev = out.device
    for owned, glob, length in runs:
        for c0 in range(0, length, chunk):
            n = min(chunk, length - c0)
            idx = torch.arange(glob + c0, glob + c0 + n, dtype=torch.int64, device=dev)
            out[owned + c0: owned + c0 + n] = master_f32(seed, idx, sigma, n_valid=n_valid)


# ----------------------------------------------------------------------------
# The same generator in C, for fast host-side generation of large inputs.
# ----------------------------------------------------------------------------

_HERE = os.path.dirname(os.path.abspath(__file__))
_CLIB_PATH = os.path.join(_HERE, "libcsynth.so")
_clib = None


def build_c(force: bool = False) -> str:
    src = os.path.join(_HERE, "csynth.c")
    if force or not os.path.exists(_CLIB_PATH) or \
            os.path.getmtime(_CLIB_PATH) < os.path.getmtime(src):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC",
                               "-shared", "-o", _CLIB_PATH, src])
    return _CLIB_PATH


def _c():
    global _clib
    if _clib is None:
        build_c()
        lib = ctypes.CDLL(_CLIB_PATH)
        lib.csynth_grad_range.argtypes = [ctypes.c_uint64] * 4 + [
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, ctypes.c_uint32,
            ctypes.c_float, ctypes.c_void_p]
        lib.csynth_grad_range.restype = None
        lib.csynth_normal_range.argtypes = [ctypes.c_uint64] * 3 + [
            ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_float, ctypes.c_void_p]
        lib.csynth_normal_range.restype = None
        _clib = lib
    return _clib


def grad_bf16_range_c(seed, step, replica, start, n, sigma, outlier_frac=0.0,
                      outlier_scale=OUTLIER_SCALE_DEFAULT, n_valid=None) -> np.ndarray:
    """bf16 bits (uint16) of replica ``replica`` at global indices [start, start+n)."""
    keys = [stream_key(seed, KIND_GRAD, step, replica, lane) for lane in range(4)]
    out = np.empty(n, dtype=np.uint16)
    nv = (1 << 62) if n_valid is None else int(n_valid)
    thr = outlier_threshold(outlier_frac) if outlier_frac > 0.0 else 0
    _c().csynth_grad_range(*keys, start, n, nv, sigma_scale(sigma), thr, outlier_scale,
                           out.ctypes.data)
    return out


def master_f32_range_c(seed, start, n, sigma=0.02, n_valid=None) -> np.ndarray:
    keys = [stream_key(seed, KIND_MASTER, 0, 0, lane) for lane in range(3)]
    out = np.empty(n, dtype=np.float32)
    nv = (1 << 62) if n_valid is None else int(n_valid)
    _c().csynth_normal_range(*keys, start, n, nv, sigma_scale(sigma), out.ctypes.data)
    return out
