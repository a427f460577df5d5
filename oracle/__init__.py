"""Oracle for the ZeRO-1/2 sharded optimizer step -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library in
``sharded_optimizer_step_zr_b200``) never touches it.

The arithmetic lives in ``zr_oracle.c`` (plain single-threaded C, built with
gcc ``-O2 -ffp-contract=off``); this module marshals numpy arrays to it and
adds the memory / communication accounting of the pages in plain Python
(``accounting.py``).  Every routine is pinned by ``tests/test_oracle_*.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import accounting  # noqa: F401  (re-exported)

FLAT = 0
WHOLE_TENSOR = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "zr_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None

SEGMENT_DTYPE = np.dtype([
    ("bucket", np.int32), ("tensor", np.int32), ("owner", np.int32), ("reserved", np.int32),
    ("offset_in_tensor", np.int64), ("length", np.int64), ("global_offset", np.int64),
    ("owned_offset", np.int64)])


class _PlanInfo(ctypes.Structure):
    _fields_ = [("total_numel", ctypes.c_int64), ("padded_numel", ctypes.c_int64),
                ("chunk", ctypes.c_int64), ("n_buckets", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("n_segments", ctypes.c_int64)]


class _HP(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in
                ("lr", "beta1", "beta2", "eps", "weight_decay", "max_grad_norm")]


class _Scalars(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in
                ("beta1", "beta2", "one_minus_beta1", "one_minus_beta2", "step_size",
                 "bc2_sqrt", "decay", "eps")]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", _LIB_PATH, _SRC, "-lm"])
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
        L.oracle_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.oracle_bf16_to_f32.restype = ctypes.c_float
        L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
        L.oracle_f32_to_bf16.restype = ctypes.c_uint16
        L.oracle_f32_to_bf16_array.argtypes = [vp, i64, vp]
        L.oracle_plan.argtypes = [i32, vp, vp, i32, i32, u64, vp, vp, vp, vp, i64,
                                  ctypes.POINTER(_PlanInfo)]
        L.oracle_plan.restype = ctypes.c_int
        L.oracle_plan_groups.argtypes = [i32, vp, vp, i32, i32, u64, vp, vp, vp, vp, vp, i64,
                                         ctypes.POINTER(_PlanInfo)]
        L.oracle_plan_groups.restype = ctypes.c_int
        L.oracle_reduce.argtypes = [i32, vp, i64, vp]
        L.oracle_adamw_scalars.argtypes = [ctypes.POINTER(_HP), i64, ctypes.POINTER(_Scalars)]
        L.oracle_adamw.argtypes = [ctypes.POINTER(_Scalars), vp, i64, vp, vp, vp]
        L.oracle_sumsq.argtypes = [vp, i64]
        L.oracle_sumsq.restype = ctypes.c_double
        L.oracle_clip_coef.argtypes = [ctypes.c_double, ctypes.c_float]
        L.oracle_clip_coef.restype = ctypes.c_float
        L.oracle_scale.argtypes = [vp, i64, ctypes.c_float]
        L.oracle_rank_step.argtypes = [i32, i32, vp, i64, vp, i64, vp, vp, vp, vp,
                                       ctypes.POINTER(_HP), i64, ctypes.c_float, ctypes.c_int, vp]
        L.oracle_ddp_step.argtypes = [i32, vp, i64, vp, vp, vp, vp, ctypes.POINTER(_HP), i64,
                                      ctypes.c_float, ctypes.c_int, vp]
        L.oracle_pad.argtypes = [i32, vp, vp, i64, vp]
        L.oracle_unpad.argtypes = [i32, vp, vp, vp]
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data


def _ptr_array(arrays):
    arr = (ctypes.c_void_p * max(1, len(arrays)))()
    for i, a in enumerate(arrays):
        arr[i] = _ptr(a)
    return arr


# ---------------------------------------------------------------------------
# bf16
# ---------------------------------------------------------------------------

def bf16_to_f32(h: int) -> float:
    return lib().oracle_bf16_to_f32(int(h))


def f32_to_bf16(x) -> int:
    return int(lib().oracle_f32_to_bf16(float(np.float32(x))))


def f32_to_bf16_array(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, dtype=np.uint16)
    lib().oracle_f32_to_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to fp32 (numpy view only)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------------------
# Plan
# ---------------------------------------------------------------------------

class Plan:
    """Partition + bucket + segment tables for all ranks.  groups (optional):
    one id per tensor, non-decreasing; then one bucket per group instead of
    the bucket_cap_bytes rule."""

    def __init__(self, shapes, world_size, mode, bucket_cap_bytes, groups=None):
        shapes = [tuple(int(d) for d in s) for s in shapes]
        n = len(shapes)
        grp = None if groups is None else np.array(list(groups) or [0], dtype=np.int32)
        ndims = np.array([len(s) for s in shapes] or [0], dtype=np.int32)
        dims = np.array([d for s in shapes for d in s] or [0], dtype=np.int64)
        owner = np.zeros(max(1, n), dtype=np.int32)
        bucket = np.zeros(max(1, n), dtype=np.int32)
        owned = np.zeros(world_size, dtype=np.int64)
        info = _PlanInfo()
        cap = 16
        while True:
            segs = np.zeros(cap, dtype=SEGMENT_DTYPE)
            if grp is None:
                rc = lib().oracle_plan(n, _ptr(ndims), _ptr(dims), world_size, mode,
                                       int(bucket_cap_bytes), _ptr(owner), _ptr(bucket),
                                       _ptr(owned), _ptr(segs), cap, ctypes.byref(info))
            else:
                rc = lib().oracle_plan_groups(n, _ptr(ndims), _ptr(dims), world_size, mode,
                                              int(bucket_cap_bytes), _ptr(grp), _ptr(owner), _ptr(bucket),
                                              _ptr(owned), _ptr(segs), cap, ctypes.byref(info))
            if rc == -2:
                cap = int(info.n_segments)
                continue
            if rc != 0:
                raise ValueError(f"oracle_plan rejected the arguments (rc={rc})")
            break
        self.shapes = shapes
        self.world_size = world_size
        self.mode = mode
        self.bucket_cap_bytes = int(bucket_cap_bytes)
        self.groups = None if groups is None else [int(g) for g in groups]
        self.total_numel = int(info.total_numel)
        self.padded_numel = int(info.padded_numel)
        self.chunk = int(info.chunk)
        self.n_buckets = int(info.n_buckets)
        self.segments = segs[: info.n_segments].copy()
        self.tensor_owner = owner[:n].copy()
        self.tensor_bucket = bucket[:n].copy()
        self.owned_numel = owned.copy()

    def rank_segments(self, rank):
        return self.segments[self.segments["owner"] == rank]

    def runs(self, rank):
        """(owned_offset, global_offset, length) for ``rank``, by owned offset."""
        s = self.rank_segments(rank)
        order = np.argsort(s["owned_offset"], kind="stable")
        return [(int(x["owned_offset"]), int(x["global_offset"]), int(x["length"]))
                for x in s[order]]

    def owned_global_index(self, rank) -> np.ndarray:
        """Global index of each of ``rank``'s owned elements, in owned order."""
        idx = np.empty(int(self.owned_numel[rank]), dtype=np.int64)
        for owned, glob, length in self.runs(rank):
            idx[owned: owned + length] = np.arange(glob, glob + length, dtype=np.int64)
        return idx


# ---------------------------------------------------------------------------
# Arithmetic
# ---------------------------------------------------------------------------

def _hp(hp):
    h = _HP()
    h.lr, h.beta1, h.beta2, h.eps, h.weight_decay, h.max_grad_norm = [float(x) for x in hp]
    return h


def reduce(grads) -> np.ndarray:
    """Fixed-order fp32 sum of W bf16 replicas (uint16 arrays), divided by W."""
    grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
    n = grads[0].size
    out = np.empty(n, dtype=np.float32)
    lib().oracle_reduce(len(grads), _ptr_array(grads), n, _ptr(out))
    return out


def adamw_scalars(hp, t) -> dict:
    s = _Scalars()
    lib().oracle_adamw_scalars(ctypes.byref(_hp(hp)), int(t), ctypes.byref(s))
    return {name: getattr(s, name) for name, _ in _Scalars._fields_}


def adamw(hp, t, g, p, m, v):
    """In-place AdamW on fp32 arrays p, m, v with gradient g."""
    s = _Scalars()
    lib().oracle_adamw_scalars(ctypes.byref(_hp(hp)), int(t), ctypes.byref(s))
    g = np.ascontiguousarray(g, dtype=np.float32)
    lib().oracle_adamw(ctypes.byref(s), _ptr(g), g.size, _ptr(p), _ptr(m), _ptr(v))


def sumsq(g: np.ndarray) -> float:
    g = np.ascontiguousarray(g, dtype=np.float32)
    return float(lib().oracle_sumsq(_ptr(g), g.size))


def clip_coef(total_sumsq: float, max_norm: float) -> float:
    return float(lib().oracle_clip_coef(float(total_sumsq), float(max_norm)))


def scale(g: np.ndarray, c: float):
    lib().oracle_scale(_ptr(g), g.size, float(c))


def rank_step(plan: Plan, rank, grads, master, m, v, param_out, hp, t, clip=None):
    """One rank's sharded step, in place.  ``grads``: W uint16 arrays in owned
    order; ``param_out``: uint16 array of plan.padded_numel (global layout);
    ``clip``: None or the fp32 clip coefficient."""
    grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in grads]
    n = int(plan.owned_numel[rank])
    scratch = np.empty(max(1, n), dtype=np.float32)
    segs = np.ascontiguousarray(plan.segments)
    lib().oracle_rank_step(plan.world_size, rank, _ptr(segs), segs.size, _ptr_array(grads), n,
                           _ptr(master), _ptr(m), _ptr(v), _ptr(param_out), ctypes.byref(_hp(hp)),
                           int(t), float(clip if clip is not None else 1.0),
                           1 if clip is not None else 0, _ptr(scratch))


def ddp_step(full_grads, master, m, v, param_out, hp, t, clip=None):
    """Unsharded data-parallel step over full replica buffers (global layout)."""
    full_grads = [np.ascontiguousarray(g, dtype=np.uint16) for g in full_grads]
    n = full_grads[0].size
    scratch = np.empty(max(1, n), dtype=np.float32)
    lib().oracle_ddp_step(len(full_grads), _ptr_array(full_grads), n, _ptr(master), _ptr(m),
                          _ptr(v), _ptr(param_out), ctypes.byref(_hp(hp)), int(t),
                          float(clip if clip is not None else 1.0),
                          1 if clip is not None else 0, _ptr(scratch))


def pad(tensors, padded_numel) -> np.ndarray:
    tensors = [np.ascontiguousarray(x, dtype=np.uint16).reshape(-1) for x in tensors]
    numels = np.array([x.size for x in tensors] or [0], dtype=np.int64)
    out = np.empty(padded_numel, dtype=np.uint16)
    lib().oracle_pad(len(tensors), _ptr_array(tensors), _ptr(numels), padded_numel, _ptr(out))
    return out


def unpad(flat, numels):
    flat = np.ascontiguousarray(flat, dtype=np.uint16)
    outs = [np.empty(int(n), dtype=np.uint16) for n in numels]
    nums = np.array(list(numels) or [0], dtype=np.int64)
    lib().oracle_unpad(len(outs), _ptr(flat), _ptr(nums), _ptr_array(outs))
    return outs
