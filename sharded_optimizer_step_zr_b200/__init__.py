"""Python binding of the fused ZeRO-1/2 sharded optimizer step (libzr.so).

Argument marshalling only: every function forwards to the C ABI declared in
``include/zr.h`` under the same name.  Device buffers are passed as integer
addresses or as torch tensors (``tensor.data_ptr()`` is taken); streams as a
``torch.cuda.Stream``, a raw ``cudaStream_t`` integer or ``None`` (the current
torch stream).  Torch is only needed when tensors or streams are passed.

The library must have been built (``python sharded_optimizer_step_zr_b200/build.py``
or ``__graft_entry__.build()``); importing this package without it raises.
There is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libzr.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python sharded_optimizer_step_zr_b200/build.py` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

ZR_OK = 0
ZR_ERR_INVALID_ARG = 1
ZR_ERR_ALIGNMENT = 2
ZR_ERR_NO_WORKSPACE = 3
ZR_ERR_CUDA = 4
ZR_ERR_UNSUPPORTED = 5
ZR_ERR_BUFFER_TOO_SMALL = 6
ZR_ERR_IO = 7
ZR_ERR_MISMATCH = 8
ZR_PARTITION_FLAT = 0
ZR_PARTITION_WHOLE_TENSOR = 1
ZR_MAX_WORLD_SIZE = 512

EXPORTED = [
    "zr_plan_create", "zr_plan_create_grouped", "zr_plan_query", "zr_plan_segments",
    "zr_plan_workspace_bytes", "zr_plan_set_workspace", "zr_plan_set_adamw",
    "zr_plan_set_device_lr", "zr_plan_set_sumsq_partials", "zr_step", "zr_step_device_count",
    "zr_step_bucket", "zr_step_finish", "zr_step_host", "zr_grad_sumsq", "zr_bucket_sumsq",
    "zr_debug_reduce", "zr_debug_average_check", "zr_step_no_alloc", "zr_state_save", "zr_state_load", "zr_state_reshard",
    "zr_state_export_params", "zr_plan_set_checked", "zr_plan_verify", "zr_plan_check_result",
    "zr_plan_set_param_layout", "zr_gather_params", "zr_plan_owner_offsets",
    "zr_plan_set_gather_targets", "zr_ipc_export", "zr_ipc_open", "zr_ipc_close", "zr_plan_destroy",
    "zr_status_string",
]
ZR_NO_ALLOC_SCRATCH_BYTES = 4 << 20


class zr_check_result(ctypes.Structure):
    _fields_ = [("bad_tiles", ctypes.c_uint64), ("first_bad", ctypes.c_int64),
                ("hash_mismatch", ctypes.c_uint32), ("tables_emptied", ctypes.c_uint32)]


class zr_adamw(ctypes.Structure):
    _fields_ = [(n, ctypes.c_float) for n in
                ("lr", "beta1", "beta2", "eps", "weight_decay", "max_grad_norm")]


class zr_segment(ctypes.Structure):
    _fields_ = [("bucket", ctypes.c_int32), ("tensor", ctypes.c_int32), ("owner", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("offset_in_tensor", ctypes.c_int64),
                ("length", ctypes.c_int64), ("global_offset", ctypes.c_int64),
                ("owned_offset", ctypes.c_int64)]


class zr_ipc_handle(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64),
                ("allocation_bytes", ctypes.c_uint64)]


_vp, _i32, _i64, _u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
_P = ctypes.POINTER
_lib.zr_plan_create.argtypes = [_i32, _vp, _vp, _i32, _i32, ctypes.c_int, _u64, _P(zr_adamw), _P(_vp)]
_lib.zr_plan_create_grouped.argtypes = [_i32, _vp, _vp, _vp, _i32, _i32, ctypes.c_int, _P(zr_adamw), _P(_vp)]
_lib.zr_plan_query.argtypes = [_vp, _P(_i64), _P(_i64), _P(_i64), _P(_i32), _P(_i64)]
_lib.zr_plan_segments.argtypes = [_vp, _vp, _i64, _P(_i64)]
_lib.zr_plan_workspace_bytes.argtypes = [_vp, _P(_u64)]
_lib.zr_plan_set_workspace.argtypes = [_vp, _vp, _u64, _vp]
_lib.zr_plan_set_sumsq_partials.argtypes = [_vp, _vp]
_lib.zr_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
_lib.zr_step_device_count.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]
_lib.zr_step_bucket.argtypes = [_vp, _i32, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
_lib.zr_step_finish.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
_lib.zr_step_host.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
_lib.zr_grad_sumsq.argtypes = [_vp, _vp, _vp, _vp]
_lib.zr_bucket_sumsq.argtypes = [_vp, _vp, _vp]
_lib.zr_debug_reduce.argtypes = [_vp, _vp, _vp, _vp]
_lib.zr_debug_average_check.argtypes = [ctypes.c_int32, ctypes.c_int32, _vp, _vp]
_lib.zr_step_no_alloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _vp]
_lib.zr_state_save.argtypes = [_vp, ctypes.c_char_p, _vp, _vp, _vp, _i64, _vp]
_lib.zr_state_load.argtypes = [_vp, ctypes.c_char_p, _vp, _vp, _vp, _P(_i64), _vp]
_lib.zr_state_reshard.argtypes = [_vp, _vp, _i32, ctypes.c_char_p]
_lib.zr_state_export_params.argtypes = [_vp, _vp, _i32, _i32, ctypes.c_char_p, _vp]
_lib.zr_plan_set_checked.argtypes = [_vp, _i32]
_lib.zr_plan_set_adamw.argtypes = [_vp, _P(zr_adamw)]
_lib.zr_plan_set_device_lr.argtypes = [_vp, _vp]
_lib.zr_plan_set_param_layout.argtypes = [_vp, _i32, _vp]
_lib.zr_gather_params.argtypes = [_vp, _i32, _i32, _vp, _vp, _i32, _vp]
_lib.zr_plan_verify.argtypes = [_vp, _vp]
_lib.zr_plan_check_result.argtypes = [_vp, _P(zr_check_result), _vp]
_lib.zr_plan_owner_offsets.argtypes = [_vp, _vp]
_lib.zr_plan_set_gather_targets.argtypes = [_vp, _vp, _vp]
_lib.zr_ipc_export.argtypes = [_vp, _P(zr_ipc_handle)]
_lib.zr_ipc_open.argtypes = [_P(zr_ipc_handle), _P(_vp)]
_lib.zr_ipc_close.argtypes = [_vp]
_lib.zr_plan_destroy.argtypes = [_vp]
_lib.zr_plan_destroy.restype = None
_lib.zr_status_string.argtypes = [ctypes.c_int]
_lib.zr_status_string.restype = ctypes.c_char_p
for _name in EXPORTED:
    if _name not in ("zr_plan_destroy", "zr_status_string"):
        getattr(_lib, _name).restype = ctypes.c_int


class ZrError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {zr_status_string(status)}")


def _check(status: int, where: str) -> int:
    if status != ZR_OK:
        raise ZrError(status, where)
    return status


def _addr(x) -> int:
    """Device or host address of a tensor (data_ptr) or a plain integer."""
    if x is None:
        return 0
    if isinstance(x, int):
        return x
    return int(x.data_ptr())


def _stream(s) -> int:
    if s is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    if isinstance(s, int):
        return s
    return int(s.cuda_stream)


def _ptr_array(xs):
    arr = (ctypes.c_void_p * max(1, len(xs)))()
    for i, x in enumerate(xs):
        arr[i] = _addr(x)
    return arr


def zr_status_string(status: int) -> str:
    return _lib.zr_status_string(int(status)).decode()


def zr_plan_create(shapes, world_size: int, rank: int, mode: int, bucket_cap_bytes: int,
                   lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1,
                   max_grad_norm=0.0, groups=None) -> int:
    """Returns the plan handle (an integer); release it with zr_plan_destroy.
    groups (one id per tensor, non-decreasing): zr_plan_create_grouped, one
    bucket per group, bucket_cap_bytes unused."""
    shapes = [tuple(int(d) for d in s) for s in shapes]
    n = len(shapes)
    ndims = (ctypes.c_int32 * max(1, n))(*[len(s) for s in shapes])
    dim_arrays = [(ctypes.c_int64 * max(1, len(s)))(*s) for s in shapes]
    shape_ptrs = (ctypes.c_void_p * max(1, n))(*[ctypes.addressof(a) for a in dim_arrays])
    hp = zr_adamw(lr, beta1, beta2, eps, weight_decay, max_grad_norm)
    out = ctypes.c_void_p()
    if groups is None:
        _check(_lib.zr_plan_create(n, ndims, shape_ptrs, world_size, rank, mode, int(bucket_cap_bytes),
                                   ctypes.byref(hp), ctypes.byref(out)), "zr_plan_create")
    else:
        groups = [int(g) for g in groups]
        if len(groups) != n:
            raise ValueError("groups: one id per tensor")
        grp = (ctypes.c_int32 * max(1, n))(*groups)
        _check(_lib.zr_plan_create_grouped(n, ndims, shape_ptrs, grp, world_size, rank, mode,
                                           ctypes.byref(hp), ctypes.byref(out)), "zr_plan_create_grouped")
    return out.value


def zr_plan_destroy(plan: int) -> None:
    _lib.zr_plan_destroy(plan)


def zr_plan_query(plan: int) -> dict:
    total, padded, owned, nseg = _i64(), _i64(), _i64(), _i64()
    nb = _i32()
    _check(_lib.zr_plan_query(plan, ctypes.byref(total), ctypes.byref(padded), ctypes.byref(owned),
                              ctypes.byref(nb), ctypes.byref(nseg)), "zr_plan_query")
    return {"total_numel": total.value, "padded_numel": padded.value, "owned_numel": owned.value,
            "n_buckets": nb.value, "n_segments": nseg.value}


def zr_plan_segments(plan: int):
    """All ranks' segments as a list of dicts (field names of zr_segment)."""
    n = _i64()
    st = _lib.zr_plan_segments(plan, None, 0, ctypes.byref(n))
    if st not in (ZR_OK, ZR_ERR_BUFFER_TOO_SMALL):
        _check(st, "zr_plan_segments")
    arr = (zr_segment * max(1, n.value))()
    _check(_lib.zr_plan_segments(plan, arr, n.value, ctypes.byref(n)), "zr_plan_segments")
    names = [f for f, _ in zr_segment._fields_]
    return [{k: getattr(arr[i], k) for k in names} for i in range(n.value)]


def zr_plan_workspace_bytes(plan: int) -> int:
    b = _u64()
    _check(_lib.zr_plan_workspace_bytes(plan, ctypes.byref(b)), "zr_plan_workspace_bytes")
    return b.value


def zr_plan_set_workspace(plan: int, workspace, nbytes: int, stream=None) -> None:
    _check(_lib.zr_plan_set_workspace(plan, _addr(workspace), int(nbytes), _stream(stream)),
           "zr_plan_set_workspace")


def zr_plan_set_sumsq_partials(plan: int, partials) -> None:
    _check(_lib.zr_plan_set_sumsq_partials(plan, _addr(partials)), "zr_plan_set_sumsq_partials")


def zr_step(plan: int, grads, master, m, v, param_out, step: int, stream=None) -> None:
    _check(_lib.zr_step(plan, _ptr_array(grads), _addr(master), _addr(m), _addr(v),
                        _addr(param_out), int(step), _stream(stream)), "zr_step")


def zr_step_device_count(plan: int, grads, master, m, v, param_out, d_step, stream=None) -> None:
    _check(_lib.zr_step_device_count(plan, _ptr_array(grads), _addr(master), _addr(m), _addr(v),
                                     _addr(param_out), _addr(d_step), _stream(stream)),
           "zr_step_device_count")


def zr_step_bucket(plan: int, bucket: int, grads, master, m, v, param_out, step: int,
                   stream=None) -> None:
    _check(_lib.zr_step_bucket(plan, int(bucket), _ptr_array(grads), _addr(master), _addr(m),
                               _addr(v), _addr(param_out), int(step), _stream(stream)),
           "zr_step_bucket")


def zr_step_finish(plan: int, grads, master, m, v, param_out, step: int, stream=None) -> None:
    _check(_lib.zr_step_finish(plan, _ptr_array(grads) if grads is not None else None, _addr(master),
                               _addr(m), _addr(v), _addr(param_out), int(step), _stream(stream)),
           "zr_step_finish")


def zr_step_host(plan: int, host_grads, dev_grads, master, m, v, param_out, host_param_out,
                 step: int, stream=None) -> None:
    _check(_lib.zr_step_host(plan, _ptr_array(host_grads), _ptr_array(dev_grads), _addr(master),
                             _addr(m), _addr(v), _addr(param_out), _addr(host_param_out), int(step),
                             _stream(stream)), "zr_step_host")


def zr_grad_sumsq(plan: int, grads, out, stream=None) -> None:
    _check(_lib.zr_grad_sumsq(plan, _ptr_array(grads), _addr(out), _stream(stream)), "zr_grad_sumsq")


def zr_debug_average_check(w_first: int, w_last: int, mismatches, stream=None) -> None:
    """Per W in [w_first, w_last]: inputs (of all 2^32 fp32 values) whose
    averaged value differs from IEEE division, into mismatches (device
    uint64 / int64 array of w_last - w_first + 1)."""
    _check(_lib.zr_debug_average_check(int(w_first), int(w_last), _addr(mismatches), _stream(stream)),
           "zr_debug_average_check")


def zr_debug_reduce(plan: int, grads, g_out, stream=None) -> None:
    _check(_lib.zr_debug_reduce(plan, _ptr_array(grads), _addr(g_out), _stream(stream)),
           "zr_debug_reduce")


def zr_bucket_sumsq(plan: int, out, stream=None) -> None:
    """This rank's S_r from the sums of squares of a bucket-by-bucket pass
    (every bucket's zr_step_bucket called), into the device double `out`."""
    _check(_lib.zr_bucket_sumsq(plan, _addr(out), _stream(stream)), "zr_bucket_sumsq")


def zr_step_no_alloc(plan: int, grads, master, m, v, param_out, sumsq_partials, step: int,
                     stream=None) -> None:
    """zr_step without a workspace: for callers that cannot allocate device
    memory.  Scratch lives in the library's fixed 4 MiB device array (see
    include/zr.h); plans too large for it raise ZR_ERR_UNSUPPORTED."""
    st = _lib.zr_step_no_alloc(plan, _ptr_array(grads), _addr(master), _addr(m), _addr(v),
                               _addr(param_out), _addr(sumsq_partials), int(step), _stream(stream))
    if st == ZR_ERR_UNSUPPORTED:
        raise ZrError(st, "zr_step_no_alloc (the plan's tile table, and clip partials, must fit "
                          f"the library's {ZR_NO_ALLOC_SCRATCH_BYTES} byte static scratch on a "
                          "compute capability 10.x device; use zr_step with a workspace)")
    _check(st, "zr_step_no_alloc")


def zr_state_save(plan: int, path: str, master, m, v, step: int, stream=None) -> None:
    _check(_lib.zr_state_save(plan, os.fsencode(path), _addr(master), _addr(m), _addr(v), int(step),
                              _stream(stream)), "zr_state_save")


def zr_state_load(plan: int, path: str, master, m, v, stream=None) -> int:
    """Loads the shard into master/m/v and returns its step."""
    step = _i64()
    _check(_lib.zr_state_load(plan, os.fsencode(path), _addr(master), _addr(m), _addr(v),
                              ctypes.byref(step), _stream(stream)), "zr_state_load")
    return step.value


def zr_state_reshard(target_plan: int, src_paths, dst_path: str) -> None:
    arr = (ctypes.c_char_p * max(1, len(src_paths)))(*[os.fsencode(p) for p in src_paths])
    _check(_lib.zr_state_reshard(target_plan, arr, len(src_paths), os.fsencode(dst_path)),
           "zr_state_reshard")


ZR_EXPORT_F32 = 0
ZR_EXPORT_BF16 = 1


def zr_state_export_params(plan: int, src_paths, dtype: int, out_path: str) -> int:
    """Writes the whole model's master weights (declaration order, raw fp32
    or bf16) from a complete shard set; returns the element count."""
    arr = (ctypes.c_char_p * max(1, len(src_paths)))(*[os.fsencode(p) for p in src_paths])
    n = _i64()
    _check(_lib.zr_state_export_params(plan, arr, len(src_paths), int(dtype), os.fsencode(out_path),
                                       ctypes.byref(n)), "zr_state_export_params")
    return n.value


def zr_plan_set_adamw(plan: int, lr=3e-4, beta1=0.9, beta2=0.999, eps=1e-8, weight_decay=0.1,
                      max_grad_norm=0.0) -> None:
    hp = zr_adamw(lr, beta1, beta2, eps, weight_decay, max_grad_norm)
    _check(_lib.zr_plan_set_adamw(plan, ctypes.byref(hp)), "zr_plan_set_adamw")


def zr_plan_set_device_lr(plan: int, d_lr) -> None:
    """d_lr: a one-element fp32 device tensor (or address), or None."""
    _check(_lib.zr_plan_set_device_lr(plan, _addr(d_lr)), "zr_plan_set_device_lr")


ZR_PARAMS_GLOBAL = 0
ZR_PARAMS_OWNED = 1


def zr_plan_set_param_layout(plan: int, layout: int, stream=None) -> None:
    _check(_lib.zr_plan_set_param_layout(plan, int(layout), _stream(stream)), "zr_plan_set_param_layout")


def zr_gather_params(plan: int, first_tensor: int, n_tensors: int, shards, dst, stream=None,
                     max_ctas: int = 0) -> None:
    arr = _ptr_array(shards)
    _check(_lib.zr_gather_params(plan, int(first_tensor), int(n_tensors), arr, _addr(dst), int(max_ctas),
                                 _stream(stream)), "zr_gather_params")


def zr_plan_set_checked(plan: int, enable: bool) -> None:
    _check(_lib.zr_plan_set_checked(plan, 1 if enable else 0), "zr_plan_set_checked")


def zr_plan_verify(plan: int, stream=None) -> None:
    _check(_lib.zr_plan_verify(plan, _stream(stream)), "zr_plan_verify")


def zr_plan_check_result(plan: int, stream=None) -> dict:
    r = zr_check_result()
    _check(_lib.zr_plan_check_result(plan, ctypes.byref(r), _stream(stream)), "zr_plan_check_result")
    return {name: getattr(r, name) for name, _ in zr_check_result._fields_}


def zr_plan_owner_offsets(plan: int, world_size: int):
    arr = (ctypes.c_int64 * (world_size + 1))()
    _check(_lib.zr_plan_owner_offsets(plan, arr), "zr_plan_owner_offsets")
    return list(arr)


def zr_plan_set_gather_targets(plan: int, targets, stream=None) -> None:
    arr = _ptr_array(targets) if targets is not None else None
    _check(_lib.zr_plan_set_gather_targets(plan, arr, _stream(stream)), "zr_plan_set_gather_targets")


def zr_ipc_export(buffer) -> bytes:
    """The handle of a device buffer (tensor or address) as bytes."""
    h = zr_ipc_handle()
    _check(_lib.zr_ipc_export(_addr(buffer), ctypes.byref(h)), "zr_ipc_export")
    return bytes(h)


def zr_ipc_open(handle: bytes) -> int:
    h = zr_ipc_handle.from_buffer_copy(handle)
    out = ctypes.c_void_p()
    _check(_lib.zr_ipc_open(ctypes.byref(h), ctypes.byref(out)), "zr_ipc_open")
    return out.value


def zr_ipc_close(address: int) -> None:
    _check(_lib.zr_ipc_close(address), "zr_ipc_close")


def raw_call(name: str, *args) -> int:
    """Call a C ABI function with already-marshalled arguments; returns the
    status code without raising (used by the error-path tests)."""
    return getattr(_lib, name)(*args)


def lib_handle():
    return _lib
