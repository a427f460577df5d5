"""C ABI of libzr.so without a GPU: the library loads, exports every function
include/zr.h declares, rejects bad arguments with the documented status
codes, and its planner's tables equal the oracle's bit for bit.

The planner runs on the host only, so table parity (the "bucket/owner tables
bit-exact" requirement) is checked here; kernels are checked in test_gpu_*.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import synth
import sharded_optimizer_step_zr_b200 as zr
from conftest import ROOT
from golden_plans import all_golden_plans

FIELDS = ("bucket", "tensor", "owner", "offset_in_tensor", "length", "global_offset", "owned_offset")


def header_functions():
    text = open(os.path.join(ROOT, "include", "zr.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(zr_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function():
    declared = header_functions()
    assert set(declared) == set(zr.EXPORTED)
    lib = zr.lib_handle()
    for name in declared:
        assert hasattr(lib, name), name


def test_only_zr_symbols_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", zr.LIB_PATH], capture_output=True, text=True).stdout
    syms = [l.split()[-1] for l in out.splitlines() if " T " in l]
    assert syms and all(s.startswith("zr_") for s in syms), syms


def test_import_without_the_library_fails_loudly(tmp_path):
    """The binding has no fallback: a copy of the package without libzr.so
    refuses to import, naming the missing file."""
    import shutil
    import subprocess
    import sys
    pkg = os.path.join(ROOT, "sharded_optimizer_step_zr_b200")
    dst = tmp_path / "sharded_optimizer_step_zr_b200"
    dst.mkdir()
    for f in os.listdir(pkg):
        if f.endswith(".py"):
            shutil.copy(os.path.join(pkg, f), dst / f)
    r = subprocess.run([sys.executable, "-c", "import sharded_optimizer_step_zr_b200"], cwd=tmp_path,
                       capture_output=True, text=True, env=dict(os.environ, PYTHONPATH=str(tmp_path)))
    assert r.returncode != 0
    assert "ImportError" in r.stderr and "libzr.so is missing" in r.stderr


def test_status_strings():
    for s in range(7):
        assert zr.zr_status_string(s).startswith("ZR_")
    assert "unknown" in zr.zr_status_string(99)


def lib_plan_table(shapes, W, rank, mode, cap, groups=None):
    h = zr.zr_plan_create(shapes, W, rank, mode, cap, groups=groups)
    try:
        segs = zr.zr_plan_segments(h)
        info = zr.zr_plan_query(h)
    finally:
        zr.zr_plan_destroy(h)
    return [tuple(s[f] for f in FIELDS) for s in segs], info


def oracle_table(shapes, W, mode, cap, groups=None):
    p = oracle.Plan(shapes, W, mode, cap, groups=groups)
    return [tuple(int(s[f]) for f in FIELDS) for s in p.segments], p


def assert_tables_equal(shapes, W, mode, cap, groups=None):
    want, p = oracle_table(shapes, W, mode, cap, groups)
    for rank in sorted({0, W - 1, W // 2}):
        got, info = lib_plan_table(shapes, W, rank, mode, cap, groups)
        assert got == want
        assert info["total_numel"] == p.total_numel
        assert info["padded_numel"] == p.padded_numel
        assert info["owned_numel"] == int(p.owned_numel[rank])
        assert info["n_buckets"] == p.n_buckets
        assert info["n_segments"] == len(want)


@pytest.mark.parametrize("g", all_golden_plans(), ids=lambda g: g["name"])
def test_tables_match_hand_derived(g):
    got, info = lib_plan_table(g["shapes"], g["world_size"], 0, g["mode"], g["cap_bytes"], g["groups"])
    assert got == g["segments"]
    assert (info["total_numel"], info["padded_numel"], info["n_buckets"]) == (g["N"], g["padded"], g["n_buckets"])


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_tables_match_oracle_workloads(name):
    wl = synth.WORKLOADS[name]
    assert_tables_equal(wl.shapes, wl.world_size, wl.mode, wl.bucket_cap_bytes)


def test_tables_match_oracle_sweep():
    for wl in synth.sweep_workloads():
        assert_tables_equal(wl.shapes, wl.world_size, wl.mode, wl.bucket_cap_bytes)


def test_tables_match_oracle_random():
    rng = np.random.default_rng(21)
    for _ in range(400):
        shapes = [tuple(int(x) for x in rng.integers(0, 30, size=int(rng.integers(0, 3))))
                  for _ in range(int(rng.integers(0, 10)))]
        W = int(rng.integers(1, 12))
        mode = int(rng.integers(0, 2))
        cap = int(rng.integers(0, 300))
        assert_tables_equal(shapes, W, mode, cap)


def test_grouped_tables_match_oracle_random():
    """Buckets given by tensor groups (one per layer): the library's tables
    equal the oracle's bit for bit on random sets, and on the GPT-2 set
    grouped by block (embeddings, 12 blocks, final norm)."""
    rng = np.random.default_rng(23)
    for _ in range(300):
        nt = int(rng.integers(0, 10))
        shapes = [tuple(int(x) for x in rng.integers(0, 30, size=int(rng.integers(0, 3))))
                  for _ in range(nt)]
        groups = np.cumsum(rng.integers(0, 2, size=nt)).tolist()
        assert_tables_equal(shapes, int(rng.integers(1, 12)), int(rng.integers(0, 2)), 0, groups)
    shapes = synth.gpt2_small_shapes()
    groups = [0, 0] + [1 + i // 12 for i in range(12 * 12)] + [13, 13]
    for mode in (0, 1):
        assert_tables_equal(shapes, 8, mode, 0, groups)
        h = zr.zr_plan_create(shapes, 8, 0, mode, 0, groups=groups)
        assert zr.zr_plan_query(h)["n_buckets"] == 14
        zr.zr_plan_destroy(h)


def test_grouped_plan_argument_errors():
    shapes = [(4,), (5,), (6,)]
    with pytest.raises(zr.ZrError) as e:
        zr.zr_plan_create(shapes, 2, 0, 0, 0, groups=[0, 1, 0])
    assert e.value.status == zr.ZR_ERR_INVALID_ARG
    hp = zr.zr_adamw(3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)
    out = ctypes.c_void_p()
    ndims = (ctypes.c_int32 * 3)(1, 1, 1)
    dims = [(ctypes.c_int64 * 1)(n) for n in (4, 5, 6)]
    ptrs = (ctypes.c_void_p * 3)(*[ctypes.addressof(d) for d in dims])
    st = zr.raw_call("zr_plan_create_grouped", 3, ndims, ptrs, None, 2, 0, 0, ctypes.byref(hp), ctypes.byref(out))
    assert st == zr.ZR_ERR_INVALID_ARG and not out.value


def test_empty_parameter_set():
    h = zr.zr_plan_create([], 4, 1, 0, 1 << 20)
    info = zr.zr_plan_query(h)
    zr.zr_plan_destroy(h)
    assert info == {"total_numel": 0, "padded_numel": 0, "owned_numel": 0, "n_buckets": 0, "n_segments": 0}


@pytest.mark.parametrize("args, status", [
    (([(4,)], 0, 0, 0, 16), zr.ZR_ERR_INVALID_ARG),          # W = 0
    (([(4,)], 2, 2, 0, 16), zr.ZR_ERR_INVALID_ARG),          # rank = W
    (([(4,)], 2, -1, 0, 16), zr.ZR_ERR_INVALID_ARG),         # negative rank
    (([(4,)], 2, 0, 3, 16), zr.ZR_ERR_INVALID_ARG),          # unknown mode
    (([(-4,)], 2, 0, 0, 16), zr.ZR_ERR_INVALID_ARG),         # negative extent
    (([(1 << 40, 1 << 40)], 2, 0, 0, 16), zr.ZR_ERR_INVALID_ARG),  # numel overflow
    (([(4,)], 513, 0, 0, 16), zr.ZR_ERR_UNSUPPORTED),        # W above the limit
])
def test_plan_create_rejects(args, status):
    with pytest.raises(zr.ZrError) as e:
        zr.zr_plan_create(*args)
    assert e.value.status == status


def test_null_arguments():
    assert zr.raw_call("zr_plan_create", 0, None, None, 1, 0, 0, 0, None, None) == zr.ZR_ERR_INVALID_ARG
    n = ctypes.c_int64()
    assert zr.raw_call("zr_plan_query", None, None, None, None, None, None) == zr.ZR_ERR_INVALID_ARG
    assert zr.raw_call("zr_plan_segments", None, None, 0, ctypes.byref(n)) == zr.ZR_ERR_INVALID_ARG
    assert zr.raw_call("zr_plan_workspace_bytes", None, None) == zr.ZR_ERR_INVALID_ARG


def test_step_checks_before_touching_the_device():
    """Without a bound workspace or with a bad step the call returns an
    error and launches nothing (no GPU needed to check this)."""
    h = zr.zr_plan_create([(64,)], 2, 0, 0, 1 << 20)
    try:
        grads = (ctypes.c_void_p * 2)(16, 32)
        assert zr.raw_call("zr_step", h, grads, 16, 16, 16, 16, 0, None) == zr.ZR_ERR_INVALID_ARG
        assert zr.raw_call("zr_step", h, grads, 16, 16, 16, 16, 1, None) == zr.ZR_ERR_NO_WORKSPACE
        assert zr.raw_call("zr_debug_reduce", h, grads, 16, None) == zr.ZR_ERR_NO_WORKSPACE
        assert zr.raw_call("zr_grad_sumsq", h, grads, 16, None) == zr.ZR_ERR_NO_WORKSPACE
        assert zr.raw_call("zr_plan_set_workspace", h, None, 0, None) == zr.ZR_ERR_INVALID_ARG
        assert zr.raw_call("zr_plan_set_workspace", h, 8, 1 << 20, None) == zr.ZR_ERR_ALIGNMENT
        assert zr.raw_call("zr_plan_set_sumsq_partials", h, 12) == zr.ZR_ERR_ALIGNMENT
        # workspace too small is detected before any CUDA call
        need = zr.zr_plan_workspace_bytes(h)
        assert zr.raw_call("zr_plan_set_workspace", h, 256, need - 1, None) == zr.ZR_ERR_NO_WORKSPACE
    finally:
        zr.zr_plan_destroy(h)


def test_segments_buffer_too_small():
    h = zr.zr_plan_create(synth.tiny_shapes(), 2, 0, 0, 1 << 20)
    try:
        n = ctypes.c_int64()
        arr = (zr.zr_segment * 2)()
        assert zr.raw_call("zr_plan_segments", h, arr, 2, ctypes.byref(n)) == zr.ZR_ERR_BUFFER_TOO_SMALL
        assert n.value == 5
    finally:
        zr.zr_plan_destroy(h)


def test_workspace_grows_with_clip_scratch():
    shapes = [(1024, 1024)]
    plain = zr.zr_plan_create(shapes, 8, 0, 0, 1 << 20)
    clip8 = zr.zr_plan_create(shapes, 8, 0, 0, 1 << 20, max_grad_norm=1.0)
    clip4 = zr.zr_plan_create(shapes, 4, 0, 0, 1 << 20, max_grad_norm=1.0)
    try:
        b_plain, b8, b4 = (zr.zr_plan_workspace_bytes(h) for h in (plain, clip8, clip4))
        owned8 = (1024 * 1024) // 8
        assert b8 - b_plain >= 4 * owned8          # fp32 g scratch for W > 4
        assert b4 - b_plain < 4 * (1024 * 1024) // 4  # W <= 4 re-reads the gradients instead
    finally:
        for h in (plain, clip8, clip4):
            zr.zr_plan_destroy(h)


def test_checked_mode_arguments_without_a_device():
    """Checked mode's calls reject a missing plan and an unbound workspace
    before touching the device."""
    import ctypes
    assert zr._lib.zr_plan_set_checked(None, 1) == zr.ZR_ERR_INVALID_ARG
    assert zr._lib.zr_plan_verify(None, None) == zr.ZR_ERR_INVALID_ARG
    r = zr.zr_check_result()
    assert zr._lib.zr_plan_check_result(None, ctypes.byref(r), None) == zr.ZR_ERR_INVALID_ARG
    h = zr.zr_plan_create([(4096,), (100,)], 2, 0, 0, 1 << 20)
    try:
        zr.zr_plan_set_checked(h, True)
        zr.zr_plan_set_checked(h, False)
        assert zr._lib.zr_plan_verify(h, None) == zr.ZR_ERR_NO_WORKSPACE
        assert zr._lib.zr_plan_check_result(h, None, None) == zr.ZR_ERR_INVALID_ARG
        assert zr._lib.zr_plan_check_result(h, ctypes.byref(r), None) == zr.ZR_ERR_NO_WORKSPACE
    finally:
        zr.zr_plan_destroy(h)


def test_plan_rejects_wrong_buffers_before_the_library():
    """ZrPlan checks tensor arguments against the plan (the C ABI sees only
    addresses): count, dtype, contiguity, size, then device -- all on the
    host, before any launch."""
    import torch
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    plan = ZrPlan([(4096,), (100,)], 2, 1, 0, 1 << 20, bind=False)
    n, P = plan.owned_numel, plan.padded_numel
    g = [torch.zeros(n, dtype=torch.bfloat16) for _ in range(2)]
    st = [torch.zeros(n, dtype=torch.float32) for _ in range(3)]
    out = torch.zeros(P, dtype=torch.bfloat16)
    cases = [
        ((g[:1], *st, out), ValueError, "W = 2"),
        (([g[0], g[1].float()], *st, out), ValueError, "dtype"),
        ((g, st[0][: n - 1], st[1], st[2], out), ValueError, "at least"),
        ((g, st[0], torch.zeros(2 * n, dtype=torch.float32)[::2], st[2], out), ValueError, "contiguous"),
        ((g, *st, out[: P - 1]), ValueError, "at least"),
        ((g, *st, out), ValueError, "must be on"),                 # host tensors, a device plan
        ((g, st[0], "m", st[2], out), TypeError, "expected a torch tensor"),
    ]
    for args, exc, text in cases:
        with pytest.raises(exc, match=text):
            plan.step(*args, 1)
        with pytest.raises(exc, match=text):
            plan.step_bucket(0, *args, 1)
    meta = torch.zeros(n, dtype=torch.bfloat16, device="meta")
    with pytest.raises(ValueError, match="host_grads\\[0\\]: must be in host memory"):
        plan.step_host([meta, meta], [None, None], None, None, None, None, out, 1)
    with pytest.raises(ValueError, match="g_out: 1 elements"):
        plan.debug_reduce(g, torch.zeros(1, dtype=torch.float32))
    with pytest.raises(ValueError, match="out: dtype"):
        plan.grad_sumsq(g, torch.zeros(1, dtype=torch.float32))
    plan.close()


def test_zero3_calls_without_a_device():
    """The parameter layout switch is host-side until a workspace is bound;
    the gather rejects bad tensor ranges, then an unbound workspace."""
    h = zr.zr_plan_create([(4096,), (0,), (100,)], 2, 0, 1, 1 << 20)
    try:
        zr.zr_plan_set_param_layout(h, zr.ZR_PARAMS_OWNED, 0)
        zr.zr_plan_set_param_layout(h, zr.ZR_PARAMS_GLOBAL, 0)
        assert zr._lib.zr_plan_set_param_layout(h, 5, None) == zr.ZR_ERR_INVALID_ARG
        arr = zr._ptr_array([0, 0])
        for first, n in ((-1, 1), (0, 4), (3, 1), (2, 2), (0, -1)):
            assert zr._lib.zr_gather_params(h, first, n, arr, None, 0, None) == zr.ZR_ERR_INVALID_ARG
        assert zr._lib.zr_gather_params(h, 0, 3, None, None, 0, None) == zr.ZR_ERR_INVALID_ARG
        assert zr._lib.zr_gather_params(h, 0, 3, arr, None, 0, None) == zr.ZR_ERR_NO_WORKSPACE
    finally:
        zr.zr_plan_destroy(h)


def test_grouped_plans_keep_the_clip_scratch():
    """With clipping a grouped plan's workspace holds the fp32 averaged
    gradient at any W (its per-layer gradients are released before the
    norm is known); a plan of the byte-cap rule holds it only for W > 4."""
    shapes = [(4096,), (100,), (2048,)]
    for W, grouped, scratch in ((2, False, False), (2, True, True), (8, False, True), (8, True, True)):
        sizes = []
        for mgn in (0.0, 1.0):
            h = zr.zr_plan_create(shapes, W, 0, 0, 1 << 20, max_grad_norm=mgn,
                                  groups=[0, 1, 2] if grouped else None)
            sizes.append((zr.zr_plan_workspace_bytes(h), zr.zr_plan_query(h)["owned_numel"]))
            zr.zr_plan_destroy(h)
        (plain, n), (clip, _) = sizes
        assert (clip - plain >= 4 * n) == scratch, (W, grouped)


def test_set_adamw_refuses_turning_clipping_on_or_off():
    h = zr.zr_plan_create([(4096,)], 2, 0, 0, 1 << 20)                     # no clipping
    hc = zr.zr_plan_create([(4096,)], 2, 0, 0, 1 << 20, max_grad_norm=1.0)
    try:
        zr.zr_plan_set_adamw(h, lr=1e-3, weight_decay=0.0)
        zr.zr_plan_set_adamw(hc, lr=1e-3, max_grad_norm=0.5)
        for plan, mgn in ((h, 1.0), (hc, 0.0)):
            with pytest.raises(zr.ZrError) as e:
                zr.zr_plan_set_adamw(plan, max_grad_norm=mgn)
            assert e.value.status == zr.ZR_ERR_UNSUPPORTED
        assert zr._lib.zr_plan_set_adamw(h, None) == zr.ZR_ERR_INVALID_ARG
    finally:
        zr.zr_plan_destroy(h)
        zr.zr_plan_destroy(hc)


def test_set_device_lr_arguments():
    h = zr.zr_plan_create([(4096,)], 2, 0, 0, 1 << 20)
    try:
        assert zr._lib.zr_plan_set_device_lr(None, None) == zr.ZR_ERR_INVALID_ARG
        assert zr._lib.zr_plan_set_device_lr(h, 2) == zr.ZR_ERR_ALIGNMENT
        zr.zr_plan_set_device_lr(h, None)
    finally:
        zr.zr_plan_destroy(h)


def test_zero_adamw_rejects_parameters_it_cannot_bind():
    import torch
    from sharded_optimizer_step_zr_b200.optim import ZeroAdamW
    with pytest.raises(ValueError, match="no parameters"):
        ZeroAdamW([])
    with pytest.raises(ValueError, match="bf16 tensors on one CUDA device"):
        ZeroAdamW([torch.nn.Parameter(torch.zeros(4, dtype=torch.float32))])
    with pytest.raises(ValueError, match="bf16 tensors on one CUDA device"):
        ZeroAdamW([torch.nn.Parameter(torch.zeros(4, dtype=torch.bfloat16))])   # host memory


def test_early_argument_errors_of_every_launching_call():
    """Each call that launches work rejects a missing plan, a bad step or
    an unbound workspace before any CUDA call (so these run without a GPU),
    and the IPC calls reject NULL arguments."""
    import ctypes
    L = zr._lib
    h = zr.zr_plan_create([(4096,), (100,)], 2, 0, 0, 1 << 20)
    try:
        g = zr._ptr_array([16, 16])
        step_like = [
            lambda p, t: L.zr_step(p, g, 16, 16, 16, 16, t, None),
            lambda p, t: L.zr_step_bucket(p, 0, g, 16, 16, 16, 16, t, None),
            lambda p, t: L.zr_step_finish(p, g, 16, 16, 16, 16, t, None),
            lambda p, t: L.zr_step_host(p, g, g, 16, 16, 16, 16, 16, t, None),
        ]
        for call in step_like:
            assert call(None, 1) == zr.ZR_ERR_INVALID_ARG
            assert call(h, 0) == zr.ZR_ERR_INVALID_ARG            # steps are 1-based
            assert call(h, 1) == zr.ZR_ERR_NO_WORKSPACE
        assert L.zr_step_device_count(h, g, 16, 16, 16, 16, None, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_step_device_count(h, g, 16, 16, 16, 16, 4, None) == zr.ZR_ERR_ALIGNMENT
        assert L.zr_step_device_count(h, g, 16, 16, 16, 16, 16, None) == zr.ZR_ERR_NO_WORKSPACE
        assert L.zr_grad_sumsq(None, g, 16, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_bucket_sumsq(None, 16, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_bucket_sumsq(h, None, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_bucket_sumsq(h, 16, None) == zr.ZR_ERR_NO_WORKSPACE
        assert L.zr_debug_reduce(None, g, 16, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_step_no_alloc(None, g, 16, 16, 16, 16, None, 1, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_step_no_alloc(h, None, 16, 16, 16, 16, None, 1, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_step_no_alloc(h, zr._ptr_array([16, 8]), 16, 16, 16, 16, None, 1, None) == zr.ZR_ERR_ALIGNMENT
        assert L.zr_plan_set_gather_targets(None, None, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_plan_set_gather_targets(h, g, None) == zr.ZR_ERR_NO_WORKSPACE
        assert L.zr_plan_owner_offsets(h, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_ipc_export(None, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_ipc_open(None, None) == zr.ZR_ERR_INVALID_ARG
        bad = zr.zr_ipc_handle()
        bad.offset, bad.allocation_bytes = 10, 10                # offset outside the allocation
        out = ctypes.c_void_p()
        assert L.zr_ipc_open(ctypes.byref(bad), ctypes.byref(out)) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_ipc_close(None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_state_save(None, b"x", 16, 16, 16, 1, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_state_load(h, None, 16, 16, 16, None, None) == zr.ZR_ERR_INVALID_ARG
        assert L.zr_state_reshard(h, None, 0, b"x") == zr.ZR_ERR_INVALID_ARG
        assert L.zr_state_export_params(h, None, 1, 1, b"x", None) == zr.ZR_ERR_INVALID_ARG
    finally:
        zr.zr_plan_destroy(h)
