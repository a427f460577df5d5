"""zr_state_reshard (host only): elastic resume on a different partition.

The ZeRO state of element g is the same whichever rank owns it (the sharded
step equals the unsharded one bit for bit -- "CS336 lecture 8", ZeRO-1
sketch), so the oracle's unsharded state after a few steps gives the
expected content of every shard of every partition.  Source shards are
written by an independent implementation of the documented format.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synth
import sharded_optimizer_step_zr_b200 as zr
from shard_format import read_shard, write_shard

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)
SHAPES = [(300, 7), (1001,), (64, 64), (17,), (5, 5, 5)]


def unsharded_state(steps=2, seed=5):
    plan = oracle.Plan(SHAPES, 1, oracle.FLAT, 1 << 30)
    N = plan.total_numel
    idx = torch.arange(N, dtype=torch.int64)
    master = synth.master_f32(seed, idx).numpy().copy()
    m, v = np.zeros(N, np.float32), np.zeros(N, np.float32)
    out = np.zeros(N, np.uint16)
    for t in range(1, steps + 1):
        reps = [synth.grad_bf16(seed, t, w, idx, 1e-2, 0.01).view(torch.int16).numpy()
                .view(np.uint16).copy() for w in range(4)]
        oracle.ddp_step(reps, master, m, v, out, HP, t)
    return N, master, m, v


def shard_of(state, plan, rank):
    N, master, m, v = state
    idx = plan.owned_global_index(rank)
    pad = idx >= N
    take = np.where(pad, 0, idx)
    return [np.where(pad, 0.0, a[take]).astype(np.float32) for a in (master, m, v)]


def write_partition(tmp_path, state, W, mode, step, tag):
    plan = oracle.Plan(SHAPES, W, mode, 4096)
    numels = [synth.numel(s) for s in SHAPES]
    paths = []
    for r in range(W):
        ma, mm, vv = shard_of(state, plan, r)
        p = os.path.join(tmp_path, f"{tag}_r{r}.zrs")
        write_shard(p, numels, W, r, mode, plan.total_numel, plan.padded_numel, ma, mm, vv, step, HP)
        paths.append(p)
    return paths


@pytest.mark.parametrize("src, dst", [((4, 0), (3, 1)), ((3, 1), (5, 0)), ((2, 0), (1, 0)),
                                      ((5, 1), (8, 1)), ((1, 0), (4, 0))])
def test_reshard_matches_the_unsharded_state(tmp_path, src, dst):
    state = unsharded_state()
    paths = write_partition(str(tmp_path), state, src[0], src[1], 2, "src")
    W2, mode2 = dst
    oplan = oracle.Plan(SHAPES, W2, mode2, 4096)
    for r in range(W2):
        h = zr.zr_plan_create(SHAPES, W2, r, mode2, 4096)
        try:
            out = os.path.join(str(tmp_path), f"dst_r{r}.zrs")
            zr.zr_state_reshard(h, paths, out)
        finally:
            zr.zr_plan_destroy(h)
        got = read_shard(out)
        assert (got["world_size"], got["rank"], got["mode"], got["step"]) == (W2, r, mode2, 2)
        want = shard_of(state, oplan, r)
        for a, b in zip((got["master"], got["m"], got["v"]), want):
            assert np.array_equal(a.view(np.uint32), b.view(np.uint32))


def test_reshard_rejects_inconsistent_sets(tmp_path):
    state = unsharded_state(steps=1)
    paths = write_partition(str(tmp_path), state, 3, 0, 1, "a")
    h = zr.zr_plan_create(SHAPES, 2, 0, 0, 4096)
    out = os.path.join(str(tmp_path), "out.zrs")
    try:
        # missing rank
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_reshard(h, paths[:2], out)
        assert e.value.status == zr.ZR_ERR_MISMATCH
        # ranks out of order
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_reshard(h, [paths[1], paths[0], paths[2]], out)
        assert e.value.status == zr.ZR_ERR_MISMATCH
        # a shard from another step
        other = write_partition(str(tmp_path), state, 3, 0, 7, "b")
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_reshard(h, [paths[0], other[1], paths[2]], out)
        assert e.value.status == zr.ZR_ERR_MISMATCH
        # a corrupted payload byte
        raw = bytearray(open(paths[1], "rb").read())
        raw[300] ^= 0x40
        bad = os.path.join(str(tmp_path), "bad.zrs")
        open(bad, "wb").write(bytes(raw))
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_reshard(h, [paths[0], bad, paths[2]], out)
        assert e.value.status == zr.ZR_ERR_MISMATCH
        # shards of other tensors
        hx = zr.zr_plan_create([(10,), (20,)], 2, 0, 0, 4096)
        try:
            with pytest.raises(zr.ZrError) as e:
                zr.zr_state_reshard(hx, paths, out)
            assert e.value.status == zr.ZR_ERR_MISMATCH
        finally:
            zr.zr_plan_destroy(hx)
        # a file that does not exist
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_reshard(h, [paths[0], os.path.join(str(tmp_path), "nope"), paths[2]], out)
        assert e.value.status == zr.ZR_ERR_IO
        assert not os.path.exists(out)
    finally:
        zr.zr_plan_destroy(h)


SPECIAL = np.array([0x3F808000, 0x3F818000, 0x3F80C000, 0x80000000, 0x00000001, 0x807FFFFF, 0x7F7FFFFF,
                    0xFF7FFFFF, 0x7F800000, 0xFF800000, 0x7FC00000, 0xFF812345, 0x7F800001, 0x3F7FFFFF],
                   dtype=np.uint32).view(np.float32)


@pytest.mark.parametrize("W, mode", [(4, 0), (3, 1), (1, 0), (8, 0)])
def test_export_params_gathers_the_whole_model(tmp_path, W, mode):
    """zr_state_export_params: the whole model's master weights in
    declaration order from a shard set, as fp32 (the unsharded state bit for
    bit) and as bf16 (the oracle's RNE of it); special values -- ties,
    signed zeros, subnormals, the largest finite values, infinities and NaNs
    -- are planted in the state to pin the rounding."""
    N, master, m, v = unsharded_state()
    master = master.copy()
    pos = np.random.default_rng(W * 10 + mode).choice(N, size=SPECIAL.size, replace=False)
    master[pos] = SPECIAL
    paths = write_partition(str(tmp_path), (N, master, m, v), W, mode, 2, "src")
    h = zr.zr_plan_create(SHAPES, 2, 1, 1 - mode, 4096)      # any plan of the same tensors
    try:
        f32 = os.path.join(str(tmp_path), "model_f32.bin")
        b16 = os.path.join(str(tmp_path), "model_bf16.bin")
        assert zr.zr_state_export_params(h, paths, zr.ZR_EXPORT_F32, f32) == N
        assert zr.zr_state_export_params(h, paths, zr.ZR_EXPORT_BF16, b16) == N
    finally:
        zr.zr_plan_destroy(h)
    got32 = np.fromfile(f32, dtype="<u4")
    got16 = np.fromfile(b16, dtype="<u2")
    assert got32.size == N and got16.size == N
    assert np.array_equal(got32, master.view(np.uint32))
    want16 = oracle.f32_to_bf16_array(master)
    nan = np.isnan(master)
    assert np.array_equal(got16[~nan], want16[~nan])
    # a NaN stays a NaN of the same sign
    assert np.all((got16[nan] & 0x7F80) == 0x7F80) and np.all(got16[nan] & 0x007F)
    assert np.array_equal(got16[nan] >> 15, want16[nan] >> 15)


def test_export_params_rejects_bad_sets(tmp_path):
    state = unsharded_state(steps=1)
    paths = write_partition(str(tmp_path), state, 3, 0, 1, "a")
    h = zr.zr_plan_create(SHAPES, 3, 0, 0, 4096)
    out = os.path.join(str(tmp_path), "model.bin")
    try:
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_export_params(h, paths[:2], zr.ZR_EXPORT_BF16, out)
        assert e.value.status == zr.ZR_ERR_MISMATCH
        with pytest.raises(zr.ZrError) as e:
            zr.zr_state_export_params(h, paths, 7, out)
        assert e.value.status == zr.ZR_ERR_INVALID_ARG
        hx = zr.zr_plan_create([(10,), (20,)], 2, 0, 0, 4096)
        try:
            with pytest.raises(zr.ZrError) as e:
                zr.zr_state_export_params(hx, paths, zr.ZR_EXPORT_F32, out)
            assert e.value.status == zr.ZR_ERR_MISMATCH
        finally:
            zr.zr_plan_destroy(hx)
        assert not os.path.exists(out)
    finally:
        zr.zr_plan_destroy(h)
