"""Checked mode on the GPU: a clean plan verifies clean and steps bit for bit
like an unchecked one; a corrupted device tile table or gather piece table
is found (by an invariant or by its hash) and emptied before a step or a
gather can use it.

No test here runs a step or a gather on a table that could send it out of
bounds: out-of-range corruptions are only verified (then the tables are
re-uploaded), and the corruptions run under checked mode keep every entry
in bounds (two tiles of equal length swap their owned offsets; a piece
reads an earlier part of the same shard)."""
import numpy as np
import pytest
import torch

import sharded_optimizer_step_zr_b200 as zr
from gpu_harness import DEV, GpuRank, bits32

pytestmark = pytest.mark.gpu

HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)
TILE = np.dtype([("owned", "<i8"), ("global", "<i8"), ("len", "<i4"), ("flags", "<i4"),
                 ("bucket", "<i4"), ("index", "<i4")])
assert TILE.itemsize == 32

CLEAN = {"bad_tiles": 0, "first_bad": -1, "hash_mismatch": 0, "tables_emptied": 0}


def read_table(ws, offset, n):
    return ws[offset:offset + 32 * n].cpu().numpy().view(TILE).copy()


def write_table(ws, offset, table):
    ws[offset:offset + table.nbytes].copy_(torch.from_numpy(table.view(np.uint8)).to(ws.device))


def rebind(plan):
    zr.zr_plan_set_workspace(plan.handle, plan.workspace, plan.workspace.numel(), None)


@pytest.mark.parametrize("shapes, W, rank, mode, clip, how", [
    ([(4096 * 3 + 5,), (17,), (64, 65)], 4, 1, 0, 0.0, "step"),
    ([(4097,), (33, 31), (5000,), (3,), (8, 8, 8)], 3, 0, 1, 1.0, "step"),
    ([(2048 * 5,), (300,), (2048 * 3 + 8,)], 2, 1, 0, 1.0, "bucket"),
    ([(2048 * 5,), (300,), (2048 * 3 + 8,)], 8, 3, 0, 0.0, "host"),
])
def test_clean_plan_checked_equals_unchecked(shapes, W, rank, mode, clip, how):
    cap = 4096 * 4
    ranks = [GpuRank(shapes, W, rank, mode, cap, HP, seed=5, max_grad_norm=clip) for _ in range(2)]
    ranks[0].plan.set_checked(True)
    P = max(ranks[0].plan.padded_numel, 8)
    outs = [torch.zeros(P, dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    host_out = [torch.zeros(P, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for g in ranks:
        if clip > 0:
            g.plan.partials.fill_(0.25)
    for t in (1, 2):
        for g, out, ho in zip(ranks, outs, host_out):
            g.fill_grads(t, 1e-2, 0.01)
            if how == "step":
                g.step(out, t)
            elif how == "bucket":
                for b in range(g.plan.n_buckets):
                    g.plan.step_bucket(b, g.grads, g.master, g.m, g.v, out, t)
                g.plan.step_finish(g.grads, g.master, g.m, g.v, out, t)
            else:
                host_grads = [x.cpu().pin_memory() for x in g.grads]
                g.plan.step_host(host_grads, g.grads, g.master, g.m, g.v, out, ho, t)
    torch.cuda.synchronize()
    for a, b in zip(ranks[0].state(), ranks[1].state()):
        assert np.array_equal(bits32(a), bits32(b))
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    if how == "host":
        assert torch.equal(host_out[0].view(torch.int16), host_out[1].view(torch.int16))
    assert ranks[0].plan.check_result() == CLEAN


def test_out_of_range_tile_found_and_tables_emptied():
    """One tile's length pushed past the tile size: the verification names
    it, both tables are emptied, and a re-upload restores a clean plan that
    steps like a fresh one."""
    shapes = [(2048 * 10,)]
    g = GpuRank(shapes, 1, 0, 0, 1 << 30, HP, seed=9)
    ref = GpuRank(shapes, 1, 0, 0, 1 << 30, HP, seed=9)
    ws = g.plan.workspace
    n, by_owned_at = 10, 512                     # ten full tiles; the second table 256-aligned after the first
    tiles = read_table(ws, 0, n)
    assert list(tiles["len"]) == [2048] * n and list(tiles["index"]) == list(range(n))
    g.plan.verify()
    assert g.plan.check_result() == CLEAN
    bad = tiles.copy()
    bad["len"][5] = 4096
    write_table(ws, 0, bad)
    g.plan.verify()                              # verification only: no step on this table
    r = g.plan.check_result()
    assert r == {"bad_tiles": 1, "first_bad": 5, "hash_mismatch": 1, "tables_emptied": 1}
    for off in (0, by_owned_at):
        t = read_table(ws, off, n)
        assert np.all(t["len"] == 0) and np.all(t["flags"] == 0) and list(t["index"]) == list(range(n))
    rebind(g.plan)
    g.plan.set_checked(True)
    out, out_ref = (torch.zeros(2048 * 10, dtype=torch.bfloat16, device=DEV) for _ in range(2))
    for x, o in ((g, out), (ref, out_ref)):
        x.fill_grads(1, 1e-2, 0.0)
        x.step(o, 1)
    torch.cuda.synchronize()
    assert g.plan.check_result() == CLEAN
    for a, b in zip(g.state(), ref.state()):
        assert np.array_equal(bits32(a), bits32(b))
    assert torch.equal(out.view(torch.int16), out_ref.view(torch.int16))


def test_in_bounds_swap_caught_by_the_hash_before_the_step():
    """Two full tiles swap their owned offsets: every invariant still holds
    (the step would silently update the wrong elements), the hash does not.
    Under checked mode the step then changes nothing."""
    shapes = [(2048 * 6,), (2048 * 6,)]
    g = GpuRank(shapes, 2, 0, 0, 1 << 30, HP, seed=3)
    g.plan.set_checked(True)
    ws = g.plan.workspace
    tiles = read_table(ws, 0, 2)
    assert tiles["len"][0] == tiles["len"][1] == 2048 and tiles["owned"][0] != tiles["owned"][1]
    bad = tiles.copy()
    bad["owned"][0], bad["owned"][1] = tiles["owned"][1], tiles["owned"][0]
    write_table(ws, 0, bad)
    before = [x.copy() for x in g.state()]
    sentinel = -16447
    out = torch.full((g.plan.padded_numel,), sentinel, dtype=torch.int16, device=DEV)
    g.fill_grads(1, 1e-2, 0.0)
    g.step(out.view(torch.bfloat16), 1)
    torch.cuda.synchronize()
    assert g.plan.check_result() == {"bad_tiles": 0, "first_bad": -1, "hash_mismatch": 1, "tables_emptied": 1}
    for a, b in zip(g.state(), before):
        assert np.array_equal(bits32(a), bits32(b))
    assert bool(torch.all(out == sentinel))


def _layout_no_clip(n_tiles, n_pieces, W):
    """Byte offsets of the workspace regions of a plan without clipping
    (each region 256-byte aligned, in this order): tile table, owned-order
    tile table, clip partials (empty), clip coefficient, own sum of squares,
    gather targets, device scalars, checked-mode status, gather pieces."""
    up = lambda x: (x + 255) // 256 * 256
    off = {"tiles": 0}
    off["by_owned"] = up(32 * max(1, n_tiles))
    partials = up(off["by_owned"] + 32 * max(1, n_tiles))
    clip_coef = partials
    own = up(clip_coef + 4)
    targets = up(own + 8)
    scalars = up(targets + 8 * W)
    check = up(scalars + 32)
    off["pieces"] = up(check + 8 * 7)
    off["total"] = up(off["pieces"] + 32 * max(1, n_pieces))
    return off


PIECE = np.dtype([("src", "<i8"), ("dst", "<i8"), ("len", "<i4"), ("owner", "<i4"), ("tensor", "<i4"),
                  ("reserved", "<i4")])


def test_gather_pieces_checked():
    """The gather piece table under checked mode: an out-of-range piece is
    found and the table emptied (only verified, never gathered from); an
    in-bounds change is caught by the hash and the checked gather writes
    nothing; a re-upload restores a clean gather."""
    shapes = [(2048 * 10,)]
    g = GpuRank(shapes, 1, 0, 0, 1 << 30, HP, seed=9)
    off = _layout_no_clip(10, 2, 1)
    assert g.plan.workspace_bytes == off["total"]
    ws = g.plan.workspace
    pieces = ws[off["pieces"]:off["pieces"] + 64].cpu().numpy().view(PIECE).copy()
    assert list(pieces["len"]) == [16384, 4096] and list(pieces["src"]) == [0, 16384]
    shard = torch.randn(2048 * 10, device=DEV).to(torch.bfloat16)
    g.plan.set_checked(True)
    dst = torch.zeros(2048 * 10, dtype=torch.bfloat16, device=DEV)
    g.plan.gather_params(0, 1, [shard], dst)
    torch.cuda.synchronize()
    assert torch.equal(dst.view(torch.int16), shard.view(torch.int16)) and g.plan.check_result() == CLEAN
    # out of range: verified only
    bad = pieces.copy()
    bad["len"][1] = 40000
    ws[off["pieces"]:off["pieces"] + 64].copy_(torch.from_numpy(bad.view(np.uint8)).to(DEV))
    g.plan.verify()
    assert g.plan.check_result() == {"bad_tiles": 1, "first_bad": 2 * 10 + 1, "hash_mismatch": 4,
                                     "tables_emptied": 1}
    emptied = ws[off["pieces"]:off["pieces"] + 64].cpu().numpy().view(PIECE)
    assert np.all(emptied["len"] == 0)
    rebind(g.plan)
    # in bounds (piece 1 now reads the shard's first 4096 elements): the hash
    moved = pieces.copy()
    moved["src"][1] = 0
    ws[off["pieces"]:off["pieces"] + 64].copy_(torch.from_numpy(moved.view(np.uint8)).to(DEV))
    sentinel = torch.full((2048 * 10,), -16447, dtype=torch.int16, device=DEV)
    g.plan.gather_params(0, 1, [shard], sentinel.view(torch.bfloat16))
    torch.cuda.synchronize()
    assert g.plan.check_result() == {"bad_tiles": 0, "first_bad": -1, "hash_mismatch": 4, "tables_emptied": 1}
    assert bool(torch.all(sentinel == -16447))
    rebind(g.plan)
    dst.zero_()
    g.plan.gather_params(0, 1, [shard], dst)
    torch.cuda.synchronize()
    assert torch.equal(dst.view(torch.int16), shard.view(torch.int16)) and g.plan.check_result() == CLEAN
