"""N > 1 host logic on the CPU: two gloo processes, each one ZeRO rank.

Each process builds libzr.so's plan for its own rank (host-only planner),
steps its owned slice with the oracle on the same seeded inputs, and the
ranks all-gather their bf16 slices ("CS336 lecture 8", ZeRO-1 sketch: the
final all-gather of the updated slices).  Rank 0 checks the gathered buffer
against the unsharded data-parallel step, and the benchmark's rank mapping
and max / sum timing reduction are exercised over the real process group.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HP = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, shapes, mode, result_q):
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    import synth
    import bench
    import sharded_optimizer_step_zr_b200 as zr
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W = world
        # the library's plan for this rank (host tables only)
        h = zr.zr_plan_create(shapes, W, rank, mode, 4096)
        info = zr.zr_plan_query(h)
        segs = zr.zr_plan_segments(h)
        zr.zr_plan_destroy(h)
        runs = synth.rank_runs(segs, rank)
        n = info["owned_numel"]
        P = info["padded_numel"]
        idx = np.zeros(n, dtype=np.int64)
        for owned, glob, length in runs:
            idx[owned: owned + length] = np.arange(glob, glob + length)
        oplan = oracle.Plan(shapes, W, mode, 4096)
        master = synth.master_f32(3, torch.from_numpy(idx), n_valid=info["total_numel"]).numpy().copy()
        m = np.zeros_like(master)
        v = np.zeros_like(master)
        out = np.zeros(P, dtype=np.uint16)
        for t in (1, 2):
            grads = [synth.grad_bf16(3, t, w, torch.from_numpy(idx), 1e-2, 0.01,
                                     n_valid=info["total_numel"]).view(torch.int16).numpy()
                     .view(np.uint16).copy() for w in range(W)]
            oracle.rank_step(oplan, rank, grads, master, m, v, out, HP, t)
        # the all-gather of this rank's positions of the parameter buffer
        mine = torch.zeros(P, dtype=torch.int32)
        mine[torch.from_numpy(idx)] = torch.from_numpy(out[idx].astype(np.int32))
        gathered = [torch.zeros(P, dtype=torch.int32) for _ in range(W)]
        dist.all_gather(gathered, mine)
        full = torch.stack(gathered).sum(0).numpy().astype(np.uint16)
        # benchmark helpers over the real group
        wl = synth.WORKLOADS["gpt2_124m_w8"]
        zr_rank = bench.shard_rank(wl, rank, world)
        ms, owned = bench.reduce_timing(dist, 10.0 + rank, 100 * (rank + 1), torch.device("cpu"))
        result_q.put((rank, zr_rank, ms, owned, full if rank == 0 else None))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("mode", [0, 1])
def test_two_ranks_gather_equals_unsharded(mode):
    import oracle
    import synth
    shapes = [(300, 7), (1001,), (64, 64), (17,)]
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, shapes, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        r, zr_rank, ms, owned, full = q.get(timeout=180)
        results[r] = (zr_rank, ms, owned, full)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # rank mapping: consecutive ZeRO ranks starting at the workload's rank
    assert [results[r][0] for r in range(world)] == [0, 1]
    # timing reduction: max of the times, sum of the work
    for r in range(world):
        assert results[r][1] == 11.0 and results[r][2] == 300.0
    # the gathered buffer equals the unsharded step
    plan = oracle.Plan(shapes, world, mode, 4096)
    P = plan.padded_numel
    idx = torch.arange(P, dtype=torch.int64)
    master = synth.master_f32(3, idx, n_valid=plan.total_numel).numpy().copy()
    m, v = np.zeros(P, np.float32), np.zeros(P, np.float32)
    out = np.zeros(P, np.uint16)
    for t in (1, 2):
        full = [synth.grad_bf16(3, t, w, idx, 1e-2, 0.01, n_valid=plan.total_numel)
                .view(torch.int16).numpy().view(np.uint16).copy() for w in range(world)]
        oracle.ddp_step(full, master, m, v, out, HP, t)
    assert np.array_equal(results[0][3], out)


def _failure_worker(rank, world, port, how, result_q):
    import sys
    import datetime
    import time
    sys.path.insert(0, ROOT)
    from sharded_optimizer_step_zr_b200.peer import PeerFailure, sync_point
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=5))
    sync_point(dist, None, "gradients ready", 1)         # step 1: everyone arrives
    if rank == 1:
        if how == "exit":
            os._exit(0)                                  # a crash between steps: no clean shutdown
        time.sleep(20)                                   # a rank that never arrives in time
        os._exit(0)
    t0 = time.time()
    try:
        sync_point(dist, None, "gradients ready", 2)
        result_q.put(("no error", time.time() - t0))
    except PeerFailure as e:
        result_q.put((str(e), time.time() - t0))
    result_q.close()
    result_q.join_thread()                               # the message is sent before the hard exit
    os._exit(0)


@pytest.mark.parametrize("how", ["exit", "hang"])
def test_missing_peer_raises_before_the_next_launch(how):
    """A peer that dies between steps, or never arrives, ends the next
    phase boundary with PeerFailure on the surviving rank (within the
    group's 5 s timeout plus slack), instead of a hang or a launch that
    would touch the peer's memory."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_failure_worker, args=(r, 2, port, how, q)) for r in range(2)]
    for p in procs:
        p.start()
    msg, waited = q.get(timeout=120)
    for p in procs:
        p.join(timeout=60)
    assert msg.startswith("step 2, gradients ready: a peer did not arrive"), msg
    assert waited < 30


def _bench_ctx_worker(rank, world, port, result_q):
    import sys
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    import synth
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    args = argparse.Namespace(backend="gloo", same_gpu=False)
    ctx = bench.ProcessContext(args, use_cuda=False)
    try:
        # the launch logic of `bench.py --gpus N`: each process one rank of
        # the peer step's W = N job over the workload's parameter set
        shapes = synth.PARAM_SETS["gpt2_124m"]()
        plan = ZrPlan(shapes, ctx.world, ctx.grank, 0, 25 << 20, bind=False)
        n, padded = plan.owned_numel, plan.padded_numel
        plan.close()
        moved = bench.peer_bytes(ctx.world, n)
        ctx.barrier()
        ms, owned = ctx.reduce(5.0 * (rank + 1), n)
        # a step that failed on one process is skipped by every process
        agreed = (ctx.all_ok(True), ctx.all_ok(rank != 1), ctx.all_ok(rank != 0))
        result_q.put((rank, ctx.grank, ctx.world, n, padded, moved, ms, owned, agreed))
    finally:
        ctx.close()


def test_bench_process_context_and_peer_accounting():
    """bench.py's N > 1 plumbing over a real gloo group on the CPU: each
    process's rank, the peer step's owned slices covering the padded set
    (flat, W = 2), the bytes each rank moves over peers, and the max / sum
    reduction of the timings, and the agreement on a step that failed on
    one process."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bench_ctx_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=180)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [res[r][1] for r in range(world)] == [0, 1] and all(res[r][2] == 2 for r in range(world))
    n0, padded = res[0][3], res[0][4]
    assert n0 + res[1][3] == padded == 124439808
    assert res[0][5] == {"peer_loads": 2 * n0, "peer_stores": 2 * n0, "local_hbm": 28 * n0}
    for r in range(world):
        assert res[r][6] == 10.0 and res[r][7] == float(padded)
        assert res[r][8] == (True, False, False)
