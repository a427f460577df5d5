"""ZeRO across processes over shared device memory (CUDA IPC), on the one
GPU this suite has: two processes, one rank each.  Each rank's fused step
reads its slice of both replicas' gradient buffers through IPC mappings (the
reduce-scatter) and stores its bf16 results into both ranks' parameter
buffers (the all-gather); barriers on the host order the phases, and no
kernel waits on the other process.  Results must equal the oracle's: the
rank's fp32 state bit for bit, and both full parameter buffers bit for bit
against the unsharded step."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, shapes, mode, max_norm, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch
    import torch.distributed as dist
    import oracle
    import synth
    from sharded_optimizer_step_zr_b200.peer import PeerZero
    import datetime
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=90))
    try:
        hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, max_norm)
        pz = PeerZero(dist.group.WORLD, shapes, mode, 4096, *hp)
        segs = pz.plan.segments()
        N, P = pz.plan.total_numel, pz.plan.padded_numel
        runs_of = [synth.rank_runs(segs, r) for r in range(world)]
        n = pz.plan.owned_numel
        master = torch.empty(max(n, 8), dtype=torch.float32, device="cuda:0")
        synth.fill_owned_master(master, runs_of[rank], 4, n_valid=N)
        m, v = torch.zeros_like(master), torch.zeros_like(master)
        oplan = oracle.Plan(shapes, world, mode, 4096)
        idx_all = torch.arange(P, dtype=torch.int64)
        o_master = synth.master_f32(4, idx_all, n_valid=N).numpy().copy()
        o_m, o_v = np.zeros(P, np.float32), np.zeros(P, np.float32)
        o_out = np.zeros(P, np.uint16)
        for t in (1, 2):
            # this process is replica `rank`: its full gradient, owner-major
            for r in range(world):
                a, b = pz.offsets[r], pz.offsets[r + 1]
                synth.fill_owned_grad(pz.grad_buffer[a:b], runs_of[r], 4, t, rank, 1e-2, 0.01, n_valid=N)
            pz.step(master, m, v, t)
            reps = [synth.grad_bf16(4, t, w, idx_all, 1e-2, 0.01, n_valid=N).view(torch.int16).numpy()
                    .view(np.uint16).copy() for w in range(world)]
            c = None
            if max_norm > 0:
                c = oracle.clip_coef(oracle.sumsq(oracle.reduce([x[:N] for x in reps])), max_norm)
            oracle.ddp_step(reps, o_master, o_m, o_v, o_out, hp, t, clip=c)
        gi = oplan.owned_global_index(rank)
        same_state = all(np.array_equal(x[:n].cpu().numpy().view(np.uint32), y[gi].view(np.uint32))
                         for x, y in ((master, o_master), (m, o_m), (v, o_v)))
        close_state = all(np.allclose(x[:n].cpu().numpy(), y[gi], rtol=2e-6, atol=1e-9)
                          for x, y in ((master, o_master), (m, o_m), (v, o_v)))
        got = pz.param_buffer[:P].cpu().view(torch.int16).numpy().view(np.uint16)
        ulp = int(np.max(np.abs(got.astype(np.int64) - o_out.astype(np.int64)))) if P else 0
        q.put((rank, bool(same_state), bool(close_state), ulp, bool(np.array_equal(got, o_out))))
        pz.close()
    except Exception as e:  # report, do not hang the other rank's barrier forever
        q.put((rank, "error", repr(e), None, None))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shapes, mode, max_norm", [
    ([(300, 7), (1001,), (64, 64), (4099,)], 0, 0.0),
    ([(300, 7), (1001,), (64, 64), (4099,), (17,)], 1, 0.0),
    ([(300, 7), (1001,), (64, 64), (4099,)], 0, 0.05),
])
def test_two_processes_share_one_gpu(shapes, mode, max_norm):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, shapes, mode, max_norm, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    for r in results:
        assert r[1] != "error", r
        rank, same_state, close_state, ulp, same_out = r
        assert close_state, r
        assert ulp <= 1, r
        if max_norm == 0:
            assert same_state and same_out, r
    assert all(p.exitcode == 0 for p in procs)


def _rank_main_stage3(rank, world, port, shapes, mode, q):
    """Stage 3 over IPC: each rank writes only its bf16 shard; after the
    step every rank gathers whole tensors from both shards (one through a
    peer mapping)."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch
    import torch.distributed as dist
    import oracle
    import synth
    from sharded_optimizer_step_zr_b200.peer import PeerZero
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=90))
    try:
        hp = (3e-4, 0.9, 0.999, 1e-8, 0.1, 0.0)
        pz = PeerZero(dist.group.WORLD, shapes, mode, 4096, *hp, stage=3)
        segs = pz.plan.segments()
        N, P = pz.plan.total_numel, pz.plan.padded_numel
        runs_of = [synth.rank_runs(segs, r) for r in range(world)]
        n = pz.plan.owned_numel
        master = torch.empty(max(n, 8), dtype=torch.float32, device="cuda:0")
        synth.fill_owned_master(master, runs_of[rank], 6, n_valid=N)
        m, v = torch.zeros_like(master), torch.zeros_like(master)
        idx_all = torch.arange(P, dtype=torch.int64)
        o_master = synth.master_f32(6, idx_all, n_valid=N).numpy().copy()
        o_m, o_v = np.zeros(P, np.float32), np.zeros(P, np.float32)
        o_out = np.zeros(P, np.uint16)
        for t in (1, 2):
            for r in range(world):
                a, b = pz.offsets[r], pz.offsets[r + 1]
                synth.fill_owned_grad(pz.grad_buffer[a:b], runs_of[r], 6, t, rank, 1e-2, 0.01, n_valid=N)
            pz.step(master, m, v, t)
            reps = [synth.grad_bf16(6, t, w, idx_all, 1e-2, 0.01, n_valid=N).view(torch.int16).numpy()
                    .view(np.uint16).copy() for w in range(world)]
            oracle.ddp_step(reps, o_master, o_m, o_v, o_out, hp, t)
        full = torch.full((max(N, 8),), -1, dtype=torch.int16, device="cuda:0")
        pz.gather(0, len(shapes), full.view(torch.bfloat16))
        numels = [int(np.prod(s)) for s in shapes]
        goff = np.concatenate([[0], np.cumsum(numels)])
        one = torch.zeros(max(numels[2], 8), dtype=torch.bfloat16, device="cuda:0")
        pz.bound_gather(2, 1, one, max_ctas=4)()
        torch.cuda.synchronize()
        got = full[:N].cpu().numpy().view(np.uint16)
        got_one = one[:numels[2]].cpu().view(torch.int16).numpy().view(np.uint16)
        gi = oracle.Plan(shapes, world, mode, 4096).owned_global_index(rank)
        shard = pz.param_shard.cpu().view(torch.int16).numpy().view(np.uint16)
        q.put((rank, bool(np.array_equal(got, o_out[:N])),
               bool(np.array_equal(got_one, o_out[goff[2]:goff[3]])),
               bool(np.array_equal(shard, o_out[gi]))))
        dist.barrier()                       # nobody unmaps a shard another rank still reads
        pz.close()
    except Exception as e:
        q.put((rank, "error", repr(e), None))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shapes, mode", [
    ([(300, 7), (1001,), (64, 64), (4099,)], 0),
    ([(300, 7), (1001,), (64, 64), (4099,), (17,)], 1),
])
def test_two_processes_stage3_gather(shapes, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_main_stage3, args=(r, 2, port, shapes, mode, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    for r in results:
        assert r[1] != "error", r
        assert r[1] and r[2] and r[3], r
    assert all(p.exitcode == 0 for p in procs)


def _rank_main_optim(rank, world, port, q, max_norm=0.0, overlap=False):
    """ZeroAdamW over a two-process group: the same bf16 model on both
    ranks, different data; after each step both models equal the oracle's
    unsharded step on the two replicas' gradients (within 1 ulp with
    clipping).  overlap: each bucket stepped as the backward fills it, its
    reduce reading the other replica's gradients through IPC."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch
    import torch.distributed as dist
    import oracle
    from sharded_optimizer_step_zr_b200.optim import ZeroAdamW
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=90))
    try:
        torch.manual_seed(5)
        model = torch.nn.Sequential(torch.nn.Linear(64, 128), torch.nn.GELU(), torch.nn.Linear(128, 24),
                                    torch.nn.LayerNorm(24)).to("cuda:0").to(torch.bfloat16)
        params = list(model.parameters())
        flat = lambda ts: torch.cat([t.detach().reshape(-1) for t in ts]).cpu().view(torch.int16).numpy() \
            .view(np.uint16).copy()
        init = flat(params)
        hp = (1e-3, 0.9, 0.999, 1e-8, 0.1, max_norm)
        opt = ZeroAdamW(params, group=dist.group.WORLD, lr=hp[0], weight_decay=hp[4], bucket_cap_mb=0.01,
                        max_grad_norm=max_norm, overlap=overlap)
        N = init.size
        o_master = (init.astype(np.uint32) << 16).view(np.float32).copy()
        o_m, o_v, o_out = np.zeros(N, np.float32), np.zeros(N, np.float32), np.zeros(N, np.uint16)
        gen = torch.Generator(device="cuda:0").manual_seed(100 + rank)
        ok = True
        for t in (1, 2, 3):
            x = torch.randn(16, 64, device="cuda:0", generator=gen).to(torch.bfloat16)
            model(x).float().pow(2).mean().backward()
            torch.cuda.synchronize()
            mine = flat([p.grad for p in params])
            reps = [None] * world
            dist.all_gather_object(reps, mine)
            c = oracle.clip_coef(oracle.sumsq(oracle.reduce(reps)), max_norm) if max_norm > 0 else None
            oracle.ddp_step(reps, o_master, o_m, o_v, o_out, hp, t, clip=c)
            opt.step()
            opt.zero_grad()
            torch.cuda.synchronize()
            got = flat(params)
            if max_norm > 0:
                d = np.abs(got.astype(np.int64) - o_out.astype(np.int64))
                ok = ok and int(d.max()) <= 1
            else:
                ok = ok and bool(np.array_equal(got, o_out))
        q.put((rank, ok, len(opt._copy_in)))
        dist.barrier()
        opt.close()
    except Exception as e:
        q.put((rank, "error", repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("max_norm, overlap", [(0.0, False), (0.0, True), (0.05, True)])
def test_zero_adamw_two_processes(max_norm, overlap):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_main_optim, args=(r, 2, port, q, max_norm, overlap)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    for r in results:
        assert r[1] is True, r
    assert all(p.exitcode == 0 for p in procs)


def _rank_main_zero3(rank, world, port, q, partition="flat", max_norm=0.0):
    """Zero3 over a two-process group: parameters gathered from both ranks'
    shards (one through IPC) before each module's forward and backward;
    after every step the gathered model equals the oracle's unsharded step
    on the two replicas' gradients.  Beside it, on a copy of the model, the
    same job with reduce_in_backward (each module's slice reduced from both
    replicas' gradient slots through IPC and applied during the backward):
    its gathered model equals the first one bit for bit after every step."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch
    import torch.distributed as dist
    import oracle
    from sharded_optimizer_step_zr_b200.optim import Zero3
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from gpu_harness import bf16_ulp_distance
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=90))
    try:
        torch.manual_seed(6)
        model = torch.nn.Sequential(torch.nn.Linear(64, 128), torch.nn.GELU(), torch.nn.Linear(128, 96),
                                    torch.nn.LayerNorm(96), torch.nn.Linear(96, 24)).to("cuda:0").to(torch.bfloat16)
        flat = lambda ts: torch.cat([t.detach().reshape(-1) for t in ts]).cpu().view(torch.int16).numpy() \
            .view(np.uint16).copy()
        init = flat(model.parameters())
        hp = (1e-3, 0.9, 0.999, 1e-8, 0.1, max_norm)
        torch.manual_seed(6)
        model2 = torch.nn.Sequential(torch.nn.Linear(64, 128), torch.nn.GELU(), torch.nn.Linear(128, 96),
                                     torch.nn.LayerNorm(96), torch.nn.Linear(96, 24)).to("cuda:0").to(torch.bfloat16)
        z = Zero3(model, group=dist.group.WORLD, lr=hp[0], weight_decay=hp[4], bucket_cap_mb=0.01,
                  partition=partition, max_grad_norm=max_norm)
        z2 = Zero3(model2, group=dist.group.WORLD, lr=hp[0], weight_decay=hp[4], partition=partition,
                   reduce_in_backward=True, max_grad_norm=max_norm)
        N = init.size
        full2 = torch.empty(N, dtype=torch.bfloat16, device="cuda:0")
        o_master = (init.astype(np.uint32) << 16).view(np.float32).copy()
        o_m, o_v, o_out = np.zeros(N, np.float32), np.zeros(N, np.float32), np.zeros(N, np.uint16)
        gen = torch.Generator(device="cuda:0").manual_seed(300 + rank)
        ok = True
        full = torch.empty(N, dtype=torch.bfloat16, device="cuda:0")
        for t in (1, 2, 3):
            x = torch.randn(16, 64, device="cuda:0", generator=gen).to(torch.bfloat16)
            model(x).float().pow(2).mean().backward()
            torch.cuda.synchronize()
            mine = flat([p.grad for p in z.params])
            reps = [None] * world
            dist.all_gather_object(reps, mine)
            c = oracle.clip_coef(oracle.sumsq(oracle.reduce(reps)), max_norm) if max_norm > 0 else None
            oracle.ddp_step(reps, o_master, o_m, o_v, o_out, hp, t, clip=c)
            z.step()
            z.zero_grad()
            z.gather_all(full)
            model2(x).float().pow(2).mean().backward()
            z2.step()
            z2.gather_all(full2)
            torch.cuda.synchronize()
            got = full.cpu().view(torch.int16).numpy().view(np.uint16)
            got2 = full2.cpu().view(torch.int16).numpy().view(np.uint16)
            if max_norm > 0:
                # the norm's fp64 sums run in other orders (oracle, byte-cap and grouped plans)
                ok = ok and int(bf16_ulp_distance(got, o_out).max()) <= 1
                ok = ok and int(bf16_ulp_distance(got2, got).max()) <= 1
            else:
                ok = ok and bool(np.array_equal(got, o_out))
                ok = ok and bool(np.array_equal(got2, got))
        q.put((rank, ok))
        dist.barrier()
        z.close()
        z2.close()
    except Exception as e:
        q.put((rank, "error", repr(e)))
        raise
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("partition, max_norm", [("flat", 0.0), ("whole", 0.0), ("flat", 0.01)])
def test_zero3_module_two_processes(partition, max_norm):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_rank_main_zero3, args=(r, 2, port, q, partition, max_norm)) for r in range(2)]
    for p in procs:
        p.start()
    results = [q.get(timeout=240) for _ in range(2)]
    for p in procs:
        p.join(timeout=60)
    for r in results:
        assert r[1] is True, r
    assert all(p.exitcode == 0 for p in procs)


def _failing_set_up_main(rank, world, port, q):
    """Rank 1 cannot map its peer's buffer (the IPC call replaced by one that
    fails, on the host); both ranks must leave the set-up with PeerFailure
    and keep a working process group."""
    import sys
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    import torch
    import torch.distributed as dist
    import sharded_optimizer_step_zr_b200.peer as peer
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        if rank == 1:
            def refuse(handle):
                raise RuntimeError("zr_ipc_open: mapping refused")
            peer.zr_ipc_open = refuse
        try:
            peer.PeerZero(dist.group.WORLD, [(300, 7), (1001,)], 0, 4096)
            outcome = "constructed"
        except peer.PeerFailure as e:
            outcome = str(e)
        dist.barrier()                       # the group still works after the failure
        q.put((rank, outcome))
    except Exception as e:                   # noqa: BLE001 -- reported to the test
        q.put((rank, f"error {type(e).__name__}: {e}"))
    finally:
        dist.destroy_process_group()


def test_set_up_failure_on_one_rank_reaches_every_rank():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _port()
    procs = [ctx.Process(target=_failing_set_up_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=240) for _ in range(2))
    for p in procs:
        p.join(timeout=60)
    assert "this rank" in results[1] and "mapping refused" in results[1], results
    assert "another rank" in results[0], results
