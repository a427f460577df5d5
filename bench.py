"""Benchmark of the fused ZeRO-1/2 sharded optimizer step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl zr|reference]
                    [--config NAME] [--no-cpu-baseline] [--no-companions]

One step = one zr_step() call on one rank's owned shard: the W-replica bf16
gradient reduce, (the global-norm clip when the workload has it), AdamW on
the fp32 master / m / v, and the bf16 write into the all-gather buffer.
Inputs are seeded synthetic data resident in HBM before the timed region;
each step's bytes exceed the 126 MB L2, so no flush is needed between steps.

The headline is the Llama-7B-shaped shard at W = 64 (105 M owned params,
154 B each); the GPT-2-small flat W = 8 shard and the 1.3B whole-tensor
clipped W = 8 shard are timed after it in the same run, each reported in
`per_config` with its own roofline, clocks and CPU baseline.

N > 1 (torchrun, one process per GPU): process i runs ZeRO rank (r0 + i) mod
W of the same workloads (r0: the workload's timed rank) on its own GPU --
independent shards, no data-path collective (weak scaling); the step time is
the max over processes.  The same run then times the real ZeRO step across
the processes (`peer`): W = N ranks of the workload's parameter set, each
reading its slice of every replica's gradient through peer loads and storing
its bf16 results into every rank's parameter buffer, beside NCCL's
reduce-scatter + local step + all-gather on the same parameters.

--impl reference times the oracle (plain C on the host, unchanged) on a
bounded sample of the same workload, split into disjoint slices stepped by
--cpu-threads host threads (default: every core the process may use), and
prints the same JSON line.  The GPU arm's cpu_baseline is the same
measurement, with the one-thread rate beside it.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "owned Gparams/s of fused reduce+AdamW step; achieved HBM GB/s vs B200 peak"
UNIT = "Gparams/s"
DEFAULT_CONFIG = "llama_7b_w64"
# timed in the same run after the headline workload, each with its own roofline, clocks and CPU baseline
COMPANIONS = ("gpt2_124m_w8", "gpt_1p3b_w8_whole_clip")
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCE = os.path.join(ROOT, "sharded_optimizer_step_zr_b200", "csrc", "zr_kernels.cu")
PROFILES = os.path.join(ROOT, "profiles")


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="zr", choices=["zr", "reference"])
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--cpu-threads", type=int, default=0,
                    help="host threads for the oracle baseline (0: every core this process may use, at most 32)")
    ap.add_argument("--per-bucket", action="store_true",
                    help="step bucket by bucket (zr_step_bucket per bucket, then zr_step_finish)")
    ap.add_argument("--overlap", action="store_true",
                    help="exposed optimizer time behind an emulated backward pass: one zr_step "
                         "after it, against zr_step_bucket as each bucket's gradients complete")
    ap.add_argument("--zero3", action="store_true",
                    help="ZeRO-3 parameter gather: bandwidth, and prefetch against an emulated forward")
    ap.add_argument("--plan-info", action="store_true",
                    help="the workload's plan and per-rank device footprint (host only, no GPU)")
    ap.add_argument("--vs-torch", action="store_true",
                    help="the optimizer step against torch's fused AdamW mixed-precision recipe (context)")
    ap.add_argument("--zero3-train", action="store_true",
                    help="training steps of an MLP stack: ZeroAdamW against Zero3 (the layer loop's cost)")
    ap.add_argument("--zero3-set", default="1p3b", choices=["1p3b", "gpt2"],
                    help="tensor set of --zero3 (gpt2: a small case, e.g. for profiling)")
    ap.add_argument("--checked", action="store_true",
                    help="checked mode: the device tile tables verified before every launch")
    ap.add_argument("--no-alloc", action="store_true",
                    help="step through zr_step_no_alloc (the library's static scratch, no workspace)")
    ap.add_argument("--gather-targets", action="store_true",
                    help="the step stores each bf16 result into W parameter buffers of this GPU (the "
                         "all-gather by stores of the step across GPUs, its HBM side); W <= 8 workloads")
    ap.add_argument("--sweep", action="store_true",
                    help="1.3B set: bucket cap x W x partition; one JSON record per point")
    ap.add_argument("--no-companions", action="store_true",
                    help="time the --config workload alone (no per_config entries)")
    ap.add_argument("--no-peer", action="store_true",
                    help="N > 1: skip the ZeRO step across the processes over peer memory")
    ap.add_argument("--peer-set", default="gpt_1p3b", choices=sorted(__import__("synth").PARAM_SETS),
                    help="parameter set of the N > 1 peer step (default: the 1.3B set of the sweep, "
                         "which with the NCCL arm's buffers fits one GPU at every N)")
    ap.add_argument("--peer-steps", type=int, default=20, help="timed steps of the N > 1 peer step")
    ap.add_argument("--backend", default="nccl", choices=["nccl", "gloo"],
                    help="process-group backend for N > 1 (gloo: tests of several processes on one GPU)")
    ap.add_argument("--same-gpu", action="store_true",
                    help="N > 1: every process on cuda:0 (a test on a one-GPU machine)")
    ap.add_argument("--write-traffic-record", metavar="CSV",
                    help="host only: turn an ncu --csv capture (dram__bytes_read.sum, dram__bytes_write.sum, "
                         "gpu__time_duration.sum) of --small-case's launches of one step into the traffic "
                         "record of --config under profiles/, scaled by owned parameters")
    ap.add_argument("--small-case", default=None, help="workload the capture ran (default: --config)")
    ap.add_argument("--sweep-w", default=None, metavar="W,W,...",
                    help="with --sweep: instead of the 40 sweep points, the 1.3B set flat, 25 MB buckets, "
                         "rank 0, at each of these replica counts (1 - 512)")
    args = ap.parse_args()
    if args.cpu_threads <= 0:
        args.cpu_threads = host_threads()
    return args


def workload(name):
    import synth
    if name in synth.WORKLOADS:
        return synth.WORKLOADS[name]
    for wl in synth.sweep_workloads():
        if wl.name == name:
            return wl
    raise SystemExit(f"unknown config {name}")


def bytes_per_owned_param(W, clip):
    """Algorithmic bytes: 2W gradient reads + 12 state reads + 12 state
    writes + 2 bf16 writes (+ the clip pass: fp32 g scratch written and read
    back when W > 4, the gradients read again when W <= 4)."""
    b = 2 * W + 26
    if clip:
        b += 8 if W > 4 else 2 * W
    return b


def shard_rank(wl, process_rank, n_processes):
    """ZeRO rank emulated by process `process_rank`: the workload's rank on a
    single process; consecutive ranks (mod W) across processes."""
    if n_processes == 1:
        return wl.ranks[0]
    return (wl.ranks[0] + process_rank) % wl.world_size


def reduce_timing(dist, elapsed_ms, owned_done, device):
    """Max of the elapsed times and sum of the owned parameters processed over
    all processes (identity without a process group)."""
    if dist is None:
        return elapsed_ms, owned_done
    import torch
    t = torch.tensor([elapsed_ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    o = torch.tensor([owned_done], dtype=torch.float64, device=device)
    dist.all_reduce(o, op=dist.ReduceOp.SUM)
    return float(t.item()), float(o.item())


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    with open(KERNEL_SOURCE, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def recorded_traffic(workload_name, clip, owned_params):
    """dram__bytes_read.sum + dram__bytes_write.sum from the committed ncu
    record of the workload, if it was taken on the current kernel source:
    per launch of zr_tile_kernel for a step without clipping, per step (all
    of its launches) with clipping -- the same unit as the line's
    `achieved`.  A record taken on a smaller case of the same kernels gives
    bytes per owned parameter, scaled here to `owned_params`.  Returns
    (bytes or None, a note on where they come from)."""
    name = f"zr_clip_step_{workload_name}" if clip else f"zr_tile_kernel_{workload_name}"
    try:
        with open(os.path.join(PROFILES, f"{name}_traffic.json")) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None, "no ncu record for this workload"
    e = d.get(workload_name)
    if not e:
        return None, "no ncu record for this workload"
    if e.get("kernel_source_sha256_16") != kernel_source_hash():
        return None, "ncu record taken on an older kernel source"
    if "bytes_per_owned_param" in e:
        small = e["small_case"]
        return (float(e["bytes_per_owned_param"]) * owned_params,
                f"ncu capture of {small['workload']} ({small['owned_params']} owned params), "
                f"scaled by owned params")
    return float(e["bytes_per_step"] if clip else e["bytes_per_launch"]), "ncu capture of this workload"


class ClockSampler:
    """NVML samples of SM clock and throttle reasons while the timed region runs."""

    def __init__(self, device_index):
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False

    def _sample(self):
        nv = self._nv
        try:
            self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
            r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
            for k, bit in self._names.items():
                if r & bit:
                    self.reasons.add(k)
        except Exception:
            pass

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)

    def _reason_bits(self):
        nv = self._nv
        return {
            "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4),
            "hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
            "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
            "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
            "hw_power_brake_slowdown": getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80),
        }

    def __enter__(self):
        if self._ok:
            self._names = self._reason_bits()
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()
            if not self.samples:
                # a region shorter than one NVML round trip: read the clocks
                # as it ends, the device having just drained the timed work
                self._sample()

    def summary(self):
        if not self._ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU arm: the oracle on a bounded sample
# ---------------------------------------------------------------------------

class OracleSample:
    """A bounded sample of one rank's shard for the oracle (test
    infrastructure, used by the CPU baseline only): the rank's first owned
    elements with the workload's gradient statistics, as their own W-replica
    flat plan of one tensor."""

    def __init__(self, wl, rank, max_elems, offset=0):
        import numpy as np
        import oracle
        import synth
        import torch
        oplan = oracle.Plan(wl.shapes, wl.world_size, wl.mode, wl.bucket_cap_bytes)
        self.owned = int(oplan.owned_numel[rank])
        offset = min(offset, self.owned)
        self.n = n = min(self.owned - offset, max_elems)
        idx = torch.from_numpy(oplan.owned_global_index(rank)[offset:offset + n])
        self.grads = [synth.grad_bf16(wl.seed, 1, w, idx, wl.grad_sigma, wl.outlier_frac,
                                      n_valid=oplan.total_numel).view(torch.int16).numpy()
                      .view(np.uint16).copy() for w in range(wl.world_size)]
        self.master = synth.master_f32(wl.seed, idx, n_valid=oplan.total_numel).numpy().copy()
        self.m = np.zeros(n, np.float32)
        self.v = np.zeros(n, np.float32)
        self.plan = oracle.Plan([(n * wl.world_size,)], wl.world_size, oracle.FLAT, 1 << 62)
        self.out = np.zeros(self.plan.padded_numel, np.uint16)
        self.wl, self.rank, self.t = wl, rank, 0

    def steps_until(self, deadline):
        """Oracle steps on the sample until perf_counter() passes `deadline`;
        returns the number of steps."""
        import oracle
        clip = 1.0 if self.wl.max_grad_norm > 0 else None
        steps = 0
        while True:
            self.t += 1
            oracle.rank_step(self.plan, 0, self.grads, self.master, self.m, self.v, self.out,
                             self.wl.hp, self.t, clip=clip)
            if clip is not None:
                oracle.sumsq(oracle.reduce(self.grads))      # the clip's extra reduce pass
            steps += 1
            if time.perf_counter() >= deadline:
                return steps


class OracleSamples:
    """`threads` disjoint samples of one rank's shard (consecutive slices of
    its owned elements), one per host thread.  The oracle's C calls release
    the interpreter lock and share no state, so the threads step their
    slices in parallel; the oracle itself is unchanged."""

    def __init__(self, wl, rank, max_elems, threads):
        self.threads = max(1, int(threads))
        per = max(1, max_elems // self.threads)
        self.samples = [OracleSample(wl, rank, per, offset=i * per) for i in range(self.threads)]
        self.samples = [x for x in self.samples if x.n > 0] or self.samples[:1]
        self.threads = len(self.samples)
        self.wl, self.rank, self.owned = wl, rank, self.samples[0].owned

    def run(self, target_seconds):
        """Every thread steps its slice until `target_seconds` have passed;
        returns (Gparams/s over all threads, description)."""
        import concurrent.futures as cf
        t0 = time.perf_counter()
        deadline = t0 + target_seconds
        if self.threads == 1:
            counts = [self.samples[0].steps_until(deadline)]
        else:
            with cf.ThreadPoolExecutor(max_workers=self.threads) as ex:
                counts = list(ex.map(lambda x: x.steps_until(deadline), self.samples))
        el = time.perf_counter() - t0
        done = sum(x.n * c for x, c in zip(self.samples, counts))
        n = sum(x.n for x in self.samples)
        desc = (f"oracle rank_step on {n} of rank {self.rank}'s {self.owned} owned params "
                f"(W={self.wl.world_size}) in {self.threads} slice(s), {min(counts)}-{max(counts)} "
                f"steps each, {el:.1f} s, {self.threads} thread(s)")
        return done / el / 1e9, desc


def host_threads():
    """Host cores this process may run on (at most 32)."""
    try:
        n = len(os.sched_getaffinity(0))
    except AttributeError:
        n = os.cpu_count() or 1
    return max(1, min(32, n))


def cpu_model():
    """The host CPU's model name, as the kernel reports it (None if unknown)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def cpu_baseline(wl, rank, seconds, threads, max_elems=1 << 21):
    """The oracle on a bounded sample of the workload: all `threads` host
    threads over disjoint slices (the reported value, `cores` = threads),
    and the same sample on one thread beside it."""
    multi = OracleSamples(wl, rank, max_elems, threads)
    rate, desc = multi.run(seconds / 2 if multi.threads > 1 else seconds)
    out = {"value": rate, "unit": UNIT, "cores": multi.threads, "kind": "oracle", "sample": desc,
           "cpu": cpu_model()}
    if multi.threads > 1:
        one = OracleSamples(wl, rank, max_elems, 1)
        r1, d1 = one.run(seconds / 2)
        out["single_thread"] = {"value": r1, "sample": d1}
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = workload(args.config)
    K, Wm = args.steps, args.warmup
    budget = max(0.05, min(2.0, 120.0 / max(1, K + Wm)))
    sample = OracleSamples(wl, wl.ranks[0], 1 << 18, args.cpu_threads)
    rates = []
    desc = ""
    for i in range(Wm + K):
        r, desc = sample.run(budget)
        if i >= Wm:
            rates.append(r)
    value = statistics.median(rates)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": K, "warmup": Wm, "ms_per_step": None, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": wl.name, "W": wl.world_size,
                   "rank": wl.ranks[0], "partition": "flat" if wl.mode == 0 else "whole_tensor",
                   "bucket_cap_mb": wl.bucket_cap_mb},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": sample.threads, "kind": "oracle",
                         "sample": desc, "cpu": cpu_model()},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------

def bound_bucket_steps(plan, buckets, grads, master, m, v, param_out, stream):
    """f(step): zr_step_bucket for every bucket this rank owns part of, in
    backward (bucket) order, then zr_step_finish; arguments marshalled once."""
    from sharded_optimizer_step_zr_b200 import _addr, _check, _lib, _ptr_array, _stream
    arr = _ptr_array(grads)
    ptrs = (_addr(master), _addr(m), _addr(v), _addr(param_out))
    s = _stream(stream)
    h = plan.handle

    def step_fn(step):
        for b in buckets:
            st = _lib.zr_step_bucket(h, b, arr, *ptrs, step, s)
            if st:
                _check(st, "zr_step_bucket")
        st = _lib.zr_step_finish(h, arr, *ptrs, step, s)
        if st:
            _check(st, "zr_step_finish")
    step_fn._keepalive = (arr, grads, master, m, v, param_out)
    return step_fn


class ProcessContext:
    """This process's place in the run: the process group (None for one
    process), its ranks and its device."""

    def __init__(self, args, use_cuda=True):
        import torch
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.grank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.dist = None
        self.backend = None
        if use_cuda:
            # --same-gpu: every process on cuda:0 (a multi-process test on a
            # one-GPU machine; the kernels never wait on another process)
            torch.cuda.set_device(0 if (self.world == 1 or args.same_gpu) else self.local)
            self.dev = torch.device("cuda", torch.cuda.current_device())
        else:
            self.dev = torch.device("cpu")     # host-side logic only (gloo tests)
        if self.world > 1:
            import datetime
            import torch.distributed as dist
            self.backend = args.backend
            kw = {"device_id": self.dev} if (self.backend == "nccl" and use_cuda) else {}
            dist.init_process_group(self.backend, timeout=datetime.timedelta(seconds=120), **kw)
            self.dist = dist

    def barrier(self):
        if self.dist is not None:
            if self.backend == "nccl":
                self.dist.barrier(device_ids=[self.dev.index])
            else:
                self.dist.barrier()

    def all_ok(self, ok):
        """True on every process when `ok` holds on every process (one
        all-reduce; the local value for one process): a step that failed on
        one rank is skipped by all of them, with no rank left waiting."""
        if self.dist is None:
            return bool(ok)
        import torch
        d = self.dev if self.backend == "nccl" else torch.device("cpu")
        flag = torch.tensor([1 if ok else 0], dtype=torch.int32, device=d)
        self.dist.all_reduce(flag, op=self.dist.ReduceOp.MIN)
        return bool(flag.item())

    def reduce(self, elapsed_ms, owned_done):
        """(max of elapsed_ms, sum of owned_done) over the processes."""
        if self.dist is None:
            return elapsed_ms, owned_done
        import torch
        d = self.dev if self.backend == "nccl" else torch.device("cpu")
        return reduce_timing(self.dist, elapsed_ms, owned_done, d)

    def close(self):
        if self.dist is not None:
            self.barrier()
            self.dist.destroy_process_group()


def measure_local(args, ctx, wl, with_e2e, with_cpu):
    """K timed steps of workload `wl` on this process's shard (ZeRO rank
    shard_rank(wl, ...)): the step time (max over processes), the roofline
    of the step's kernels, the clocks, and optionally the end-to-end rate
    through zr_step_host and the oracle's CPU rate.  Returns the entry as
    rank 0 reports it (identical keys on every process)."""
    import torch
    import synth
    from sharded_optimizer_step_zr_b200.plan import ZrPlan

    dev = ctx.dev
    W = wl.world_size
    zr_rank = shard_rank(wl, ctx.grank, ctx.world)
    clip = wl.max_grad_norm > 0
    plan = ZrPlan(wl.shapes, W, zr_rank, wl.mode, wl.bucket_cap_bytes, *wl.hp, device=dev)
    n = plan.owned_numel
    runs = plan.runs()
    stream = torch.cuda.current_stream()

    grads = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(W)]
    for w in range(W):
        synth.fill_owned_grad(grads[w], runs, wl.seed, 1, w, wl.grad_sigma, wl.outlier_frac,
                              n_valid=plan.total_numel)
    master = torch.empty(n, dtype=torch.float32, device=dev)
    synth.fill_owned_master(master, runs, wl.seed, n_valid=plan.total_numel)
    m = torch.zeros_like(master)
    v = torch.zeros_like(master)
    param_out = torch.zeros(plan.padded_numel, dtype=torch.bfloat16, device=dev)
    if clip:
        # the scalar exchange of the clip: this rank's S_r, and the other
        # ranks' entries set to the same value (their gradients have the same
        # statistics), so the norm has its real magnitude, S ~ W * S_r
        plan.grad_sumsq(grads, plan.partials[zr_rank:zr_rank + 1])
        plan.partials.fill_(float(plan.partials[zr_rank].item()))
    torch.cuda.synchronize()

    step_no = 0
    if args.checked:
        plan.set_checked(True)
    run_step = plan.bound_step(grads, master, m, v, param_out, stream)   # arguments marshalled once
    my_buckets = sorted({s["bucket"] for s in plan.segments() if s["owner"] == zr_rank})
    if args.per_bucket:
        run_step = bound_bucket_steps(plan, my_buckets, grads, master, m, v, param_out, stream)
    if args.no_alloc:
        run_step = bound_no_alloc_steps(plan, grads, master, m, v, param_out, stream)
    targets = None
    if args.gather_targets:
        if W > 8:
            raise SystemExit("--gather-targets: W parameter buffers of the full set fit one GPU only for W <= 8")
        from sharded_optimizer_step_zr_b200 import zr_plan_set_gather_targets
        targets = [param_out] + [torch.zeros_like(param_out) for _ in range(W - 1)]
        zr_plan_set_gather_targets(plan.handle, targets, stream)
        run_step = plan.bound_step(grads, master, m, v, None, stream)

    for _ in range(args.warmup):
        step_no += 1
        run_step(step_no)
    torch.cuda.synchronize()

    K = args.steps
    sampler = ClockSampler(dev.index)
    ctx.barrier()
    torch.cuda.synchronize()
    with sampler:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record(stream)
        for i in range(K):
            step_no += 1
            run_step(step_no)
        t_end.record(stream)
        torch.cuda.synchronize()
    ctx.barrier()
    local_ms = t_start.elapsed_time(t_end)
    total_ms, owned_total = ctx.reduce(local_ms, n * K)
    value = owned_total / (total_ms * 1e-3) / 1e9
    ms_per_step = total_ms / K

    # roofline: without clipping the step is one launch of zr_tile_kernel, so
    # its average launch duration is this process's timed region / K; with
    # clipping the step's launches are taken together.
    bpp = bytes_per_owned_param(W, clip)
    if args.no_alloc and clip and W > 4:
        bpp = 2 * W + 26 + 2 * W        # pass 2 reads the gradients again instead of an fp32 copy
    if args.gather_targets:
        bpp += 2 * (W - 1)              # the bf16 result stored into W buffers instead of one
    alg_bytes = n * bpp
    avg_ms = local_ms / K
    achieved = alg_bytes / (avg_ms * 1e-3) / 1e9
    peak, peak_kind = measured_peak()
    # (bucket-by-bucket or checked steps launch more kernels: no per-launch record)
    traffic = None
    traffic_note = None
    if not (args.per_bucket or args.checked or args.no_alloc or args.gather_targets):
        traffic, traffic_note = recorded_traffic(wl.name, clip, n)

    # the ceiling at this size: a plain device copy (torch) moving the step's
    # algorithmic bytes (half read, half written), timed the same way
    copy_ref = None
    if not (args.per_bucket or args.checked):
        half = (alg_bytes // 2) // 16 * 16
        src = torch.empty(half, dtype=torch.uint8, device=dev)
        dst = torch.empty(half, dtype=torch.uint8, device=dev)
        reps = max(3, min(K, 200))
        for _ in range(3):
            dst.copy_(src)
        torch.cuda.synchronize()
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(reps):
            dst.copy_(src)
        c1.record(stream)
        torch.cuda.synchronize()
        copy_ms = c0.elapsed_time(c1) / reps
        # the same bytes through a kernel (torch's vectorised elementwise
        # kernel, bf16 x 1): a copy that ncu sees, for its DRAM figures
        # beside the step's (the driver copy above is not a kernel)
        sb, db = src.view(torch.bfloat16), dst.view(torch.bfloat16)
        for _ in range(3):
            torch.mul(sb, 1, out=db)
        torch.cuda.synchronize()
        c0.record(stream)
        for _ in range(reps):
            torch.mul(sb, 1, out=db)
        c1.record(stream)
        torch.cuda.synchronize()
        kcopy_ms = c0.elapsed_time(c1) / reps
        copy_ref = {"bytes": 2 * half, "ms": copy_ms, "gbs": 2 * half / (copy_ms * 1e-3) / 1e9, "reps": reps,
                    "step_speed_vs_copy": copy_ms / avg_ms,
                    "kernel_copy": {"ms": kcopy_ms, "gbs": 2 * half / (kcopy_ms * 1e-3) / 1e9,
                                    "step_speed_vs_kernel_copy": kcopy_ms / avg_ms,
                                    "kernel": "torch elementwise mul (bf16, x 1)"}}
        del src, dst, sb, db
        torch.cuda.empty_cache()

    # end to end through zr_step_host: pinned host gradients in, result out
    e2e = None
    pinned = None
    if with_e2e and not args.gather_targets:
        try:
            host_grads = [g.cpu().pin_memory() for g in grads]
            host_out = torch.empty(plan.padded_numel, dtype=torch.bfloat16).pin_memory()
        except (RuntimeError, MemoryError) as e:     # pinned host memory is a host resource
            host_grads = host_out = None
            pinned = f"{type(e).__name__}: {e}"
        if not ctx.all_ok(pinned is None):
            e2e = {"unavailable": f"pinned host buffers could not be allocated on every process"
                                  f"{' (here: ' + pinned + ')' if pinned else ''}",
                   "h2d_bytes_per_step": 2 * W * n, "d2h_bytes_per_step": 2 * n}
    if with_e2e and not args.gather_targets and e2e is None:
        for _ in range(3):
            step_no += 1
            plan.step_host(host_grads, grads, master, m, v, param_out, host_out, step_no, stream)
        torch.cuda.synchronize()
        K2 = max(3, min(K, 50))
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ctx.barrier()
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(K2):
            step_no += 1
            plan.step_host(host_grads, grads, master, m, v, param_out, host_out, step_no, stream)
        b.record(stream)
        torch.cuda.synchronize()
        e2e_ms, e2e_owned = ctx.reduce(a.elapsed_time(b), n * K2)
        e2e = {"value": e2e_owned / (e2e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": 2 * W * n, "d2h_bytes_per_step": 2 * n,
               "steps": K2, "api": "zr_step_host"}
        del host_grads, host_out

    cpu = None
    if with_cpu and ctx.grank == 0 and ctx.world == 1:
        cpu = cpu_baseline(wl, zr_rank, args.cpu_seconds, args.cpu_threads)

    launches_per_step = launches_per_clip_step() if clip else 1
    if args.per_bucket:
        # pass 1 per bucket with clipping; zr_step_finish: the coefficient, then pass 2
        launches_per_step = len(my_buckets) + (2 if clip else 0)
    if args.checked:
        launches_per_step += (len(my_buckets) + (1 if clip else 0)) if args.per_bucket else 1
    entry = {
        "workload": wl.name, "value": value, "unit": UNIT, "ms_per_step": ms_per_step, "steps": K,
        "config": {"workload": wl.name, "W": W, "rank": zr_rank,
                   "partition": "flat" if wl.mode == 0 else "whole_tensor",
                   "bucket_cap_mb": wl.bucket_cap_mb, "clip": clip, "owned_params": n,
                   "per_bucket": bool(args.per_bucket), "buckets_stepped": len(my_buckets),
                   "checked": bool(args.checked), "no_alloc": bool(args.no_alloc),
                   "gather_targets": W if args.gather_targets else 0,
                   "bytes_per_owned_param": bpp,
                   "l2": f"no flush: each step touches {alg_bytes / 1e6:.0f} MB > 126 MB L2"},
        "hbm_gbs": achieved,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "traffic_source": traffic_note,
                     "peak_source": peak_kind,
                     "kernel": "zr_tile_kernel" if not clip else
                     f"zr_step ({launches_per_clip_step()} kernels)"},
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": launches_per_step * K,
        "clocks": sampler.summary(),
        "copy_reference": copy_ref,
    }
    plan.close()
    del grads, master, m, v, param_out, run_step, targets
    torch.cuda.empty_cache()
    return entry


def launches_per_clip_step():
    """Kernel launches of one clipped zr_step: pass 1, the combine (S_r, S,
    the coefficient) and pass 2."""
    return 3


def peer_bytes(W, n):
    """Bytes one rank of a W-rank peer-memory step moves per step for its
    n owned parameters: gradient loads from the W - 1 peers' replicas (the
    reduce-scatter), bf16 stores into the W - 1 peers' parameter buffers
    (the all-gather), and its local HBM traffic (own replica, fp32 state
    read and written, own parameter buffer)."""
    return {"peer_loads": 2 * (W - 1) * n, "peer_stores": 2 * (W - 1) * n,
            "local_hbm": 2 * n + 24 * n + 2 * n}


def measure_peer(args, ctx):
    """The ZeRO step across the processes of this run (one rank each, W =
    the number of processes): PeerZero over CUDA IPC, the step reading every
    replica's slice through peer loads and storing the bf16 results into
    every rank's parameter buffer.  Beside it, on the same parameters, the
    library-collective recipe: NCCL reduce-scatter (average) of the bf16
    gradients, the local step on the owned chunk (one replica), NCCL
    all-gather of the bf16 chunk.  Returns the entry (identical keys on
    every process)."""
    import torch
    import synth
    from sharded_optimizer_step_zr_b200.peer import PeerFailure, PeerZero
    from sharded_optimizer_step_zr_b200.plan import ZrPlan

    wl = workload(args.config)
    set_name = args.peer_set
    shapes = synth.PARAM_SETS[set_name]()
    W, rank, dev = ctx.world, ctx.grank, ctx.dev
    hp = wl.hp[:5] + (0.0,)
    try:
        pz = PeerZero(ctx.dist.group.WORLD, shapes, 0, wl.bucket_cap_bytes, *hp, device=dev, stage=2)
    except PeerFailure as e:
        # every rank gets it together (the set-up agrees before anyone steps):
        # the line keeps the independent-shard measurements
        return {"mode": "peer", "W": W, "param_set": set_name, "unavailable": str(e)}
    n = pz.plan.owned_numel
    N = pz.plan.total_numel
    segs = pz.plan.segments()
    runs_of = [synth.rank_runs(segs, r) for r in range(W)]
    # this process is replica `rank`: its full gradient in the owner-major layout
    for r in range(W):
        a, b = pz.offsets[r], pz.offsets[r + 1]
        synth.fill_owned_grad(pz.grad_buffer[a:b], runs_of[r], wl.seed, 1, rank, wl.grad_sigma,
                              wl.outlier_frac, n_valid=N)
    master = torch.empty(max(n, 8), dtype=torch.float32, device=dev)
    synth.fill_owned_master(master, runs_of[rank], wl.seed, n_valid=N)
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    stream = torch.cuda.current_stream()
    t = 0
    for _ in range(args.warmup):
        t += 1
        pz.step(master, m, v, t)
    K = max(1, args.peer_steps)
    ctx.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        t += 1
        pz.step(master, m, v, t)
    e1.record(stream)
    torch.cuda.synchronize()
    ms, owned = ctx.reduce(e0.elapsed_time(e1), n * K)
    entry = {"mode": "peer", "W": W, "param_set": set_name, "partition": "flat",
             "bucket_cap_mb": wl.bucket_cap_mb, "total_params": N, "owned_params": n,
             "steps": K, "ms_per_step": ms / K, "value": owned / (ms * 1e-3) / 1e9, "unit": UNIT,
             "per_gpu_value": n / (ms / K * 1e-3) / 1e9,
             "bytes_per_step_per_rank": peer_bytes(W, n),
             "same_gpu": bool(args.same_gpu), "backend": ctx.backend,
             "timing": "CUDA events over K steps, host barriers between the phases included; max over ranks"}

    # the library-collective arm (flat partitions whose owner-major layout is the global one)
    C = pz.plan.padded_numel // W
    aligned = all(pz.offsets[r] == r * C for r in range(W + 1))
    if ctx.backend != "nccl" or args.same_gpu:
        entry["nccl_arm"] = {"skipped": "needs NCCL with one GPU per process"}
    elif not aligned:
        entry["nccl_arm"] = {"skipped": "owner-major layout differs from the global layout"}
    else:
        dist = ctx.dist
        full_grad = pz.grad_buffer[:W * C]
        shard_grad = torch.empty(C, dtype=torch.bfloat16, device=dev)
        shard_out = torch.empty(C, dtype=torch.bfloat16, device=dev)
        full_param = torch.empty(W * C, dtype=torch.bfloat16, device=dev)
        one = ZrPlan([(C,)], 1, 0, 0, 1 << 40, *hp, device=dev)
        mb = master[:n].clone() if C == n else torch.zeros(C, dtype=torch.float32, device=dev)
        mmb, vvb = torch.zeros_like(mb), torch.zeros_like(mb)
        local_step = one.bound_step([shard_grad], mb, mmb, vvb, shard_out, stream)

        def nccl_step(tt):
            dist.reduce_scatter_tensor(shard_grad, full_grad, op=dist.ReduceOp.AVG)
            local_step(tt)
            dist.all_gather_into_tensor(full_param, shard_out)

        tt = 0
        for _ in range(args.warmup):
            tt += 1
            nccl_step(tt)
        ctx.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for _ in range(K):
            tt += 1
            nccl_step(tt)
        e1.record(stream)
        torch.cuda.synchronize()
        ms2, owned2 = ctx.reduce(e0.elapsed_time(e1), C * K)
        entry["nccl_arm"] = {"ms_per_step": ms2 / K, "value": owned2 / (ms2 * 1e-3) / 1e9, "unit": UNIT,
                             "recipe": "reduce_scatter_tensor(bf16, AVG) + zr_step on the chunk (W = 1) "
                                       "+ all_gather_into_tensor(bf16)"}
        one.close()
        del full_grad, shard_grad, shard_out, full_param, mb, mmb, vvb, local_step
    pz.close()
    del master, m, v
    torch.cuda.empty_cache()
    return entry


def bound_no_alloc_steps(plan, grads, master, m, v, param_out, stream):
    """f(step): zr_step_no_alloc on fixed buffers, arguments marshalled once
    (its scratch is the library's static array; the plan's partials array,
    if any, is passed as the sums-of-squares array)."""
    from sharded_optimizer_step_zr_b200 import _addr, _check, _lib, _ptr_array, _stream
    arr = _ptr_array(grads)
    args = (plan.handle, arr, _addr(master), _addr(m), _addr(v), _addr(param_out),
            _addr(plan.partials) if plan.partials is not None else None)
    s = _stream(stream)
    fn = _lib.zr_step_no_alloc

    def step_fn(step):
        st = fn(*args, step, s)
        if st:
            _check(st, "zr_step_no_alloc")
    step_fn._keepalive = (arr, grads, master, m, v, param_out)
    return step_fn


def run_zr(args):
    ctx = ProcessContext(args)
    head = measure_local(args, ctx, workload(args.config), with_e2e=not args.no_e2e,
                         with_cpu=not args.no_cpu_baseline)
    per_config = []
    if not (args.no_companions or args.per_bucket or args.checked):
        for name in COMPANIONS:
            if name != args.config:
                per_config.append(measure_local(args, ctx, workload(name), with_e2e=False,
                                                with_cpu=not args.no_cpu_baseline))
    peer = None
    if ctx.world > 1 and not args.no_peer:
        peer = measure_peer(args, ctx)
    ctx.close()
    if ctx.grank != 0:
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": UNIT, "n_gpus": ctx.world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": head["config"],
        "hbm_gbs": head["hbm_gbs"],
        "roofline": head["roofline"],
        "cpu_baseline": head["cpu_baseline"],
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "clocks": head["clocks"],
        "copy_reference": head["copy_reference"],
        "per_config": per_config,
    }
    if peer is not None:
        line["peer"] = peer
    print(json.dumps(line), flush=True)


def run_sweep(args):
    """Every point of the 1.3B sweep (bucket cap {1,5,25,100,400} MB x W
    {2,8,32,64} x {flat, whole-tensor}); rank 0, plus the most-loaded rank
    for whole-tensor points -- or, with --sweep-w, the flat 25 MB point at
    each listed W.  Prints one JSON record per point."""
    import torch
    import synth
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream()
    peak, peak_kind = measured_peak()
    points = synth.sweep_workloads()
    if args.sweep_w:
        points = [synth.Workload(f"sweep_1p3b_flat_w{w}_cap25", "gpt_1p3b", w, (0,), 0, 25, 1e-3, 0.01)
                  for w in (int(x) for x in args.sweep_w.split(","))]
    for wl in points:
        probe = ZrPlan(wl.shapes, wl.world_size, 0, wl.mode, wl.bucket_cap_bytes, *wl.hp, bind=False)
        loads = {}
        for s in probe.segments():
            loads[s["owner"]] = loads.get(s["owner"], 0) + s["length"]
        probe.close()
        ranks = [0]
        if wl.mode == 1:
            heavy = max(loads, key=lambda r: (loads[r], -r))
            if heavy != 0:
                ranks.append(heavy)
        for rank in ranks:
            plan = ZrPlan(wl.shapes, wl.world_size, rank, wl.mode, wl.bucket_cap_bytes, *wl.hp, device=dev)
            n, W = plan.owned_numel, wl.world_size
            runs = plan.runs()
            grads = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(W)]
            for w in range(W):
                synth.fill_owned_grad(grads[w], runs, wl.seed, 1, w, wl.grad_sigma, wl.outlier_frac,
                                      n_valid=plan.total_numel)
            master = torch.empty(n, dtype=torch.float32, device=dev)
            synth.fill_owned_master(master, runs, wl.seed, n_valid=plan.total_numel)
            m, v = torch.zeros_like(master), torch.zeros_like(master)
            out = torch.zeros(plan.padded_numel, dtype=torch.bfloat16, device=dev)
            run_step = plan.bound_step(grads, master, m, v, out, stream)
            for t in range(args.warmup):
                run_step(t + 1)
            torch.cuda.synchronize()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for t in range(args.steps):
                run_step(args.warmup + t + 1)
            b.record(stream)
            torch.cuda.synchronize()
            ms = a.elapsed_time(b) / args.steps
            bpp = bytes_per_owned_param(W, False)
            gbs = n * bpp / (ms * 1e-3) / 1e9
            print(json.dumps({"point": wl.name, "W": W, "rank": rank,
                              "partition": "flat" if wl.mode == 0 else "whole_tensor",
                              "bucket_cap_mb": wl.bucket_cap_mb, "n_buckets": plan.n_buckets,
                              "owned_params": n, "ms_per_step": ms,
                              "gparams_per_s": n / (ms * 1e-3) / 1e9, "hbm_gbs": gbs,
                              "frac_of_peak": gbs / peak, "peak_source": peak_kind}), flush=True)
            plan.close()
            del grads, master, m, v, out, run_step
            torch.cuda.empty_cache()


def run_overlap(args):
    """Bucket-by-bucket stepping overlapped with the backward pass.

    The backward pass is emulated by one bf16 matmul per bucket on a compute
    stream, in bucket (backward) order, each sized in proportion to the
    bucket's parameter count and together about 20 times the optimizer
    step; an event marks each bucket's gradients as ready.  Measured:
    (a) the backward alone; (b) the backward, then one zr_step; (c) the
    backward with zr_step_bucket launched on a second stream as each bucket
    completes (then zr_step_finish).  The optimizer time left exposed is
    (b) - (a) against (c) - (a)."""
    import torch
    import synth
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    wl = workload(args.config)
    W, rank = wl.world_size, wl.ranks[0]
    plan = ZrPlan(wl.shapes, W, rank, wl.mode, wl.bucket_cap_bytes, *wl.hp, device=dev)
    n = plan.owned_numel
    runs = plan.runs()
    grads = [torch.empty(n, dtype=torch.bfloat16, device=dev) for _ in range(W)]
    for w in range(W):
        synth.fill_owned_grad(grads[w], runs, wl.seed, 1, w, wl.grad_sigma, wl.outlier_frac,
                              n_valid=plan.total_numel)
    master = torch.empty(n, dtype=torch.float32, device=dev)
    synth.fill_owned_master(master, runs, wl.seed, n_valid=plan.total_numel)
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    out = torch.zeros(plan.padded_numel, dtype=torch.bfloat16, device=dev)
    if wl.max_grad_norm > 0:
        plan.grad_sumsq(grads, plan.partials[rank:rank + 1])
        plan.partials.fill_(float(plan.partials[rank].item()))
    segs = plan.segments()
    bucket_params = [0] * plan.n_buckets
    for sgm in segs:
        bucket_params[sgm["bucket"]] += sgm["length"]
    compute, opt = torch.cuda.Stream(), torch.cuda.Stream()
    step_no = [0]

    def step_once(stream):
        step_no[0] += 1
        with torch.cuda.stream(stream):
            plan.step(grads, master, m, v, out, step_no[0], stream)

    # size the emulated backward: total ~20x one optimizer step
    for _ in range(3):
        step_once(compute)
    torch.cuda.synchronize()
    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_.record(compute)
    for _ in range(5):
        step_once(compute)
    b_.record(compute)
    torch.cuda.synchronize()
    opt_ms = a_.elapsed_time(b_) / 5
    x = torch.randn(4096, 4096, dtype=torch.bfloat16, device=dev)
    with torch.cuda.stream(compute):
        for _ in range(3):
            torch.matmul(x, x)
    torch.cuda.synchronize()
    a_.record(compute)
    for _ in range(10):
        with torch.cuda.stream(compute):
            torch.matmul(x, x)
    b_.record(compute)
    torch.cuda.synchronize()
    mm_ms = a_.elapsed_time(b_) / 10
    total = sum(bucket_params)
    reps = [max(1, round(20.0 * opt_ms / mm_ms * p / total)) for p in bucket_params]
    ready = [torch.cuda.Event() for _ in range(plan.n_buckets)]

    def backward():
        with torch.cuda.stream(compute):
            for b in range(plan.n_buckets):
                for _ in range(reps[b]):
                    torch.matmul(x, x)
                ready[b].record(compute)

    my_buckets = sorted({sgm["bucket"] for sgm in segs if sgm["owner"] == rank})

    def time_it(fn, iters=args.steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(compute)
        for _ in range(iters):
            fn()
        opt.wait_stream(compute)
        compute.wait_stream(opt)
        t1.record(compute)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1) / iters

    def sequential():
        backward()
        step_once(compute)

    def overlapped():
        backward()
        step_no[0] += 1
        for b in my_buckets:
            opt.wait_event(ready[b])
            with torch.cuda.stream(opt):
                plan.step_bucket(b, grads, master, m, v, out, step_no[0], opt)
        with torch.cuda.stream(opt):
            plan.step_finish(grads, master, m, v, out, step_no[0], opt)
        compute.wait_stream(opt)      # the next backward reads the new parameters

    back_ms = time_it(backward)
    seq_ms = time_it(sequential)
    ovl_ms = time_it(overlapped)
    print(json.dumps({"mode": "overlap", "workload": wl.name, "rank": rank, "owned_params": n,
                      "buckets_stepped": len(my_buckets), "optimizer_step_ms": opt_ms,
                      "backward_ms": back_ms, "backward_then_step_ms": seq_ms,
                      "backward_with_bucket_steps_ms": ovl_ms,
                      "exposed_ms_single_step": seq_ms - back_ms,
                      "exposed_ms_per_bucket": ovl_ms - back_ms}), flush=True)


def run_zero3(args):
    """ZeRO-3 parameter gather on the 1.3B set (or the GPT-2 set), flat,
    W = 8: every rank's bf16 shard resident on this GPU (standing in for
    peer mappings).

    Measured: (a) one zr_gather_params of the whole model and of one
    transformer block, against the copy roofline (2 bytes read + 2 written
    per element); (b) an emulated forward -- per block one bf16 matmul of
    about the block's FLOPs at 8192 tokens -- run with the block's gather
    in front of it on the same stream (in line), or with block i + 1's
    gather issued on a side stream while block i computes (prefetch).  The
    gather time left exposed is the difference from the forward alone.
    Prints one JSON record."""
    import torch
    import synth
    from sharded_optimizer_step_zr_b200 import ZR_PARAMS_OWNED
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    if args.zero3_set == "gpt2":
        wl = synth.WORKLOADS["gpt2_124m_w8"]
    else:
        wl = next(w for w in synth.sweep_workloads() if w.name == "sweep_1p3b_flat_w8_cap25")
    W = wl.world_size
    plans = [ZrPlan(wl.shapes, W, r, wl.mode, wl.bucket_cap_bytes, *wl.hp, device=dev, bind=(r == 0))
             for r in range(W)]
    plan = plans[0]
    plan.set_param_layout(ZR_PARAMS_OWNED)
    gen = torch.Generator(device=dev)
    gen.manual_seed(wl.seed)
    shards = [torch.randn(p.owned_numel, device=dev, generator=gen).to(torch.bfloat16) for p in plans]
    for p in plans[1:]:
        p.close()
    numels = [int(math.prod(s)) for s in wl.shapes]
    # GPT blocks: tensors 2 + 12 i .. 2 + 12 i + 11 (wte and wpe first, ln_f last)
    per_block = 12
    n_blocks = (len(numels) - 4) // per_block
    d_model = int(wl.shapes[1][1])
    block_params = sum(numels[2:2 + per_block])
    layer_buf = [torch.empty(block_params, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    full = torch.empty(sum(numels), dtype=torch.bfloat16, device=dev)
    peak, peak_kind = measured_peak()

    def timed(fn, reps, stream=None):
        stream = stream or torch.cuda.current_stream()
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(reps):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e3    # us

    # arguments marshalled once per call site (bound_gather): the loops time the GPU, not Python
    whole_us = timed(plan.bound_gather(0, len(numels), shards, full), 20)
    block_us = timed(plan.bound_gather(2, per_block, shards, layer_buf[0]), 200)
    gb = lambda elems, us: 4 * elems / (us * 1e-6) / 1e9

    def graph_us(bind, reps):
        """Per-launch device time of `reps` launches replayed from one CUDA
        graph: no host launch gap between them (a 6 us gather issued from
        Python one call at a time waits on the host)."""
        s = torch.cuda.Stream()
        fn = bind(s)
        with torch.cuda.stream(s):
            for _ in range(3):
                fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            for _ in range(reps):
                fn()
        with torch.cuda.stream(s):                     # replay() launches on the current stream
            g.replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(s):
            e0.record(s)
            g.replay()
            e1.record(s)
        torch.cuda.synchronize()
        del g
        return e0.elapsed_time(e1) / reps * 1e3

    # the same bytes moved by a plain device copy (torch), for the ceiling at each size
    src_block = torch.empty(block_params, dtype=torch.bfloat16, device=dev)
    src_whole = torch.empty(sum(numels), dtype=torch.bfloat16, device=dev)
    graph = {
        "gather_block_us": graph_us(lambda st: plan.bound_gather(2, per_block, shards, layer_buf[0], st), 100),
        "copy_block_us": graph_us(lambda st: (lambda: layer_buf[1].copy_(src_block)), 100),
        "gather_whole_model_us": graph_us(lambda st: plan.bound_gather(0, len(numels), shards, full, st), 10),
        "copy_whole_model_us": graph_us(lambda st: (lambda: full.copy_(src_whole)), 10),
    }
    del src_whole

    # emulated forward: per block [8192, d] x [d, 12 d] bf16, 2 * 8192 * 12 * d^2 flops -- a
    # block's forward (12 d^2 weights) at 8192 tokens
    x = torch.randn(8192, d_model, dtype=torch.bfloat16, device=dev)
    w_ = torch.randn(d_model, 12 * d_model, dtype=torch.bfloat16, device=dev)
    compute = torch.cuda.Stream()
    lo, hi = torch.cuda.Stream.priority_range() if hasattr(torch.cuda.Stream, "priority_range") else (0, -1)
    side_streams = {"default": torch.cuda.Stream(), "high": torch.cuda.Stream(priority=hi)}
    side = side_streams["default"]

    def forward_only():
        with torch.cuda.stream(compute):
            for _ in range(n_blocks):
                torch.matmul(x, w_)

    in_line = [plan.bound_gather(2 + per_block * i, per_block, shards, layer_buf[i % 2], compute)
               for i in range(n_blocks)]

    def forward_sequential():
        with torch.cuda.stream(compute):
            for i in range(n_blocks):
                in_line[i]()
                torch.matmul(x, w_)

    ready = [torch.cuda.Event() for _ in range(n_blocks)]
    done = [torch.cuda.Event() for _ in range(n_blocks)]

    prefetch = []

    def forward_prefetch():
        side.wait_stream(compute)
        with torch.cuda.stream(side):
            prefetch[0]()
            ready[0].record(side)
        for i in range(n_blocks):
            if i + 1 < n_blocks:
                with torch.cuda.stream(side):
                    if i >= 1:
                        side.wait_event(done[i - 1])          # buffer (i + 1) % 2 was block i - 1's
                    prefetch[i + 1]()
                    ready[i + 1].record(side)
            with torch.cuda.stream(compute):
                compute.wait_event(ready[i])
                torch.matmul(x, w_)
                done[i].record(compute)

    t_fwd = timed(forward_only, 10, compute)
    t_seq = timed(forward_sequential, 10, compute)
    t_pre = {}
    for name, st, c in (("default", side_streams["default"], 0), ("high", side_streams["high"], 0),
                        ("high_16_ctas", side_streams["high"], 16), ("high_32_ctas", side_streams["high"], 32)):
        side = st
        prefetch[:] = [plan.bound_gather(2 + per_block * i, per_block, shards, layer_buf[i % 2], st, c)
                       for i in range(n_blocks)]
        t_pre[name] = timed(forward_prefetch, 10, compute)
    capped_us = {c: timed(plan.bound_gather(2, per_block, shards, layer_buf[0], None, c), 50) for c in (16, 32)}
    line = {
        "mode": "zero3_gather", "workload": f"{wl.name} (flat W={W}), all ranks' shards on one GPU",
        "params": sum(numels), "block_params": block_params, "unit": "us",
        "gather_whole_model_us": whole_us, "gather_whole_model_gbs": gb(sum(numels), whole_us),
        "gather_block_us": block_us, "gather_block_gbs": gb(block_params, block_us),
        "roofline": {"bound": "hbm", "peak": peak, "peak_source": peak_kind, "unit": "GB/s",
                     "bytes_per_element": 4, "frac_whole_model": gb(sum(numels), whole_us) / peak,
                     "frac_block": gb(block_params, block_us) / peak},
        "forward_only_us": t_fwd, "forward_gather_in_line_us": t_seq,
        "gather_block_16_ctas_us": capped_us[16], "gather_block_32_ctas_us": capped_us[32],
        "forward_gather_prefetched_us": t_pre,
        "exposed_gather_in_line_us": t_seq - t_fwd,
        "exposed_gather_prefetched_us": {k: v - t_fwd for k, v in t_pre.items()},
        "blocks": n_blocks,
        "graph_replay": dict(graph, **{
            "frac_block": gb(block_params, graph["gather_block_us"]) / peak,
            "frac_whole_model": gb(sum(numels), graph["gather_whole_model_us"]) / peak,
            "gather_over_copy_block": graph["copy_block_us"] / graph["gather_block_us"],
            "gather_over_copy_whole_model": graph["copy_whole_model_us"] / graph["gather_whole_model_us"]}),
    }
    print(json.dumps(line), flush=True)
    plan.close()


def run_zero3_train(args):
    """Training steps of a stack of MLP blocks (12 x [Linear(d, 4d), GELU,
    Linear(4d, d)], d = 2048: 403 M bf16 parameters; 4096 tokens) with
    ZeroAdamW (every parameter resident), with Zero3 (each layer gathered
    from the shard before its forward and again before its backward, the
    next layer's forward gather prefetched) and with Zero3's
    reduce_in_backward (each layer's gradients reduced and applied as its
    backward ends, two layer-sized gradient slots instead of a full
    gradient buffer), one rank.  All take the same steps (checked); the
    differences in step time are what the layer loop costs on one GPU.
    Prints one JSON record."""
    import torch
    from sharded_optimizer_step_zr_b200.optim import Zero3, ZeroAdamW
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    d, n_blocks, tokens = 2048, 12, 4096

    def model(seed):
        torch.manual_seed(seed)
        layers = []
        for _ in range(n_blocks):
            layers += [torch.nn.Linear(d, 4 * d), torch.nn.GELU(), torch.nn.Linear(4 * d, d)]
        return torch.nn.Sequential(*layers).to(dev).to(torch.bfloat16)

    a, b, c, e, f = model(1), model(1), model(1), model(1), model(1)
    n_params = sum(p.numel() for p in a.parameters())
    z2 = ZeroAdamW(list(a.parameters()), lr=1e-4)
    z2_overlap = ZeroAdamW(list(f.parameters()), lr=1e-4, overlap=True)
    z3 = Zero3(b, lr=1e-4)
    z3_fwd_only = Zero3(c, lr=1e-4, backward_prefetch=False)
    z3_rib = Zero3(e, lr=1e-4, reduce_in_backward=True)
    x = torch.randn(tokens, d, device=dev, dtype=torch.bfloat16)

    def step(m, opt):
        m(x).float().pow(2).mean().backward()
        opt.step()
        opt.zero_grad()

    def timed(m, opt, reps):
        for _ in range(2):
            step(m, opt)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            step(m, opt)
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    t2 = timed(a, z2, 5)
    t2o = timed(f, z2_overlap, 5)
    t3 = timed(b, z3, 5)
    t3f = timed(c, z3_fwd_only, 5)
    t3r = timed(e, z3_rib, 5)
    full = torch.empty(n_params, dtype=torch.bfloat16, device=dev)
    z3.gather_all(full)
    resident = torch.cat([p.detach().reshape(-1) for p in a.parameters()])
    same = bool(torch.equal(full.view(torch.int16), resident.view(torch.int16)))
    overlap_same = bool(torch.equal(torch.cat([p.detach().reshape(-1) for p in f.parameters()]).view(torch.int16),
                                    resident.view(torch.int16)))
    full_r = torch.empty(n_params, dtype=torch.bfloat16, device=dev)
    z3_rib.gather_all(full_r)
    same_rib = bool(torch.equal(full.view(torch.int16), full_r.view(torch.int16)))
    flops = 6 * tokens * n_params
    line = {"mode": "zero3_train", "params": n_params, "tokens": tokens, "blocks": n_blocks, "unit": "ms",
            "zero_adamw_step_ms": t2, "zero3_step_ms": t3, "layer_loop_overhead_ms": t3 - t2,
            "zero3_forward_prefetch_only_step_ms": t3f,
            "gathers_per_step": 2 * len(z3.units), "gathered_bytes_per_step": 2 * 2 * n_params,
            "model_tflops_zero_adamw": flops / (t2 * 1e-3) / 1e12, "same_parameters": same,
            "zero3_reduce_in_backward_step_ms": t3r, "reduce_in_backward_same_parameters": same_rib,
            "zero_adamw_overlap_step_ms": t2o, "overlap_same_parameters": overlap_same,
            "gradient_bytes": {"zero3": 2 * z3.grad_buffer.numel(),
                               "zero3_reduce_in_backward": 2 * sum(g.numel() for g in z3_rib.grad_slots)}}
    print(json.dumps(line), flush=True)
    z2.close()
    z2_overlap.close()
    z3.close()
    z3_fwd_only.close()
    z3_rib.close()


def run_vs_torch(args):
    """The optimizer step alone, one rank, on the 403 M-parameter MLP stack
    of --zero3-train, against PyTorch's own mixed-precision recipe: fused
    torch.optim.AdamW on fp32 master parameters (gradients cast from the
    bf16 ones), then the masters copied back into the bf16 model.  Context,
    not a target: both are memory-bound, and the fused step moves fewer
    bytes (2 gradient + 24 state + 2 parameter per element at W = 1).
    Prints one JSON record."""
    import torch
    from sharded_optimizer_step_zr_b200.optim import ZeroAdamW
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    d, n_blocks = 2048, 12
    shapes = [(4 * d, d), (4 * d,), (d, 4 * d), (d,)] * n_blocks
    torch.manual_seed(0)
    model = [torch.nn.Parameter(torch.randn(s, device=dev).mul_(0.02).to(torch.bfloat16)) for s in shapes]
    grads = [torch.randn(s, device=dev).mul_(1e-3).to(torch.bfloat16) for s in shapes]
    n = sum(p.numel() for p in model)
    z = ZeroAdamW(model, lr=1e-4)
    for p, g in zip(model, grads):
        p.grad.copy_(g)
    masters = [torch.nn.Parameter(p.detach().float()) for p in model]
    opt = torch.optim.AdamW(masters, lr=1e-4, weight_decay=0.1, fused=True)

    def torch_step():
        for mp, g in zip(masters, grads):
            mp.grad = g.float()
        opt.step()
        with torch.no_grad():
            for p, mp in zip(model, masters):
                p.copy_(mp)

    def timed(fn, reps=20):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            fn()
        e1.record()
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    t_zr = timed(z.step)
    t_torch = timed(torch_step)
    line = {"mode": "vs_torch_adamw", "params": n, "unit": "ms", "zr_step_ms": t_zr,
            "torch_fused_adamw_step_ms": t_torch, "speedup": t_torch / t_zr,
            "zr_gbs_algorithmic": 28 * n / (t_zr * 1e-3) / 1e9}
    print(json.dumps(line), flush=True)
    z.close()


def plan_info(name):
    """A workload's plan and this rank's device footprint, host only (no
    GPU): element counts, buckets, tiles, the workspace and the buffers the
    step reads and writes."""
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    wl = workload(name)
    plan = ZrPlan(wl.shapes, wl.world_size, wl.ranks[0], wl.mode, wl.bucket_cap_bytes, *wl.hp, bind=False)
    n, W = plan.owned_numel, wl.world_size
    info = {"workload": wl.name, "W": W, "rank": wl.ranks[0], "partition": "flat" if wl.mode == 0 else "whole_tensor",
            "tensors": len(wl.shapes), "total_numel": plan.total_numel, "padded_numel": plan.padded_numel,
            "owned_numel": n, "buckets": plan.n_buckets, "segments": len(plan.segments()),
            "bytes": {"gradients": 2 * W * n, "master_m_v": 12 * n, "param_out": 2 * plan.padded_numel,
                      "workspace": plan.workspace_bytes},
            "bytes_per_owned_param": bytes_per_owned_param(W, wl.max_grad_norm > 0)}
    info["bytes"]["total"] = sum(info["bytes"].values())
    plan.close()
    return info


def _owned_params(name):
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    wl = workload(name)
    plan = ZrPlan(wl.shapes, wl.world_size, wl.ranks[0], wl.mode, wl.bucket_cap_bytes, *wl.hp, bind=False)
    n = plan.owned_numel
    plan.close()
    return n


def write_traffic_record(csv_path, full_name, small_name):
    """The record `recorded_traffic` reads: the DRAM bytes of the captured
    launches of one step of `small_name` (an ncu --csv log of
    dram__bytes_read.sum, dram__bytes_write.sum and gpu__time_duration.sum,
    one row per launch and metric), per owned parameter, scaled to
    `full_name`'s owned parameters, with the hash of the kernel source it
    was taken on.  Host only."""
    import csv
    with open(csv_path) as f:
        rows = list(csv.reader(line for line in f if not line.startswith("==")))
    head = rows[0]
    ki, mi, vi, ii = (head.index(k) for k in ("Kernel Name", "Metric Name", "Metric Value", "ID"))
    metrics = {}
    for r in rows[1:]:
        metrics.setdefault((int(r[ii]), r[ki]), {})[r[mi]] = float(r[vi].replace(",", ""))
    launches = []
    for (_, name), m in sorted(metrics.items()):
        short = name
        for k in ("zr_tile_kernel", "zr_clip_combine_small_kernel", "zr_clip_combine_kernel"):
            if k in name:
                a = name.index(k)
                short = name[a:name.index(">", a) + 1] if k == "zr_tile_kernel" else k
                break
        launches.append({"kernel": short, "dram_bytes_read": int(m["dram__bytes_read.sum"]),
                         "dram_bytes_write": int(m["dram__bytes_write.sum"]),
                         "gpu_time_duration_ns": int(m["gpu__time_duration.sum"])})
    full = workload(full_name)
    clip = full.max_grad_norm > 0
    n_small, n_full = _owned_params(small_name), _owned_params(full_name)
    total = sum(x["dram_bytes_read"] + x["dram_bytes_write"] for x in launches)
    stem = f"zr_clip_step_{full_name}" if clip else f"zr_tile_kernel_{full_name}"
    summary = "profiles/zr_clip_step_gpt_1p3b_w8_whole.md" if clip else f"profiles/zr_tile_kernel_{full_name}.md"
    entry = {"kernel": " + ".join(x["kernel"] for x in launches), "launches_per_step": len(launches),
             "small_case": {"workload": small_name, "owned_params": n_small, "per_launch": launches,
                            "dram_bytes": total},
             "bytes_per_owned_param": total / n_small,
             "full_size": {"owned_params": n_full, "scaled_bytes_per_step": total / n_small * n_full,
                           "algorithmic_bytes_per_step": n_full * bytes_per_owned_param(full.world_size, clip)},
             "kernel_source_sha256_16": kernel_source_hash(), "summary": summary}
    out = os.path.join(PROFILES, f"{stem}_traffic.json")
    with open(out, "w") as f:
        json.dump({full_name: entry}, f, indent=2)
        f.write("\n")
    return out, entry


def main():
    args = parse()
    if args.write_traffic_record:
        out, entry = write_traffic_record(args.write_traffic_record, args.config, args.small_case or args.config)
        print(json.dumps({"record": os.path.relpath(out, ROOT), "full_size": entry["full_size"],
                          "bytes_per_owned_param": entry["bytes_per_owned_param"]}), flush=True)
        return
    if args.plan_info:
        print(json.dumps(plan_info(args.config)), flush=True)
        return
    if args.vs_torch:
        run_vs_torch(args)
        return
    if args.zero3_train:
        run_zero3_train(args)
        return
    if args.overlap:
        run_overlap(args)
        return
    if args.zero3:
        run_zero3(args)
        return
    if args.sweep:
        run_sweep(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_zr(args)


if __name__ == "__main__":
    main()
