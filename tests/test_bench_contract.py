"""bench.py's output contract, checked on the CPU through its reference arm
(the oracle timed on a bounded sample) and its helpers."""
import json
import os
import subprocess
import sys

import bench
import synth
from conftest import ROOT


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "1", "--cpu-threads", "2"], capture_output=True, text=True,
                         timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "scaling",
              "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e", "impl"):
        assert k in d, k
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "Gparams/s"
    assert d["config"]["workload"] == bench.DEFAULT_CONFIG
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 2
    assert "2 thread(s)" in d["cpu_baseline"]["sample"] and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"]
    assert d["value"] > 0


def test_algorithmic_bytes_per_param():
    # 2W gradient reads + 12 state reads + 12 state writes + 2 bf16 writes
    assert bench.bytes_per_owned_param(8, False) == 42
    assert bench.bytes_per_owned_param(64, False) == 154
    assert bench.bytes_per_owned_param(8, True) == 50     # + fp32 g scratch write and read
    assert bench.bytes_per_owned_param(2, True) == 34     # + gradients read again


def test_shard_rank_and_workloads():
    wl = synth.WORKLOADS["gpt_1p3b_w8_whole_clip"]
    assert bench.shard_rank(wl, 0, 1) == 3
    assert [bench.shard_rank(wl, i, 8) for i in range(8)] == [3, 4, 5, 6, 7, 0, 1, 2]
    assert bench.workload("gpt2_124m_w8").world_size == 8
    assert len(synth.sweep_workloads()) == 40


def test_threaded_oracle_sample_covers_disjoint_slices():
    wl = synth.WORKLOADS["tiny"]
    multi = bench.OracleSamples(wl, 0, 1 << 12, 4)
    assert multi.threads == 4 and [x.n for x in multi.samples] == [1024] * 4
    # consecutive, disjoint slices of the rank's owned elements
    import oracle
    oplan = oracle.Plan(wl.shapes, wl.world_size, wl.mode, wl.bucket_cap_bytes)
    idx = oplan.owned_global_index(0)
    one = bench.OracleSample(wl, 0, 4096)
    for i, x in enumerate(multi.samples):
        assert (x.master == one.master[i * 1024:(i + 1) * 1024]).all()
    rate, desc = multi.run(0.2)
    assert rate > 0 and "4 thread(s)" in desc
    assert idx.size == multi.owned


class _FakeNvml:
    """Stands in for pynvml: a fixed SM clock and throttle-reason mask."""
    NVML_CLOCK_SM = 1
    nvmlClocksEventReasonSwPowerCap = 0x4
    nvmlClocksEventReasonHwSlowdown = 0x8

    def __init__(self, mhz, reasons):
        self.mhz, self.mask, self.calls = mhz, reasons, 0

    def nvmlInit(self):
        pass

    def nvmlDeviceGetHandleByIndex(self, i):
        return i

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        self.calls += 1
        return self.mhz

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return self.mask


def test_clock_sampler_against_a_fake_nvml(monkeypatch):
    import time
    fake = _FakeNvml(1800, 0x4 | 0x8)
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    with bench.ClockSampler(0) as s:
        time.sleep(0.05)
    out = s.summary()
    assert out["sm_mhz"] == 1800 and out["sm_max_mhz"] == 1965 and out["samples"] >= 1
    assert out["reasons"] == ["hw_slowdown", "sw_power_cap"]
    # a region too short for the thread's first read still gets one, at its end
    fake2 = _FakeNvml(1965, 0)
    monkeypatch.setitem(sys.modules, "pynvml", fake2)
    s2 = bench.ClockSampler(0)
    s2._run = lambda: None
    with s2:
        pass
    assert s2.summary()["samples"] == 1 and s2.summary()["reasons"] == []


def test_recorded_traffic_is_close_to_the_algorithmic_bytes():
    """The committed ncu DRAM records stay within a few percent of the
    algorithmic bytes (no re-reads; a write-back still in L2 when the kernel
    ends makes them a little lower).  A record taken on an older kernel
    source is not used: the bench then reports traffic as null."""
    from sharded_optimizer_step_zr_b200.plan import ZrPlan
    for name, clip in (("gpt2_124m_w8", False), ("llama_7b_w64", False), ("gpt_1p3b_w8_whole_clip", True)):
        wl = synth.WORKLOADS[name]
        plan = ZrPlan(wl.shapes, wl.world_size, wl.ranks[0], wl.mode, wl.bucket_cap_bytes, *wl.hp, bind=False)
        t, note = bench.recorded_traffic(name, clip, plan.owned_numel)
        alg = plan.owned_numel * bench.bytes_per_owned_param(wl.world_size, clip)
        plan.close()
        if t is None:
            assert note in ("ncu record taken on an older kernel source", "no ncu record for this workload")
            continue
        assert 0.88 * alg <= t <= 1.02 * alg, (name, t, alg, note)


def test_reference_arm_other_ranks_exit_quietly():
    """Under torchrun (N > 1) only rank 0 runs and prints the reference
    arm; the other ranks exit 0 without work or output."""
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=300,
                         cwd=ROOT, env=env)
    assert out.returncode == 0, out.stderr[-2000:]
    assert out.stdout.strip() == ""


def test_plan_info_footprints():
    """--plan-info on the host: the footprints stated for the GPT-2 and
    Llama-7B workloads (249 MB of gradients and 187 MB of state at W = 8;
    about 28 GB in all at W = 64)."""
    g = bench.plan_info("gpt2_124m_w8")
    assert g["owned_numel"] == 15554976 and g["bytes"]["gradients"] == 248879616
    assert g["bytes"]["master_m_v"] == 186659712 and g["bytes_per_owned_param"] == 42
    ll = bench.plan_info("llama_7b_w64")
    assert ll["owned_numel"] == 105287744 and ll["total_numel"] == 6738415616
    assert 27e9 < ll["bytes"]["total"] < 29e9
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--plan-info", "--config", "tiny"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0 and json.loads(out.stdout)["total_numel"] == 1441792
