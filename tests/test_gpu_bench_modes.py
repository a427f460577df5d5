"""The benchmark's extra modes run on the GPU and print their record: the
ZeRO-3 gather (GPT-2 set), the layer-loop training comparison (whose
Zero3 and ZeroAdamW runs must end with the same parameters) and the
comparison with PyTorch's fused AdamW recipe."""
import json
import os
import subprocess
import sys

import pytest

from conftest import ROOT

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def run_mode(*flags):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *flags], capture_output=True,
                         text=True, timeout=900, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_zero3_gather_mode():
    d = run_mode("--zero3", "--zero3-set", "gpt2")
    assert d["mode"] == "zero3_gather" and d["params"] == 124439808
    assert 0.3 < d["roofline"]["frac_whole_model"] < 1.3
    assert set(d["exposed_gather_prefetched_us"]) == {"default", "high", "high_16_ctas", "high_32_ctas"}


def test_zero3_train_mode_takes_identical_steps():
    d = run_mode("--zero3-train")
    assert d["mode"] == "zero3_train" and d["same_parameters"] is True
    assert d["reduce_in_backward_same_parameters"] is True and d["overlap_same_parameters"] is True
    assert d["gradient_bytes"]["zero3_reduce_in_backward"] < d["gradient_bytes"]["zero3"] / 4
    assert d["zero3_step_ms"] > 0 and d["zero_adamw_step_ms"] > 0


def test_vs_torch_mode():
    d = run_mode("--vs-torch")
    assert d["mode"] == "vs_torch_adamw" and d["zr_step_ms"] > 0 and d["torch_fused_adamw_step_ms"] > 0


def test_peer_mode_two_processes_one_gpu():
    """`bench.py --gpus 2` as torchrun launches it, both processes on this
    machine's one GPU (gloo for the host barriers; the kernels never wait on
    the other process): the headline line, and the peer step of a W = 2 job
    whose gradient loads and parameter stores cross into the other
    process's memory through CUDA IPC.  The NCCL arm needs one GPU per
    process and reports that it was skipped."""
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes", "1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.join(ROOT, "bench.py"),
           "--gpus", "2", "--backend", "gloo", "--same-gpu", "--config", "gpt2_124m_w8", "--no-companions",
           "--no-cpu-baseline", "--no-e2e", "--peer-set", "gpt2_124m", "--steps", "20", "--warmup", "3",
           "--peer-steps", "5"]
    out = subprocess.run(["timeout", "-k", "30", "600"] + cmd, capture_output=True, text=True, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-3000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["config"]["workload"] == "gpt2_124m_w8" and d["value"] > 0
    p = d["peer"]
    assert p["W"] == 2 and p["param_set"] == "gpt2_124m" and p["value"] > 0
    assert p["owned_params"] == 124439808 // 2
    assert p["bytes_per_step_per_rank"]["peer_loads"] == 2 * p["owned_params"]
    assert "skipped" in p["nccl_arm"]


def test_gather_targets_and_no_alloc_modes():
    """The step with W parameter buffers as gather targets (56 B per owned
    parameter at W = 8) and through zr_step_no_alloc report their lines."""
    base = ["--config", "gpt2_124m_w8", "--no-companions", "--no-e2e", "--no-cpu-baseline",
            "--steps", "20", "--warmup", "3"]
    d = run_mode(*base, "--gather-targets")
    assert d["config"]["gather_targets"] == 8 and d["config"]["bytes_per_owned_param"] == 56
    assert d["value"] > 0 and d["roofline"]["traffic"] is None
    d = run_mode(*base, "--no-alloc")
    assert d["config"]["no_alloc"] is True and d["value"] > 0
