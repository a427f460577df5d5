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
    assert d["zero3_step_ms"] > 0 and d["zero_adamw_step_ms"] > 0


def test_vs_torch_mode():
    d = run_mode("--vs-torch")
    assert d["mode"] == "vs_torch_adamw" and d["zr_step_ms"] > 0 and d["torch_fused_adamw_step_ms"] > 0
