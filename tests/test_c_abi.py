"""The C ABI from plain C: tests/c/zr_c_abi_test.c is compiled with gcc
against include/zr.h and linked to libzr.so (compiled on any machine; run
on a GPU)."""
import os
import subprocess

import pytest

import sharded_optimizer_step_zr_b200 as zr
from conftest import ROOT

CUDA = "/usr/local/cuda"


def build_c_test(tmp_path):
    exe = os.path.join(str(tmp_path), "zr_c_abi_test")
    lib_dir = os.path.dirname(zr.LIB_PATH)
    subprocess.check_call(["gcc", "-std=c11", "-O1", "-Wall", "-Werror",
                           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                           os.path.join(ROOT, "tests", "c", "zr_c_abi_test.c"), "-o", exe,
                           "-L", lib_dir, "-lzr", f"-Wl,-rpath,{lib_dir}",
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{CUDA}/lib64",
                           "-lm"])
    return exe


def test_c_program_compiles_and_links(tmp_path):
    assert os.path.exists(build_c_test(tmp_path))


@pytest.mark.gpu
def test_c_program_runs(tmp_path):
    exe = build_c_test(tmp_path)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "mismatches 0" in out.stdout
