"""Host logic of the block-scaled GEMM: its work schedule, checked on the CPU.

tests/schedule_check.cu includes the library's host source and checks build_schedule on the
64-layer stack, single matrices and 300 random stacks (coverage of every k-tile exactly once,
split bookkeeping, k order of split parts, workspace limits, balance). It is compiled for the
host with nvcc (device code is compiled but never launched)."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _nvcc():
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", shutil.which("nvcc")):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_block_scaled_schedule(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not available")
    exe = tmp_path / "schedule_check"
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "-O1",
                    "-I", os.path.join(ROOT, "include"), "-o", str(exe),
                    os.path.join(ROOT, "tests", "schedule_check.cu"), "-lcuda"],
                   check=True, capture_output=True, timeout=600)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    assert "bad=0" in out.stdout
