"""The stream-K partition arithmetic of the tensor-core GEMMs and the row
groups of their epilogues, checked on the CPU: stream_k_check.cu includes the
kernels' own headers, calls their host-callable index helpers over the launch
shapes the library uses and checks that every unit and row is covered once,
that each tile's contributors and fix-up slots agree between the producing
CTAs and the reducing ones, and that the part slots fit their allocation."""

import os
import shutil
import subprocess

import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


def _nvcc():
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return None


def test_stream_k_partition_and_row_groups(tmp_path):
    nvcc = _nvcc()
    if nvcc is None:
        pytest.skip("nvcc not found")
    exe = str(tmp_path / "stream_k_check")
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-O2",
                    "-diag-suppress", "550", "-I", os.path.join(ROOT, "include"), "-o", exe,
                    os.path.join(HERE, "stream_k_check.cu")], check=True, timeout=600)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout[-3000:]
