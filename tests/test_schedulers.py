"""The kernels' work schedulers, checked on the host (no GPU): tests/sched_check.cu
includes the kernel headers and calls the same __host__ __device__ functions the
kernels call (tile decoding, key-block trip counts, key splits)."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_schedulers_cover_every_tile_once(tmp_path):
    nvcc = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = tmp_path / "sched_check"
    subprocess.run([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "exact_io_aware_100_b200", "csrc"),
                    "-o", str(exe), os.path.join(ROOT, "tests", "sched_check.cu")], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip().endswith("OK"), out.stdout + out.stderr
