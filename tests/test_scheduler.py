"""The forward kernel's work schedule, checked on the CPU with the kernel's
own decode functions (tests/c/sched_check.cu compiles them for the host).

For plain and causal calls every (batch, head, Q tile) is scheduled exactly
once with the KV tile count its rows need (brute force over the rows), and
within a chunk of heads the heaviest Q-tile pairs come first.  Under a band
every visible key of every valid row lies in its tile's KV range and both
ends of the range are used.  Under split-KV the slices of every (batch,
head, Q-tile pair) cover its KV tiles exactly once.  Several chunk sizes."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not os.path.exists(NVCC) and shutil.which("nvcc") is None, reason="needs nvcc")
def test_schedule_covers_every_tile_once(tmp_path):
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    exe = tmp_path / "sched_check"
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(ROOT, "tiled_attention_13_b200", "csrc"),
           "-o", str(exe), os.path.join(ROOT, "tests", "c", "sched_check.cu")]
    r = subprocess.run(cmd, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0 and "sched ok" in r.stdout, r.stdout[-3000:]
