"""The kernels' scheduling arithmetic (common.cuh), checked on the CPU: nvcc
compiles tests/c/sched_check.cu as host code against the real header and the
program compares FastDiv with plain division and the tile schedule (ranges per
CTA, owner of a tile, CTAs per segment, partial-slot indices) with a
brute-force count on the workloads' shapes and random ones."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "linear_attention_video_relu_b200", "csrc")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc (host compilation only)")
def test_schedule_arithmetic(tmp_path):
    exe = tmp_path / "sched_check"
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
                           "-O1", "-I", CSRC,
                           os.path.join(ROOT, "tests", "c", "sched_check.cu"), "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="needs nvcc (host compilation only)")
def test_shared_memory_plans(tmp_path):
    # every state, apply and causal plan fits its budget with at least two
    # stages; two half-budget apply CTAs fit an SM; the 480p plans are the
    # intended ones
    exe = tmp_path / "plan_check"
    subprocess.check_call(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
                           "-O1", "--expt-relaxed-constexpr", "-I", CSRC,
                           "-I", os.path.join(ROOT, "include"),
                           os.path.join(ROOT, "tests", "c", "plan_check.cu"), "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=600)
    assert r.returncode == 0 and r.stdout.startswith("ok"), r.stdout + r.stderr
