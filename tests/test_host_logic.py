"""Host-side logic of the CUDA path, checked without a GPU."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_row_range_schedule(tmp_path):
    """Compiles the kernels' schedule code (sa_internal.h) for the host and
    checks coverage, slot uniqueness and finalize ownership on thousands of
    random ragged batches."""
    exe = tmp_path / "schedule_check"
    cuda_inc = "/usr/local/cuda/include"
    subprocess.run(["g++", "-O1", "-std=c++17",
                    "-I", os.path.join(ROOT, "sketch_attention_compression_b200", "csrc"),
                    "-I", os.path.join(ROOT, "include"),
                    "-I", cuda_inc, os.path.join(ROOT, "tests", "host", "schedule_check.cpp"),
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("OK")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs g++")
def test_shared_memory_plan(tmp_path):
    """Compiles the fused pass's shared-memory plan (sa_plan.h) for the host
    and checks that its regions are disjoint and that every MMA2 operand
    reads its chunks (X boxes, then the block of ones) at its stride."""
    exe = tmp_path / "plan_check"
    subprocess.run(["g++", "-O1", "-std=c++17",
                    "-I", os.path.join(ROOT, "sketch_attention_compression_b200", "csrc"),
                    "-I", os.path.join(ROOT, "include"),
                    "-I", "/usr/local/cuda/include", os.path.join(ROOT, "tests", "host", "plan_check.cpp"),
                    "-o", str(exe)], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0, out.stdout + out.stderr
    assert out.stdout.startswith("OK")

