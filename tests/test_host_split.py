"""Host logic of the kernels, checked by small C++ programs compiled with the
kernels' own sources (nvcc is needed; no GPU): the M <= 8 GEMV's work split
and shared-memory plans, and the batched GEMM's level decode, A-stage layout
and stream-K split."""
import os
import shutil
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_gemv_work_split_and_layouts():
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "split_check")
        subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
                               "--expt-relaxed-constexpr", "-w", "-I", os.path.join(ROOT, "include"),
                               "-I", os.path.join(ROOT, "nested_bit_weight_b200", "csrc"),
                               os.path.join(ROOT, "tests", "host", "gemv_split_check.cu"), "-o", exe],
                              timeout=600)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    checked = int(out.stdout.split("checked=")[1].split()[0])
    assert checked > 1000 and "bad=0" in out.stdout, out.stdout


@pytest.mark.skipif(not (os.path.exists(NVCC) or shutil.which("nvcc")), reason="nvcc not found")
def test_gemm_decode_and_work_split():
    # the batched GEMM's natural-order level decode against the level
    # definition, its A-stage layout and its stream-K split
    nvcc = NVCC if os.path.exists(NVCC) else shutil.which("nvcc")
    with tempfile.TemporaryDirectory() as d:
        exe = os.path.join(d, "gemm_check")
        subprocess.check_call([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-std=c++17",
                               "--expt-relaxed-constexpr", "-w", "-I", os.path.join(ROOT, "include"),
                               "-I", os.path.join(ROOT, "nested_bit_weight_b200", "csrc"),
                               os.path.join(ROOT, "tests", "host", "gemm_decode_check.cu"), "-o", exe],
                              timeout=600)
        out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stdout + out.stderr
    checked = int(out.stdout.split("checked=")[1].split()[0])
    assert checked > 100000 and "bad=0" in out.stdout, out.stdout
