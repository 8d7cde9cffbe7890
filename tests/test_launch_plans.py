"""moe_expert_gemm's launch arguments for every token count, on the CPU.

tests/launch_plan_check.cu includes the library's host-only launch header
(the path choice, the token chunk, the E4M3 term counts, the workspace
carve-up and both kernels' pipeline plans) and checks, for the V4 and tiny
shapes and T = 1 .. 8192: every argument points at its buffer, the workspace
regions are disjoint and inside moe_expert_gemm_workspace_size(), the size
never shrinks as T grows, and every plan fits TMEM, shared memory and one CTA
per SM.  No GPU and no CUDA call: it only compiles host code with nvcc.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_expert_launch_arguments_for_every_token_count(tmp_path):
    nvcc = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc) and shutil.which(nvcc) is None:
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "launch_plan_check")
    subprocess.check_call([nvcc, "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
                           "-I", os.path.join(ROOT, "include"),
                           "-I", os.path.join(ROOT, "mxfp4_routed_expert_sqrt_b200", "csrc"),
                           "-o", exe, os.path.join(ROOT, "tests", "launch_plan_check.cu")])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout[-4000:]
    assert r.stdout.strip().startswith("ok ")
