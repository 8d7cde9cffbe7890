"""Build step for the CUDA library (sm_100a) and the device input generator.

    python -m mxfp4_routed_expert_sqrt_b200.build [--force]
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
NVCC = os.environ.get("NVCC", "nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC", "--expt-relaxed-constexpr"]


def _stale(target: str, sources) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_libmoe(force: bool = False, debug: bool = False) -> str:
    """libmoe.so, or with debug=True libmoe_debug.so: the same library built
    with -DMOE_DEBUG, whose kernels check the indices they otherwise trust and
    report a bad one through moe_device_error() instead of touching memory
    out of bounds."""
    out = os.path.join(PKG, "libmoe_debug.so" if debug else "libmoe.so")
    srcs = glob.glob(os.path.join(PKG, "csrc", "*")) + [os.path.join(ROOT, "include", "moe.h")]
    if force or _stale(out, srcs):
        cmd = [NVCC, *ARCH, *FLAGS, *(["-DMOE_DEBUG"] if debug else []), "-I", os.path.join(ROOT, "include"),
               os.path.join(PKG, "csrc", "moe.cu"), "-o", out]
        subprocess.check_call(cmd)
    return out


def build_gen(force: bool = False) -> str:
    src = os.path.join(ROOT, "gen", "gen_device.cu")
    out = os.path.join(ROOT, "gen", "libmoegen.so")
    if force or _stale(out, [src]):
        subprocess.check_call([NVCC, *ARCH, *FLAGS, src, "-o", out])
    return out


def build_all(force: bool = False) -> None:
    build_libmoe(force)
    build_libmoe(force, debug=True)
    build_gen(force)


if __name__ == "__main__":
    build_all(force="--force" in sys.argv)
