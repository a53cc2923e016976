"""Build libnvfp4.so in-tree with nvcc for sm_100a (cross-compiles without a GPU).

Also builds libnvfp4_testhooks.so, the same sources with NVFP4_TEST_HOOKS defined: the tests use it to
make a device-side wait run out on purpose (see nvfp4_test_withhold_split_ready in nvfp4_api.cu); the
product library has no such hook.

    python -m epilogue_gemm_nvfp4_b200.build [--force] [--ptxas-verbose]
"""
from __future__ import annotations

import argparse
import glob
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libnvfp4.so")
TEST_LIB = os.path.join(PKG, "libnvfp4_testhooks.so")
MAIN = os.path.join(CSRC, "nvfp4_api.cu")


def nvcc() -> str:
    path = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(path):
        raise RuntimeError("nvcc not found: the NVFP4 library needs the CUDA toolkit to build")
    return path


def sources() -> list[str]:
    return sorted(glob.glob(os.path.join(CSRC, "*.cu*")) + [os.path.join(ROOT, "include", "nvfp4.h")])


def up_to_date() -> bool:
    if not (os.path.exists(LIB) and os.path.exists(TEST_LIB)):
        return False
    t = min(os.path.getmtime(LIB), os.path.getmtime(TEST_LIB))
    return all(os.path.getmtime(s) <= t for s in sources())


def command(ptxas_verbose: bool = False, test_hooks: bool = False) -> list[str]:
    cmd = [nvcc(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "--expt-relaxed-constexpr", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-shared",
           "-I", os.path.join(ROOT, "include"), "-o", TEST_LIB if test_hooks else LIB, MAIN]
    if test_hooks:
        cmd[1:1] = ["-DNVFP4_TEST_HOOKS"]
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    return cmd


def build(force: bool = False, ptxas_verbose: bool = False, quiet: bool = False) -> str:
    """Compile both libraries (in parallel); returns the product library's path."""
    if not force and not ptxas_verbose and up_to_date():
        return LIB
    cmds = [command(ptxas_verbose), command(False, test_hooks=True)]
    procs = [subprocess.Popen(c, stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True) for c in cmds]
    for cmd, p in zip(cmds, procs):
        out, err = p.communicate()
        if p.returncode != 0:
            raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + out + err)
        if (ptxas_verbose and cmd is cmds[0]) or not quiet:
            text = (out + err).strip()
            if text:
                print(text, file=sys.stderr)
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--ptxas-verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, ptxas_verbose=a.ptxas_verbose))
