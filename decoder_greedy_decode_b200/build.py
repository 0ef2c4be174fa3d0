"""Build libdec.so in-tree with nvcc for sm_100a (B200)."""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libdec.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def sources():
    return sorted(glob.glob(os.path.join(HERE, "csrc", "*.cu")))


def deps():
    return sources() + glob.glob(os.path.join(HERE, "csrc", "*.h*")) + \
        [os.path.join(ROOT, "include", "dec.h")]


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(p) <= t for p in deps())


def build(force: bool = False, verbose: bool = False, profile: bool = False) -> str:
    """profile=True builds libdec_prof.so with per-phase device timestamps."""
    lib = LIB if not profile else os.path.join(HERE, "libdec_prof.so")
    if not force and not profile and up_to_date():
        return LIB
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [NVCC, "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "--expt-relaxed-constexpr",
           "-I", os.path.join(ROOT, "include"), "-o", tmp] + sources()
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    if profile:
        cmd.insert(1, "-DDEC_PROFILE")
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose="-v" in sys.argv,
                profile="--profile" in sys.argv))
