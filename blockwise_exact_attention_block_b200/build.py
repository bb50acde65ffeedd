"""Build libra_b200.so (the C-ABI library) in-tree with nvcc for sm_100a.

    python blockwise_exact_attention_block_b200/build.py [--verbose-ptxas] [--debug-bounds]

(run as a file: importing the package loads the library it builds)

csrc/api.cu is the main translation unit (it includes every kernel);
csrc/noalloc.cu adds the entry point whose scratch is a fixed device array.
--debug-bounds builds the checked variant libra_b200_debug.so instead
(-DRA_DEBUG_BOUNDS: every run-time-indexed global access is checked; the
binding loads it when RA_DEBUG_BOUNDS=1 is set in the environment).
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRCS = [os.path.join(PKG, "csrc", "api.cu"), os.path.join(PKG, "csrc", "noalloc.cu")]
OUT = os.path.join(PKG, "libra_b200.so")
OUT_DEBUG = os.path.join(PKG, "libra_b200_debug.so")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def sources():
    d = os.path.join(PKG, "csrc")
    return [os.path.join(d, f) for f in sorted(os.listdir(d)) if f.endswith((".cu", ".cuh"))] + [
        os.path.join(ROOT, "include", "ra.h")]


def up_to_date(out: str = OUT) -> bool:
    if not os.path.exists(out):
        return False
    t = os.path.getmtime(out)
    return all(os.path.getmtime(s) <= t for s in sources())


def build(force: bool = False, ptxas_verbose: bool = False, debug_bounds: bool = False) -> str:
    out = OUT_DEBUG if debug_bounds else OUT
    if not force and up_to_date(out):
        return out
    cmd = [nvcc_path(), "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
           "-Xcompiler", "-fPIC", "-shared", "-I", os.path.join(ROOT, "include"), *SRCS, "-o", out + ".tmp"]
    if debug_bounds:
        cmd.insert(1, "-DRA_DEBUG_BOUNDS")
    if ptxas_verbose:
        cmd[1:1] = ["-Xptxas", "-v"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + res.stdout + res.stderr)
    if ptxas_verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True, ptxas_verbose="--verbose-ptxas" in sys.argv, debug_bounds="--debug-bounds" in sys.argv))
