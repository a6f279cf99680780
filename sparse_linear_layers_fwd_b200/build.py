"""Build step of libsbn.so: nvcc for sm_100a, in-tree, no JIT cache.

    python -m sparse_linear_layers_fwd_b200.build [--verbose]
"""

from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libsbn.so")
SOURCES = [os.path.join(CSRC, "sbn.cu")]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _deps():
    files = list(SOURCES)
    for d in (CSRC, INCLUDE):
        for f in os.listdir(d):
            if f.endswith((".cuh", ".h", ".cu")):
                files.append(os.path.join(d, f))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _deps())


def nvcc_command(out=LIB, ptxas_verbose=False):
    cmd = [
        NVCC, "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC", "-shared", "--cudart", "static",
        "-I", INCLUDE, "-I", CSRC,
        "-o", out,
    ] + SOURCES
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    return cmd


def build(force: bool = False, verbose: bool = False) -> str:
    """Compile libsbn.so next to this file (skipped when up to date)."""
    if not force and up_to_date():
        return LIB
    cmd = nvcc_command(ptxas_verbose=verbose)
    tmp = LIB + ".tmp"
    cmd[cmd.index("-o") + 1] = tmp
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("nvcc failed:\n" + " ".join(cmd) + "\n" + r.stdout + r.stderr)
    if verbose:
        sys.stderr.write(r.stdout + r.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
