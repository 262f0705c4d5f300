"""Build the C-ABI library libflashmap_b200.so for sm_100a with nvcc.

Usage: python -m step_flow_map_b200.build [--verbose]
The library lands next to this file, so it travels with the source tree.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "libflashmap_b200.so")
SRC = os.path.join(HERE, "csrc", "fm_api.cu")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def command(out: str = LIB, extra=()) -> list:
    return [
        nvcc(), "-O3", "-std=c++17", "-shared", "-Xcompiler", "-fPIC",
        "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(HERE, "csrc"),
        "--expt-relaxed-constexpr", "--extended-lambda",
        *extra, SRC, "-o", out,
    ]


def sources() -> list:
    csrc = os.path.join(HERE, "csrc")
    files = [os.path.join(csrc, f) for f in os.listdir(csrc)]
    files.append(os.path.join(ROOT, "include", "flashmap.h"))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in sources())


def build(force: bool = False, verbose: bool = False, extra=()) -> str:
    if not force and up_to_date():
        return LIB
    cmd = command(extra=extra)
    if verbose:
        print(" ".join(cmd), flush=True)
    tmp = LIB + ".tmp"
    cmd[cmd.index(LIB)] = tmp
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed building libflashmap_b200.so")
    if verbose and (res.stdout or res.stderr):
        sys.stderr.write(res.stdout + res.stderr)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    v = "--verbose" in sys.argv
    extra = ["-Xptxas", "-v"] if "--ptxas" in sys.argv else []
    print(build(force=True, verbose=v, extra=extra))
