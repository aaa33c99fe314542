"""Build libfa.so in-tree for sm_100a with nvcc.

    python -m exact_attention_119_b200.build [--verbose]

The shared library lands next to this file so it travels with the source
tree; the Python binding loads it from there and nowhere else.
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
LIB = os.path.join(HERE, "libfa.so")
SOURCES = ["fa_api.cu"]
HEADERS = ["sm100.cuh", "fwd_kernel.cuh", "bwd_kernels.cuh", "decode_kernels.cuh"]
INCLUDE = os.path.join(os.path.dirname(HERE), "include")


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    return "nvcc"


def command(verbose: bool = False, out: str = LIB) -> list:
    cmd = [
        nvcc(), "-std=c++17", "-O3", "-lineinfo",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-shared", "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
        "--expt-relaxed-constexpr",
        "-I", INCLUDE,
        "-o", out,
    ]
    if verbose:
        cmd += ["-Xptxas", "-v"]
    cmd += [os.path.join(CSRC, s) for s in SOURCES]
    return cmd


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS] + [os.path.join(INCLUDE, "fa.h")]
    return all(os.path.getmtime(p) <= t for p in deps if os.path.exists(p))


def build(verbose: bool = False, force: bool = False) -> str:
    if force or not up_to_date():
        cmd = command(verbose)
        res = subprocess.run(cmd, capture_output=True, text=True)
        if verbose or res.returncode != 0:
            sys.stderr.write(res.stdout + res.stderr)
        if res.returncode != 0:
            raise RuntimeError("nvcc failed building libfa.so:\n" + " ".join(cmd))
    return LIB


if __name__ == "__main__":
    build(verbose="--verbose" in sys.argv, force=True)
    print(LIB)
