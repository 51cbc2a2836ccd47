"""Compile the CPU oracle (plain C, fp64, OpenMP) into oracle/liboracle_paged_decode.so.

Test infrastructure: the CUDA library never links or loads this.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "paged_decode_oracle.c")
LIB = os.path.join(HERE, "liboracle_paged_decode.so")
GEMV_SRC = os.path.join(HERE, "gemv_oracle.c")
GEMV_LIB = os.path.join(HERE, "liboracle_gemv.so")
PREFILL_SRC = os.path.join(HERE, "paged_prefill_oracle.c")
PREFILL_LIB = os.path.join(HERE, "liboracle_paged_prefill.so")


def _build_one(src: str, lib: str, force: bool, verbose: bool) -> str:
    if not force and os.path.exists(lib) and os.path.getmtime(lib) >= os.path.getmtime(src):
        return lib
    # -O2 without -ffast-math: IEEE double arithmetic in program order.
    tmp = lib + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-fPIC",
           "-shared", "-Wall", "-Wextra", "-o", tmp, src, "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(tmp, lib)
    return lib


def build(force: bool = False, verbose: bool = False) -> str:
    """Build every oracle library; returns the decode-attention one."""
    _build_one(GEMV_SRC, GEMV_LIB, force, verbose)
    _build_one(PREFILL_SRC, PREFILL_LIB, force, verbose)
    return _build_one(SRC, LIB, force, verbose)


def build_gemv(force: bool = False, verbose: bool = False) -> str:
    return _build_one(GEMV_SRC, GEMV_LIB, force, verbose)


def build_prefill(force: bool = False, verbose: bool = False) -> str:
    return _build_one(PREFILL_SRC, PREFILL_LIB, force, verbose)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True))
