"""Builds liboracle.so (plain C, fp64, OpenMP) next to its source.

Test infrastructure: the product never builds against or loads this library.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SOURCES = ["attention_oracle.c", "gemm_oracle.c", "vector_add_oracle.c"]


def library_path() -> str:
    return os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    srcs = [os.path.join(HERE, f) for f in SOURCES]
    out = library_path()
    if not force and os.path.exists(out) and all(
            os.path.getmtime(out) >= os.path.getmtime(s) for s in srcs):
        return out
    tmp = out + ".tmp"
    # -O2 without -ffast-math: IEEE fp64, sums taken in the written order.
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                           "-fno-fast-math", "-ffp-contract=off", *srcs, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True))
