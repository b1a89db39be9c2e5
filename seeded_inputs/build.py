"""Builds libseeded_inputs.so (plain C, OpenMP) next to its source."""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(HERE, "libseeded_inputs.so")


def build(force: bool = False) -> str:
    src = os.path.join(HERE, "philox_normal.c")
    out = library_path()
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp"
    subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-std=c11",
                           src, "-o", tmp, "-lm"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True))
