"""Builds libfa_b200.so, the sm_100a attention library, in-tree with nvcc.

The library is self-contained: CUDA runtime linked statically, the driver's
tensor-map encoder fetched at run time, no torch symbols.
"""
from __future__ import annotations

import glob
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")

NVCC_FLAGS = [
    "-gencode", "arch=compute_100a,code=sm_100a",
    "-O3", "-std=c++17", "-lineinfo",
    "-Xcompiler", "-fPIC", "-shared",
    "-Xptxas", "-v",
]


def library_path() -> str:
    return os.path.join(HERE, "libfa_b200.so")


def _sources():
    return [os.path.join(CSRC, f) for f in
            ("fa_fwd.cu", "fa_fwd_sched_d128.cu", "fa_fwd_sched_d64.cu", "row_softmax.cu",
             "gemm_bias_gelu.cu", "vector_add.cu")]


def _deps():
    return (_sources() + glob.glob(os.path.join(CSRC, "*.cuh"))
            + glob.glob(os.path.join(CSRC, "*.h"))
            + glob.glob(os.path.join(ROOT, "include", "*.h")))


def build(force: bool = False, verbose: bool = False) -> str:
    out = library_path()
    if (not force and os.path.exists(out)
            and all(os.path.getmtime(out) >= os.path.getmtime(p) for p in _deps())):
        return out
    nvcc = os.environ.get("NVCC", "nvcc")
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include")]
    flags = [f for f in NVCC_FLAGS if f != "-shared"]

    def compile_one(src):
        obj = os.path.join(objdir, os.path.basename(src) + ".o")
        cmd = [nvcc, *flags, *inc, "-c", src, "-o", obj]
        res = subprocess.run(cmd, capture_output=True, text=True)
        return obj, " ".join(cmd) + "\n" + res.stdout + res.stderr, res.returncode

    # the translation units compile independently; run them side by side
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as pool:
        results = list(pool.map(compile_one, _sources()))
    log = "".join(r[1] for r in results)
    failed = any(r[2] != 0 for r in results)
    tmp = out + ".tmp"
    if not failed:
        cmd = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a",
               *[r[0] for r in results], "-o", tmp]
        res = subprocess.run(cmd, capture_output=True, text=True)
        log += " ".join(cmd) + "\n" + res.stdout + res.stderr
        failed = res.returncode != 0
    with open(os.path.join(HERE, "build.log"), "w") as f:
        f.write(log)
    if failed:
        sys.stderr.write(log)
        raise RuntimeError("nvcc failed building libfa_b200.so")
    if verbose:
        sys.stdout.write(log)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force=True, verbose=True))
