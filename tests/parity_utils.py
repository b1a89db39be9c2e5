"""Shared helpers of the GPU parity tests: seeded inputs on the device, the
kernel call, and the tolerance check against the fp64 oracle."""
from __future__ import annotations

import json
import math
import os

import numpy as np

import seeded_inputs as si

# Tolerances on O (bf16 output) and LSE (fp32) against the fp64 oracle.  P is
# rounded to bf16 (relative error <= 2^-9) before the P.V product and O is
# stored as bf16 (relative error <= 2^-9 of |O|), so O errors sit well inside
# 2e-2 absolute and 1e-2 relative-L2; LSE only carries fp32 rounding of the
# running max and of the normaliser, far inside 1e-3.
O_MAX_ABS = 2e-2
O_REL_L2 = 1e-2
LSE_MAX_ABS = 1e-3


def to_device(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def inputs(B, H, N, d, seed=0, sigma_qk=1.0, sigma_v=1.0):
    q, k, v = si.make_qkv(B, H, N, d, seed=seed, sigma_qk=sigma_qk, sigma_v=sigma_v)
    return (q, k, v), tuple(to_device(x) for x in (q, k, v))


def run(qt, kt, vt, causal, scale=None):
    import torch
    import attention_forward_17_b200 as fa
    o, lse = fa.fa_fwd(qt, kt, vt, causal=causal, scale=scale)
    torch.cuda.synchronize()
    return o, lse


def o_f64(o) -> np.ndarray:
    import torch
    return o.float().cpu().numpy().astype(np.float64)


def check(o_gpu: np.ndarray, lse_gpu: np.ndarray, o_ref: np.ndarray, lse_ref: np.ndarray, what: str):
    """Assert the tolerances; return the metrics."""
    assert o_gpu.shape == o_ref.shape and lse_gpu.shape == lse_ref.shape, what
    assert np.all(np.isfinite(o_gpu)), f"{what}: non-finite O"
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isfinite(lse_gpu), fin), f"{what}: LSE finiteness differs"
    err = np.abs(o_gpu - o_ref)
    max_abs = float(err.max()) if err.size else 0.0
    denom = float(np.linalg.norm(o_ref))
    rel_l2 = float(np.linalg.norm(o_gpu - o_ref) / denom) if denom > 0 else float(np.linalg.norm(o_gpu))
    lse_err = float(np.abs(lse_gpu[fin] - lse_ref[fin]).max()) if fin.any() else 0.0
    m = dict(o_max_abs=max_abs, o_rel_l2=rel_l2, lse_max_abs=lse_err)
    log = os.environ.get("FA_PARITY_LOG")
    if log:     # one JSON line per comparison, for the record of a GPU run
        with open(log, "a") as f:
            f.write(json.dumps(dict(what=what, rows=int(o_ref.size // max(1, o_ref.shape[-1])), **m)) + "\n")
    assert max_abs <= O_MAX_ABS, f"{what}: O max-abs {max_abs:.3e} > {O_MAX_ABS} ({m})"
    assert rel_l2 <= O_REL_L2, f"{what}: O rel-L2 {rel_l2:.3e} > {O_REL_L2} ({m})"
    assert lse_err <= LSE_MAX_ABS, f"{what}: LSE max-abs {lse_err:.3e} > {LSE_MAX_ABS} ({m})"
    return m


def sample_rows(B, H, N, count, seed=0):
    """Flat row indices bh * N + i: tile edges of a few slices plus random rows."""
    rng = np.random.default_rng(seed)
    BH = B * H
    rows = set()
    for bh in {0, BH - 1, BH // 2}:
        for i in (0, 1, 127, 128, 129, 255, 256, N // 2, N - 129, N - 128, N - 1):
            if 0 <= i < N:
                rows.add(bh * N + i)
    while len(rows) < count:
        rows.add(int(rng.integers(0, BH * N)))
    return np.array(sorted(rows), dtype=np.int64)


def default_scale(d):
    return 1.0 / math.sqrt(d)
