"""fp64 CPU oracle for the attention forward pass.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``, never by the product package.  It
shares no code with the CUDA path; the only thing both sides use is the
seeded input generator in ``seeded_inputs``.

``attention_fwd`` returns, per (b, h) and query row i, the plain definition
  S = scale * Q K^T (fp64), S[i, j] = -inf for j > i when causal,
  P = row softmax of S,  O = P V,  LSE_i = ln sum_j exp(S[i, j])
as in the FlashAttention section of the TileLang tutorial (fused forward over
Q/K/V tiles, validated against scaled-dot-product attention, causal and
non-causal).  ``attention_fwd_strips`` computes the same definition with
fp64 library matrix products (torch on the CPU) as its steps, a strip of
complete query rows at a time, so whole outputs of the large workloads finish
in seconds; it is pinned against ``attention_fwd``.  ``row_softmax`` is the tutorial's row-wise softmax, ``gemm`` its
tiled matrix multiplication with the optional fused bias / bias + GELU
epilogue, ``vector_add`` its elementwise addition.  Every function here is
pinned by ``tests/test_oracle.py`` or ``tests/test_oracle_gemm.py``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build, library_path

_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            _build()
        lib = ctypes.CDLL(path)
        lib.oracle_attention_fwd.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int64] * 4 + [
            ctypes.c_int, ctypes.c_double, ctypes.c_int]
        lib.oracle_attention_fwd.restype = ctypes.c_int
        lib.oracle_attention_rows.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 4 + [
            ctypes.c_int, ctypes.c_double, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int]
        lib.oracle_attention_rows.restype = ctypes.c_int
        lib.oracle_row_softmax.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                           ctypes.c_int64, ctypes.c_double, ctypes.c_int]
        lib.oracle_row_softmax.restype = ctypes.c_int
        lib.oracle_gemm.argtypes = [ctypes.c_void_p] * 4 + [ctypes.c_int64] * 3 + [
            ctypes.c_int, ctypes.c_int]
        lib.oracle_gemm.restype = ctypes.c_int
        lib.oracle_gemm_entries.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64] * 3 + [
            ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_void_p, ctypes.c_int]
        lib.oracle_gemm_entries.restype = ctypes.c_int
        lib.oracle_vector_add.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int64, ctypes.c_int]
        lib.oracle_vector_add.restype = ctypes.c_int
        lib.oracle_threads.argtypes = []
        lib.oracle_threads.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def _bits(a) -> np.ndarray:
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("oracle inputs are bf16 bit patterns (uint16)")
    return a


def default_threads() -> int:
    return int(_lib().oracle_threads())


def attention_fwd(q, k, v, causal: bool, scale: float, threads: int = 0):
    """O (fp64 [B,H,N,d]) and LSE (fp64 [B,H,N]) for bf16-bit inputs [B,H,N,d]."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, H, N, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape
    o = np.zeros((B, H, N, d), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    rc = _lib().oracle_attention_fwd(q.ctypes.data, k.ctypes.data, v.ctypes.data, o.ctypes.data,
                                     lse.ctypes.data, B, H, N, d, int(bool(causal)),
                                     float(scale), int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_fwd failed ({rc})")
    return o, lse


def attention_rows(q, k, v, causal: bool, scale: float, rows, threads: int = 0):
    """O and LSE for selected rows only; rows are flat indices bh * N + i."""
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, H, N, d = q.shape
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.zeros((len(r), d), dtype=np.float64)
    lse = np.zeros(len(r), dtype=np.float64)
    rc = _lib().oracle_attention_rows(q.ctypes.data, k.ctypes.data, v.ctypes.data, B, H, N, d,
                                      int(bool(causal)), float(scale), r.ctypes.data, len(r),
                                      o.ctypes.data, lse.ctypes.data, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_attention_rows failed ({rc})")
    return o, lse


def attention_fwd_strips(q, k, v, causal: bool, scale: float, strip: int = 1024):
    """The definition of ``attention_fwd`` with fp64 matrix products as steps.

    For each (b, h) and each strip of up to ``strip`` complete query rows
    [r0, r1):
      S = scale * Q[r0:r1] K^T              (fp64 matrix product; under the causal
                                             mask only keys j < r1 can be visible)
      S[i, j] = -inf where j > i (causal)
      m = max_j S,  E = exp(S - m),  l = sum_j E
      O = (E V) / l,  LSE = m + ln l
    Every row sees its complete score row, as in ``attention_fwd``; only the
    summation order inside the products differs (a library fp64 product).
    Returns fp64 O [B,H,N,d] and LSE [B,H,N].  Rows whose keys are all masked
    cannot occur with the top-left mask and equal lengths.
    """
    import torch
    q, k, v = _bits(q), _bits(k), _bits(v)
    B, H, N, d = q.shape
    assert k.shape == q.shape and v.shape == q.shape

    def widen(b):
        # bf16 bits -> fp32 (exact: the bits are the upper half of the fp32) -> fp64
        u = torch.from_numpy(b.astype(np.int32) << 16)
        return u.view(torch.float32).to(torch.float64)

    o = np.zeros((B, H, N, d), dtype=np.float64)
    lse = np.zeros((B, H, N), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            qh, kh, vh = widen(q[b, h]), widen(k[b, h]), widen(v[b, h])
            for r0 in range(0, N, strip):
                r1 = min(N, r0 + strip)
                nk = r1 if causal else N
                s = scale * (qh[r0:r1] @ kh[:nk].T)
                if causal:
                    i = torch.arange(r0, r1).unsqueeze(1)
                    j = torch.arange(nk).unsqueeze(0)
                    s.masked_fill_(j > i, float("-inf"))
                m = s.max(dim=1, keepdim=True).values
                e = torch.exp(s - m)
                l = e.sum(dim=1, keepdim=True)
                o[b, h, r0:r1] = ((e @ vh[:nk]) / l).numpy()
                lse[b, h, r0:r1] = (m + torch.log(l)).squeeze(1).numpy()
    return o, lse


def row_softmax(x, scale: float = 1.0, threads: int = 0):
    """fp64 row-wise softmax of bf16 bits x [rows, cols]: exp(scale*x - max) / sum."""
    x = _bits(x)
    rows, cols = x.shape
    y = np.zeros((rows, cols), dtype=np.float64)
    rc = _lib().oracle_row_softmax(x.ctypes.data, y.ctypes.data, rows, cols, float(scale),
                                   int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_row_softmax failed ({rc})")
    return y


GEMM_PLAIN, GEMM_BIAS, GEMM_BIAS_GELU = 0, 1, 2


def _ptr(a):
    return a.ctypes.data if a is not None and a.size else None


def gemm(a, b, bias=None, mode: int = GEMM_BIAS_GELU, threads: int = 0):
    """fp64 C [M, N] = epilogue(A B) for bf16 bits A [M, K], B [K, N], bias [N]."""
    a, b = _bits(a), _bits(b)
    M, K = a.shape
    K2, N = b.shape
    assert K == K2
    bias = None if bias is None else _bits(bias)
    if mode and bias is not None:
        assert bias.shape == (N,)
    c = np.zeros((M, N), dtype=np.float64)
    rc = _lib().oracle_gemm(_ptr(a), _ptr(b), _ptr(bias), c.ctypes.data, M, N, K, int(mode),
                            int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm failed ({rc})")
    return c


def gemm_entries(a, b, bias, idx, mode: int = GEMM_BIAS_GELU, threads: int = 0):
    """C entries at flat indices idx (i * N + j), arithmetic as ``gemm``."""
    a, b = _bits(a), _bits(b)
    M, K = a.shape
    N = b.shape[1]
    bias = None if bias is None else _bits(bias)
    r = np.ascontiguousarray(np.asarray(idx, dtype=np.int64))
    out = np.zeros(len(r), dtype=np.float64)
    rc = _lib().oracle_gemm_entries(_ptr(a), _ptr(b), _ptr(bias), M, N, K, int(mode),
                                    r.ctypes.data, len(r), out.ctypes.data, int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_gemm_entries failed ({rc})")
    return out


def vector_add(x, y, threads: int = 0):
    """fp64 z = x + y for float32 x, y of equal length."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    y = np.ascontiguousarray(y, dtype=np.float32)
    assert x.shape == y.shape
    z = np.zeros(x.shape, dtype=np.float64)
    rc = _lib().oracle_vector_add(x.ctypes.data, y.ctypes.data, z.ctypes.data, x.size,
                                  int(threads))
    if rc != 0:
        raise RuntimeError(f"oracle_vector_add failed ({rc})")
    return z
