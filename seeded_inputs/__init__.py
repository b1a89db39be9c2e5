"""Seeded synthetic inputs shared by the oracle and the CUDA path.

The generator (Philox4x32-10 counter-based bits, Box-Muller normals, one
round-to-nearest-even step to bf16) lives in ``philox_normal.c``; this module
only builds and calls it.  It holds none of the kernels' arithmetic, so
importing it from both sides couples nothing but the input bytes.

bf16 tensors are returned as numpy ``uint16`` arrays of bit patterns, fp32
tensors as ``float32`` arrays.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from .build import build as _build, library_path

_LIB = None

TENSOR_Q, TENSOR_K, TENSOR_V = 0, 1, 2
TENSOR_GEMM_A, TENSOR_GEMM_B, TENSOR_GEMM_BIAS = 3, 4, 5
TENSOR_ADD_X, TENSOR_ADD_Y = 6, 7


def _lib():
    global _LIB
    if _LIB is None:
        path = library_path()
        if not os.path.exists(path):
            _build()
        lib = ctypes.CDLL(path)
        lib.seeded_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                           ctypes.c_uint32, ctypes.c_double]
        lib.seeded_normal_bf16.restype = None
        lib.seeded_normal_f32.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64,
                                          ctypes.c_uint32, ctypes.c_double]
        lib.seeded_normal_f32.restype = None
        lib.seeded_philox4x32.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int,
                                          ctypes.c_void_p]
        lib.seeded_philox4x32.restype = None
        lib.seeded_round_bf16.argtypes = [ctypes.c_double]
        lib.seeded_round_bf16.restype = ctypes.c_uint16
        _LIB = lib
    return _LIB


def philox4x32(counter, key, rounds: int = 10):
    """One Philox4x32-R block: four 32-bit words from a 4-word counter and 2-word key."""
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    _lib().seeded_philox4x32(c.ctypes.data, k.ctypes.data, int(rounds), out.ctypes.data)
    return out


def round_bf16(x: float) -> int:
    """Bit pattern of the bf16 nearest to ``x`` (ties to even)."""
    return int(_lib().seeded_round_bf16(float(x)))


def normal_bf16(shape, seed: int, tensor_id: int, sigma: float = 1.0) -> np.ndarray:
    """bf16 bits of iid N(0, sigma^2) draws for (seed, tensor_id), in flat index order."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.uint16)
    if n:
        _lib().seeded_normal_bf16(out.ctypes.data, n, int(seed) & (2**64 - 1),
                                  int(tensor_id), float(sigma))
    return out.reshape(shape)


def normal_f32(shape, seed: int, tensor_id: int, sigma: float = 1.0) -> np.ndarray:
    """float32 iid N(0, sigma^2): the draws of ``normal_bf16`` rounded to fp32 instead."""
    n = int(np.prod(shape)) if len(shape) else 1
    out = np.empty(n, dtype=np.float32)
    if n:
        _lib().seeded_normal_f32(out.ctypes.data, n, int(seed) & (2**64 - 1), int(tensor_id),
                                 float(sigma))
    return out.reshape(shape)


def make_gemm(M: int, N: int, K: int, seed: int = 0):
    """A [M, K], B [K, N], bias [N] as bf16 bits: A ~ N(0, 1), B ~ N(0, 1/K), bias ~ N(0, 1).

    B's scale keeps the pre-activation A B + bias near unit variance, so the
    GELU epilogue acts on values where it is far from linear."""
    a = normal_bf16((M, K), seed, TENSOR_GEMM_A, 1.0)
    b = normal_bf16((K, N), seed, TENSOR_GEMM_B, 1.0 / max(K, 1) ** 0.5)
    bias = normal_bf16((N,), seed, TENSOR_GEMM_BIAS, 1.0)
    return a, b, bias


def make_add(n: int, seed: int = 0):
    """x, y float32 [n], iid N(0, 1)."""
    return normal_f32((n,), seed, TENSOR_ADD_X), normal_f32((n,), seed, TENSOR_ADD_Y)


def make_qkv(B: int, H: int, N: int, d: int, seed: int = 0, sigma_qk: float = 1.0,
             sigma_v: float = 1.0):
    """Q, K, V as bf16 bits, each [B, H, N, d], contiguous."""
    shape = (B, H, N, d)
    q = normal_bf16(shape, seed, TENSOR_Q, sigma_qk)
    k = normal_bf16(shape, seed, TENSOR_K, sigma_qk)
    v = normal_bf16(shape, seed, TENSOR_V, sigma_v)
    return q, k, v


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)
