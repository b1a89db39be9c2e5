"""Pins for the GEMM (+ bias, + GELU) and vector-add oracles, none of which reuse
their code:

- tabulated values of the standard normal distribution function
  (tests/golden/normal_cdf_values.json) for the exact GELU x * Phi(x);
- numpy's fp64 matmul with scipy's ``ndtr`` for Phi, on non-square shapes (a
  transposed operand or a dropped bias fails);
- a pure-Python brute force on tiny shapes using the erfc form of Phi;
- identities: GELU(x) - GELU(-x) = x, the identity matrix, K = 0, the relations
  between the three epilogue modes;
- the selected-entries entry point against the full product;
- vector add against numpy's IEEE fp32 addition, bit for bit.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle
import seeded_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "normal_cdf_values.json")


def bits(x) -> np.ndarray:
    import torch
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f64(b) -> np.ndarray:
    return si.bf16_bits_to_f32(b).astype(np.float64)


def gelu_ref(x):
    return x * scipy.special.ndtr(x)


def test_gelu_tabulated_values():
    cases = json.load(open(GOLDEN))["cases"]
    xs = np.array([c["x"] for c in cases])
    a = bits(xs[:, None])                      # [n, 1]
    b = bits(np.ones((1, 1)))                  # [1, 1]
    bias = bits(np.zeros(1))
    c = oracle.gemm(a, b, bias, oracle.GEMM_BIAS_GELU)[:, 0]
    expect = np.array([cc["x"] * cc["Phi"] for cc in cases])
    np.testing.assert_allclose(c, expect, rtol=0, atol=2e-15)


@pytest.mark.parametrize("M,N,K", [(33, 48, 40), (7, 130, 65), (64, 24, 1)])
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_against_numpy_scipy(M, N, K, mode):
    a, b, bias = si.make_gemm(M, N, K, seed=M + N + K)
    acc = f64(a) @ f64(b)
    ref = acc if mode == 0 else acc + f64(bias)[None, :]
    if mode == 2:
        ref = gelu_ref(ref)
    c = oracle.gemm(a, b, bias, mode)
    np.testing.assert_allclose(c, ref, rtol=1e-12, atol=1e-13)


def test_brute_force_tiny():
    a, b, bias = si.make_gemm(3, 5, 4, seed=11)
    af, bf, biasf = f64(a), f64(b), f64(bias)
    c = oracle.gemm(a, b, bias)
    for i in range(3):
        for j in range(5):
            x = math.fsum(af[i, k] * bf[k, j] for k in range(4)) + biasf[j]
            want = x * 0.5 * math.erfc(-x / math.sqrt(2.0))
            assert abs(c[i, j] - want) <= 1e-14 * max(1.0, abs(want))


def test_gelu_odd_part_is_identity():
    # GELU(x) - GELU(-x) = x (Phi(x) + Phi(-x) = 1): with zero bias, C(A) - C(-A) = A B
    a, b, _ = si.make_gemm(20, 24, 16, seed=3)
    neg = (a ^ np.uint16(0x8000)).astype(np.uint16)
    zero = bits(np.zeros(24))
    d = oracle.gemm(a, b, zero) - oracle.gemm(neg, b, zero)
    np.testing.assert_allclose(d, oracle.gemm(a, b, None, oracle.GEMM_PLAIN), rtol=1e-12, atol=1e-13)


def test_identity_matrix_and_modes():
    K = 24
    _, b, bias = si.make_gemm(K, 40, K, seed=5)
    eye = bits(np.eye(K))
    c1 = oracle.gemm(eye, b, bias, oracle.GEMM_BIAS)
    np.testing.assert_array_equal(c1, f64(b) + f64(bias)[None, :])
    c2 = oracle.gemm(eye, b, bias, oracle.GEMM_BIAS_GELU)
    np.testing.assert_allclose(c2, gelu_ref(c1), rtol=1e-13, atol=1e-15)


def test_empty_k():
    bias = bits(np.array([-1.0, 0.0, 2.0, 0.5]))
    c = oracle.gemm(np.zeros((3, 0), np.uint16), np.zeros((0, 4), np.uint16), bias)
    np.testing.assert_allclose(c, np.broadcast_to(gelu_ref(f64(bias)), (3, 4)), rtol=1e-14)


def test_entries_match_full():
    a, b, bias = si.make_gemm(37, 45, 50, seed=9)
    full = oracle.gemm(a, b, bias)
    rng = np.random.default_rng(0)
    idx = rng.integers(0, 37 * 45, size=200)
    np.testing.assert_array_equal(oracle.gemm_entries(a, b, bias, idx), full.reshape(-1)[idx])


def test_thread_count_does_not_change_result():
    a, b, bias = si.make_gemm(30, 20, 70, seed=2)
    np.testing.assert_array_equal(oracle.gemm(a, b, bias, threads=1), oracle.gemm(a, b, bias, threads=3))


def test_vector_add_matches_ieee_fp32():
    x, y = si.make_add(100_003, seed=4)
    z = oracle.vector_add(x, y)
    np.testing.assert_array_equal(z.astype(np.float32), x + y)
    # the fp64 sum is the exact sum for these operands
    np.testing.assert_array_equal(z - x.astype(np.float64), y.astype(np.float64))


def test_vector_add_closed_forms():
    x, _ = si.make_add(1000, seed=1)
    np.testing.assert_array_equal(oracle.vector_add(x, np.zeros_like(x)), x.astype(np.float64))
    np.testing.assert_array_equal(oracle.vector_add(x, -x), np.zeros(1000))
    big = np.full(4, 2.0 ** 40, np.float32)
    tiny = np.full(4, 2.0 ** -20, np.float32)
    # the fp32 result rounds back to the larger operand
    np.testing.assert_array_equal(oracle.vector_add(big, tiny).astype(np.float32), big)
    assert oracle.vector_add(np.zeros(0, np.float32), np.zeros(0, np.float32)).size == 0
