"""Pins for the fp64 oracle, none of which reuse its own code:

- hand-derived closed forms (tests/golden/worked_examples.json);
- an independent pure-Python brute force on tiny shapes (log-sum-exp form, math.fsum);
- torch's fp64 scaled_dot_product_attention and logsumexp on CPU (a library routine the
  oracle does not use);
- the invariants of softmax attention: rows of P sum to one, constant V, causal row 0,
  Q = 0 / K = 0 give (prefix) means with LSE = ln(count), permutation equivariance, shift
  invariance, a dominant key, slice independence;
- the selected-rows entry point against the full pass.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import seeded_inputs as si

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_examples.json")


def bits(x) -> np.ndarray:
    """float array -> bf16 bits (values must already be bf16-exact or are rounded RNE)."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def f64(b) -> np.ndarray:
    return si.bf16_bits_to_f32(b).astype(np.float64)


def rand_qkv(B, H, N, d, seed=0, sigma=1.0):
    return si.make_qkv(B, H, N, d, seed=seed, sigma_qk=sigma)


# ---------------------------------------------------------------- closed forms
def test_worked_examples():
    cases = json.load(open(GOLDEN))["cases"]
    env = {"e": math.e, "log": math.log}
    for c in cases:
        q = bits(np.array(c["q"])[None, None])
        k = bits(np.array(c["k"])[None, None])
        v = bits(np.array(c["v"])[None, None])
        o, lse = oracle.attention_fwd(q, k, v, c["causal"], c["scale"])
        exp_o = np.array([[eval(x, env) for x in row] for row in c["O"]])
        exp_l = np.array([eval(x, env) for x in c["LSE"]])
        np.testing.assert_allclose(o[0, 0], exp_o, rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(lse[0, 0], exp_l, rtol=0, atol=1e-13, err_msg=c["name"])


# ---------------------------------------------------------------- brute force
def brute_force(qf, kf, vf, causal, scale):
    """Scalar pure-Python attention written in log-sum-exp form (no max subtraction)."""
    B, H, N, d = qf.shape
    O = np.zeros((B, H, N, d))
    L = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                keys = range(i + 1) if causal else range(N)
                sc = {j: scale * math.fsum(qf[b, h, i, t] * kf[b, h, j, t] for t in range(d)) for j in keys}
                lse = math.log(math.fsum(math.exp(s) for s in sc.values()))
                L[b, h, i] = lse
                for t in range(d):
                    O[b, h, i, t] = math.fsum(math.exp(sc[j] - lse) * vf[b, h, j, t] for j in keys)
    return O, L


@pytest.mark.parametrize("N", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("d", [1, 2, 4])
@pytest.mark.parametrize("causal", [False, True])
def test_brute_force_tiny(N, d, causal):
    q, k, v = rand_qkv(2, 2, N, d, seed=N * 10 + d)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention_fwd(q, k, v, causal, scale)
    O, L = brute_force(f64(q), f64(k), f64(v), causal, scale)
    np.testing.assert_allclose(o, O, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, L, rtol=0, atol=1e-12)


# ---------------------------------------------------------------- torch fp64 SDPA
@pytest.mark.parametrize("shape", [(1, 1, 128, 64), (2, 3, 200, 64), (1, 2, 512, 128), (1, 1, 129, 128)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sigma", [1.0, 3.0])
def test_against_torch_sdpa_fp64(shape, causal, sigma):
    B, H, N, d = shape
    q, k, v = rand_qkv(B, H, N, d, seed=1, sigma=sigma)
    scale = 1.0 / math.sqrt(d)
    o, lse = oracle.attention_fwd(q, k, v, causal, scale)
    tq, tk, tv = (torch.from_numpy(f64(x)) for x in (q, k, v))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=causal, scale=scale)
    s = scale * tq @ tk.transpose(-1, -2)
    if causal:
        s = s.masked_fill(torch.ones(N, N, dtype=torch.bool).triu(1), float("-inf"))
    ref_lse = torch.logsumexp(s, dim=-1)
    np.testing.assert_allclose(o, ref.numpy(), rtol=0, atol=1e-10)
    np.testing.assert_allclose(lse, ref_lse.numpy(), rtol=0, atol=1e-10)


# ---------------------------------------------------------------- invariants
@pytest.mark.parametrize("causal", [False, True])
def test_rows_sum_to_one(causal):
    # V = all ones => O = sum_j P_ij = 1 for every row and column
    q, k, _ = rand_qkv(1, 2, 300, 64, seed=2, sigma=3.0)
    v = bits(np.ones((1, 2, 300, 64)))
    o, _ = oracle.attention_fwd(q, k, v, causal, 0.125)
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v(causal):
    q, k, _ = rand_qkv(1, 1, 257, 64, seed=3)
    row = np.linspace(-2, 2, 64).astype(np.float32)
    v = bits(np.broadcast_to(row, (1, 1, 257, 64)))
    o, _ = oracle.attention_fwd(q, k, v, causal, 0.125)
    np.testing.assert_allclose(o, np.broadcast_to(f64(v)[0, 0, 0], o.shape), rtol=0, atol=1e-12)


def test_causal_row_zero():
    q, k, v = rand_qkv(2, 2, 64, 128, seed=4)
    scale = 1 / math.sqrt(128)
    o, lse = oracle.attention_fwd(q, k, v, True, scale)
    qf, kf, vf = f64(q), f64(k), f64(v)
    np.testing.assert_array_equal(o[:, :, 0], vf[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], scale * np.einsum("bhd,bhd->bh", qf[:, :, 0], kf[:, :, 0]),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("zero", ["q", "k"])
def test_uniform_weights(zero):
    N = 100
    q, k, v = rand_qkv(1, 1, N, 64, seed=5)
    if zero == "q":
        q = np.zeros_like(q)
    else:
        k = np.zeros_like(k)
    vf = f64(v)[0, 0]
    o, lse = oracle.attention_fwd(q, k, v, False, 0.125)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(vf.mean(0), (N, 64)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], math.log(N), rtol=0, atol=1e-12)
    o, lse = oracle.attention_fwd(q, k, v, True, 0.125)
    prefix = np.cumsum(vf, axis=0) / np.arange(1, N + 1)[:, None]
    np.testing.assert_allclose(o[0, 0], prefix, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], np.log(np.arange(1, N + 1)), rtol=0, atol=1e-12)


def test_permutation_equivariance():
    N = 150
    q, k, v = rand_qkv(1, 1, N, 64, seed=6)
    o, lse = oracle.attention_fwd(q, k, v, False, 0.125)
    perm = np.random.default_rng(0).permutation(N)
    # joint permutation of key/value rows leaves the result unchanged
    o2, lse2 = oracle.attention_fwd(q, k[:, :, perm], v[:, :, perm], False, 0.125)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse, rtol=0, atol=1e-12)
    # permuting query rows permutes the outputs
    o3, lse3 = oracle.attention_fwd(q[:, :, perm], k, v, False, 0.125)
    np.testing.assert_allclose(o3, o[:, :, perm], rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse3, lse[:, :, perm], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_shift_invariance(causal):
    # an extra feature column, 1 in every query and c in every key, adds scale*c to every score:
    # O is unchanged and LSE moves by scale*c
    N, d, c, scale = 90, 63, 4.0, 0.125
    q, k, v = rand_qkv(1, 1, N, d, seed=7)
    o, lse = oracle.attention_fwd(q, k, v, causal, scale)
    q2 = np.concatenate([q, bits(np.ones((1, 1, N, 1)))], axis=-1)
    k2 = np.concatenate([k, bits(np.full((1, 1, N, 1), c))], axis=-1)
    v2 = np.concatenate([v, bits(np.zeros((1, 1, N, 1)))], axis=-1)
    o2, lse2 = oracle.attention_fwd(q2, k2, v2, causal, scale)
    np.testing.assert_allclose(o2[..., :d], o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse2, lse + scale * c, rtol=0, atol=1e-12)


def test_dominant_key():
    N, d, jstar, i = 64, 64, 17, 40
    q, k, v = rand_qkv(1, 1, N, d, seed=8)
    k = k.copy()
    k[0, 0, jstar] = bits(8.0 * f64(q)[0, 0, i])  # score ~ 8 |q|^2 / 8 ~ 64 above the rest
    o, _ = oracle.attention_fwd(q, k, v, False, 1 / 8)
    np.testing.assert_allclose(o[0, 0, i], f64(v)[0, 0, jstar], rtol=0, atol=1e-9)


def test_slices_independent():
    q, k, v = rand_qkv(2, 3, 70, 64, seed=9)
    o, lse = oracle.attention_fwd(q, k, v, True, 0.125)
    o1, lse1 = oracle.attention_fwd(q[1:2, 2:3], k[1:2, 2:3], v[1:2, 2:3], True, 0.125)
    np.testing.assert_array_equal(o1[0, 0], o[1, 2])
    np.testing.assert_array_equal(lse1[0, 0], lse[1, 2])


def test_rows_entry_matches_full():
    B, H, N, d = 2, 2, 130, 64
    q, k, v = rand_qkv(B, H, N, d, seed=10)
    rng = np.random.default_rng(1)
    rows = rng.choice(B * H * N, 37, replace=False)
    for causal in (False, True):
        o, lse = oracle.attention_fwd(q, k, v, causal, 0.125)
        ro, rl = oracle.attention_rows(q, k, v, causal, 0.125, rows)
        np.testing.assert_array_equal(ro, o.reshape(-1, d)[rows])
        np.testing.assert_array_equal(rl, lse.reshape(-1)[rows])


# ---------------------------------------------------------------- strip form (fp64 matrix products)
@pytest.mark.parametrize("N,strip", [(130, 64), (700, 256), (257, 1024), (1, 16)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("sigma", [1.0, 3.0])
def test_strips_match_plain_loops(N, strip, causal, sigma):
    # the strip form against the per-row loops: strip edges inside and past N,
    # wide and narrow score ranges, both masks
    q, k, v = rand_qkv(2, 2, N, 64, seed=N + strip, sigma=sigma)
    o, lse = oracle.attention_fwd(q, k, v, causal, 0.125)
    so, sl = oracle.attention_fwd_strips(q, k, v, causal, 0.125, strip=strip)
    np.testing.assert_allclose(so, o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(sl, lse, rtol=1e-13, atol=1e-12)


def test_strips_worked_examples():
    cases = json.load(open(GOLDEN))["cases"]
    env = {"e": math.e, "log": math.log}
    for c in cases:
        q = bits(np.array(c["q"])[None, None])
        k = bits(np.array(c["k"])[None, None])
        v = bits(np.array(c["v"])[None, None])
        o, lse = oracle.attention_fwd_strips(q, k, v, c["causal"], c["scale"], strip=2)
        exp_o = np.array([[eval(x, env) for x in row] for row in c["O"]])
        exp_l = np.array([eval(x, env) for x in c["LSE"]])
        np.testing.assert_allclose(o[0, 0], exp_o, rtol=0, atol=1e-13, err_msg=c["name"])
        np.testing.assert_allclose(lse[0, 0], exp_l, rtol=0, atol=1e-13, err_msg=c["name"])


@pytest.mark.parametrize("causal", [False, True])
def test_strips_zero_q_prefix_means(causal):
    # Q = 0: uniform weights over the visible keys (closed form, strips of 100 rows)
    N, d = 333, 8
    q, k, v = rand_qkv(1, 1, N, d, seed=21)
    q = np.zeros_like(q)
    o, lse = oracle.attention_fwd_strips(q, k, v, causal, 0.5, strip=100)
    vf = f64(v)[0, 0]
    if causal:
        ref = np.cumsum(vf, 0) / np.arange(1, N + 1)[:, None]
        ref_l = np.log(np.arange(1, N + 1))
    else:
        ref = np.broadcast_to(vf.mean(0), (N, d))
        ref_l = np.full(N, math.log(N))
    np.testing.assert_allclose(o[0, 0], ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], ref_l, rtol=0, atol=1e-12)


def test_thread_count_does_not_change_result():
    q, k, v = rand_qkv(1, 2, 200, 64, seed=11)
    a = oracle.attention_fwd(q, k, v, False, 0.125, threads=1)
    b = oracle.attention_fwd(q, k, v, False, 0.125, threads=4)
    np.testing.assert_array_equal(a[0], b[0])
    np.testing.assert_array_equal(a[1], b[1])


# ---------------------------------------------------------------- row softmax
def row_bits(rows, cols, seed, sigma=1.0):
    return si.normal_bf16((rows, cols), seed=seed, tensor_id=7, sigma=sigma)


@pytest.mark.parametrize("cols", [1, 3, 8, 100, 1000])
@pytest.mark.parametrize("scale", [1.0, 0.3])
def test_row_softmax_brute_force(cols, scale):
    x = row_bits(5, cols, seed=cols)
    y = oracle.row_softmax(x, scale)
    xf = f64(x)
    for r in range(5):
        lse = math.log(math.fsum(math.exp(scale * v) for v in xf[r]))
        ref = [math.exp(scale * v - lse) for v in xf[r]]
        np.testing.assert_allclose(y[r], ref, rtol=1e-12, atol=0)


def test_row_softmax_against_torch():
    x = row_bits(64, 777, seed=1, sigma=4.0)
    y = oracle.row_softmax(x, 0.7)
    ref = torch.softmax(0.7 * torch.from_numpy(f64(x)), dim=-1).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-12, atol=1e-300)


def test_row_softmax_invariants():
    x = row_bits(16, 513, seed=2, sigma=3.0)
    y = oracle.row_softmax(x)
    np.testing.assert_allclose(y.sum(axis=1), 1.0, rtol=0, atol=1e-12)      # rows sum to one
    # shift invariance: integer-valued rows plus 16 stay exact in bf16 and give the same softmax
    xi = np.random.default_rng(4).integers(-20, 20, size=(8, 300)).astype(np.float64)
    np.testing.assert_allclose(oracle.row_softmax(bits(xi + 16.0)), oracle.row_softmax(bits(xi)),
                               rtol=1e-14, atol=0)
    xs = bits(np.full((2, 40), 3.0))                                         # equal entries: uniform
    np.testing.assert_allclose(oracle.row_softmax(xs), 1.0 / 40, rtol=1e-15)
    xo = bits(np.where(np.arange(50) == 17, 100.0, 0.0)[None])               # one dominant entry
    yo = oracle.row_softmax(xo)
    assert abs(yo[0, 17] - 1.0) < 1e-40 + 1e-15 and yo[0, :17].max() < 1e-40
    # permuting columns permutes the output
    perm = np.random.default_rng(3).permutation(513)
    np.testing.assert_allclose(oracle.row_softmax(x[:, perm]), y[:, perm], rtol=1e-14, atol=0)
