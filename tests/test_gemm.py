"""GPU parity of the tcgen05 GEMM with its fused epilogues against the fp64
oracle on the same seeded bf16 inputs: single tiles, ragged M / N / K tails,
more tiles than SMs (each CTA cycles through both tensor-memory accumulators
and the shared-memory ring several times), K = 0, all three epilogues, and
sampled entries of the 8192^3 problem the benchmark times.  Problems of at
most 128 rows (and K = 0) run the one-SM kernel; the others run 256-row tiles
over SM pairs, including pairs whose second CTA holds one valid row or none.

Bound per element: C is rounded to bf16 (relative error <= 2^-9); fp32
accumulation of at most K exact bf16 products and erff add well under 1e-3
absolute at these magnitudes (|A B + bias| is O(1) by construction of the
inputs), so |C - C_ref| <= 2^-8 |C_ref| + 1e-3, and the relative L2 error
over the whole output stays below 4e-3."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu


def dev(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run(a, b, bias, mode, status=None):
    import torch
    import attention_forward_17_b200 as fa
    c = fa.gemm(dev(a), dev(b), dev(bias), epilogue=mode, status=status)
    torch.cuda.synchronize()
    return c.float().cpu().numpy().astype(np.float64)


def check(c, ref, what):
    assert np.all(np.isfinite(c)), what
    err = np.abs(c - ref)
    bad = err > 2.0 ** -8 * np.abs(ref) + 1e-3
    assert not bad.any(), f"{what}: {bad.sum()} of {c.size} off, worst {err.max():.3e}"
    rel = np.linalg.norm(c - ref) / max(np.linalg.norm(ref), 1e-30)
    assert rel < 4e-3, f"{what}: relative L2 {rel:.3e}"


SHAPES = [
    (128, 256, 64),      # exactly one tile, one K block
    (1, 8, 8),           # smallest legal problem
    (300, 520, 200),     # ragged M, N (last column block is 8 wide), K (last block 8 deep)
    (257, 264, 72),
    (129, 136, 24),      # one 256-row pair tile: the second CTA holds a single valid row
    (300, 8, 8),         # pair tiles whose second CTA's columns of B all lie past N
    (520, 24, 1032),     # 17 K blocks, the last 8 deep, on a two-block pair grid
    (640, 768, 1024),    # 16 K blocks: the stage rings wrap several times
]


@pytest.mark.parametrize("M,N,K", SHAPES)
@pytest.mark.parametrize("mode", [0, 1, 2])
def test_gemm_parity(cuda_device, M, N, K, mode):
    a, b, bias = si.make_gemm(M, N, K, seed=M * 7 + N + K)
    check(run(a, b, bias, mode), oracle.gemm(a, b, bias, mode), f"{M}x{N}x{K} mode {mode}")


@pytest.mark.parametrize("M,N,K", [(2048, 2560, 256), (4096, 2560, 128)])
def test_more_tiles_than_sms(cuda_device, M, N, K):
    # 160 and 320 tiles of 128 x 256 on 148 SMs: CTAs take 1 to 3 tiles
    a, b, bias = si.make_gemm(M, N, K, seed=K)
    check(run(a, b, bias, 2), oracle.gemm(a, b, bias, 2), f"{M}x{N}x{K}")


def test_k_zero_gives_epilogue_of_zero(cuda_device):
    import torch
    import attention_forward_17_b200 as fa
    bias = si.normal_bf16((264,), seed=1, tensor_id=5)
    a = torch.empty((130, 0), dtype=torch.bfloat16, device="cuda")
    b = torch.empty((0, 264), dtype=torch.bfloat16, device="cuda")
    c = fa.gemm(a, b, dev(bias), epilogue=2).float().cpu().numpy().astype(np.float64)
    ref = oracle.gemm(np.zeros((130, 0), np.uint16), np.zeros((0, 264), np.uint16), bias, 2)
    check(c, ref, "K = 0")


def test_status_word_stays_clear(cuda_device):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    a, b, bias = si.make_gemm(256, 512, 256, seed=3)
    run(a, b, bias, 2, status=status)
    assert int(status.item()) == 0


def test_repeat_calls_identical(cuda_device):
    a, b, bias = si.make_gemm(384, 768, 512, seed=4)
    assert np.array_equal(run(a, b, bias, 2), run(a, b, bias, 2))


def test_full_size_sampled(cuda_device):
    # the benchmark's problem: M = N = K = 8192, bias + GELU
    M = N = K = 8192
    a, b, bias = si.make_gemm(M, N, K, seed=0)
    c = run(a, b, bias, 2)
    rng = np.random.default_rng(0)
    idx = np.concatenate([rng.integers(0, M * N, 3000),
                          [0, N - 1, (M - 1) * N, M * N - 1]])   # the four corners
    ref = oracle.gemm_entries(a, b, bias, idx, 2)
    got = c.reshape(-1)[idx]
    err = np.abs(got - ref)
    assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 1e-3), f"worst {err.max():.3e}"
    # every entry is finite and the GELU range holds: C >= min GELU ~ -0.17
    assert np.all(np.isfinite(c)) and c.min() >= -0.1705
