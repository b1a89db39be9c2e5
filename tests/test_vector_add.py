"""GPU parity of the fp32 vector addition against the oracle: bit for bit,
for lengths around the vector width, the 16-byte vector path and the scalar
path (offset pointers), in place, and sampled at the benchmark's length."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu


def run(x, y, offset=0, inplace=False):
    import torch
    import attention_forward_17_b200 as fa
    n = x.size
    xs = torch.empty(n + offset, dtype=torch.float32, device="cuda")[offset:]
    ys = torch.empty(n + offset, dtype=torch.float32, device="cuda")[offset:]
    xs.copy_(torch.from_numpy(x))
    ys.copy_(torch.from_numpy(y))
    z = fa.vector_add(xs, ys, out=xs if inplace else None)
    torch.cuda.synchronize()
    return z.cpu().numpy()


@pytest.mark.parametrize("n", [1, 3, 4, 5, 1023, 4096, 1_000_003, 1 << 22])
def test_bit_exact(cuda_device, n):
    x, y = si.make_add(n, seed=n)
    want = oracle.vector_add(x, y).astype(np.float32)
    assert np.array_equal(run(x, y).view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("offset", [1, 2, 3])
def test_unaligned_scalar_path(cuda_device, offset):
    x, y = si.make_add(100_001, seed=offset)
    want = oracle.vector_add(x, y).astype(np.float32)
    assert np.array_equal(run(x, y, offset=offset).view(np.uint32), want.view(np.uint32))


def test_in_place(cuda_device):
    x, y = si.make_add(65_537, seed=9)
    want = oracle.vector_add(x, y).astype(np.float32)
    assert np.array_equal(run(x, y, inplace=True).view(np.uint32), want.view(np.uint32))


def test_benchmark_length_sampled(cuda_device):
    n = 1 << 28
    x, y = si.make_add(n, seed=0)
    z = run(x, y)
    idx = np.random.default_rng(0).integers(0, n, 100_000)
    idx = np.concatenate([idx, [0, n - 1]])
    want = oracle.vector_add(x[idx], y[idx]).astype(np.float32)
    assert np.array_equal(z[idx].view(np.uint32), want.view(np.uint32))
