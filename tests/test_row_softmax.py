"""GPU parity of the row-wise softmax kernel against the fp64 oracle on the
same seeded bf16 rows: every fast-path width class, ragged widths and
unaligned rows (general path), negative and zero scale, wide value ranges,
plus properties at a size the oracle is not run on.

Bound: y is rounded to bf16 (relative error <= 2^-9); the fp32 exponentials
and sum add ~1e-6 relative; so |y - y_ref| <= 2^-8 |y_ref| + 1e-30."""
import numpy as np
import pytest

import oracle
import seeded_inputs as si

pytestmark = pytest.mark.gpu


def run(bits, scale, offset=0):
    import torch
    import attention_forward_17_b200 as fa
    rows, cols = bits.shape
    flat = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()
    if offset:
        buf = torch.empty(rows * cols + offset, dtype=torch.bfloat16, device="cuda")
        x = buf[offset:].view(rows, cols)
        x.copy_(flat.view(rows, cols))
        out_buf = torch.empty(rows * cols + offset, dtype=torch.bfloat16, device="cuda")
        y = out_buf[offset:].view(rows, cols)
        fa.row_softmax(x, scale, out=y)
    else:
        y = fa.row_softmax(flat.view(rows, cols), scale)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64)


def check(y, ref, what):
    assert np.all(np.isfinite(y)), what
    err = np.abs(y - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 1e-30
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst {err.max():.3e}"


@pytest.mark.parametrize("cols", [8, 200, 256, 264, 512, 1000, 1024, 2048, 3000, 4096, 8192, 16384])
def test_fast_path_widths(cuda_device, cols):
    x = si.normal_bf16((37, cols), seed=cols, tensor_id=7, sigma=2.0)
    check(run(x, 1.0), oracle.row_softmax(x, 1.0), f"cols={cols}")


@pytest.mark.parametrize("cols", [1, 3, 7, 13, 1001, 16390, 40000])
def test_general_path_widths(cuda_device, cols):
    x = si.normal_bf16((9, cols), seed=cols, tensor_id=7, sigma=2.0)
    check(run(x, 0.5), oracle.row_softmax(x, 0.5), f"cols={cols}")


def test_unaligned_rows_use_general_path(cuda_device):
    x = si.normal_bf16((11, 512), seed=5, tensor_id=7)
    check(run(x, 1.0, offset=1), oracle.row_softmax(x, 1.0), "2-byte offset")


@pytest.mark.parametrize("scale", [-1.5, 0.0, 0.125, 8.0])
def test_scales(cuda_device, scale):
    x = si.normal_bf16((64, 1024), seed=9, tensor_id=7, sigma=3.0)
    check(run(x, scale), oracle.row_softmax(x, scale), f"scale={scale}")


def test_large_rows_properties(cuda_device):
    import torch
    import attention_forward_17_b200 as fa
    rows, cols = 8192, 4096
    x = torch.randn(rows, cols, device="cuda").bfloat16()
    y = fa.row_softmax(x).float()
    torch.cuda.synchronize()
    s = y.sum(dim=1)
    assert (s - 1).abs().max().item() < cols * 2.0 ** -9 / cols ** 0.5 + 1e-2
    assert (y >= 0).all().item() and (y <= 1).all().item()
    # the largest input of each row gets the largest output (ties in bf16 allowed)
    at_argmax = y.gather(1, x.float().argmax(dim=1, keepdim=True)).squeeze(1)
    assert torch.equal(at_argmax, y.max(dim=1).values)
