"""Device-side failure detection without faulting the GPU: a pipeline wait on
an mbarrier nothing arrives at gives up after its limit, reports
FA_ERR_TIMEOUT through the caller's status word, and the context stays usable
for a normal forward pass afterwards."""
import time

import numpy as np
import pytest

import attention_forward_17_b200 as fa

pytestmark = pytest.mark.gpu


def test_wait_times_out_and_reports(cuda_device):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    fa.selftest_wait_timeout(status, limit_us=20_000)
    torch.cuda.synchronize()
    dt = time.perf_counter() - t0
    assert status.item() == fa.FA_ERR_TIMEOUT
    assert 0.015 < dt < 5.0


def test_completed_wait_leaves_status_clear(cuda_device):
    import torch
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fa.selftest_wait_timeout(status, limit_us=20_000, arrive=True)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_context_usable_after_timeout(cuda_device):
    import torch
    import parity_utils as pu
    import oracle
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fa.selftest_wait_timeout(status, limit_us=5_000)
    torch.cuda.synchronize()
    assert status.item() == fa.FA_ERR_TIMEOUT
    (q, k, v), (qt, kt, vt) = pu.inputs(1, 2, 300, 64, seed=12)
    o, lse = pu.run(qt, kt, vt, True)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, True, pu.default_scale(64))
    pu.check(pu.o_f64(o), lse.cpu().numpy().astype(np.float64), o_ref, lse_ref, "after timeout")
