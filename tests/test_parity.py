"""GPU parity of the sm_100a attention kernel against the fp64 oracle, on the
same seeded inputs, through the C ABI.

Small problems (several tiles plus ragged tails) are compared element by
element over the whole output; the full-size workloads are compared on
sampled rows the oracle computes one by one, plus properties that hold at any
size (finite outputs; each O row is a convex combination of V rows)."""
import math

import numpy as np
import pytest

import oracle
import parity_utils as pu

pytestmark = pytest.mark.gpu


def full_case(B, H, N, d, causal, sigma=1.0, seed=0):
    (q, k, v), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=seed, sigma_qk=sigma)
    scale = pu.default_scale(d)
    o, lse = pu.run(qt, kt, vt, causal)
    o_ref, lse_ref = oracle.attention_fwd(q, k, v, causal, scale)
    return pu.check(pu.o_f64(o), lse.cpu().numpy().astype(np.float64), o_ref, lse_ref,
                    f"B{B} H{H} N{N} d{d} causal={causal} sigma={sigma}")


# --------------------------------------------------------------- whole-output parity
@pytest.mark.parametrize("causal", [False, True])
def test_small_config(cuda_device, causal):
    # B=1, H=1, N=128, d=64, N(0,1), scale 1/sqrt(d), both modes, seed 0
    full_case(1, 1, 128, 64, causal)


def test_four_by_eight_heads_1024_d64(cuda_device):
    # B=4, H=8, N=1024, d=64, N(0,1), non-causal
    full_case(4, 8, 1024, 64, False)


@pytest.mark.parametrize("N", [1, 2, 7, 64, 127, 129, 255, 256, 257, 383, 640, 1000])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(cuda_device, N, d, causal):
    full_case(1, 2, N, d, causal, seed=N)


@pytest.mark.parametrize("sigma", [3.0, 3.0 ** 0.5])
@pytest.mark.parametrize("causal", [False, True])
def test_wide_score_range_small(cuda_device, sigma, causal):
    # the wide-range (N(0,3)) inputs at a size the oracle runs whole
    full_case(1, 4, 2048, 128, causal, sigma=sigma)


def test_several_slices_and_ctas(cuda_device):
    full_case(2, 3, 700, 128, True, seed=3)
    full_case(3, 2, 513, 64, False, seed=4)


# --------------------------------------------------------------- full sizes, sampled rows
def sampled_case(B, H, N, d, causal, sigma=1.0, count=192, seed=0):
    (q, k, v), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=seed, sigma_qk=sigma)
    scale = pu.default_scale(d)
    o, lse = pu.run(qt, kt, vt, causal)
    rows = pu.sample_rows(B, H, N, count, seed=seed + 1)
    o_ref, lse_ref = oracle.attention_rows(q, k, v, causal, scale, rows)
    o_all = o.view(-1, d)
    o_s = o_all[rows].float().cpu().numpy().astype(np.float64)
    lse_s = lse.view(-1)[rows].cpu().numpy().astype(np.float64)
    m = pu.check(o_s, lse_s, o_ref, lse_ref, f"B{B} H{H} N{N} d{d} causal={causal} sigma={sigma}")
    # properties of the whole output: finite, and each O row inside the hull of V
    import torch
    assert torch.isfinite(o).all().item() and torch.isfinite(lse).all().item()
    vmax = vt.float().abs().amax().item()
    assert o.float().abs().amax().item() <= vmax * (1 + 2 ** -8) + 1e-6
    return m


# --------------------------------------------------------------- full sizes, every element
def whole_case(B, H, N, d, causal, sigma=1.0, seed=0):
    """Every element of O and LSE at a full workload size against the strip
    form of the oracle (fp64 matrix products), rel-L2 over the whole tensor."""
    (q, k, v), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=seed, sigma_qk=sigma)
    scale = pu.default_scale(d)
    o, lse = pu.run(qt, kt, vt, causal)
    o_g, l_g = pu.o_f64(o), lse.cpu().numpy().astype(np.float64)
    del o, lse, qt, kt, vt
    o_ref, lse_ref = oracle.attention_fwd_strips(q, k, v, causal, scale)
    m = pu.check(o_g, l_g, o_ref, lse_ref,
                 f"whole B{B} H{H} N{N} d{d} causal={causal} sigma={sigma:.4g}")
    print(f"whole-output parity B={B} H={H} N={N} d={d} causal={causal} sigma={sigma:.4g}: {m}")
    return m


def test_b2_h16_n4096_d128_causal_whole(cuda_device):
    whole_case(2, 16, 4096, 128, True)


@pytest.mark.parametrize("sigma", [3.0, 3.0 ** 0.5])
@pytest.mark.parametrize("causal", [False, True])
def test_b1_h32_n16384_d128_wide_whole(cuda_device, sigma, causal):
    whole_case(1, 32, 16384, 128, causal, sigma=sigma)


@pytest.mark.parametrize("causal", [False, True])
def test_d64_default_path_whole(cuda_device, causal):
    # d = 64 at a length where the table picks three query tiles per CTA: 40
    # query tiles per slice, so the last tile group holds a lone tile, and the
    # wide score range
    import attention_forward_17_b200 as fa
    sid, _ = fa.pick_schedule(5000, 64, causal)
    print("schedule", fa.schedules()[sid])
    whole_case(2, 8, 5000, 64, causal, sigma=3.0)


def test_b2_h16_n4096_d128_causal(cuda_device):
    sampled_case(2, 16, 4096, 128, True)


@pytest.mark.parametrize("N", [512, 1024, 2048, 4096, 8192, 16384, 32768])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_sequence_sweep(cuda_device, N, d, causal):
    B = max(1, 16384 // N)
    sampled_case(B, 16, N, d, causal, count=96, seed=N + d)


# --------------------------------------------------------------- invariants through the kernel
@pytest.mark.parametrize("causal", [False, True])
def test_ones_v_gives_ones(cuda_device, causal):
    import torch
    (_, _, _), (qt, kt, _) = pu.inputs(1, 2, 1000, 128, sigma_qk=3.0)
    vt = torch.ones_like(qt)
    o, _ = pu.run(qt, kt, vt, causal)
    assert (o.float() - 1).abs().max().item() <= 2 ** -7


def test_causal_row_zero_is_v0(cuda_device):
    (q, k, v), (qt, kt, vt) = pu.inputs(2, 2, 300, 64)
    o, lse = pu.run(qt, kt, vt, True)
    assert torch_equal(o[:, :, 0], vt[:, :, 0])
    qf = qt[:, :, 0].double()
    kf = kt[:, :, 0].double()
    ref = (qf * kf).sum(-1) / 8.0
    assert (lse[:, :, 0].double() - ref).abs().max().item() <= 1e-4


def torch_equal(a, b):
    import torch
    return torch.equal(a, b)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_q_uniform_weights(cuda_device, causal):
    import torch
    N = 777
    (_, _, v), (qt, kt, vt) = pu.inputs(1, 1, N, 128)
    qt = torch.zeros_like(qt)
    o, lse = pu.run(qt, kt, vt, causal)
    vf = vt[0, 0].double()
    if causal:
        ref = torch.cumsum(vf, 0) / torch.arange(1, N + 1, device=vf.device, dtype=torch.float64)[:, None]
        ref_lse = torch.log(torch.arange(1, N + 1, device=vf.device, dtype=torch.float64))
    else:
        ref = vf.mean(0, keepdim=True).expand(N, -1)
        ref_lse = torch.full((N,), math.log(N), dtype=torch.float64, device=vf.device)
    assert (o[0, 0].double() - ref).abs().max().item() <= 2e-2
    assert (lse[0, 0].double() - ref_lse).abs().max().item() <= 1e-3


# --------------------------------------------------------------- determinism, bounds, slices
def test_bitwise_deterministic(cuda_device):
    import torch
    (_, _, _), (qt, kt, vt) = pu.inputs(2, 4, 2000, 128, seed=5)
    for causal in (False, True):
        o1, l1 = pu.run(qt, kt, vt, causal)
        o2, l2 = pu.run(qt, kt, vt, causal)
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


@pytest.mark.parametrize("N,d", [(300, 64), (129, 128), (1024, 128)])
def test_writes_stay_in_bounds(cuda_device, N, d):
    import torch
    import attention_forward_17_b200 as fa
    B, H, pad = 1, 3, 4096
    (_, _, _), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=6)
    n_o = B * H * N * d
    n_l = B * H * N
    o_buf = torch.full((n_o + 2 * pad,), 7.0, dtype=torch.bfloat16, device="cuda")
    l_buf = torch.full((n_l + 2 * pad,), 7.0, dtype=torch.float32, device="cuda")
    o = o_buf[pad:pad + n_o].view(B, H, N, d)
    lse = l_buf[pad:pad + n_l].view(B, H, N)
    for causal in (False, True):
        fa.fa_fwd(qt, kt, vt, causal=causal, out=o, lse=lse)
        torch.cuda.synchronize()
        assert (o_buf[:pad] == 7).all() and (o_buf[pad + n_o:] == 7).all()
        assert (l_buf[:pad] == 7).all() and (l_buf[pad + n_l:] == 7).all()


def test_slices_independent(cuda_device):
    import torch
    (_, _, _), (qt, kt, vt) = pu.inputs(2, 3, 600, 128, seed=8)
    o, lse = pu.run(qt, kt, vt, True)
    s = (slice(1, 2), slice(2, 3))
    o1, l1 = pu.run(qt[s].contiguous(), kt[s].contiguous(), vt[s].contiguous(), True)
    assert torch.equal(o1, o[s]) and torch.equal(l1, lse[s])


def test_host_entry_matches_device_entry(cuda_device):
    import torch
    import attention_forward_17_b200 as fa
    B, H, N, d = 1, 4, 1500, 128
    (_, _, _), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=9)
    o_dev, l_dev = pu.run(qt, kt, vt, True)
    q_h, k_h, v_h = (t.cpu().pin_memory() for t in (qt, kt, vt))
    o_h = torch.empty_like(q_h).pin_memory()
    l_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    q_d, k_d, v_d = (torch.empty_like(qt) for _ in range(3))
    o_d = torch.empty_like(qt)
    l_d = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    fa.fa_fwd_host(q_h, k_h, v_h, o_h, l_h, q_d, k_d, v_d, o_d, l_d, causal=True)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(l_h, l_dev.cpu())


@pytest.mark.parametrize("B,H,N,d", [(2, 32, 2048, 64), (3, 7, 4096, 128), (1, 250, 640, 64)])
def test_host_entry_pipelined_chunks(cuda_device, B, H, N, d):
    # enough (b, h) slices that the host entry splits them into several chunks
    # (uploads, kernels and downloads on different streams); a ragged last chunk
    # in the second and third cases.  Must equal the device entry bit for bit,
    # also when the stream already holds other work, and match sampled oracle rows.
    import torch
    import attention_forward_17_b200 as fa
    (q, k, v), (qt, kt, vt) = pu.inputs(B, H, N, d, seed=B + H + N)
    q_h, k_h, v_h = (t.cpu().pin_memory() for t in (qt, kt, vt))
    o_h = torch.empty_like(q_h).pin_memory()
    l_h = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    q_d, k_d, v_d, o_d = (torch.zeros_like(qt) for _ in range(4))
    l_d = torch.empty((B, H, N), dtype=torch.float32, device="cuda")
    for causal in (False, True):
        o_dev, l_dev = pu.run(qt, kt, vt, causal)
        o_h.zero_()
        busy = torch.randn(4096, 4096, device="cuda")
        busy = busy @ busy                      # queued work ahead of the call on the same stream
        fa.fa_fwd_host(q_h, k_h, v_h, o_h, l_h, q_d, k_d, v_d, o_d, l_d, causal=causal)
        torch.cuda.current_stream().synchronize()
        assert torch.equal(o_h, o_dev.cpu()) and torch.equal(l_h, l_dev.cpu()), f"causal={causal}"
        rows = pu.sample_rows(B, H, N, 48, seed=N)
        o_ref, l_ref = oracle.attention_rows(q, k, v, causal, pu.default_scale(d), rows)
        o_g = pu.o_f64(o_h).reshape(-1, d)[rows]
        l_g = l_h.double().numpy().reshape(-1)[rows]
        pu.check(o_g, l_g, o_ref, l_ref, f"host entry B={B} H={H} N={N} d={d} causal={causal}")


def test_status_word_stays_clear(cuda_device):
    import torch
    import attention_forward_17_b200 as fa
    (_, _, _), (qt, kt, vt) = pu.inputs(1, 2, 1024, 64, seed=10)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    fa.fa_fwd(qt, kt, vt, causal=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0


def test_misaligned_pointer_rejected(cuda_device):
    import torch
    import attention_forward_17_b200 as fa
    (_, _, _), (qt, kt, vt) = pu.inputs(1, 1, 128, 64)
    base = torch.empty(128 * 64 + 8, dtype=torch.bfloat16, device="cuda")
    q_off = base[1:1 + 128 * 64].view(1, 1, 128, 64)   # 2-byte offset
    with pytest.raises(fa.FaError) as e:
        fa.fa_fwd(q_off, kt, vt)
    assert e.value.status == fa.FA_ERR_ALIGN
