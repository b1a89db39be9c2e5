"""Seeded input generator: Philox4x32-10 known answers, determinism, moments,
and round-to-nearest-even bf16 conversion."""
import numpy as np
import pytest
import torch

import seeded_inputs as si


# Known-answer vectors published with Random123 (Salmon et al., SC'11) for philox4x32-10.
KAT = [
    ([0, 0, 0, 0], [0, 0], [0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8]),
    ([0xFFFFFFFF] * 4, [0xFFFFFFFF] * 2, [0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD]),
    ([0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344], [0xA4093822, 0x299F31D0],
     [0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1]),
]


@pytest.mark.parametrize("ctr,key,expect", KAT)
def test_philox_known_answers(ctr, key, expect):
    assert list(si.philox4x32(ctr, key, 10)) == expect


def test_same_seed_same_bytes():
    a = si.normal_bf16((3, 1000), seed=7, tensor_id=1)
    b = si.normal_bf16((3, 1000), seed=7, tensor_id=1)
    assert np.array_equal(a, b)


def test_streams_differ_by_tensor_and_seed():
    a = si.normal_bf16((4096,), seed=0, tensor_id=0)
    b = si.normal_bf16((4096,), seed=0, tensor_id=1)
    c = si.normal_bf16((4096,), seed=1, tensor_id=0)
    assert (a != b).mean() > 0.9 and (a != c).mean() > 0.9


def test_prefix_stable():
    # element i depends only on (seed, tensor, i): a longer tensor extends a shorter one
    a = si.normal_bf16((1001,), seed=3, tensor_id=2)
    b = si.normal_bf16((5000,), seed=3, tensor_id=2)
    assert np.array_equal(a, b[:1001])


@pytest.mark.parametrize("sigma", [1.0, 3.0, 3.0 ** 0.5])
def test_moments(sigma):
    x = si.bf16_bits_to_f32(si.normal_bf16((1_000_000,), seed=0, tensor_id=0, sigma=sigma)).astype(np.float64)
    n = x.size
    assert abs(x.mean()) < 5 * sigma / np.sqrt(n)
    assert abs(x.std() / sigma - 1) < 5e-3
    # fourth standardised moment of a normal is 3
    k4 = np.mean((x / x.std()) ** 4)
    assert abs(k4 - 3) < 0.05
    # tail mass beyond 3 sigma ~ 0.0027
    assert abs(np.mean(np.abs(x) > 3 * sigma) - 0.0027) < 0.0006


def test_bf16_rne_halfway_cases():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even mantissa (1.0)
    assert si.round_bf16(1 + 2 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 1+2^-7 (odd) and 1+2^-6 (even)
    assert si.round_bf16(1 + 3 * 2 ** -8) == 0x3F82
    # just above the halfway point rounds up
    assert si.round_bf16(1 + 2 ** -8 + 2 ** -30) == 0x3F81
    assert si.round_bf16(-(1 + 2 ** -8)) == 0xBF80
    assert si.round_bf16(0.0) == 0 and si.round_bf16(-0.0) == 0x8000


def test_bf16_matches_torch_on_float32_values():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(200_000) * np.exp(rng.uniform(-20, 20, 200_000))).astype(np.float32)
    ours = np.array([si.round_bf16(float(t)) for t in x[:20_000]], dtype=np.uint16)
    ref = torch.from_numpy(x[:20_000]).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_values_are_bf16_of_sigma_z():
    # the stored value must be the bf16 of a plausible normal draw: re-rounding is the identity
    bits = si.normal_bf16((512,), seed=5, tensor_id=0, sigma=3.0)
    f = si.bf16_bits_to_f32(bits)
    again = np.array([si.round_bf16(float(t)) for t in f], dtype=np.uint16)
    assert np.array_equal(bits, again)


def test_f32_stream_is_the_bf16_stream_unrounded():
    # the fp32 and bf16 tensors of one (seed, tensor) come from the same draws
    x = si.normal_f32((200_000,), seed=5, tensor_id=6)
    b = si.bf16_bits_to_f32(si.normal_bf16((200_000,), seed=5, tensor_id=6))
    assert np.all(np.abs(b - x) <= 2.0 ** -8 * np.abs(x) + 1e-30)
    x_b = torch.as_tensor(x).to(torch.bfloat16).float().numpy()
    # rounding the fp32 value to bf16 differs from the direct rounding only at double-rounding ties
    assert (x_b == b).mean() > 0.999


def test_gemm_inputs_scale():
    a, b, bias = si.make_gemm(64, 64, 256, seed=0)
    assert a.shape == (64, 256) and b.shape == (256, 64) and bias.shape == (64,)
    assert abs(si.bf16_bits_to_f32(b).std() * 16 - 1) < 0.05
