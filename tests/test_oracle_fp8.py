"""Oracle FP8 pins: e4m3 decode and the activation quantiser against torch's cast."""

import numpy as np
import pytest
import torch

from dsa_inputs import bf16_bits_to_f32, f32_to_bf16_bits, make_inputs
from oracle import fp8


def test_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ours = fp8.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6


@pytest.mark.parametrize("scale", [1.0, 0.21, 2.0 / 448.0])
def test_encode_all_bf16_values_match_torch(scale):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = bf16_bits_to_f32(bits)
    v = v[np.isfinite(v)]
    with np.errstate(over="ignore"):
        y = (v / np.float32(scale)).astype(np.float32)
    y = y[np.abs(y) <= 464.0]
    ours = fp8.encode_e4m3_from_f32(y)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_encode_saturates_and_keeps_sign_of_zero():
    y = np.array([1000.0, -1000.0, 0.0, -0.0, 2.0 ** -10, 3 * 2.0 ** -10], np.float32)
    # 2^-10 is half of the smallest subnormal: ties to even (0); 3*2^-10 ties up to 2*2^-9
    assert fp8.encode_e4m3_from_f32(y).tolist() == [0x7E, 0xFE, 0x00, 0x80, 0x00, 0x02]


def test_oracle_quantiser_reproduces_generator_bytes():
    x = make_inputs("tiny_prefill_512", keep_raw=True)
    qc, qs = fp8.act_quant(bf16_bits_to_f32(x.q_idx_bf16))
    kc, ks = fp8.act_quant(bf16_bits_to_f32(x.k_idx_bf16))
    assert np.array_equal(qc, x.q8) and np.array_equal(qs, x.q_scale)
    assert np.array_equal(kc, x.k8) and np.array_equal(ks, x.k_scale)


def test_quantisation_error_is_within_half_ulp():
    rng = np.random.default_rng(4)
    x = bf16_bits_to_f32(f32_to_bf16_bits(rng.standard_normal((64, 128)).astype(np.float32)))
    codes, scale = fp8.act_quant(x)
    back = fp8.dequant(codes, scale)
    # e4m3 has 3 mantissa bits: relative rounding error <= 2^-4 for normals,
    # absolute <= 2^-10 * scale in the subnormal range
    err = np.abs(back - x)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scale[:, None]) * (1 + 1e-6)
    assert np.all(err <= bound)
