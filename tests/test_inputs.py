"""The seeded generator: storage encodings against torch, determinism, shapes."""

import numpy as np
import pytest
import torch

from dsa_inputs import (WORKLOADS, Batch, bf16_bits_to_f32, e4m3_encode, f32_to_bf16_bits,
                        make_inputs, quantize_fp8_blocks)
from dsa_inputs.workloads import make_batch


def _all_bf16_f32():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    v = bf16_bits_to_f32(bits)
    return v[np.isfinite(v)]


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.standard_normal(200_000).astype(np.float32),
                        (rng.standard_normal(1000) * 1e30).astype(np.float32),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875], np.float32)])
    ours = f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


@pytest.mark.parametrize("scale", [1.0, 0.37, 3.0 / 448.0, 1e-3])
def test_e4m3_encoder_matches_torch_cast(scale):
    v = _all_bf16_f32()
    with np.errstate(over="ignore"):
        y = (v / np.float32(scale)).astype(np.float32)
    y = y[np.abs(y) <= 464.0]          # torch's cast is non-saturating above 464 (-> NaN)
    ours = e4m3_encode(y)
    ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ours, ref)


def test_e4m3_encoder_saturates():
    y = np.array([448.0, 470.0, 1e6, -1e6], np.float32)
    assert e4m3_encode(y).tolist() == [0x7E, 0x7E, 0x7E, 0xFE]


def test_block_quantiser_hits_448_once_per_block():
    rng = np.random.default_rng(2)
    x = f32_to_bf16_bits(rng.standard_normal((50, 3, 128)).astype(np.float32))
    codes, scale = quantize_fp8_blocks(x)
    assert codes.shape == x.shape and scale.shape == (50, 3)
    assert np.all((codes & 0x7F).max(axis=-1) == 0x7E)     # |max code| = 448
    assert np.all(scale > 0)


def test_generator_is_deterministic_and_seeded():
    a = make_inputs("tiny_prefill_512", seed=0)
    b = make_inputs("tiny_prefill_512", seed=0)
    c = make_inputs("tiny_prefill_512", seed=1)
    for name in ["q8", "q_scale", "w", "k8", "k_scale", "q_mla", "latent"]:
        assert np.array_equal(getattr(a, name), getattr(b, name)), name
    assert not np.array_equal(a.k8, c.k8)


def test_tiny_prefill_shapes_and_layout():
    x = make_inputs("tiny_prefill_512")
    b = x.batch
    assert b.total_q == 512 and b.total_keys == 512 and b.num_seqs == 1
    assert x.q8.shape == (512, 64, 128) and x.q8.dtype == np.uint8
    assert x.q_scale.shape == (512, 64) and x.w.shape == (512, 64)
    assert x.k8.shape == (512, 128) and x.k_scale.shape == (512,)
    assert x.q_mla.shape == (512, 16, 576) and x.latent.shape == (512, 576)
    assert np.array_equal(b.q_pos, np.arange(512))
    assert x.k_sel == 64 and abs(x.sm_scale - 192 ** -0.5) < 1e-15
    # w ~ N(0, 1/64)
    assert abs(float(np.std(x.w)) - 0.125) < 0.01


def test_ragged_batch_layout():
    b = Batch.from_lengths([5, 9, 3], [2, 9, 1])
    assert b.cu_q.tolist() == [0, 2, 11, 12]
    assert b.kv_start.tolist() == [0, 5, 14]
    assert b.q_pos.tolist() == [3, 4] + list(range(9)) + [2]
    assert b.q_seq.tolist() == [0, 0] + [1] * 9 + [2]
    with pytest.raises(ValueError):
        Batch.from_lengths([3], [4])


def test_decode_context_lengths_in_range():
    b = make_batch(WORKLOADS["decode_64x16k_32k"], 0)
    assert b.num_seqs == 64 and b.total_q == 64
    assert b.kv_len.min() >= 16384 and b.kv_len.max() <= 32768
    assert np.array_equal(b.q_pos, b.kv_len.astype(np.int64) - 1)


def test_heavy_rows_keep_fp8_bytes_and_scale_by_four():
    from dsa_inputs import custom_workload
    wl = custom_workload("heavy_small", [4000], [8], k_sel=64, n_heads=16, heavy_frac=0.05)
    x = make_inputs(wl, seed=3, keep_raw=True)
    h = x.heavy_rows
    assert h.shape[0] == 200
    raw = x.k_idx_bf16[h]
    unscaled = f32_to_bf16_bits(bf16_bits_to_f32(raw) / np.float32(4.0))
    codes, scale = quantize_fp8_blocks(unscaled)
    assert np.array_equal(codes, x.k8[h])
    assert np.array_equal(scale * np.float32(4.0), x.k_scale[h])
