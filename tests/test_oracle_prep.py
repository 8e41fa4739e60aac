"""Pins of the oracle's indexer input chain (oracle/prep.py): RoPE on the pe
dims, the normalised Walsh-Hadamard transform, and their composition with the
FP8 quantiser."""

import numpy as np
import pytest
import scipy.linalg

from oracle import fp8, prep


def _bf16(rng, shape, scale=1.0):
    return prep.to_bf16(rng.standard_normal(shape).astype(np.float32) * np.float32(scale))


def test_hadamard_matches_the_library_matrix():
    rng = np.random.default_rng(1)
    x = _bf16(rng, (50, 128))
    H = scipy.linalg.hadamard(128).astype(np.float64)            # Sylvester order
    ref = x.astype(np.float64) @ H.T
    got = prep.hadamard_f32(x).astype(np.float64)
    assert np.allclose(got, ref, rtol=0, atol=1e-4 * np.abs(x).sum(axis=1, keepdims=True).max())
    # normalised: an involution (up to fp32 / bf16 rounding) that keeps the norm
    y = prep.hadamard_f32(x) * np.float32(128 ** -0.5)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-5)
    back = prep.hadamard_f32(y) * np.float32(128 ** -0.5)
    assert np.allclose(back, x, atol=1e-5)


def test_hadamard_of_a_unit_vector_is_a_row_of_signs():
    e = np.zeros((1, 128), np.float32)
    e[0, 5] = 1.0
    H = scipy.linalg.hadamard(128)
    assert np.array_equal(prep.hadamard_f32(e)[0], H[:, 5].astype(np.float32))


def test_rope_is_identity_at_angle_zero_and_pairs_i_with_i_plus_32():
    rng = np.random.default_rng(2)
    x = _bf16(rng, (8, 128))
    one, zero = np.ones((8, 32), np.float32), np.zeros((8, 32), np.float32)
    assert np.array_equal(prep.rope_non_interleaved(x, one, zero), x)
    # a quarter turn on frequency 3 only: (x3, x35) -> (-x35, x3); all else fixed
    c, s = one.copy(), zero.copy()
    c[:, 3], s[:, 3] = 0.0, 1.0
    y = prep.rope_non_interleaved(x, c, s)
    assert np.array_equal(y[:, 3], -x[:, 35]) and np.array_equal(y[:, 35], x[:, 3])
    keep = [d for d in range(128) if d not in (3, 35)]
    assert np.array_equal(y[:, keep], x[:, keep])


def test_rope_matches_complex_rotation_and_keeps_the_nope_dims():
    rng = np.random.default_rng(3)
    x = _bf16(rng, (40, 128))
    pos = rng.integers(0, 5000, 40)
    freq = 10000.0 ** (-np.arange(32) / 32.0)
    ang = pos[:, None] * freq[None, :]
    cos, sin = np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)
    y = prep.rope_non_interleaved(x, cos, sin)
    z = (x[:, :32] + 1j * x[:, 32:64]).astype(np.complex128) * (cos + 1j * sin).astype(np.complex128)
    assert np.allclose(y[:, :32], z.real, atol=1e-2) and np.allclose(y[:, 32:64], z.imag, atol=1e-2)
    assert np.array_equal(y[:, 64:], x[:, 64:])
    # an interleaved pairing would rotate (0, 1) together instead: it differs
    inter = x.copy()
    a, b = x[:, 0:64:2], x[:, 1:64:2]
    inter[:, 0:64:2] = a * cos - b * sin
    inter[:, 1:64:2] = b * cos + a * sin
    assert not np.allclose(prep.to_bf16(inter), y)


def test_chain_quantises_the_rotated_vector():
    rng = np.random.default_rng(4)
    x = _bf16(rng, (16, 128), scale=3.0)
    cos = np.cos(rng.uniform(0, 6.3, (16, 32))).astype(np.float32)
    sin = np.sqrt(np.maximum(0.0, 1.0 - cos.astype(np.float64) ** 2)).astype(np.float32)
    codes, scales = prep.indexer_inputs(x, cos, sin)
    r = prep.rotate_activation(prep.rope_non_interleaved(x, cos, sin))
    c2, s2 = fp8.act_quant(r)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2)
    # the dequantised result is the fp64 chain within the FP8 step
    ref = (np.asarray(prep.rope_non_interleaved(x, cos, sin), np.float64)
           @ scipy.linalg.hadamard(128).T) / np.sqrt(128.0)
    deq = fp8.dequant(codes, scales)
    assert np.all(np.abs(deq - ref) <= 0.07 * np.abs(ref) + scales[:, None] * 2 ** -6 + 1e-2)
