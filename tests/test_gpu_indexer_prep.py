"""dsa_indexer_prep (RoPE on the pe dims -> normalised Walsh-Hadamard -> per-128
FP8) against the oracle's step-by-step chain: the same fp32 arithmetic in the
same order, so codes and scales must agree bit for bit."""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import f32_to_bf16_bits
from oracle import prep

pytestmark = pytest.mark.gpu


def _tables(n_pos, theta=10000.0):
    freq = theta ** (-np.arange(32, dtype=np.float64) / 32.0)
    ang = np.arange(n_pos, dtype=np.float64)[:, None] * freq[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def _run(x_bits, pos, vecs_per_pos, cos, sin):
    n = x_bits.shape[0]
    x = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).cuda()
    codes = torch.empty((n, 128), dtype=torch.uint8, device="cuda")
    scales = torch.empty(n, dtype=torch.float32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dsa.indexer_prep(x, torch.from_numpy(pos).cuda(), torch.from_numpy(cos).cuda(), torch.from_numpy(sin).cuda(),
                     codes, scales, ws, vecs_per_pos)
    return codes.cpu().numpy(), scales.cpu().numpy(), ws


@pytest.mark.parametrize("vecs_per_pos,n_tok,scale", [(64, 7, 1.0), (1, 300, 1.0), (64, 3, 900.0), (1, 64, 1e-4)])
def test_prep_chain_bit_exact(vecs_per_pos, n_tok, scale):
    rng = np.random.default_rng(61 + n_tok)
    n = n_tok * vecs_per_pos
    xf = (rng.standard_normal((n, 128)) * scale).astype(np.float32)
    xf[0] = 0.0                                      # an all-zero vector: scale 1
    bits = f32_to_bf16_bits(xf)
    cos, sin = _tables(40000)
    pos = rng.integers(0, 40000, n_tok).astype(np.int32)
    pos[0] = 0                                        # angle zero
    codes, scales, ws = _run(bits, pos, vecs_per_pos, cos, sin)
    dsa.check_device_error(ws)
    xv = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    rows = np.repeat(pos, vecs_per_pos)
    ref_c, ref_s = prep.indexer_inputs(xv, cos[rows], sin[rows])
    assert np.array_equal(scales, ref_s)
    assert np.array_equal(codes, ref_c)


def test_position_outside_the_table_is_a_bounds_error():
    rng = np.random.default_rng(70)
    bits = f32_to_bf16_bits(rng.standard_normal((4, 128)).astype(np.float32))
    cos, sin = _tables(100)
    pos = np.array([5, 100, 7, -1], np.int32)
    codes, scales, ws = _run(bits, pos, 1, cos, sin)
    with pytest.raises(dsa.DSAError) as e:
        dsa.check_device_error(ws)
    assert e.value.status == 6
    assert np.all(codes[[1, 3]] == 0) and np.all(scales[[1, 3]] == 1.0)
    xv = (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)
    ref_c, ref_s = prep.indexer_inputs(xv[[0, 2]], cos[[5, 7]], sin[[5, 7]])
    assert np.array_equal(codes[[0, 2]], ref_c) and np.array_equal(scales[[0, 2]], ref_s)
