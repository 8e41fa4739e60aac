"""Oracle pins for sparse MLA in MQA mode."""

import json
import os

import numpy as np
import pytest
import torch

from dsa_inputs import custom_workload, make_inputs
from oracle import brute, indexer, mla, topk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
SM = 1.0 / np.sqrt(192.0)


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def test_sparse_equals_dense_masked():
    rng = np.random.default_rng(20)
    lat = _rand(rng, 300, 576)
    q = _rand(rng, 16, 576)
    t = 250
    idx = np.full(64, -1)
    idx[:40] = rng.choice(t + 1, 40, replace=False)
    o1, l1 = mla.sparse_token(q, lat, idx, SM)
    o2, l2 = mla.dense_masked(q, lat, idx, t, SM)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-13)
    assert np.allclose(l1, l2, rtol=1e-13)


def test_full_selection_is_causal_attention_sdpa():
    # With k >= n_valid every position is selected and sparse MLA reduces to
    # plain causal MQA attention; compare against torch's SDPA in fp64.
    rng = np.random.default_rng(21)
    lat = _rand(rng, 40, 576)
    q = _rand(rng, 8, 576)
    t = 33
    idx = np.concatenate([np.arange(t + 1), -np.ones(64 - t - 1, dtype=np.int64)])
    o, lse = mla.sparse_token(q, lat, idx, SM)
    Q = torch.from_numpy(q)[None, :, None, :]                      # [1, H, 1, 576]
    K = torch.from_numpy(lat[: t + 1])[None, None].expand(1, 8, t + 1, 576)
    V = torch.from_numpy(lat[: t + 1, :512])[None, None].expand(1, 8, t + 1, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=SM)[0, :, 0].numpy()
    assert np.allclose(o, ref, rtol=1e-12, atol=1e-13)
    ref_lse = torch.logsumexp(SM * torch.from_numpy(q) @ torch.from_numpy(lat[: t + 1]).T, dim=1).numpy()
    assert np.allclose(lse, ref_lse, rtol=1e-13)


def test_matches_brute_loops():
    rng = np.random.default_rng(22)
    D, Dv = 12, 8
    lat = _rand(rng, 10, D)
    q = _rand(rng, 3, D)
    idx = np.array([7, 2, -1, 5, 0])
    sm = 0.3
    sel = [7, 2, 5, 0]
    ref_o, ref_l = brute.attend(q.tolist(), [lat[s].tolist() for s in sel], sm, Dv)
    # the oracle hard-codes a 512-wide value slice; emulate by padding
    latp = np.zeros((10, 600))
    latp[:, :D] = lat
    latp[:, 512:512 + D] = 0.0
    qp = np.zeros((3, 600))
    qp[:, :D] = q
    o, l = mla.sparse_token(qp, latp, idx, sm)
    assert np.allclose(o[:, :Dv], np.array(ref_o), rtol=1e-12, atol=1e-14)
    assert np.allclose(l, ref_l, rtol=1e-13)


def test_index_order_and_padding_invariance():
    rng = np.random.default_rng(23)
    lat = _rand(rng, 100, 576)
    q = _rand(rng, 4, 576)
    idx = rng.choice(100, 30, replace=False)
    o1, l1 = mla.sparse_token(q, lat, idx, SM)
    shuf = rng.permutation(idx)
    padded = np.concatenate([[-1, -1], shuf[:10], [-1], shuf[10:], [-1] * 5])
    o2, l2 = mla.sparse_token(q, lat, padded, SM)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14) and np.allclose(l1, l2, rtol=1e-14)


def test_empty_selection():
    o, l = mla.sparse_token(np.ones((2, 576)), np.ones((5, 576)), np.full(8, -1), SM)
    assert np.all(o == 0) and np.all(np.isneginf(l))


def test_single_entry_returns_its_value():
    rng = np.random.default_rng(24)
    lat = _rand(rng, 6, 576)
    o, l = mla.sparse_token(_rand(rng, 3, 576), lat, np.array([4, -1]), SM)
    assert np.allclose(o, np.broadcast_to(lat[4, :512], (3, 512)), rtol=0, atol=1e-15)


def test_pipeline_on_ragged_batch_is_dense_masked_attention():
    x = make_inputs(custom_workload("pipe", [90, 30], [6, 4], k_sel=16, n_heads=16), seed=9)
    idx = np.full((x.batch.total_q, 16), -1, np.int32)
    for r, t, I, B in indexer.scores(x):
        idx[r] = topk.padded(topk.select(I, 16)[0], 16)
    res = mla.sparse(x, idx)
    for r in range(x.batch.total_q):
        seq = x.batch.q_seq[r]
        k0, kv = x.batch.kv_start[seq], x.batch.kv_len[seq]
        lat = mla.bf16_to_f64(x.latent[k0:k0 + kv])
        q = mla.bf16_to_f64(x.q_mla[r])
        o, l = mla.dense_masked(q, lat, idx[r], int(x.batch.q_pos[r]), x.sm_scale)
        assert np.allclose(res[r][0], o, rtol=1e-11, atol=1e-12)


def test_flop_count_and_page_figures():
    assert mla.flops_per_token(128, 2048) == 570_425_344
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        g = json.load(f)["fp32_score_matrix_128k_bytes"]
    assert g["context"] ** 2 * 4 == pytest.approx(g["value"], rel=1e-3)


def test_bf16_output_rounding_matches_torch():
    # The rounding every output comparison runs through (fp64 -> fp32 -> bf16,
    # nearest even) against torch's own float32 -> bfloat16 cast: random
    # values over many binades, exact ties between two bf16 neighbours (odd
    # and even lower neighbour), values next to the largest finite bf16, bf16
    # subnormals, signed zeros.
    import torch
    rng = np.random.default_rng(23)
    parts = [rng.standard_normal(20000) * np.exp2(rng.integers(-40, 40, 20000))]
    hi = (rng.integers(0, 1 << 16, 4000, dtype=np.uint32) << np.uint32(16))
    hi = hi[np.isfinite(hi.view(np.float32))]
    ties = (hi | np.uint32(0x8000)).view(np.float32)                   # halfway between neighbours
    parts.append(ties[np.isfinite(ties)].astype(np.float64))
    parts.append(np.array([3.3895313892515355e38, 3.38e38, -3.3895e38, 1e-40, -1e-40, 9.2e-41,
                           1.1754942e-38, 0.0, -0.0, 1.0, -1.0, 65504.0, 6.103515625e-05]))
    x = np.concatenate(parts)
    x = x[np.isfinite(x.astype(np.float32))]
    got = mla.bf16_output(x)
    ref = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, ref)
    assert np.array_equal(np.signbit(got), np.signbit(ref))
