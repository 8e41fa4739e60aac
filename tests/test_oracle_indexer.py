"""Oracle pins for the Lightning-Indexer scores (Eq. (1) of "详解DSA")."""

import json
import os

import numpy as np
import pytest

from dsa_inputs import custom_workload, make_inputs
from oracle import brute, fp8, indexer

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_fp8(rng, shape):
    x = rng.standard_normal(shape).astype(np.float32)
    return fp8.act_quant(x)


def test_scores_match_brute_force_loops():
    rng = np.random.default_rng(10)
    q8, qs = _rand_fp8(rng, (3, 64, 128))
    k8, ks = _rand_fp8(rng, (7, 128))
    w = (rng.standard_normal((3, 64)) * 0.125).astype(np.float32)
    qd = fp8.dequant(q8, qs)
    kd = fp8.dequant(k8, ks)
    for r in range(3):
        I, B = indexer.scores_for_row(q8[r], qs[r], w[r], k8, ks)
        for s in range(7):
            ref = brute.index_score(qd[r].tolist(), w[r].tolist(), kd[s].tolist())
            assert abs(I[s] - ref) <= 1e-12 * max(1.0, B[s])


def test_single_head_unit_weight_is_relu_of_dot():
    # H_I = 1, w = 1: I = ReLU(q . k).  Exact FP8 values: q = e_0 * 1.0,
    # k rows = (+2, ...) * 0.5 and (-3, ...) * 0.5, so q . k = +1 and -1.5.
    q8 = np.zeros((1, 128), np.uint8)
    q8[0, 0] = 0x38                        # 1.0
    k8 = np.zeros((2, 128), np.uint8)
    k8[0, 0] = 0x40                        # 2.0
    k8[1, 0] = 0xC4                        # -3.0
    k8[:, 5] = 0x38                        # orthogonal to q
    I, B = indexer.scores_for_row(q8, np.array([1.0], np.float32), np.array([1.0], np.float32),
                                  k8, np.array([0.5, 0.5], np.float32))
    assert I.tolist() == [1.0, 0.0]
    assert B.tolist() == [1.0, 1.5]


def test_negative_dots_give_exact_zero():
    rng = np.random.default_rng(11)
    q8, qs = _rand_fp8(rng, (64, 128))
    k8 = (q8 ^ np.uint8(0x80))[:1]         # k = -q_0: every head with q_j . k < 0 is cut
    ks = qs[:1].copy()
    w = np.ones(64, np.float32)
    q8[1:] = q8[0]
    qs[1:] = qs[0]
    I, _ = indexer.scores_for_row(q8, qs, w, k8, ks)
    assert I[0] == 0.0


def test_equal_key_rows_give_a_constant_row():
    x = make_inputs(custom_workload("eqk", [300], [4], k_sel=64, n_heads=16), seed=5)
    x.k8[:] = x.k8[17]
    x.k_scale[:] = x.k_scale[17]
    for r, t, I, _ in indexer.scores(x):
        assert np.all(I == I[0])


def test_scale_folding_identity():
    # k_scale * sum_j (w * q_scale) * ReLU(q8 . k8) equals Eq. (1) on dequantised
    # values because the scales are positive and ReLU is positively homogeneous.
    rng = np.random.default_rng(12)
    q8, qs = _rand_fp8(rng, (64, 128))
    k8, ks = _rand_fp8(rng, (50, 128))
    w = (rng.standard_normal(64) * 0.125).astype(np.float32)
    I, _ = indexer.scores_for_row(q8, qs, w, k8, ks)
    raw = fp8.decode_e4m3(q8) @ fp8.decode_e4m3(k8).T            # [64, 50]
    folded = ks.astype(np.float64) * ((w.astype(np.float64) * qs)[:, None] * np.maximum(raw, 0)).sum(0)
    assert np.allclose(I, folded, rtol=1e-13, atol=1e-12)


def test_causal_range_per_row():
    x = make_inputs(custom_workload("rag", [40, 9], [5, 9], k_sel=8, n_heads=16), seed=6)
    rows = indexer.scores(x)
    for r, t, I, B in rows:
        assert I.shape[0] == t + 1 and B.shape[0] == t + 1
        assert np.all(B >= np.abs(I))


def test_flop_ratio_against_page_figures():
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        g = json.load(f)
    ratio = indexer.flops_per_pair(64, 128) / indexer.mla_flops_per_pair(128, 576)
    assert ratio == pytest.approx(g["indexer_to_mla_compute_ratio"]["value"])


def test_tolerance_formula():
    B = np.array([0.0, 1.0, 1000.0])
    assert np.allclose(indexer.tolerance(B), [1e-6, 1e-3 + 1e-6, 1.0 + 1e-6])


def test_ragged_batch_offsets_every_score_against_brute_loops():
    # Three sequences of different lengths, one or more query rows each, in
    # flat caches: every score of every row must come from its own sequence's
    # key rows (kv_start offset) and cover exactly s = 0..t (t = kv_len -
    # q_len + i).  A wrong offset, a wrong causal end or a row mapped to the
    # wrong sequence changes values or lengths here.
    x = make_inputs(custom_workload("pin_ragged", [9, 5, 12], [2, 5, 3], k_sel=4, n_heads=16), seed=13)
    b = x.batch
    assert b.kv_start.tolist() == [0, 9, 14]
    qd = fp8.dequant(x.q8, x.q_scale)
    kd = fp8.dequant(x.k8, x.k_scale)
    expect_t = [7, 8, 0, 1, 2, 3, 4, 9, 10, 11]
    got = indexer.scores(x)
    assert [t for _, t, _, _ in got] == expect_t
    starts = [0, 0, 9, 9, 9, 9, 9, 14, 14, 14]
    for (r, t, I, B), k0 in zip(got, starts):
        assert I.shape == (t + 1,) and B.shape == (t + 1,)
        for s in range(t + 1):
            ref = brute.index_score(qd[r].tolist(), x.w[r].tolist(), kd[k0 + s].tolist())
            assert abs(I[s] - ref) <= 1e-12 * max(1.0, B[s]), (r, s)
