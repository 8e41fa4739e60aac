"""GPU top-k on crafted score rows against the oracle's selection, exactly.

The scores here are fed straight to dsa_topk (no indexer in between), so the
selection must equal the oracle's bit for bit: the selected positions in
ascending order, then -1 padding.  The rows cover the three kernel shapes
(rows up to 8192, up to 32768 and longer), persistent CTAs that walk many rows
of mixed lengths, and the value patterns that push the value-bin selection onto
its exact radix fallback: a crowded boundary bin, a far outlier, infinities,
signed zeros and wholesale ties.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from oracle import topk as o_topk

pytestmark = pytest.mark.gpu


def _run(kv, q, rows_fn, k, seed=0):
    """kv, q: per-sequence lengths; rows_fn(rng, n) -> float32 scores of one row
    with n valid positions.  Returns (gpu idx [total_q, k], expected [total_q, k])."""
    rng = np.random.default_rng(seed)
    kv = np.asarray(kv, np.int32)
    q = np.asarray(q, np.int32)
    cu_q = np.concatenate([[0], np.cumsum(q)]).astype(np.int32)
    total_q = int(cu_q[-1])
    ld = ((int(kv.max()) + 3) // 4) * 4
    scores = np.full((total_q, ld), np.nan, np.float32)       # beyond t: never read
    expect = np.full((total_q, k), -1, np.int32)
    for b in range(len(kv)):
        for i in range(int(q[b])):
            r = int(cu_q[b]) + i
            n = int(kv[b]) - int(q[b]) + i + 1
            row = rows_fn(rng, n).astype(np.float32)
            scores[r, :n] = row
            sel, _ = o_topk.select(row.astype(np.float64), k)
            expect[r] = o_topk.padded(sel, k)
    kv_start = np.concatenate([[0], np.cumsum(kv)[:-1]]).astype(np.int64)
    dev = lambda a: torch.from_numpy(a).cuda()
    batch = dsa.Batch(dev(cu_q), dev(kv), dev(kv_start), total_q, int(q.max()), int(kv.max()), int(kv.sum()))
    s = dev(scores)
    idx = torch.full((total_q, k), -7, dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_TOPK, batch, k)
    dsa.topk(batch, s, k, idx, ws)
    dsa.check_device_error(ws)
    return idx.cpu().numpy(), expect


def _assert_equal(got, expect):
    bad = np.nonzero(np.any(got != expect, axis=1))[0]
    assert bad.size == 0, f"{bad.size} rows differ, first {bad[0]}: " \
        f"{np.setdiff1d(got[bad[0]], expect[bad[0]])[:8]} vs {np.setdiff1d(expect[bad[0]], got[bad[0]])[:8]}"


normal = lambda rng, n: rng.standard_normal(n)


@pytest.mark.parametrize("L", [5000, 20000, 40000])
def test_normal_rows_each_kernel_shape(L):
    got, exp = _run([L, L // 2], [5, 3], normal, 2048, seed=L)
    _assert_equal(got, exp)


@pytest.mark.parametrize("L,R", [(7000, 700), (12000, 400)])
def test_persistent_ctas_walk_many_rows(L, R):
    got, exp = _run([L], [R], normal, 2048, seed=R)
    _assert_equal(got, exp)


def test_mixed_lengths_between_short_and_long_rows():
    kv = [100, 9000, 50, 15000, 3000, 2048, 2049, 30000, 1] * 40
    got, exp = _run(kv, [1] * len(kv), normal, 2048, seed=9)
    _assert_equal(got, exp)


@pytest.mark.parametrize("L", [6000, 25000, 50000])
def test_crowded_and_tied_rows(L):
    pats = [
        lambda rng, n: np.round(rng.standard_normal(n) * 2) / 2,                # few levels: big tie groups
        lambda rng, n: np.concatenate([[1e30], 1 + 1e-4 * rng.standard_normal(n - 1)]),   # far outlier
        lambda rng, n: np.where(rng.random(n) < 0.01, np.inf,
                                np.where(rng.random(n) < 0.01, -np.inf, rng.standard_normal(n))),
        lambda rng, n: np.where(rng.random(n) < 0.03, rng.random(n) + 1,
                                np.where(rng.random(n) < 0.5, 0.0, -0.0)),        # signed zeros tie
        lambda rng, n: np.full(n, 3.5),                                            # all equal
        lambda rng, n: rng.integers(0, 1000, n).astype(np.float64),               # small tie groups
    ]
    for j, pat in enumerate(pats):
        got, exp = _run([L], [3], pat, 2048, seed=100 + j)
        _assert_equal(got, exp)


@pytest.mark.parametrize("k", [1, 7, 300])
def test_small_k(k):
    got, exp = _run([20000, 900, 6000], [2, 3, 2], normal, k, seed=k)
    _assert_equal(got, exp)


@pytest.mark.parametrize("kv,q", [([131072, 70000], [2, 2]), ([65536 + 100, 32768 + 5], [1, 2]),
                                  ([150000, 40000], [1, 1])])
def test_rows_over_32768_in_segments(kv, q):
    # rows longer than one register row go through per-segment selections and
    # a merge (150000 positions make 5 segments); a last segment shorter than k
    # contributes all its positions
    got, exp = _run(kv, q, normal, 2048, seed=kv[0] % 97)
    _assert_equal(got, exp)


@pytest.mark.parametrize("k", [7, 300, 2048])
def test_long_rows_mixed_with_short_ones(k):
    # one batch of short, register-sized and long rows; k = 7 (not a multiple
    # of 4) takes the single-CTA path for the long rows, the others the segments
    kv = [40000, 100, 33000, 2049, 90000]
    got, exp = _run(kv, [2, 1, 1, 1, 1], normal, k, seed=k + 3)
    _assert_equal(got, exp)
