"""Oracle pins for the token-wise top-k (Eq. (2) of "详解DSA")."""

import json
import os

import numpy as np
import pytest

from dsa_inputs import custom_workload, make_inputs
from oracle import brute, indexer, topk

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.mark.parametrize("n,k", [(50, 10), (200, 64), (1000, 999), (37, 37), (5, 64)])
def test_select_matches_full_stable_sort(n, k):
    rng = np.random.default_rng(n + k)
    I = np.round(rng.standard_normal(n), 1)           # many exact ties
    sel, vk = topk.select(I, k)
    ref = np.argsort(-I, kind="stable")[: min(n, k)]
    assert set(sel.tolist()) == set(ref.tolist())
    if n > k:
        assert vk == I[ref[-1]]
        assert sel.tolist() == ref.tolist()
    else:
        assert vk is None and sel.tolist() == list(range(n))


def test_select_matches_brute_selection():
    rng = np.random.default_rng(3)
    for n, k in [(9, 4), (16, 5), (12, 12), (3, 8)]:
        I = rng.integers(-3, 4, n).astype(np.float64)
        sel, _ = topk.select(I, k)
        assert sel.tolist() == brute.topk_positions(I.tolist(), k)


def test_short_rows_select_everything_and_pad():
    x = make_inputs(custom_workload("short", [70], [70], k_sel=64, n_heads=16), seed=2)
    for r, t, I, B in indexer.scores(x):
        sel, vk = topk.select(I, 64)
        row = topk.padded(sel, 64)
        if t + 1 <= 64:
            assert vk is None
            assert row[: t + 1].tolist() == list(range(t + 1))
            assert np.all(row[t + 1:] == -1)
        else:
            assert np.all(row >= 0) and np.all(row <= t)       # causal: no s > t
            assert len(set(row.tolist())) == 64


def test_permutation_equivariance():
    rng = np.random.default_rng(8)
    I = rng.standard_normal(500)
    perm = rng.permutation(500)
    sel, _ = topk.select(I, 40)
    sel_p, _ = topk.select(I[perm], 40)
    assert set(perm[sel_p].tolist()) == set(sel.tolist())


def test_ties_prefer_lower_positions():
    I = np.array([1.0, 3.0, 2.0, 3.0, 2.0, 2.0, 0.0])
    sel, vk = topk.select(I, 4)
    assert sel.tolist() == [1, 3, 2, 4] and vk == 2.0


def test_near_threshold_set():
    I = np.array([5.0, 4.0, 3.0005, 3.0, 2.9995, 1.0])
    tol = np.full(6, 1e-3)
    sel, vk = topk.select(I, 3)
    assert vk == 3.0005
    near = topk.near_threshold(I, tol, vk, sel)
    assert near.tolist() == [2, 3, 4]


def test_selected_fraction_page_figure():
    with open(os.path.join(GOLDEN, "page_figures.json")) as f:
        g = json.load(f)["selected_fraction_128k"]
    assert g["k"] / g["context"] == pytest.approx(g["value"], abs=5e-5)
