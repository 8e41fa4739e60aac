"""Token-wise top-k selection (oracle).

Eq. (2) of "详解DSA": S_t = { s : I[t, s] in Top-k(I[t, :]) }, over the causal
range s <= t; the demo indexer takes ``topk(min(index_topk, end_pos))`` so a row
with no more than k valid positions keeps all of them ("详解DSA", prefill
analysis: below k the whole sequence is kept and the indexer can be bypassed).

Readings taken where the pages leave the contract open ("DeepSeek V3.2
稀疏注意力", section on top-k as the algorithm/kernel interface, asks for the
tie rule, the padding and the ragged rule to be defined):

* ties: higher score first, then the lower position s;
* output: a set of sequence-relative positions, stored valid-first and padded
  with -1 up to k.
"""

from __future__ import annotations

import numpy as np


def select(I_row: np.ndarray, k: int):
    """Top-k of one row of scores over its valid prefix.

    Returns (sel, v_k): ``sel`` the selected positions in selection order
    (score descending, position ascending), ``v_k`` the k-th score (None when
    the row has at most k positions and everything is kept).
    """
    I_row = np.asarray(I_row, dtype=np.float64)
    n = I_row.shape[0]
    if n <= k:
        return np.arange(n, dtype=np.int64), None
    order = np.lexsort((np.arange(n), -I_row))   # primary: -I ascending, secondary: s ascending
    sel = order[:k].astype(np.int64)
    return sel, float(I_row[sel[-1]])


def padded(sel: np.ndarray, k: int) -> np.ndarray:
    """Selection as a fixed-width int32 row: the set in ascending order, then -1."""
    out = np.full(k, -1, dtype=np.int32)
    s = np.sort(np.asarray(sel, dtype=np.int64))
    out[: s.shape[0]] = s
    return out


def near_threshold(I_row: np.ndarray, tol_row: np.ndarray, v_k, sel: np.ndarray) -> np.ndarray:
    """Positions whose score lies within tolerance of the k-th value.

    A position s is near the threshold when |I[s] - v_k| <= tol[s] + tol_k,
    tol_k being the largest tolerance among positions scoring exactly v_k
    (both the position's score and the k-th score carry an error).
    """
    if v_k is None:
        return np.zeros(0, dtype=np.int64)
    I_row = np.asarray(I_row, dtype=np.float64)
    tol_row = np.asarray(tol_row, dtype=np.float64)
    tol_k = float(tol_row[I_row == v_k].max())
    return np.nonzero(np.abs(I_row - v_k) <= tol_row + tol_k)[0].astype(np.int64)
