"""Lightning-Indexer scores (oracle).

Eq. (1) of "详解DSA" (restated on "DeepSeek V3.2 稀疏注意力", data-flow section,
and "NSA 与 DSA" §3.2):

    I[t, s] = sum_{j < H_I} w[t, j] * ReLU(q[t, j] . k[s])

with H_I = 64 indexer heads of dim 128 and a single key per position shared by
all heads.  The indexer consumes q and k in FP8 with per-128 scales (the demo
code quantises both, then calls the FP8 index kernel), so the oracle evaluates
Eq. (1) literally on the *dequantised* values q = code(q8) * q_scale and
k = code(k8) * k_scale, in float64, for the causal range s <= t ("DeepSeek V3.2
稀疏注意力": the indexer scores every history position s <= t).

Alongside each score it returns the magnitude bound

    B[t, s] = sum_j |w[t, j]| * |q[t, j] . k[s]|

that the parity tolerance ``1e-3 * B + 1e-6`` is stated in.
"""

from __future__ import annotations

import numpy as np

from .fp8 import dequant

SCORE_RTOL = 1e-3
SCORE_ATOL = 1e-6


def scores_for_row(q8_row, q_scale_row, w_row, k8_rows, k_scale_rows):
    """Scores of one query row against the given key rows.

    q8_row [H_I, d] uint8, q_scale_row [H_I], w_row [H_I],
    k8_rows [n, d] uint8, k_scale_rows [n]  ->  (I [n], B [n]) float64.
    """
    q = dequant(q8_row, q_scale_row)                       # [H_I, d]
    k = dequant(k8_rows, k_scale_rows)                     # [n, d]
    dots = q @ k.T                                         # [H_I, n]   q[t,j] . k[s]
    w = np.asarray(w_row, dtype=np.float64)[:, None]
    I = (w * np.maximum(dots, 0.0)).sum(axis=0)
    B = (np.abs(w) * np.abs(dots)).sum(axis=0)
    return I, B


def scores(inputs, rows=None):
    """Scores for query rows ``rows`` (default: all) of a ``DSAInputs`` batch.

    Returns a list of (row, t, I[0..t], B[0..t]) tuples: one entry per query
    row, covering exactly its causal range s = 0..t of its own sequence.
    """
    b = inputs.batch
    rows = range(b.total_q) if rows is None else rows
    out = []
    for r in rows:
        r = int(r)
        seq = int(b.q_seq[r])
        t = int(b.q_pos[r])
        k0 = int(b.kv_start[seq])
        I, B = scores_for_row(inputs.q8[r], inputs.q_scale[r], inputs.w[r],
                              inputs.k8[k0:k0 + t + 1], inputs.k_scale[k0:k0 + t + 1])
        out.append((r, t, I, B))
    return out


def tolerance(B: np.ndarray) -> np.ndarray:
    """Per-score parity tolerance |dI| <= 1e-3 * sum_j |w q k| + 1e-6."""
    return SCORE_RTOL * np.asarray(B, dtype=np.float64) + SCORE_ATOL


def flops_per_pair(h_index: int = 64, d_index: int = 128) -> int:
    """Multiply-add work of one (t, s) score: H_I dot products of length d_I."""
    return 2 * h_index * d_index


def mla_flops_per_pair(n_heads: int = 128, latent_dim: int = 576) -> int:
    """The corresponding score work of MLA in MQA mode for one (t, s) pair."""
    return 2 * n_heads * latent_dim
