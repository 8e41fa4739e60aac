"""Sparse MLA in MQA mode over the selected latent entries (oracle).

"DeepSeek V3.2 稀疏注意力" (section on how DSA sits inside MLA) and "NSA 与
DSA" §3.1: DSA runs MLA in its MQA mode, where all query heads of a token share
the same selected latent KV entries c_s; Eq. (2) of "详解DSA" restricts the
attention of token t to { c_s : s in S_t }.  For each head h:

    logit[h, i] = sm_scale * q[h] . c[s_i]            (576-d: 512 latent + 64 RoPE)
    o[h]        = sum_i softmax_i(logit[h, :]) * c[s_i][0:512]
    lse[h]      = log sum_i exp(logit[h, i])           (natural log)

with sm_scale = 1/sqrt(192) applied to the whole 576-d product, over the
entries of the index row that are >= 0 (-1 marks padding).  An empty set gives
o = 0 and lse = -inf.

``dense_masked`` restates the official demo's prefill form ("详解DSA", MLA
forward: an index mask of -inf scattered to 0 at the top-k positions, added to
the causal mask, then softmax over all positions and the product with V).
The page notes it saves no compute; it is kept only as an independent check.
"""

from __future__ import annotations

import numpy as np

VALUE_DIM = 512

OUT_MAX_ABS = 2e-2      # parity bound on the bf16 attention output
OUT_MEAN_REL = 1e-3     # parity bound on sum|d| / sum|ref|


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def attend(q: np.ndarray, c: np.ndarray, sm_scale: float):
    """All heads of one token over the gathered entries c [n, 576] (float64)."""
    H = q.shape[0]
    if c.shape[0] == 0:
        return np.zeros((H, VALUE_DIM)), np.full(H, -np.inf)
    logits = sm_scale * (q @ c.T)                         # [H, n]
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    o = (p / l) @ c[:, :VALUE_DIM]
    lse = (m + np.log(l))[:, 0]
    return o, lse


def sparse_token(q: np.ndarray, latent_seq: np.ndarray, idx_row: np.ndarray, sm_scale: float):
    """One query token.

    q [H, 576] float64, latent_seq [kv_len, 576] float64 (this sequence's
    rows), idx_row [k] int (positions, -1 = padding)  ->  (o [H, 512], lse [H]).
    """
    sel = np.asarray(idx_row, dtype=np.int64)
    sel = sel[sel >= 0]
    return attend(q, latent_seq[sel], sm_scale)          # gather of the selected entries


def dense_masked(q: np.ndarray, latent_seq: np.ndarray, idx_row: np.ndarray, t: int,
                 sm_scale: float):
    """Same result through a dense [H, kv_len] score matrix and an additive mask."""
    kv_len = latent_seq.shape[0]
    sel = np.asarray(idx_row, dtype=np.int64)
    sel = sel[sel >= 0]
    index_mask = np.full(kv_len, -np.inf)
    index_mask[sel] = 0.0
    causal = np.where(np.arange(kv_len) <= t, 0.0, -np.inf)
    scores = sm_scale * (q @ latent_seq.T) + (index_mask + causal)[None, :]
    H = q.shape[0]
    if not np.isfinite(scores).any():
        return np.zeros((H, VALUE_DIM)), np.full(H, -np.inf)
    m = scores.max(axis=1, keepdims=True)
    e = np.exp(scores - m)
    s = e.sum(axis=1, keepdims=True)
    o = (e / s) @ latent_seq[:, :VALUE_DIM]
    return o, (m + np.log(s))[:, 0]


def sparse(inputs, idx: np.ndarray, rows=None):
    """Sparse MLA for query rows ``rows`` of a ``DSAInputs`` batch.

    ``idx`` is an [n_rows, k] index array (sequence-relative positions, -1 or
    out-of-range = skipped), row i of ``idx`` belonging to query row rows[i]
    (default: all rows, idx[r] for row r).  Returns {row: (o [H, 512], lse [H])}.
    """
    b = inputs.batch
    rows = list(range(b.total_q)) if rows is None else [int(r) for r in rows]
    out = {}
    for i, r in enumerate(rows):
        seq = int(b.q_seq[r])
        k0 = int(b.kv_start[seq])
        kv = int(b.kv_len[seq])
        sel = np.asarray(idx[i], dtype=np.int64)
        sel = sel[(sel >= 0) & (sel < kv)]
        c = bf16_to_f64(inputs.latent[k0 + sel])
        q = bf16_to_f64(inputs.q_mla[r])
        out[r] = attend(q, c, inputs.sm_scale)
    return out


def flops_per_token(n_heads: int, n_sel: int, latent_dim: int = 576, value_dim: int = VALUE_DIM) -> int:
    """Tensor-core work of one token: QK^T over 576 dims and PV over 512."""
    return 2 * n_heads * n_sel * (latent_dim + value_dim)


def bf16_output(o: np.ndarray) -> np.ndarray:
    """The output in the path's storage format: fp64 -> fp32 -> bf16, round to
    nearest even (the attention output is bf16).  Returned as float64 values."""
    f = np.ascontiguousarray(o, dtype=np.float32)
    u = f.view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)) << np.uint32(16)
    return r.astype(np.uint32).view(np.float32).astype(np.float64)
