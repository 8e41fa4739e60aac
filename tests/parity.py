"""Parity helpers shared by the GPU tests: run the CUDA path through the C ABI and
compare it with the fp64 oracle at the tolerances the hot path is specified to.

* scores:  |I_gpu - I| <= 1e-3 * sum_j |w q k| + 1e-6 for every valid (t, s);
* top-k:   the selected sets are equal except for positions whose oracle score
           lies within tolerance of the k-th value (counts must match);
* output:  against the oracle rounded to the bf16 output format, max |d| <= 2e-2
           and sum |d| / sum |ref| <= 1e-3.
"""

from __future__ import annotations

import numpy as np
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs.torch_io import device_tensors
from oracle import indexer as o_indexer
from oracle import mla as o_mla
from oracle import topk as o_topk


class GpuRun:
    """Device copies of a DSAInputs batch plus the ABI batch descriptor."""

    def __init__(self, x, device="cuda"):
        self.x = x
        self.t = device_tensors(x, device)
        b = x.batch
        self.batch = dsa.Batch(self.t["cu_q"], self.t["kv_len"], self.t["kv_start"], b.total_q, b.max_q_per_seq,
                               b.max_kv_len, b.total_keys)
        self.ld = ((b.max_kv_len + 3) // 4) * 4

    def scores(self, fill=float("nan")):
        b = self.x.batch
        s = torch.full((b.total_q, self.ld), fill, dtype=torch.float32, device="cuda")
        ws = dsa.workspace(dsa.OP_INDEXER, self.batch)
        dsa.indexer_scores(self.batch, self.t["q8"], self.t["q_scale"], self.t["w"], self.t["k8"],
                           self.t["k_scale"], s, ws)
        dsa.check_device_error(ws)
        return s

    def topk(self, scores, k_sel):
        idx = torch.full((self.x.batch.total_q, k_sel), -7, dtype=torch.int32, device="cuda")
        ws = dsa.workspace(dsa.OP_TOPK, self.batch, k_sel)
        dsa.topk(self.batch, scores, k_sel, idx, ws)
        dsa.check_device_error(ws)
        return idx

    def mla(self, idx, k_sel, with_lse=True):
        b = self.x.batch
        H = self.x.n_heads
        out = torch.full((b.total_q, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((b.total_q, H), float("nan"), dtype=torch.float32, device="cuda") if with_lse else None
        ws = dsa.workspace(dsa.OP_SPARSE_MLA, self.batch, k_sel, H)
        dsa.sparse_mla(self.batch, self.t["q_mla"], self.t["latent"], idx, k_sel, self.x.sm_scale, out, lse, ws)
        dsa.check_device_error(ws)
        return out, lse

    def forward(self, k_sel):
        b = self.x.batch
        H = self.x.n_heads
        idx = torch.full((b.total_q, k_sel), -7, dtype=torch.int32, device="cuda")
        out = torch.full((b.total_q, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((b.total_q, H), float("nan"), dtype=torch.float32, device="cuda")
        ws = dsa.workspace(dsa.OP_FORWARD, self.batch, k_sel, H)
        dsa.forward(self.batch, self.t["q8"], self.t["q_scale"], self.t["w"], self.t["k8"], self.t["k_scale"], k_sel,
                    self.t["q_mla"], self.t["latent"], self.x.sm_scale, idx, out, lse, ws)
        dsa.check_device_error(ws)
        return idx, out, lse


def check_scores(x, scores_gpu: np.ndarray, rows):
    """scores_gpu: [len(rows), ld] host copy of the GPU rows."""
    worst = 0.0
    for i, (r, t, I, B) in enumerate(o_indexer.scores(x, rows)):
        g = scores_gpu[i, : t + 1].astype(np.float64)
        tol = o_indexer.tolerance(B)
        err = np.abs(g - I)
        bad = np.nonzero(~(err <= tol))[0]
        assert bad.size == 0, f"row {r} (t={t}): {bad.size} scores out of tolerance, first s={bad[0]} " \
                              f"gpu={g[bad[0]]} ref={I[bad[0]]} tol={tol[bad[0]]}"
        worst = max(worst, float((err / tol).max()))
    return worst


def check_topk(x, idx_gpu: np.ndarray, rows, k_sel):
    """idx_gpu: [len(rows), k_sel] host copy.  Returns the number of tie swaps seen."""
    swaps = 0
    for i, (r, t, I, B) in enumerate(o_indexer.scores(x, rows)):
        row = idx_gpu[i]
        n = t + 1
        valid = row[row >= 0]
        assert np.all(row[: valid.size] >= 0) and np.all(row[valid.size:] == -1), f"row {r}: valid entries first"
        assert valid.size == min(n, k_sel), f"row {r}: {valid.size} selected, expected {min(n, k_sel)}"
        assert np.unique(valid).size == valid.size, f"row {r}: duplicate positions"
        assert valid.max(initial=-1) <= t, f"row {r}: position beyond t={t}"
        sel, vk = o_topk.select(I, k_sel)
        g, o = set(valid.tolist()), set(sel.tolist())
        diff = np.array(sorted(g ^ o), dtype=np.int64)
        if diff.size:
            near = set(o_topk.near_threshold(I, o_indexer.tolerance(B), vk, sel).tolist())
            far = [int(s) for s in diff if int(s) not in near]
            assert not far, f"row {r}: positions {far[:5]} differ but are not near the threshold"
            swaps += diff.size // 2
    return swaps


def check_mla(x, out_gpu: np.ndarray, lse_gpu, idx_rows: np.ndarray, rows, max_abs=o_mla.OUT_MAX_ABS,
              mean_rel=o_mla.OUT_MEAN_REL, value_scale=1.0, ulp_floor=False):
    """out_gpu [len(rows), H, 512] float (from bf16), lse_gpu [len(rows), H] or None,
    idx_rows [len(rows), k] -- the index rows the GPU attended over.

    ``value_scale``: the factor the latent entries were scaled by (1 for the
    configs' N(0,1) draws).  The output is linear in the values, so the max-abs
    bound applies to the difference divided by it; the mean relative error is
    scale-free.  ``ulp_floor``: an element may also differ by one bf16 step --
    when a peaky softmax makes outputs as large as the values themselves
    (|o| >= 4 value scales, where one bf16 step exceeds the bound), an fp32
    result and the fp64 one may round to neighbouring bf16 numbers."""
    ref = o_mla.sparse(x, idx_rows, rows)
    sum_abs = sum_ref = 0.0
    worst = 0.0
    where = None
    for i, r in enumerate(rows):
        o, lse = ref[int(r)]
        rb = o_mla.bf16_output(o)
        g = out_gpu[i].astype(np.float64)
        d = np.abs(g - rb)
        assert np.all(np.isfinite(out_gpu[i])), f"row {r}: non-finite output"
        dm = d / value_scale
        if ulp_floor:
            # one bf16 step at the larger of the two magnitudes (the two may sit
            # on either side of a power of two)
            big = np.maximum(np.abs(rb), np.abs(g))
            step = np.where(big == 0, 0.0, np.ldexp(1.0, np.frexp(big)[1] - 8))
            dm = np.where(d <= step, np.minimum(dm, max_abs), dm)
        j = np.unravel_index(int(np.argmax(dm)), dm.shape)
        if float(dm[j]) > worst or where is None:
            worst = max(worst, float(dm[j]))
            where = (int(r), tuple(int(v) for v in j), float(rb[j]), float(g[j]))
        sum_abs += float(d.sum())
        sum_ref += float(np.abs(rb).sum())
        if lse_gpu is not None:
            fin = np.isfinite(lse)
            assert np.array_equal(np.isfinite(lse_gpu[i]), fin), f"row {r}: lse finiteness differs"
            assert np.allclose(lse_gpu[i][fin], lse[fin], rtol=1e-4, atol=2e-3), f"row {r}: lse"
    rel = sum_abs / max(sum_ref, 1e-300)
    assert worst <= max_abs, f"max |d| = {worst} at (row, (head, dim), ref, gpu) = {where}"
    assert rel <= mean_rel, f"mean relative error = {rel}"
    return worst, rel


def sample_rows(x, n, seed=0):
    """n query rows spread over the batch: first, last, and seeded picks."""
    total = x.batch.total_q
    if total <= n:
        return list(range(total))
    rng = np.random.default_rng(seed)
    picks = set([0, total - 1]) | set(rng.choice(total, n - 2, replace=False).tolist())
    return sorted(picks)[:n]
