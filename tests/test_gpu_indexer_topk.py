"""The fused decode indexer + top-k (dsa_indexer_topk) against the two-kernel
path and the fp64 oracle.

For decode batches (1-2 query tokens per sequence) one cluster of CTAs per
sequence scores the row into shared memory and selects on chip.  Its output
must equal dsa_topk over dsa_indexer_scores bit for bit (same scores, same
exact selection rule and order), and the oracle's selection up to
near-threshold swaps.  The batches cover cluster sizes from 1 to 16, CTAs
whose chunk is empty or holds no valid position, rows of at most k positions,
two-token groups with a lone last token, k not a multiple of 4, and a row of
equal scores (the threshold ties are split across CTAs by position).
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import custom_workload, make_inputs
from tests.parity import GpuRun, check_topk

pytestmark = pytest.mark.gpu


def _fused(g, k_sel):
    b = g.x.batch
    idx = torch.full((b.total_q, k_sel), -7, dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER_TOPK, g.batch, k_sel)
    assert ws.numel() == 256, "the decode batch takes the fused kernel"
    dsa.indexer_topk(g.batch, g.t["q8"], g.t["q_scale"], g.t["w"], g.t["k8"], g.t["k_scale"], k_sel, idx, ws)
    dsa.check_device_error(ws)
    return idx


CASES = [
    # (kv_lens, q_lens, k_sel)
    ([4000, 3100, 5000, 257], [1, 1, 1, 1], 2048),               # short row (n <= k) next to long ones
    ([6000, 4100, 2049, 3000], [2, 2, 2, 2], 2048),              # two-token groups
    ([5000, 3000, 4100], [2, 1, 2], 1024),                       # a one-token sequence in a two-token batch
    ([2100 + 37 * i for i in range(40)], [1] * 40, 2048),        # 40 sequences
    ([40000, 300, 1500], [1, 1, 1], 64),                         # 16-CTA clusters: empty chunks on short rows
    ([70000, 9000], [2, 2], 2048),                               # 70K positions, two tokens
    ([3000, 2500], [1, 1], 7),                                   # k not a multiple of 4
    ([3000, 2500], [2, 2], 1),                                   # k = 1
]


@pytest.mark.parametrize("kv,q,k_sel", CASES)
def test_fused_equals_two_kernels_and_oracle(kv, q, k_sel):
    x = make_inputs(custom_workload("fused", kv, q, k_sel=k_sel, n_heads=16), seed=31)
    g = GpuRun(x)
    idx = _fused(g, k_sel)
    ref = g.topk(g.scores(), k_sel)
    assert torch.equal(idx, ref)
    rows = list(range(x.batch.total_q))
    check_topk(x, idx.cpu().numpy(), rows, k_sel)


def test_fused_equal_scores_split_ties_by_position():
    # every key the same: every score of a row ties, so the threshold value is
    # shared by all positions and the lowest k positions win -- across the
    # CTAs of each cluster
    x = make_inputs(custom_workload("fused_ties", [20000, 6000], [1, 2], k_sel=2048, n_heads=16), seed=32)
    x.k8[:] = x.k8[0]
    x.k_scale[:] = x.k_scale[0]
    g = GpuRun(x)
    idx = _fused(g, 2048).cpu().numpy()
    for r in range(x.batch.total_q):
        assert idx[r].tolist() == list(range(2048))


def test_forward_on_decode_uses_no_score_matrix():
    # one-token decode rows over enough sequences to fill the GPU: the forward
    # takes the fused kernel (its workspace has no room for the scores), and
    # its selection equals the two-kernel one
    x = make_inputs(custom_workload("fused_fwd", [3000 + 17 * i for i in range(64)], [1] * 64, k_sel=2048,
                                    n_heads=16), seed=33)
    g = GpuRun(x)
    ws_fwd = dsa.workspace_size(dsa.OP_FORWARD, g.batch, 2048, 16)
    assert ws_fwd == dsa.workspace_size(dsa.OP_SPARSE_MLA, g.batch, 2048, 16)
    idx_f, _, _ = g.forward(2048)
    assert torch.equal(idx_f, g.topk(g.scores(), 2048))
