"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Small cases are compared on every row; the full-size workloads on sampled rows,
in the same launch configuration the benchmark times (dsa_forward), plus a
bit-exact check that dsa_forward equals the three standalone stages.
"""

import numpy as np
import pytest
import torch

from dsa_inputs import custom_workload, make_inputs
from tests.parity import GpuRun, check_mla, check_scores, check_topk, sample_rows

pytestmark = pytest.mark.gpu


def _host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _full_check(x, rows=None, k_sel=None):
    g = GpuRun(x)
    k_sel = k_sel or x.k_sel
    rows = list(range(x.batch.total_q)) if rows is None else rows
    s = g.scores()
    sh = _host(s)
    check_scores(x, sh[rows], rows)
    # positions beyond t stay untouched
    for r in rows[:8]:
        t = int(x.batch.q_pos[r])
        assert np.all(np.isnan(sh[r, t + 1:])), f"row {r}: wrote beyond t"
    idx = g.topk(s, k_sel)
    ih = _host(idx)
    check_topk(x, ih[rows], rows, k_sel)
    out, lse = g.mla(idx, k_sel)
    oh, lh = _host(out), _host(lse)
    check_mla(x, oh[rows], lh[rows], ih[rows], rows)
    idx2, out2, lse2 = g.forward(k_sel)
    assert torch.equal(idx2, idx)
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
    assert torch.equal(lse2, lse)
    return g, ih, oh


def test_tiny_prefill_512_every_row():
    _full_check(make_inputs("tiny_prefill_512"))


@pytest.mark.parametrize("kv,q,k_sel,H", [
    ([300, 1000, 77, 2500, 129], [5, 130, 77, 3, 1], 256, 64),     # 8-token indexer blocks, ragged tails
    ([4000, 3100, 5000, 257], [1, 1, 1, 1], 2048, 128),            # decode: 1 token, selection split in 4
    ([6000, 4100, 2049, 3000], [2, 2, 2, 2], 2048, 128),           # speculative pairs, split in 4
    ([700, 900], [5, 4], 512, 32),                                 # 4-token indexer blocks
    ([2100 + 37 * i for i in range(40)], [1] * 40, 2048, 128),      # 40 decode tokens, one pair each
    ([9000, 700], [1, 1], 1024, 64),                               # 2 tokens, 16 tiles: split in 2
    ([128, 256, 384], [128, 17, 256], 64, 16),                     # exact tile multiples
    ([3000], [100], 2048, 64),                                     # one sequence over more tokens than CTA pairs
    ([5000], [80], 1024, 128),                                     # the same with 16-tile selections
])
def test_ragged_batches(kv, q, k_sel, H):
    x = make_inputs(custom_workload("ragged", kv, q, k_sel=k_sel, n_heads=H), seed=11)
    _full_check(x)


def test_short_rows_and_k_sel_one():
    x = make_inputs(custom_workload("short", [1, 5, 40], [1, 5, 40], k_sel=64, n_heads=16), seed=3)
    _, ih, _ = _full_check(x)
    for r in range(x.batch.total_q):
        t = int(x.batch.q_pos[r])
        assert ih[r, : t + 1].tolist() == list(range(t + 1))
    x1 = make_inputs(custom_workload("k1", [300], [50], k_sel=1, n_heads=16), seed=4)
    _full_check(x1, k_sel=1)


def test_equal_keys_break_ties_by_position():
    x = make_inputs(custom_workload("ties", [3000], [6], k_sel=512, n_heads=16), seed=5)
    x.k8[:] = x.k8[0]
    x.k_scale[:] = x.k_scale[0]
    g = GpuRun(x)
    s = g.scores()
    idx = _host(g.topk(s, 512))
    for r in range(6):
        assert sorted(idx[r].tolist()) == list(range(512))


def test_mla_index_edge_cases():
    x = make_inputs(custom_workload("mlaedge", [500, 300], [3, 2], k_sel=128, n_heads=128), seed=6)
    g = GpuRun(x)
    idx = np.full((5, 128), -1, np.int32)
    idx[0, :70] = np.arange(0, 140, 2)                 # plain
    idx[1, 5:20] = np.arange(15)                       # -1 before and after
    idx[1, 40] = 499
    idx[2, :10] = [3, 600, -5, 7, 499, 1000000, 2, 9, 11, 13]   # out-of-range entries are skipped
    idx[3, :] = -1                                     # nothing selected
    idx[4, 127] = 0                                    # a single entry at the very end
    out, lse = g.mla(torch.from_numpy(idx).cuda(), 128)
    oh, lh = _host(out), _host(lse)
    assert np.all(oh[3] == 0) and np.all(np.isneginf(lh[3]))
    rows = [0, 1, 2, 4]
    check_mla(x, oh[rows], lh[rows], idx[rows], rows)


@pytest.mark.parametrize("name,n_rows", [
    ("decode_64x16k_32k", 12),
    ("prefill_8k", 10),
    ("chunked_prefill_28k_4k", 10),
    ("spec_decode_8x2_128k", 8),
])
def test_full_size_workloads_sampled(name, n_rows):
    x = make_inputs(name)
    rows = sample_rows(x, n_rows, seed=1)
    g = GpuRun(x)
    s = g.scores()
    check_scores(x, _host(s[rows]), rows)
    idx = g.topk(s, x.k_sel)
    ih = _host(idx[rows])
    check_topk(x, ih, rows, x.k_sel)
    out, lse = g.mla(idx, x.k_sel)
    check_mla(x, _host(out[rows]), _host(lse[rows]), ih, rows)
    del s
    idx2, out2, lse2 = g.forward(x.k_sel)
    assert torch.equal(idx2, idx)
    assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
