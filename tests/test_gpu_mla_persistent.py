"""Sparse MLA persistent grid: many (token, split) items per CTA pair.

The kernel launches one CTA pair per resident cluster slot and each pair walks
its share of the items, carrying barrier phases, ring slots and TMEM contents
from one item to the next.  The configs' small batches give each pair one
item, so these tests cap the grid (DSA_MLA_MAX_PAIRS, read at every launch)
to push 10-200 items through each pair and check, against the fp64 oracle
and bit for bit against the uncapped launch:

* both kernel paths: the fp16-copy kernel of prefill-shaped batches and the
  bf16-cache kernel of decode-shaped ones, unsplit and split;
* head counts below, at and above 64 (the RoPE rows of a Q slice travel in
  one or two ring stages) and not a multiple of 8;
* items whose selection holds no valid position (a Q slice and no tiles:
  out = 0, lse = -inf) next to ordinary ones, and short selections.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import custom_workload, make_inputs
from oracle import indexer as o_indexer
from oracle import topk as o_topk
from tests.parity import GpuRun, check_mla

pytestmark = pytest.mark.gpu

# (name, kv_lens, q_lens, k_sel, n_heads)
SHAPES = {
    "prefill_h128": ([2048], [192], 512, 128),
    "prefill_h100": ([1600, 900], [96, 64], 256, 100),
    "prefill_h64": ([2048], [160], 384, 64),
    "prefill_h24": ([3000], [128], 256, 24),
    "decode_unsplit": ([2100 + 37 * i for i in range(40)], [1] * 40, 2048, 128),
    "decode_split": ([4000, 3100, 5000, 2600], [1, 1, 1, 1], 2048, 128),
}
CAPS = [1, 3, 7]


def _oracle_idx(x):
    rows = list(range(x.batch.total_q))
    idx = np.full((len(rows), x.k_sel), -1, np.int32)
    for i, (_, t, I, _) in enumerate(o_indexer.scores(x, rows)):
        sel, _ = o_topk.select(I, x.k_sel)
        idx[i, : sel.size] = sel
    return idx


def _host(t):
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def _run(g, idx, k, monkeypatch, cap):
    if cap:
        monkeypatch.setenv("DSA_MLA_MAX_PAIRS", str(cap))
    else:
        monkeypatch.delenv("DSA_MLA_MAX_PAIRS", raising=False)
    out, lse = g.mla(torch.from_numpy(idx).cuda(), k)
    torch.cuda.synchronize()
    return out, lse


@pytest.mark.parametrize("shape", list(SHAPES))
def test_many_items_per_pair(shape, monkeypatch):
    kv, q, k_sel, H = SHAPES[shape]
    x = make_inputs(custom_workload(f"persist_{shape}", kv, q, k_sel=k_sel, n_heads=H), seed=61)
    g = GpuRun(x)
    idx = _oracle_idx(x)
    n = x.batch.total_q
    # every fifth row selects nothing valid (a Q slice, no tiles), every
    # seventh keeps only its first 40 slots (a ragged last tile)
    empty = list(range(2, n, 5))
    idx[empty] = -1
    for r in range(3, n, 7):
        if r not in empty:
            idx[r, 40:] = -1
    rows = list(range(n))
    ref_out, ref_lse = _run(g, idx, k_sel, monkeypatch, 0)
    check_mla(x, _host(ref_out), _host(ref_lse), idx, rows)
    ho, hl = _host(ref_out), _host(ref_lse)
    assert np.all(ho[empty] == 0.0)
    assert np.all(np.isneginf(hl[empty]))
    for cap in CAPS:
        out, lse = _run(g, idx, k_sel, monkeypatch, cap)
        # the same arithmetic per item, whichever pair runs it
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16)), cap
        assert torch.equal(lse, ref_lse), cap


def test_forward_capped_matches_uncapped(monkeypatch):
    x = make_inputs(custom_workload("persist_fwd", [3000, 1700], [40, 24], k_sel=512, n_heads=128), seed=62)
    g = GpuRun(x)
    monkeypatch.delenv("DSA_MLA_MAX_PAIRS", raising=False)
    idx0, out0, lse0 = g.forward(x.k_sel)
    monkeypatch.setenv("DSA_MLA_MAX_PAIRS", "2")
    idx1, out1, lse1 = g.forward(x.k_sel)
    torch.cuda.synchronize()
    assert torch.equal(idx0, idx1)
    assert torch.equal(out0.view(torch.int16), out1.view(torch.int16))
    assert torch.equal(lse0, lse1)


# (name, kv_lens, q_lens, k_sel): the bf16-cache kernel unsplit, the same split
# (one-token rows), and the fp16-copy kernel of a prefill-shaped batch
GAP_SHAPES = {
    "unsplit": ([3000, 2000], [5, 4], 256),
    "split": ([4000, 3100, 5000, 2600], [1, 1, 1, 1], 2048),
    "fp16_copy": ([2048], [192], 512),
}


@pytest.mark.parametrize("shape", list(GAP_SHAPES))
def test_row_outside_every_sequence(shape, monkeypatch):
    # cu_q stops one row short of total_q: that row lies in no sequence.  The
    # kernel records DSA_ERR_DEVICE_BOUNDS and gives the row out = 0 and
    # lse = -inf (split partials: lse = -inf, so the merge cannot pick up a
    # stale partial); every other row is computed as usual.
    monkeypatch.delenv("DSA_MLA_MAX_PAIRS", raising=False)
    kv, q, k_sel = GAP_SHAPES[shape]
    x = make_inputs(custom_workload(f"persist_gap_{shape}", kv, q, k_sel=k_sel, n_heads=128), seed=63)
    g = GpuRun(x)
    idx = _oracle_idx(x)
    n, H = x.batch.total_q, x.n_heads
    g.t["cu_q"][-1] -= 1
    out = torch.full((n, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((n, H), float("nan"), dtype=torch.float32, device="cuda")
    ws = dsa.workspace(dsa.OP_SPARSE_MLA, g.batch, k_sel, H)
    ws.zero_()
    dsa.sparse_mla(g.batch, g.t["q_mla"], g.t["latent"], torch.from_numpy(idx).cuda(), k_sel, x.sm_scale, out,
                   lse, ws)
    with pytest.raises(dsa.DSAError) as e:
        dsa.check_device_error(ws)
    assert e.value.status == 6
    oh, lh = _host(out), _host(lse)
    assert np.all(oh[n - 1] == 0.0) and np.all(np.isneginf(lh[n - 1]))
    rows = list(range(n - 1))
    check_mla(x, oh[: n - 1], lh[: n - 1], idx[: n - 1], rows)
