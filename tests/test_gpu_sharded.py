"""Key-sharded selection on one GPU: the keys of every sequence split into
contiguous shards (emulated one after another, as separate ranks would run
them), each shard's local top k as global candidates (dsa_topk_candidates),
then the merge (dsa_topk_merge).  The result must equal the unsharded
selection bit for bit -- the same exact rule over the same scores -- for
decode rows (one query token per sequence, so every shard position is
visible to it)."""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import custom_workload, make_inputs
from long_context_sparse_lightning_b200 import sharded
from tests.parity import GpuRun, check_topk

pytestmark = pytest.mark.gpu


def _sharded_topk(g, R, k):
    x = g.x
    b = x.batch
    pos_l, val_l = [], []
    for r in range(R):
        starts, lens = sharded.shard_bounds(b.kv_len, R, r)
        kv_len_r = torch.tensor(lens, dtype=torch.int32, device="cuda")
        kv_start_r = torch.from_numpy(b.kv_start + np.asarray(starts, np.int64)).cuda()
        off = torch.tensor(starts, dtype=torch.int32, device="cuda")
        batch_r = dsa.Batch(g.t["cu_q"], kv_len_r, kv_start_r, b.total_q, b.max_q_per_seq, max(lens), b.total_keys)
        ld = ((max(lens) + 3) // 4) * 4
        sc = torch.empty((b.total_q, ld), dtype=torch.float32, device="cuda")
        ws = dsa.workspace(dsa.OP_TOPK, batch_r, k)
        dsa.indexer_scores(batch_r, g.t["q8"], g.t["q_scale"], g.t["w"], g.t["k8"], g.t["k_scale"], sc, ws)
        cp = torch.empty((b.total_q, k), dtype=torch.int32, device="cuda")
        cv = torch.empty((b.total_q, k), dtype=torch.float32, device="cuda")
        dsa.topk_candidates(batch_r, sc, k, cp, cv, ws, pos_offset=off)
        dsa.check_device_error(ws)
        pos_l.append(cp)
        val_l.append(cv)
    cand_pos = torch.stack(pos_l, dim=1).contiguous()
    cand_val = torch.stack(val_l, dim=1).contiguous()
    idx = torch.full((b.total_q, k), -7, dtype=torch.int32, device="cuda")
    dsa.topk_merge(cand_pos, cand_val, k, idx)
    return idx


@pytest.mark.parametrize("kv,k,R", [
    ([9000, 5000, 12000, 3000], 2048, 3),
    ([40000, 2100], 2048, 4),          # shards shorter than k on the short row
    ([700, 5000], 256, 8),
])
def test_emulated_key_shards_merge_to_the_unsharded_selection(kv, k, R):
    x = make_inputs(custom_workload("sharded", kv, [1] * len(kv), k_sel=k, n_heads=16), seed=51)
    g = GpuRun(x)
    ref = g.topk(g.scores(), k)
    idx = _sharded_topk(g, R, k)
    assert torch.equal(idx, ref)
    check_topk(x, idx.cpu().numpy(), list(range(x.batch.total_q)), k)


def test_equal_scores_across_shards_keep_the_lowest_positions():
    x = make_inputs(custom_workload("sharded_ties", [6000, 3000], [1, 1], k_sel=1024, n_heads=16), seed=52)
    x.k8[:] = x.k8[0]
    x.k_scale[:] = x.k_scale[0]
    g = GpuRun(x)
    idx = _sharded_topk(g, 4, 1024).cpu().numpy()
    for r in range(2):
        assert idx[r].tolist() == list(range(1024))
