"""Paged KV caches on the GPU: the same batch with its caches scattered over a
page pool (block tables) must give the flat-cache results bit for bit -- the
indexer's key tiles, the fused decode selection, the sparse MLA gather and the
cache write only change where rows are read or written -- and the oracle's
results on the logical sequences rebuilt through its own page map.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import custom_workload, make_inputs
from dsa_inputs.paged import paged_layout
from oracle import paged as o_paged
from tests.parity import GpuRun, check_mla, check_topk

pytestmark = pytest.mark.gpu


class PagedRun(GpuRun):
    """GpuRun whose key, scale and latent caches are page pools."""

    def __init__(self, x, page_size, seed=0):
        super().__init__(x)
        self.pc = paged_layout(x, page_size, seed=seed)
        b = x.batch
        self.t["k8"] = torch.from_numpy(self.pc.k8).cuda()
        self.t["k_scale"] = torch.from_numpy(self.pc.k_scale).cuda()
        self.t["latent"] = torch.from_numpy(self.pc.latent.view(np.int16)).view(torch.bfloat16).cuda()
        self.table = torch.from_numpy(self.pc.block_table).cuda()
        self.batch = dsa.Batch(self.t["cu_q"], self.t["kv_len"], None, b.total_q, b.max_q_per_seq, b.max_kv_len,
                               self.pc.total_keys, block_table=self.table, page_size=page_size)


CASES = [
    # (kv_lens, q_lens, k_sel, n_heads, page)
    ([9000, 7000, 12000], [1, 1, 1], 2048, 128, 64),          # decode: fused indexer + top-k
    ([6000, 4100, 2049], [2, 2, 2], 2048, 128, 128),          # speculative pairs
    ([300, 1000, 77, 2500], [5, 130, 77, 3], 256, 64, 64),    # 8-token indexer blocks, ragged
    ([2048], [192], 512, 128, 256),                           # prefill-shaped: fp16 copy of the pool
]


@pytest.mark.parametrize("kv,q,k_sel,H,page", CASES)
def test_paged_forward_equals_flat(kv, q, k_sel, H, page):
    x = make_inputs(custom_workload("paged", kv, q, k_sel=k_sel, n_heads=H), seed=41)
    flat = GpuRun(x)
    pg = PagedRun(x, page, seed=7)
    i_f, o_f, l_f = flat.forward(k_sel)
    i_p, o_p, l_p = pg.forward(k_sel)
    assert torch.equal(i_p, i_f)
    assert torch.equal(o_p.view(torch.int16), o_f.view(torch.int16))
    assert torch.equal(l_p, l_f)
    # the standalone stages on the pool too
    s_p = pg.scores()
    s_f = flat.scores()
    rows = list(range(x.batch.total_q))
    for r in rows:
        t = int(x.batch.q_pos[r])
        assert torch.equal(s_p[r, : t + 1], s_f[r, : t + 1])


def test_paged_parity_with_the_oracle_through_its_page_map():
    x = make_inputs(custom_workload("paged_o", [3000, 1700], [2, 1], k_sel=512, n_heads=32), seed=42)
    pg = PagedRun(x, 64, seed=8)
    idx, out, lse = pg.forward(512)
    # the logical caches, rebuilt from the pool by the oracle's own map
    b = x.batch
    k8 = np.concatenate([o_paged.logical_view(pg.pc.k8, pg.pc.block_table, 64, s, int(b.kv_len[s]))
                         for s in range(b.num_seqs)])
    ks = np.concatenate([o_paged.logical_view(pg.pc.k_scale, pg.pc.block_table, 64, s, int(b.kv_len[s]))
                         for s in range(b.num_seqs)])
    lat = np.concatenate([o_paged.logical_view(pg.pc.latent, pg.pc.block_table, 64, s, int(b.kv_len[s]))
                          for s in range(b.num_seqs)])
    x.k8, x.k_scale, x.latent = k8, ks, lat
    rows = list(range(b.total_q))
    ih = idx.cpu().numpy()
    check_topk(x, ih, rows, 512)
    check_mla(x, out.float().cpu().numpy(), lse.cpu().numpy(), ih, rows)


@pytest.mark.parametrize("page", [64, 128])
def test_paged_cache_write(page):
    x = make_inputs(custom_workload("paged_w", [500, 260, 130], [3, 1, 2], k_sel=64, n_heads=16), seed=43)
    pg = PagedRun(x, page, seed=9)
    b = x.batch
    g = torch.Generator(device="cuda").manual_seed(3)
    k_new = torch.randn((b.total_q, 128), generator=g, device="cuda").to(torch.bfloat16)
    lat_new = torch.randn((b.total_q, 576), generator=g, device="cuda").to(torch.bfloat16)
    k8, ks, lat = pg.t["k8"].clone(), pg.t["k_scale"].clone(), pg.t["latent"].clone()
    ws = dsa.workspace(dsa.OP_CACHE_WRITE, pg.batch, 0, 0)
    dsa.cache_write(pg.batch, k_new, lat_new, k8, ks, lat, ws)
    dsa.check_device_error(ws)
    # the same write on the flat caches, then compared row by row through the page map
    flat = GpuRun(x)
    fk8, fks, flat_lat = flat.t["k8"].clone(), flat.t["k_scale"].clone(), flat.t["latent"].clone()
    wsf = dsa.workspace(dsa.OP_CACHE_WRITE, flat.batch, 0, 0)
    dsa.cache_write(flat.batch, k_new, lat_new, fk8, fks, flat_lat, wsf)
    dsa.check_device_error(wsf)
    k8h, ksh, lath = k8.cpu().numpy(), ks.cpu().numpy(), lat.view(torch.int16).cpu().numpy()
    fk8h, fksh, flath = fk8.cpu().numpy(), fks.cpu().numpy(), flat_lat.view(torch.int16).cpu().numpy()
    for s in range(b.num_seqs):
        k0, kv = int(b.kv_start[s]), int(b.kv_len[s])
        for pos in range(kv):
            r = o_paged.pool_row(pg.pc.block_table, page, s, pos)
            assert np.array_equal(k8h[r], fk8h[k0 + pos]) and ksh[r] == fksh[k0 + pos]
            assert np.array_equal(lath[r], flath[k0 + pos])
    # rows no sequence owns are untouched
    owned = {o_paged.pool_row(pg.pc.block_table, page, s, pos)
             for s in range(b.num_seqs) for pos in range(int(b.kv_len[s]))}
    spare = np.array(sorted(set(range(pg.pc.total_keys)) - owned))
    assert np.array_equal(k8h[spare], pg.pc.k8[spare])


def test_page_id_outside_the_pool_is_a_bounds_error():
    # the kernels check every page id before using it: a bad entry is reported
    # as DSA_ERR_DEVICE_BOUNDS and no row is read through it
    x = make_inputs(custom_workload("paged_bad", [3000, 2000], [1, 1], k_sel=256, n_heads=16), seed=44)
    pg = PagedRun(x, 64, seed=10)
    pg.table[1, 3] = pg.pc.num_pages + 5
    idx = torch.empty((2, 256), dtype=torch.int32, device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER_TOPK, pg.batch, 256)
    dsa.indexer_topk(pg.batch, pg.t["q8"], pg.t["q_scale"], pg.t["w"], pg.t["k8"], pg.t["k_scale"], 256, idx, ws)
    with pytest.raises(dsa.DSAError) as e:
        dsa.check_device_error(ws)
    assert e.value.status == 6
    # the context stays usable: a correct table afterwards gives the flat result
    pg.table[1, 3] = int(pg.pc.block_table[1, 3])
    ws.zero_()
    dsa.indexer_topk(pg.batch, pg.t["q8"], pg.t["q_scale"], pg.t["w"], pg.t["k8"], pg.t["k_scale"], 256, idx, ws)
    dsa.check_device_error(ws)
    flat = GpuRun(x)
    assert torch.equal(idx, flat.topk(flat.scores(), 256))
