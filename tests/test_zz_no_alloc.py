"""dsa_sparse_mla_no_alloc: sparse MLA for callers that cannot allocate device memory.

Callers such as an engine plugin restricted to the buffers its host hands it,
or a latency-critical loop that cannot afford cudaMalloc's implicit device
synchronisation, have no workspace to give dsa_sparse_mla.  The no-alloc entry
point keeps the split-selection partials in a fixed library-owned device array
instead.  These tests call it through the C ABI and check it against the
workspace-based entry point.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import custom_workload, make_inputs

SCRATCH_BYTES = 32 * 1024 * 1024


def _no_alloc(batch, q, kv, idx, k_sel, sm_scale, out, lse):
    lib = dsa.library()
    return lib.dsa_sparse_mla_no_alloc(batch.ref, ctypes.c_void_p(q.data_ptr()), int(q.shape[1]),
                                       ctypes.c_void_p(kv.data_ptr()), ctypes.c_void_p(idx.data_ptr()), k_sel,
                                       float(sm_scale), ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(lse.data_ptr()),
                                       ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _compare(out, lse, out_ref, lse_ref):
    o = out.float().cpu().numpy().astype(np.float64)
    r = out_ref.float().cpu().numpy().astype(np.float64)
    d = np.abs(o - r)
    assert d.max() <= 2e-2
    assert d.sum() / np.abs(r).sum() <= 1e-3
    assert torch.allclose(lse, lse_ref, rtol=1e-4, atol=2e-3)


@pytest.mark.gpu
def test_no_alloc_matches_workspace_entry_point_on_two_calls():
    # decode-shaped batch: few tokens, so the selection is split over several
    # CTA pairs and the partial results go through the scratch array
    x = make_inputs(custom_workload("noalloc", [4100, 3000, 5000, 2600, 6100, 3333, 4444, 2900],
                                    [1] * 8, k_sel=2048, n_heads=128), seed=21)
    from dsa_inputs.torch_io import device_tensors
    t = device_tensors(x)
    b = x.batch
    batch = dsa.Batch(t["cu_q"], t["kv_len"], t["kv_start"], b.total_q, b.max_q_per_seq, b.max_kv_len,
                      b.total_keys)
    assert dsa.workspace_size(dsa.OP_SPARSE_MLA, batch, 2048, 128) > 256   # the split path is taken
    rng = np.random.default_rng(5)
    results = []
    for call in range(2):
        # a different selection per call, so stale scratch from call 1 cannot pass for call 2
        idx = np.full((b.total_q, 2048), -1, np.int32)
        for r in range(b.total_q):
            kv = int(b.kv_len[r])
            n = 2048 - 300 * call
            idx[r, :n] = rng.choice(kv, n, replace=False)
        idx_d = torch.from_numpy(idx).cuda()
        out_ref = torch.empty((b.total_q, 128, 512), dtype=torch.bfloat16, device="cuda")
        lse_ref = torch.empty((b.total_q, 128), dtype=torch.float32, device="cuda")
        ws = dsa.workspace(dsa.OP_SPARSE_MLA, batch, 2048, 128)
        dsa.sparse_mla(batch, t["q_mla"], t["latent"], idx_d, 2048, x.sm_scale, out_ref, lse_ref, ws)
        dsa.check_device_error(ws)
        out = torch.full_like(out_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        assert _no_alloc(batch, t["q_mla"], t["latent"], idx_d, 2048, x.sm_scale, out, lse) == 0
        torch.cuda.synchronize()
        _compare(out, lse, out_ref, lse_ref)
        results.append(out)
    assert not torch.equal(results[0], results[1])


def test_no_alloc_scratch_covers_every_split_batch():
    # Only small batches have their selections split over several CTA pairs
    # (total_q * nsplit within one wave of 74 pairs; the only case with partial
    # results); the largest such batch must fit the fixed scratch array, so the
    # over-size rejection stays a guard that valid batches never reach.  Sizes
    # come from the library's own workspace rule, without touching the device.
    lib = dsa.library()
    worst = 0
    for total_q in range(1, 80):
        for k_sel in (64, 256, 1024, 2048):
            c = dsa._BatchC()
            c.num_seqs, c.total_q, c.max_q_per_seq, c.max_kv_len, c.total_keys = total_q, total_q, 1, 32768, total_q * 32768
            c.cu_q = c.kv_len = c.kv_start = 0x1000
            need = lib.dsa_workspace_size(dsa.OP_SPARSE_MLA, ctypes.byref(c), k_sel, 128)
            assert need > 0
            worst = max(worst, need)
    assert worst <= SCRATCH_BYTES
