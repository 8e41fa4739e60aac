"""dsa_sparse_mla_no_alloc: sparse MLA for callers that cannot allocate device memory.

Callers such as an engine plugin restricted to the buffers its host hands it,
or a latency-critical loop that cannot afford cudaMalloc's implicit device
synchronisation, have no workspace to give dsa_sparse_mla.  The no-alloc entry
point keeps the split-selection partials in a fixed library-owned device array
instead.  These tests call it through the C ABI, twice in a row on different
selections, and check it against the fp64 oracle and against the
workspace-based entry point, at the parity tolerances of the other tests.

This file is named so that pytest collects it last.
"""

import ctypes

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import custom_workload, make_inputs
from dsa_inputs.torch_io import device_tensors
from tests.parity import check_mla

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


def _setup(x):
    t = device_tensors(x)
    b = x.batch
    batch = dsa.Batch(t["cu_q"], t["kv_len"], t["kv_start"], b.total_q, b.max_q_per_seq, b.max_kv_len,
                      b.total_keys)
    return t, batch


def _random_selection(x, rng, n_drop):
    b = x.batch
    k = x.k_sel
    idx = np.full((b.total_q, k), -1, np.int32)
    for r in range(b.total_q):
        t = int(b.q_pos[r])
        n = min(k - n_drop, t + 1)
        idx[r, :n] = rng.choice(t + 1, n, replace=False)
    return idx


def _two_calls(x, seed):
    """Two calls in a row on different selections: each against the oracle and
    against dsa_sparse_mla with a workspace."""
    t, batch = _setup(x)
    b = x.batch
    H, k = x.n_heads, x.k_sel
    rng = np.random.default_rng(seed)
    rows = list(range(b.total_q))
    results = []
    for call in range(2):
        # a different selection per call, so stale scratch from call 1 cannot pass for call 2
        idx = _random_selection(x, rng, n_drop=(k // 7) * call)
        idx_d = torch.from_numpy(idx).cuda()
        out_ref = torch.empty((b.total_q, H, 512), dtype=torch.bfloat16, device="cuda")
        lse_ref = torch.empty((b.total_q, H), dtype=torch.float32, device="cuda")
        ws = dsa.workspace(dsa.OP_SPARSE_MLA, batch, k, H)
        dsa.sparse_mla(batch, t["q_mla"], t["latent"], idx_d, k, x.sm_scale, out_ref, lse_ref, ws)
        dsa.check_device_error(ws)
        out = torch.full_like(out_ref, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        assert _no_alloc(batch, t["q_mla"], t["latent"], idx_d, k, x.sm_scale, out, lse) == 0
        torch.cuda.synchronize()
        check_mla(x, out.float().cpu().numpy(), lse.cpu().numpy(), idx, rows)
        _compare(out, lse, out_ref, lse_ref)
        results.append(out)
    assert not torch.equal(results[0], results[1])


@pytest.mark.gpu
def test_no_alloc_split_decode_two_calls():
    # decode-shaped batch: few tokens, so the selection is split over several
    # CTA pairs and the partial results go through the scratch array
    x = make_inputs(custom_workload("noalloc", [4100, 3000, 5000, 2600, 6100, 3333, 4444, 2900],
                                    [1] * 8, k_sel=2048, n_heads=128), seed=21)
    _, batch = _setup(x)
    assert dsa.workspace_size(dsa.OP_SPARSE_MLA, batch, 2048, 128) > 256   # the split path is taken
    _two_calls(x, seed=5)


@pytest.mark.gpu
def test_no_alloc_unsplit_prefill_two_calls():
    # prefill-shaped batch: one CTA pair per token, no partial results; here
    # dsa_sparse_mla would gather from an fp16 copy of the cache while the
    # no-alloc entry point gathers bf16 rows -- both within the tolerances
    x = make_inputs("tiny_prefill_512", seed=22)
    _, batch = _setup(x)
    assert dsa.workspace_size(dsa.OP_SPARSE_MLA, batch, x.k_sel, x.n_heads) >= 256 + x.batch.total_keys * 1152
    _two_calls(x, seed=6)


@pytest.mark.gpu
def test_no_alloc_out_of_range_sequence_leaves_no_stale_rows():
    # A first call fills the scratch array with split partials.  The second
    # call's batch gives one sequence a kv_start that runs past the cache: the
    # kernel's own bounds check skips that sequence (no access through it) and
    # its row must come out as out = 0, lse = -inf -- not as the first call's
    # partials merged again.  The other rows are checked against the oracle.
    x = make_inputs(custom_workload("noalloc_bad", [4100, 3000, 5000, 2600], [1] * 4, k_sel=2048, n_heads=128),
                    seed=23)
    t, batch = _setup(x)
    b = x.batch
    rng = np.random.default_rng(7)
    idx = _random_selection(x, rng, n_drop=0)
    idx_d = torch.from_numpy(idx).cuda()
    out = torch.empty((b.total_q, 128, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((b.total_q, 128), dtype=torch.float32, device="cuda")
    assert _no_alloc(batch, t["q_mla"], t["latent"], idx_d, 2048, x.sm_scale, out, lse) == 0
    torch.cuda.synchronize()
    bad = 2
    ks = t["kv_start"].clone()
    ks[bad] = b.total_keys - 100              # kv_start + kv_len > total_keys
    batch2 = dsa.Batch(t["cu_q"], t["kv_len"], ks, b.total_q, b.max_q_per_seq, b.max_kv_len, b.total_keys)
    out.fill_(float("nan"))
    lse.fill_(float("nan"))
    assert _no_alloc(batch2, t["q_mla"], t["latent"], idx_d, 2048, x.sm_scale, out, lse) == 0
    torch.cuda.synchronize()
    oh, lh = out.float().cpu().numpy(), lse.cpu().numpy()
    assert np.all(oh[bad] == 0) and np.all(np.isneginf(lh[bad]))
    good = [r for r in range(b.total_q) if r != bad]
    check_mla(x, oh[good], lh[good], idx[good], good)


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
