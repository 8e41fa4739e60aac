"""The C ABI without a GPU: the library loads, exports every declared entry point,
sizes workspaces, describes statuses and rejects bad arguments before any launch."""

import ctypes
import os
import re

import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from long_context_sparse_lightning_b200 import _BatchC

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    txt = open(os.path.join(ROOT, "include", "dsa.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z0-9_]+)\s*\(", txt)))


def test_library_exports_every_declared_symbol():
    lib = dsa.library()
    names = declared_functions()
    assert set(names) == set(dsa.EXPORTS)
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings():
    assert dsa.version() == 200
    lib = dsa.library()
    for code in range(7):
        assert lib.dsa_status_string(code).decode()
    assert lib.dsa_status_string(99) == b"unknown status"


def _host_batch(B=2, total_q=10, max_q=6, max_kv=100, total_keys=180):
    c = _BatchC()
    c.num_seqs, c.total_q, c.max_q_per_seq, c.max_kv_len, c.total_keys = B, total_q, max_q, max_kv, total_keys
    c.cu_q = c.kv_len = c.kv_start = 0x1000   # never dereferenced on the host
    return c


def test_workspace_sizes():
    lib = dsa.library()
    c = _host_batch()
    ref = ctypes.byref(c)
    assert lib.dsa_workspace_size(dsa.OP_INDEXER, ref, 64, 16) == 256
    assert lib.dsa_workspace_size(dsa.OP_TOPK, ref, 64, 16) == 256
    fwd = lib.dsa_workspace_size(dsa.OP_FORWARD, ref, 64, 16)
    assert fwd >= 256 + 10 * 100 * 4
    assert lib.dsa_workspace_size(dsa.OP_FORWARD, ref, 4096, 16) == 0       # k_sel too large
    assert lib.dsa_workspace_size(dsa.OP_SPARSE_MLA, ref, 64, 256) == 0     # too many heads
    bad = _host_batch(B=0)
    assert lib.dsa_workspace_size(dsa.OP_TOPK, ctypes.byref(bad), 64, 16) == 0
    # rows longer than 32768 positions: the two-phase top-k keeps k candidates
    # (position + score) per 32768-position segment of every row
    # (4 segments for 131072 positions)
    long = _host_batch(max_kv=131072, total_keys=131072 * 3)
    extra = lib.dsa_workspace_size(dsa.OP_TOPK, ctypes.byref(long), 2048, 128) - 256
    per_seg = long.total_q * 2048 * 4            # one array of [total_q, k] (a multiple of 256 B here)
    assert extra == 2 * 4 * per_seg
    assert lib.dsa_workspace_size(dsa.OP_TOPK, ctypes.byref(long), 7, 128) == 256       # single-CTA rows
    assert lib.dsa_workspace_size(dsa.OP_FORWARD, ctypes.byref(long), 2048, 128) >= 256 + extra


def test_forward_launch_counts():
    lib = dsa.library()
    # short rows, few gathers per cache row: indexer, top-k, sparse MLA
    c = _host_batch()
    assert lib.dsa_forward_launches(ctypes.byref(c), 64, 16) == 3
    # one long-context sequence of many queries: + the fp16 latent copy
    pre = _host_batch(B=1, total_q=4096, max_q=4096, max_kv=32768, total_keys=32768)
    assert lib.dsa_forward_launches(ctypes.byref(pre), 2048, 128) == 4
    # a few two-token groups at 128K: two-phase top-k and split selections + merge
    dec = _host_batch(B=8, total_q=16, max_q=2, max_kv=131072, total_keys=8 * 131072)
    assert lib.dsa_forward_launches(ctypes.byref(dec), 2048, 128) == 5
    assert lib.dsa_forward_launches(ctypes.byref(dec), 4096, 128) == 0      # k_sel too large
    # 64 one-token decode rows: the fused indexer + top-k, then the sparse MLA
    dec1 = _host_batch(B=64, total_q=64, max_q=1, max_kv=32768, total_keys=64 * 32768)
    assert lib.dsa_forward_launches(ctypes.byref(dec1), 2048, 128) == 2


def test_fused_decode_workspace_holds_no_scores():
    lib = dsa.library()
    # decode: scores stay on chip, the indexer + top-k needs only the error word
    dec = _host_batch(B=64, total_q=64, max_q=1, max_kv=32768, total_keys=64 * 32768)
    assert lib.dsa_workspace_size(dsa.OP_INDEXER_TOPK, ctypes.byref(dec), 2048, 128) == 256
    fwd = lib.dsa_workspace_size(dsa.OP_FORWARD, ctypes.byref(dec), 2048, 128)
    assert fwd == lib.dsa_workspace_size(dsa.OP_SPARSE_MLA, ctypes.byref(dec), 2048, 128)
    # prefill: the [total_q, ld] fp32 score matrix
    pre = _host_batch(B=1, total_q=4096, max_q=4096, max_kv=32768, total_keys=32768)
    n = lib.dsa_workspace_size(dsa.OP_INDEXER_TOPK, ctypes.byref(pre), 2048, 128)
    assert n == 256 + 4096 * 32768 * 4
    # rows too long for 16 CTAs of 16384 positions: unfused
    huge = _host_batch(B=1, total_q=1, max_q=1, max_kv=300000, total_keys=300000)
    assert lib.dsa_workspace_size(dsa.OP_INDEXER_TOPK, ctypes.byref(huge), 2048, 128) > 256 + 300000 * 4


def test_rejections_happen_before_any_launch():
    lib = dsa.library()
    c = _host_batch()
    ref = ctypes.byref(c)
    P = ctypes.c_void_p
    fake = P(0x10000)                   # aligned, never dereferenced
    # null pointers
    assert lib.dsa_indexer_scores(ref, None, fake, fake, fake, fake, fake, 100, fake, 4096, None) == 1
    assert lib.dsa_topk(ref, fake, 100, 64, None, fake, 4096, None) == 1
    # misaligned pointer
    assert lib.dsa_topk(ref, P(0x10004), 100, 64, fake, fake, 4096, None) == 1
    # leading dimension too small / not a multiple of 4
    assert lib.dsa_topk(ref, fake, 99, 64, fake, fake, 4096, None) == 1
    assert lib.dsa_topk(ref, fake, 102, 64, fake, fake, 4096, None) == 1
    # unsupported k_sel / heads
    assert lib.dsa_topk(ref, fake, 100, 4096, fake, fake, 4096, None) == 2
    assert lib.dsa_sparse_mla(ref, fake, 200, fake, fake, 64, 0.07, fake, None, fake, 4096, None) == 2
    # bad scale
    assert lib.dsa_sparse_mla(ref, fake, 16, fake, fake, 64, -1.0, fake, None, fake, 4096, None) == 1
    # workspace too small
    assert lib.dsa_topk(ref, fake, 100, 64, fake, fake, 16, None) == 4
    need = lib.dsa_workspace_size(dsa.OP_FORWARD, ref, 64, 16)
    assert lib.dsa_forward(ref, fake, fake, fake, fake, fake, 64, fake, 16, fake, 0.07, fake, fake, None, fake,
                           need - 1, None) == 4
    # inconsistent batch
    bad = _host_batch(max_q=20)          # max_q_per_seq > total_q
    assert lib.dsa_topk(ctypes.byref(bad), fake, 100, 64, fake, fake, 4096, None) == 1


def test_empty_batch_is_a_no_op():
    lib = dsa.library()
    c = _host_batch(total_q=0, max_q=0)
    fake = ctypes.c_void_p(0x10000)
    assert lib.dsa_topk(ctypes.byref(c), fake, 100, 64, fake, fake, 4096, None) == 0


def test_binding_fails_loudly_without_library(monkeypatch):
    monkeypatch.setattr(dsa, "LIB_PATH", "/nonexistent/libdsa.so")
    monkeypatch.setattr(dsa, "_LIB", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        dsa.library()


def test_prep_entry_points_reject_bad_arguments():
    lib = dsa.library()
    c = _host_batch()
    ref = ctypes.byref(c)
    P = ctypes.c_void_p
    fake = P(0x10000)
    # quantiser: negative count, null or misaligned pointers; an empty call is a no-op
    assert lib.dsa_quantize_fp8(fake, -1, fake, fake, None) == 1
    assert lib.dsa_quantize_fp8(None, 4, fake, fake, None) == 1
    assert lib.dsa_quantize_fp8(fake, 4, P(0x10004), fake, None) == 1
    assert lib.dsa_quantize_fp8(fake, 0, fake, fake, None) == 0
    # cache write: workspace size, null / misaligned caches, empty batch
    assert lib.dsa_workspace_size(dsa.OP_CACHE_WRITE, ref, 0, 0) == 256
    assert lib.dsa_cache_write(ref, fake, fake, fake, fake, None, fake, 256, None) == 1
    assert lib.dsa_cache_write(ref, fake, P(0x10008), fake, fake, fake, fake, 256, None) == 1
    assert lib.dsa_cache_write(ref, fake, fake, fake, fake, fake, fake, 16, None) == 4
    empty = _host_batch(total_q=0, max_q=0)
    assert lib.dsa_cache_write(ctypes.byref(empty), fake, fake, fake, fake, fake, fake, 256, None) == 0


def test_quantize_binding_checks_shapes_before_the_call():
    x = torch.zeros((3, 128), dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        dsa.quantize_fp8(x, torch.zeros((3, 128), dtype=torch.uint8), torch.zeros(2, dtype=torch.float32))
    with pytest.raises(ValueError):
        dsa.quantize_fp8(x.float(), torch.zeros((3, 128), dtype=torch.uint8), torch.zeros(3, dtype=torch.float32))
    with pytest.raises(ValueError):
        dsa.quantize_fp8(torch.zeros((3, 64), dtype=torch.bfloat16), torch.zeros((3, 64), dtype=torch.uint8),
                         torch.zeros(3, dtype=torch.float32))


def test_paged_batch_checks():
    lib = dsa.library()

    def paged(page, blocks, total_keys=64 * 40, max_kv=1000):
        c = _host_batch(max_kv=max_kv, total_keys=total_keys)
        c.kv_start = None                    # ignored (may be null) with a block table
        c.block_table = 0x2000
        c.page_size, c.blocks_per_seq = page, blocks
        return c

    ok = paged(64, 16)
    assert lib.dsa_workspace_size(dsa.OP_INDEXER, ctypes.byref(ok), 64, 16) == 256
    for bad in (paged(32, 32), paged(96, 11), paged(64, 15),          # page not a multiple of 64; table too short
                paged(64, 16, total_keys=64 * 40 + 1)):               # pool not a whole number of pages
        assert lib.dsa_workspace_size(dsa.OP_INDEXER, ctypes.byref(bad), 64, 16) == 0
    flat_null = _host_batch()
    flat_null.kv_start = None                # flat caches need kv_start
    assert lib.dsa_workspace_size(dsa.OP_INDEXER, ctypes.byref(flat_null), 64, 16) == 0
