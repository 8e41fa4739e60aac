"""Python binding of libdsa.so, the B200 (sm_100a) DeepSeek Sparse Attention hot path.

Argument marshalling only: every stage runs in the library's CUDA kernels on
the caller's current torch stream; torch provides device memory and streams.
There is no CPU fallback -- if the shared library is missing, importing the
binding's entry points raises.

    import long_context_sparse_lightning_b200 as dsa
    batch = dsa.Batch(cu_q, kv_len, kv_start, max_q_per_seq, max_kv_len, total_keys)
    ws = dsa.workspace(dsa.OP_FORWARD, batch, k_sel=2048, n_heads=128)
    dsa.forward(batch, q8, q_scale, w, k8, k_scale, 2048, q, kv, sm_scale, idx, out, lse, ws)
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdsa.so")

OP_INDEXER, OP_TOPK, OP_SPARSE_MLA, OP_FORWARD, OP_CACHE_WRITE, OP_INDEXER_TOPK = 0, 1, 2, 3, 4, 5
INDEX_HEADS, INDEX_DIM, LATENT_DIM, VALUE_DIM, MAX_K_SEL = 64, 128, 576, 512, 2048

STATUS = {
    0: "DSA_OK",
    1: "DSA_ERR_INVALID_ARG",
    2: "DSA_ERR_UNSUPPORTED",
    3: "DSA_ERR_CUDA",
    4: "DSA_ERR_WORKSPACE",
    5: "DSA_ERR_DEVICE_TIMEOUT",
    6: "DSA_ERR_DEVICE_BOUNDS",
}

# every entry point declared in include/dsa.h
EXPORTS = [
    "dsa_workspace_size",
    "dsa_indexer_scores",
    "dsa_topk",
    "dsa_indexer_topk",
    "dsa_topk_candidates",
    "dsa_topk_merge",
    "dsa_sparse_mla",
    "dsa_forward",
    "dsa_sparse_mla_no_alloc",
    "dsa_check_device_error",
    "dsa_status_string",
    "dsa_version",
    "dsa_forward_launches",
    "dsa_quantize_fp8",
    "dsa_indexer_prep",
    "dsa_cache_write",
]


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({_lib().dsa_status_string(status).decode()})")


class _BatchC(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int32),
        ("total_q", ctypes.c_int32),
        ("max_q_per_seq", ctypes.c_int32),
        ("max_kv_len", ctypes.c_int32),
        ("total_keys", ctypes.c_int64),
        ("cu_q", ctypes.c_void_p),
        ("kv_len", ctypes.c_void_p),
        ("kv_start", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("page_size", ctypes.c_int32),
        ("blocks_per_seq", ctypes.c_int32),
    ]


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m long_context_sparse_lightning_b200.build` "
                "(there is no fallback implementation)")
        lib = ctypes.CDLL(LIB_PATH)
        P, I32, I64, SZ, F = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
        BP = ctypes.POINTER(_BatchC)
        lib.dsa_workspace_size.argtypes = [ctypes.c_int, BP, I32, I32]
        lib.dsa_workspace_size.restype = SZ
        lib.dsa_indexer_scores.argtypes = [BP, P, P, P, P, P, P, I64, P, SZ, P]
        lib.dsa_indexer_scores.restype = ctypes.c_int
        lib.dsa_topk.argtypes = [BP, P, I64, I32, P, P, SZ, P]
        lib.dsa_topk.restype = ctypes.c_int
        lib.dsa_indexer_topk.argtypes = [BP, P, P, P, P, P, I32, P, P, SZ, P]
        lib.dsa_indexer_topk.restype = ctypes.c_int
        lib.dsa_topk_candidates.argtypes = [BP, P, I64, I32, P, P, P, P, SZ, P]
        lib.dsa_topk_candidates.restype = ctypes.c_int
        lib.dsa_topk_merge.argtypes = [I32, I32, I32, P, P, P, P]
        lib.dsa_topk_merge.restype = ctypes.c_int
        lib.dsa_sparse_mla.argtypes = [BP, P, I32, P, P, I32, F, P, P, P, SZ, P]
        lib.dsa_sparse_mla.restype = ctypes.c_int
        lib.dsa_forward.argtypes = [BP, P, P, P, P, P, I32, P, I32, P, F, P, P, P, P, SZ, P]
        lib.dsa_forward.restype = ctypes.c_int
        lib.dsa_sparse_mla_no_alloc.argtypes = [BP, P, I32, P, P, I32, F, P, P, P]
        lib.dsa_sparse_mla_no_alloc.restype = ctypes.c_int
        lib.dsa_check_device_error.argtypes = [P, P, ctypes.POINTER(ctypes.c_uint32), ctypes.POINTER(ctypes.c_uint32)]
        lib.dsa_check_device_error.restype = ctypes.c_int
        lib.dsa_status_string.argtypes = [ctypes.c_int]
        lib.dsa_status_string.restype = ctypes.c_char_p
        lib.dsa_version.argtypes = []
        lib.dsa_version.restype = I32
        lib.dsa_forward_launches.argtypes = [BP, I32, I32]
        lib.dsa_forward_launches.restype = I32
        lib.dsa_quantize_fp8.argtypes = [P, I64, P, P, P]
        lib.dsa_quantize_fp8.restype = ctypes.c_int
        lib.dsa_indexer_prep.argtypes = [P, I64, I32, P, P, P, I32, P, P, P, SZ, P]
        lib.dsa_indexer_prep.restype = ctypes.c_int
        lib.dsa_cache_write.argtypes = [BP, P, P, P, P, P, P, SZ, P]
        lib.dsa_cache_write.restype = ctypes.c_int
        _LIB = lib
    return _LIB


def library():
    """The loaded ctypes library (raises if it was not built)."""
    return _lib()


def _ptr(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise DSAError(status, where)


class Batch:
    """Ragged batch: device arrays cu_q [B+1] int32, kv_len [B] int32, kv_start [B] int64,
    plus the host-side sizes that shape the launch grids.

    Paged caches: pass ``block_table`` (int32 [B, blocks_per_seq] page ids) and
    ``page_size`` (a multiple of 64); ``kv_start`` may then be None and
    ``total_keys`` is the pool's row count."""

    def __init__(self, cu_q: torch.Tensor, kv_len: torch.Tensor, kv_start: Optional[torch.Tensor], total_q: int,
                 max_q_per_seq: int, max_kv_len: int, total_keys: int, block_table: Optional[torch.Tensor] = None,
                 page_size: int = 0):
        if cu_q.dtype != torch.int32 or kv_len.dtype != torch.int32 or \
                (kv_start is not None and kv_start.dtype != torch.int64):
            raise TypeError("cu_q/kv_len must be int32 and kv_start int64")
        if block_table is not None and (block_table.dtype != torch.int32 or block_table.dim() != 2
                                        or not block_table.is_contiguous()):
            raise TypeError("block_table must be a contiguous int32 [num_seqs, blocks_per_seq] tensor")
        self.cu_q, self.kv_len, self.kv_start, self.block_table = cu_q, kv_len, kv_start, block_table
        self.num_seqs = int(kv_len.shape[0])
        self.total_q = int(total_q)
        self.c = _BatchC()
        self.c.num_seqs = self.num_seqs
        self.c.total_q = self.total_q
        self.c.max_q_per_seq = int(max_q_per_seq)
        self.c.max_kv_len = int(max_kv_len)
        self.c.total_keys = int(total_keys)
        self.c.cu_q = cu_q.data_ptr()
        self.c.kv_len = kv_len.data_ptr()
        self.c.kv_start = kv_start.data_ptr() if kv_start is not None else None
        if block_table is not None:
            self.c.block_table = block_table.data_ptr()
            self.c.page_size = int(page_size)
            self.c.blocks_per_seq = int(block_table.shape[1])

    @staticmethod
    def from_host(cu_q, kv_len, kv_start, device="cuda", total_keys: Optional[int] = None):
        """Build from host sequences / numpy arrays; copies the arrays to `device`."""
        import numpy as np
        cu = np.asarray(cu_q, dtype=np.int32)
        kl = np.asarray(kv_len, dtype=np.int32)
        ks = np.asarray(kv_start, dtype=np.int64)
        q_len = np.diff(cu)
        if total_keys is None:
            total_keys = int((ks + kl).max()) if kl.size else 0
        return Batch(torch.from_numpy(cu).to(device), torch.from_numpy(kl).to(device),
                     torch.from_numpy(ks).to(device), int(cu[-1]), int(q_len.max()) if q_len.size else 0,
                     int(kl.max()) if kl.size else 0, int(total_keys))

    @property
    def ref(self):
        return ctypes.byref(self.c)


def workspace_size(op: int, batch: Batch, k_sel: int = MAX_K_SEL, n_heads: int = 128) -> int:
    return int(_lib().dsa_workspace_size(op, batch.ref, k_sel, n_heads))


def workspace(op: int, batch: Batch, k_sel: int = MAX_K_SEL, n_heads: int = 128, device="cuda") -> torch.Tensor:
    """A zeroed device workspace (the zero error word is part of the contract)."""
    n = workspace_size(op, batch, k_sel, n_heads)
    if n == 0:
        raise DSAError(1, "dsa_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def indexer_scores(batch: Batch, q_fp8, q_scale, w, k_fp8, k_scale, scores, ws, stream=None):
    _check(_lib().dsa_indexer_scores(batch.ref, _ptr(q_fp8), _ptr(q_scale), _ptr(w), _ptr(k_fp8), _ptr(k_scale),
                                     _ptr(scores), scores.shape[-1], _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_indexer_scores")


def topk(batch: Batch, scores, k_sel: int, idx, ws, stream=None):
    _check(_lib().dsa_topk(batch.ref, _ptr(scores), scores.shape[-1], k_sel, _ptr(idx), _ptr(ws), ws.numel(),
                           _stream(stream)), "dsa_topk")


def indexer_topk(batch: Batch, q_fp8, q_scale, w, k_fp8, k_scale, k_sel: int, idx, ws, stream=None):
    """Indexer scores and top-k in one call (fused on chip for decode batches)."""
    _check(_lib().dsa_indexer_topk(batch.ref, _ptr(q_fp8), _ptr(q_scale), _ptr(w), _ptr(k_fp8), _ptr(k_scale), k_sel,
                                   _ptr(idx), _ptr(ws), ws.numel(), _stream(stream)), "dsa_indexer_topk")


def topk_candidates(batch: Batch, scores, k_sel: int, cand_pos, cand_val, ws, pos_offset=None, stream=None):
    """One key shard's top k as global positions (+ pos_offset per sequence) and their scores."""
    _check(_lib().dsa_topk_candidates(batch.ref, _ptr(scores), scores.shape[-1], k_sel, _ptr(pos_offset),
                                      _ptr(cand_pos), _ptr(cand_val), _ptr(ws), ws.numel(), _stream(stream)),
           "dsa_topk_candidates")


def topk_merge(cand_pos, cand_val, k_sel: int, idx, stream=None):
    """Top k per row over [n_rows, n_src, k_sel] candidate lists (shards in position order)."""
    if cand_pos.dim() != 3 or cand_pos.shape != cand_val.shape or cand_pos.shape[2] != k_sel:
        raise ValueError("topk_merge: cand_pos / cand_val [n_rows, n_src, k_sel]")
    _check(_lib().dsa_topk_merge(int(cand_pos.shape[0]), int(cand_pos.shape[1]), k_sel, _ptr(cand_pos),
                                 _ptr(cand_val), _ptr(idx), _stream(stream)), "dsa_topk_merge")


def sparse_mla(batch: Batch, q, kv, idx, k_sel: int, sm_scale: float, out, lse, ws, stream=None):
    n_heads = int(q.shape[1])
    _check(_lib().dsa_sparse_mla(batch.ref, _ptr(q), n_heads, _ptr(kv), _ptr(idx), k_sel, float(sm_scale), _ptr(out),
                                 _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)), "dsa_sparse_mla")


def forward(batch: Batch, q_fp8, q_scale, w, k_fp8, k_scale, k_sel: int, q, kv, sm_scale: float, idx, out, lse, ws,
            stream=None):
    n_heads = int(q.shape[1])
    _check(_lib().dsa_forward(batch.ref, _ptr(q_fp8), _ptr(q_scale), _ptr(w), _ptr(k_fp8), _ptr(k_scale), k_sel,
                              _ptr(q), n_heads, _ptr(kv), float(sm_scale), _ptr(idx), _ptr(out), _ptr(lse), _ptr(ws),
                              ws.numel(), _stream(stream)), "dsa_forward")


def quantize_fp8(x, codes, scales, stream=None):
    """Per-128 FP8 e4m3 quantisation: x bf16 [..., 128] -> codes uint8 [..., 128], scales fp32 [...]."""
    if x.dtype != torch.bfloat16 or x.shape[-1] != INDEX_DIM or codes.dtype != torch.uint8 \
            or codes.numel() != x.numel() or scales.dtype != torch.float32 or scales.numel() * INDEX_DIM != x.numel():
        raise ValueError("quantize_fp8: x bf16 [..., 128], codes uint8 of the same size, scales fp32 [...]")
    n_vec = x.numel() // INDEX_DIM
    _check(_lib().dsa_quantize_fp8(_ptr(x), n_vec, _ptr(codes), _ptr(scales), _stream(stream)), "dsa_quantize_fp8")


def indexer_prep(x, pos, rope_cos, rope_sin, codes, scales, ws, vecs_per_pos: int, stream=None):
    """Non-interleaved RoPE on dims 0..63, normalised Walsh-Hadamard, per-128 FP8: x bf16 [..., 128]."""
    if x.dtype != torch.bfloat16 or x.shape[-1] != INDEX_DIM or codes.dtype != torch.uint8 \
            or codes.numel() != x.numel() or scales.dtype != torch.float32 or scales.numel() * INDEX_DIM != x.numel() \
            or pos.dtype != torch.int32 or rope_cos.dtype != torch.float32 or rope_sin.shape != rope_cos.shape \
            or rope_cos.shape[-1] != 32:
        raise ValueError("indexer_prep: x bf16 [..., 128], pos int32, rope tables fp32 [n_pos, 32]")
    n_vec = x.numel() // INDEX_DIM
    _check(_lib().dsa_indexer_prep(_ptr(x), n_vec, int(vecs_per_pos), _ptr(pos), _ptr(rope_cos), _ptr(rope_sin),
                                   int(rope_cos.shape[0]), _ptr(codes), _ptr(scales), _ptr(ws), ws.numel(),
                                   _stream(stream)), "dsa_indexer_prep")


def cache_write(batch: Batch, k, latent, k_cache, k_scale, latent_cache, ws, stream=None):
    """New tokens' keys (FP8 + scale) and latent rows into the flat caches at their positions."""
    _check(_lib().dsa_cache_write(batch.ref, _ptr(k), _ptr(latent), _ptr(k_cache), _ptr(k_scale), _ptr(latent_cache),
                                  _ptr(ws), ws.numel(), _stream(stream)), "dsa_cache_write")


def check_device_error(ws, stream=None):
    """Synchronise, read and clear the workspace's device error word; raise if set."""
    site = ctypes.c_uint32(0)
    info = ctypes.c_uint32(0)
    st = _lib().dsa_check_device_error(_ptr(ws), _stream(stream), ctypes.byref(site), ctypes.byref(info))
    if st != 0:
        err = DSAError(st, f"device error (site {site.value}, info {info.value})")
        err.site, err.info = site.value, info.value
        raise err


def forward_launches(batch: Batch, k_sel: int, n_heads: int) -> int:
    """Kernel launches one dsa_forward call makes for this batch (host only)."""
    return int(_lib().dsa_forward_launches(batch.ref, k_sel, n_heads))


def version() -> int:
    return int(_lib().dsa_version())
