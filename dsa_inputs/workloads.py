"""Workload definitions and the seeded generator for the DSA hot path.

Every tensor is drawn from its own child of ``numpy.random.SeedSequence(seed)``
(PCG64), in fixed-size chunks that each get their own grandchild seed, so the
bytes do not depend on how many threads draw them.

Storage formats (what the CUDA path and the oracle both consume):

* bf16 tensors are ``uint16`` arrays holding bf16 bit patterns, made from
  float32 draws by round-to-nearest-even.
* FP8 tensors are ``uint8`` arrays of e4m3 codes (1 sign, 4 exponent bits with
  bias 7, 3 mantissa bits, no infinities, 0x7F/0xFF = NaN, max 448), one fp32
  scale per 128-element vector.  The quantisation follows the activation
  quantiser the indexer code on the "详解DSA" page applies to q and k before
  the FP8 index kernel (block size 128 = the indexer head dim, so one scale per
  head vector of q and one per key row of k): ``scale = fp32(amax / 448)``,
  ``code = e4m3_rne_saturating(fp32(x / scale))``.

The five workloads follow the pages' own settings (64 indexer heads of dim 128,
top-k 2048, 128 MLA heads over a 576-d latent = 512 value + 64 RoPE dims) at
the sizes named below; all inputs are N(0,1) draws (w ~ N(0, 1/64)).
"""

from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Optional

import numpy as np

INDEX_HEADS = 64      # H_I: indexer heads ("DeepSeek V3.2 稀疏注意力", data-flow section; luowle "NSA 与 DSA" §3.2)
INDEX_DIM = 128       # d_I: indexer head dim, also the FP8 scale block
LATENT_DIM = 576      # MLA latent entry: 512 latent + 64 RoPE dims
VALUE_DIM = 512       # value = first 512 dims of the latent entry
FP8_MAX = 448.0       # largest finite e4m3 magnitude

_CHUNK = 1 << 22      # elements per independently seeded chunk


@dataclasses.dataclass(frozen=True)
class Workload:
    """A synthetic DSA workload.

    Each sequence b holds ``kv_len[b]`` cached keys; its ``q_len`` query rows
    are the last ``q_len`` positions, so query i sits at
    ``t = kv_len[b] - q_len + i`` and may attend to positions ``0..t``.
    """

    name: str
    description: str
    num_seqs: int
    q_len: int
    k_sel: int
    n_heads: int
    kv_len: Optional[int] = None                       # fixed context per sequence
    kv_len_range: Optional[tuple[int, int]] = None     # inclusive uniform range per sequence
    heavy_frac: float = 0.0                            # fraction of indexer key rows scaled x4 (in bf16, before FP8)

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(192.0)


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload(
            name="tiny_prefill_512",
            description="1 sequence, 512 causal queries over 512 keys, top-64, 16 MLA heads",
            num_seqs=1, q_len=512, kv_len=512, k_sel=64, n_heads=16,
        ),
        Workload(
            name="decode_64x16k_32k",
            description="64 sequences x 1 query token, context U{16384..32768}, top-2048, 128 MLA heads",
            num_seqs=64, q_len=1, kv_len_range=(16384, 32768), k_sel=2048, n_heads=128,
        ),
        Workload(
            name="prefill_8k",
            description="1 sequence, 8192 causal queries over 8192 keys, top-2048, 128 MLA heads",
            num_seqs=1, q_len=8192, kv_len=8192, k_sel=2048, n_heads=128,
        ),
        Workload(
            name="chunked_prefill_28k_4k",
            description="1 sequence, 4096 new queries after a 28672-token prefix (32768 keys), "
                        "5% of indexer key rows x4, top-2048, 128 MLA heads",
            num_seqs=1, q_len=4096, kv_len=32768, k_sel=2048, n_heads=128, heavy_frac=0.05,
        ),
        Workload(
            name="spec_decode_8x2_128k",
            description="8 sequences x 2 query tokens at 131072 context, top-2048, 128 MLA heads",
            num_seqs=8, q_len=2, kv_len=131072, k_sel=2048, n_heads=128,
        ),
        # smaller shapes of the same kinds, for profiling captures
        Workload(
            name="chunked_prefill_32k_512",
            description="1 sequence, 512 new queries ending at position 32767 (32768 keys), top-2048, 128 MLA heads",
            num_seqs=1, q_len=512, kv_len=32768, k_sel=2048, n_heads=128, heavy_frac=0.05,
        ),
        Workload(
            name="decode_16x32k",
            description="16 sequences x 1 query token at 32768 context, top-2048, 128 MLA heads",
            num_seqs=16, q_len=1, kv_len=32768, k_sel=2048, n_heads=128,
        ),
    ]
}


def custom_workload(name: str, kv_lens, q_lens, k_sel: int, n_heads: int,
                    heavy_frac: float = 0.0) -> "Workload":
    """A ragged workload with explicit per-sequence context and query counts.

    ``q_lens`` may differ per sequence; it is stored in ``kv_len_range`` form
    only for the record, the explicit lists travel through ``make_inputs``.
    """
    w = Workload(name=name, description="custom", num_seqs=len(kv_lens), q_len=-1,
                 k_sel=k_sel, n_heads=n_heads, heavy_frac=heavy_frac)
    object.__setattr__(w, "_kv_lens", tuple(int(x) for x in kv_lens))
    object.__setattr__(w, "_q_lens", tuple(int(x) for x in q_lens))
    return w


@dataclasses.dataclass
class Batch:
    """Ragged batch layout shared by every stage.

    ``cu_q`` are query-row offsets, ``kv_start`` the first row of each
    sequence in the flat key / latent caches, ``q_pos`` the absolute position t
    of every query row inside its own sequence.
    """

    kv_len: np.ndarray      # int32 [B]
    q_len: np.ndarray       # int32 [B]
    cu_q: np.ndarray        # int32 [B+1]
    kv_start: np.ndarray    # int64 [B]
    q_seq: np.ndarray       # int32 [n_q]
    q_pos: np.ndarray       # int64 [n_q]

    @property
    def num_seqs(self) -> int:
        return int(self.kv_len.shape[0])

    @property
    def total_q(self) -> int:
        return int(self.cu_q[-1])

    @property
    def total_keys(self) -> int:
        return int(self.kv_len.astype(np.int64).sum())

    @property
    def max_q_per_seq(self) -> int:
        return int(self.q_len.max()) if self.num_seqs else 0

    @property
    def max_kv_len(self) -> int:
        return int(self.kv_len.max()) if self.num_seqs else 0

    @staticmethod
    def from_lengths(kv_lens, q_lens) -> "Batch":
        kv = np.asarray(kv_lens, dtype=np.int32)
        ql = np.asarray(q_lens, dtype=np.int32)
        if kv.shape != ql.shape or np.any(ql > kv) or np.any(ql < 0) or np.any(kv < 0):
            raise ValueError("need 0 <= q_len <= kv_len per sequence")
        cu_q = np.zeros(kv.shape[0] + 1, dtype=np.int32)
        cu_q[1:] = np.cumsum(ql, dtype=np.int64)
        kv_start = np.zeros(kv.shape[0], dtype=np.int64)
        if kv.shape[0] > 1:
            kv_start[1:] = np.cumsum(kv.astype(np.int64))[:-1]
        q_seq = np.repeat(np.arange(kv.shape[0], dtype=np.int32), ql)
        q_pos = np.concatenate(
            [np.arange(int(k) - int(q), int(k), dtype=np.int64) for k, q in zip(kv, ql)]
        ) if kv.shape[0] else np.zeros(0, np.int64)
        return Batch(kv, ql, cu_q, kv_start, q_seq, q_pos)


@dataclasses.dataclass
class DSAInputs:
    workload: Workload
    seed: int
    batch: Batch
    k_sel: int
    n_heads: int
    sm_scale: float
    q8: np.ndarray          # uint8  [n_q, 64, 128] e4m3 codes
    q_scale: np.ndarray     # f32    [n_q, 64]
    w: np.ndarray           # f32    [n_q, 64]
    k8: np.ndarray          # uint8  [n_keys, 128] e4m3 codes
    k_scale: np.ndarray     # f32    [n_keys]
    q_mla: np.ndarray       # uint16 [n_q, H, 576] bf16 bits
    latent: np.ndarray      # uint16 [n_keys, 576] bf16 bits
    q_idx_bf16: Optional[np.ndarray] = None   # uint16 [n_q, 64, 128] before FP8 (kept on request)
    k_idx_bf16: Optional[np.ndarray] = None   # uint16 [n_keys, 128] before FP8 (kept on request)
    heavy_rows: Optional[np.ndarray] = None   # int64 key rows scaled x4


# ----------------------------------------------------------------------------
# bit-level helpers (storage encodings only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _e4m3_positive_grid() -> np.ndarray:
    """The 127 finite non-negative e4m3 values, indexed by their code 0..126."""
    vals = np.empty(127, dtype=np.float64)
    for code in range(127):
        e, m = code >> 3, code & 7
        vals[code] = m * 2.0 ** -9 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


_E4M3_GRID = _e4m3_positive_grid()


def e4m3_encode(y: np.ndarray) -> np.ndarray:
    """float32 -> e4m3 code: round to nearest, ties to the even code, saturate at 448."""
    y = np.asarray(y, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    flat_in, flat_out = y.reshape(-1), out.reshape(-1)
    grid = _E4M3_GRID
    for s in range(0, flat_in.size, _CHUNK):
        v = flat_in[s:s + _CHUNK]
        a = np.abs(v.astype(np.float64))
        i = np.searchsorted(grid, a, side="right") - 1          # grid[i] <= a
        i = np.minimum(i, 126)
        top = i >= 126                                         # >= 448: saturate
        j = np.minimum(i + 1, 126)
        d_lo = a - grid[i]
        d_hi = grid[j] - a
        up = (d_hi < d_lo) | ((d_hi == d_lo) & (j % 2 == 0))
        code = np.where(top, 126, np.where(up, j, i)).astype(np.uint8)
        sign = np.signbit(v).astype(np.uint8) << np.uint8(7)
        flat_out[s:s + _CHUNK] = code | sign
    return out


def quantize_fp8_blocks(x_bf16: np.ndarray, block: int = INDEX_DIM):
    """Per-``block`` e4m3 quantisation of bf16 data along the last axis.

    Returns (codes uint8 same shape, scales float32 shape[:-1] + (n_blocks,)
    squeezed when there is exactly one block per row).
    """
    x = bf16_bits_to_f32(x_bf16)
    shp = x.shape
    assert shp[-1] % block == 0
    xb = x.reshape(shp[:-1] + (shp[-1] // block, block))
    amax = np.max(np.abs(xb), axis=-1)                        # float32, exact
    scale = np.where(amax == 0, np.float32(1.0), amax / np.float32(FP8_MAX)).astype(np.float32)
    y = (xb / scale[..., None]).astype(np.float32)
    codes = e4m3_encode(y).reshape(shp)
    if scale.shape[-1] == 1:
        scale = scale[..., 0]
    return codes, scale


# ----------------------------------------------------------------------------
# seeded draws
# ----------------------------------------------------------------------------

def _threads() -> int:
    return max(1, min(16, os.cpu_count() or 1))


def _normal_chunks(ss: np.random.SeedSequence, n: int, convert):
    nchunks = max(1, -(-n // _CHUNK))
    kids = ss.spawn(nchunks)

    def one(i):
        m = min(_CHUNK, n - i * _CHUNK)
        g = np.random.Generator(np.random.PCG64(kids[i]))
        return i, convert(g.standard_normal(m, dtype=np.float32))

    return nchunks, one


def normal_bf16(ss: np.random.SeedSequence, n: int, scale: float = 1.0) -> np.ndarray:
    """n draws of N(0, scale^2) as bf16 bits (scale must be a power of two)."""
    out = np.empty(n, dtype=np.uint16)
    conv = (lambda a: f32_to_bf16_bits(a * np.float32(scale))) if scale != 1.0 else f32_to_bf16_bits
    nchunks, one = _normal_chunks(ss, n, conv)
    with ThreadPoolExecutor(_threads()) as ex:
        for i, part in ex.map(one, range(nchunks)):
            out[i * _CHUNK:i * _CHUNK + part.size] = part
    return out


def normal_f32(ss: np.random.SeedSequence, n: int, scale: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    conv = (lambda a: a * np.float32(scale)) if scale != 1.0 else (lambda a: a)
    nchunks, one = _normal_chunks(ss, n, conv)
    with ThreadPoolExecutor(_threads()) as ex:
        for i, part in ex.map(one, range(nchunks)):
            out[i * _CHUNK:i * _CHUNK + part.size] = part
    return out


def _quantize_threaded(x_bf16: np.ndarray):
    rows = x_bf16.reshape(-1, INDEX_DIM)
    codes = np.empty(rows.shape, dtype=np.uint8)
    scales = np.empty(rows.shape[0], dtype=np.float32)
    step = max(1, _CHUNK // INDEX_DIM)

    def one(s):
        c, sc = quantize_fp8_blocks(rows[s:s + step])
        codes[s:s + step] = c
        scales[s:s + step] = sc

    with ThreadPoolExecutor(_threads()) as ex:
        list(ex.map(one, range(0, rows.shape[0], step)))
    return codes.reshape(x_bf16.shape), scales.reshape(x_bf16.shape[:-1])


def make_batch(workload: Workload, seed: int = 0) -> Batch:
    ss = np.random.SeedSequence(seed).spawn(8)
    if hasattr(workload, "_kv_lens"):
        return Batch.from_lengths(workload._kv_lens, workload._q_lens)
    if workload.kv_len is not None:
        kv = [workload.kv_len] * workload.num_seqs
    else:
        lo, hi = workload.kv_len_range
        g = np.random.Generator(np.random.PCG64(ss[0]))
        kv = g.integers(lo, hi, size=workload.num_seqs, endpoint=True).tolist()
    return Batch.from_lengths(kv, [workload.q_len] * workload.num_seqs)


def make_inputs(workload: Workload | str, seed: int = 0, keep_raw: bool = False) -> DSAInputs:
    """Draw every input of the hot path for ``workload`` with ``seed``."""
    if isinstance(workload, str):
        workload = WORKLOADS[workload]
    ss = np.random.SeedSequence(seed).spawn(8)
    batch = make_batch(workload, seed)
    n_q, n_k, H = batch.total_q, batch.total_keys, workload.n_heads

    q_idx = normal_bf16(ss[1], n_q * INDEX_HEADS * INDEX_DIM).reshape(n_q, INDEX_HEADS, INDEX_DIM)
    k_idx = normal_bf16(ss[2], n_k * INDEX_DIM).reshape(n_k, INDEX_DIM)
    heavy = None
    if workload.heavy_frac > 0 and n_k > 0:
        n_heavy = int(round(workload.heavy_frac * n_k))
        g = np.random.Generator(np.random.PCG64(ss[6]))
        heavy = np.sort(g.permutation(n_k)[:n_heavy]).astype(np.int64)
        k_idx[heavy] = f32_to_bf16_bits(bf16_bits_to_f32(k_idx[heavy]) * np.float32(4.0))
    w = normal_f32(ss[3], n_q * INDEX_HEADS, scale=0.125).reshape(n_q, INDEX_HEADS)
    q_mla = normal_bf16(ss[4], n_q * H * LATENT_DIM).reshape(n_q, H, LATENT_DIM)
    latent = normal_bf16(ss[5], n_k * LATENT_DIM).reshape(n_k, LATENT_DIM)

    q8, q_scale = _quantize_threaded(q_idx)
    k8, k_scale = _quantize_threaded(k_idx)
    return DSAInputs(
        workload=workload, seed=seed, batch=batch, k_sel=workload.k_sel, n_heads=H,
        sm_scale=workload.sm_scale, q8=q8, q_scale=q_scale, w=w, k8=k8, k_scale=k_scale,
        q_mla=q_mla, latent=latent,
        q_idx_bf16=q_idx if keep_raw else None, k_idx_bf16=k_idx if keep_raw else None,
        heavy_rows=heavy,
    )
