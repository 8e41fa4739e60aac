"""Paged cache layouts for tests and benchmarks: the same logical caches moved
into pools of fixed-size pages in a seeded random order (data movement only).

Position s of sequence b lands in pool row
``block_table[b, s // page_size] * page_size + s % page_size``.  Pool rows no
sequence owns (spare pages, the tail of each sequence's last page) hold random
bytes, so a kernel that reads through a wrong mapping sees garbage.
"""

from __future__ import annotations

import dataclasses

import numpy as np


@dataclasses.dataclass
class PagedCaches:
    page_size: int
    block_table: np.ndarray     # int32 [B, blocks_per_seq], -1 past a sequence's pages
    num_pages: int
    k8: np.ndarray              # uint8  [num_pages * page_size, 128]
    k_scale: np.ndarray         # f32    [num_pages * page_size]
    latent: np.ndarray          # uint16 [num_pages * page_size, 576] bf16 bits

    @property
    def total_keys(self) -> int:
        return self.num_pages * self.page_size


def paged_layout(x, page_size: int, seed: int = 0, spare_pages: int = 3) -> PagedCaches:
    """Move the flat caches of DSAInputs ``x`` into a page pool."""
    b = x.batch
    kv = b.kv_len.astype(np.int64)
    n_pages_seq = (kv + page_size - 1) // page_size
    num_pages = int(n_pages_seq.sum()) + spare_pages
    g = np.random.Generator(np.random.PCG64(np.random.SeedSequence(seed)))
    order = g.permutation(num_pages).astype(np.int32)
    blocks = int(max(1, n_pages_seq.max()))
    table = np.full((b.num_seqs, blocks), -1, np.int32)
    rows = num_pages * page_size
    k8 = g.integers(0, 256, size=(rows, x.k8.shape[1]), dtype=np.uint8)
    ks = g.uniform(0.5, 2.0, size=rows).astype(np.float32)
    lat = g.integers(0, 1 << 16, size=(rows, x.latent.shape[1]), dtype=np.uint16)
    nxt = 0
    for s_ in range(b.num_seqs):
        k0 = int(b.kv_start[s_])
        for i in range(int(n_pages_seq[s_])):
            pg = int(order[nxt])
            nxt += 1
            table[s_, i] = pg
            lo = i * page_size
            n = min(page_size, int(kv[s_]) - lo)
            dst = pg * page_size
            k8[dst:dst + n] = x.k8[k0 + lo:k0 + lo + n]
            ks[dst:dst + n] = x.k_scale[k0 + lo:k0 + lo + n]
            lat[dst:dst + n] = x.latent[k0 + lo:k0 + lo + n]
    return PagedCaches(page_size, table, num_pages, k8, ks, lat)
