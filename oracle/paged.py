"""Logical view of a paged cache (oracle side; test infrastructure only).

"DeepSeek V3.2 稀疏注意力" (decode and top-k sections) names the map from a
logical top-k position to a physical KV page and offset as something a paged
kernel must define.  The reading taken here: position s of sequence b lives at
page ``block_table[b][s // page_size]``, offset ``s % page_size``, i.e. pool
row page * page_size + offset.  These functions restate that map on their own
(no code shared with the input generator or the CUDA path) so that a paged run
can be checked against the oracle on the logical, flat sequence.
"""

from __future__ import annotations

import numpy as np


def pool_row(block_table, page_size: int, b: int, s: int) -> int:
    """Pool row of position s of sequence b."""
    page = int(block_table[b][s // page_size])
    if page < 0:
        raise IndexError(f"sequence {b} has no page for position {s}")
    return page * page_size + (s % page_size)


def logical_view(pool: np.ndarray, block_table, page_size: int, b: int, kv_len: int) -> np.ndarray:
    """Rows 0 .. kv_len-1 of sequence b, gathered from the pool in position order."""
    rows = [pool_row(block_table, page_size, b, s) for s in range(kv_len)]
    return pool[np.asarray(rows, dtype=np.int64)] if rows else pool[:0]
