"""Key-sharded top-k across ranks: local candidates, all-gather, merge.

"DeepSeek V3.2 稀疏注意力" (top-k section) raises selecting a local top k per
shard and merging the shards' candidates when the keys are split across
devices.  Here the keys of every sequence are split into contiguous position
ranges, one per rank (``shard_bounds``); rank r scores its range and selects
its local top k as global positions with their scores (dsa_topk_candidates);
the candidate lists are all-gathered in rank order (so positions ascend across
the lists) and every rank merges them into the row's global top k
(dsa_topk_merge).  Each of a row's top k lies in the top k of its own shard,
so the merge equals a selection over the whole row.  The exchange is one
all-gather of 8 * k_sel bytes per query row and rank.

Host plumbing only: the selection and the merge run in the library's kernels.
"""

from __future__ import annotations

from typing import Callable, Optional

import torch

from . import topk_merge


def shard_bounds(kv_len, world: int, rank: int):
    """Contiguous split of each sequence's positions over `world` ranks: the
    (first position, length) lists of rank `rank` (ranks in position order;
    the first kv_len % world ranks get one position more)."""
    starts, lens = [], []
    for n in (int(v) for v in kv_len):
        base, extra = divmod(n, world)
        lo = rank * base + min(rank, extra)
        starts.append(lo)
        lens.append(base + (1 if rank < extra else 0))
    return starts, lens


def gather_candidates(cand_pos: torch.Tensor, cand_val: torch.Tensor, group=None):
    """All-gather each rank's [rows, k] candidates into [rows, world, k] (rank order)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    pos = [torch.empty_like(cand_pos) for _ in range(world)]
    val = [torch.empty_like(cand_val) for _ in range(world)]
    dist.all_gather(pos, cand_pos.contiguous(), group=group)
    dist.all_gather(val, cand_val.contiguous(), group=group)
    return torch.stack(pos, dim=1).contiguous(), torch.stack(val, dim=1).contiguous()


def key_sharded_topk(cand_pos: torch.Tensor, cand_val: torch.Tensor, k_sel: int, group=None,
                     merge: Optional[Callable] = None) -> torch.Tensor:
    """The global top k of every query row from this rank's local candidates
    (dsa_topk_candidates output); every rank gets the same [rows, k_sel] result.
    `merge(pos [rows, R, k], val [rows, R, k], k_sel, idx)` defaults to the
    library's dsa_topk_merge."""
    pos_all, val_all = gather_candidates(cand_pos, cand_val, group)
    idx = torch.empty((cand_pos.shape[0], k_sel), dtype=torch.int32, device=cand_pos.device)
    (merge or topk_merge)(pos_all, val_all, k_sel, idx)
    return idx
