"""The key-sharded selection's host flow on CPU: two gloo ranks each hold a
contiguous shard of every sequence's keys, select their local top k (here the
fp64 oracle stands in for the kernels, which need a GPU), all-gather the
candidates through the package's plumbing and merge them.  The result must be
the oracle's top k over the whole row."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_sparse_lightning_b200 import sharded


def test_shard_bounds_cover_every_position_once():
    kv = [7, 1, 0, 100, 33]
    for world in (1, 2, 3, 4):
        for b, n in enumerate(kv):
            got = []
            for r in range(world):
                s, l = sharded.shard_bounds(kv, world, r)
                got.extend(range(s[b], s[b] + l[b]))
            assert got == list(range(n))


def _oracle_local(scores_row, lo, n, k):
    """Top k of positions [lo, lo + n) of a score row: global positions ascending + scores."""
    part = scores_row[lo:lo + n]
    order = np.lexsort((np.arange(n), -part))[:k]
    sel = np.sort(order)
    pos = np.full(k, -1, np.int32)
    val = np.full(k, np.nan, np.float32)
    pos[: sel.size] = lo + sel
    val[: sel.size] = part[sel]
    return pos, val


def _oracle_merge(pos, val, k, idx):
    """Reference merge: top k of the valid candidates by (score desc, position asc)."""
    p, v = pos.numpy(), val.numpy()
    out = np.full((p.shape[0], k), -1, np.int32)
    for r in range(p.shape[0]):
        pp, vv = p[r].reshape(-1), v[r].reshape(-1)
        ok = pp >= 0
        pp, vv = pp[ok], vv[ok]
        order = np.lexsort((pp, -vv.astype(np.float64)))[:k]
        sel = np.sort(pp[order])
        out[r, : sel.size] = sel
    idx.copy_(torch.from_numpy(out))


def _rank(rank, world, port, rows, k, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        kv = [len(r) for r in rows]
        starts, lens = sharded.shard_bounds(kv, world, rank)
        pos = np.zeros((len(rows), k), np.int32)
        val = np.zeros((len(rows), k), np.float32)
        for b, row in enumerate(rows):
            pos[b], val[b] = _oracle_local(row, starts[b], lens[b], k)
        idx = sharded.key_sharded_topk(torch.from_numpy(pos), torch.from_numpy(val), k, merge=_oracle_merge)
        for b, row in enumerate(rows):
            full = np.sort(np.lexsort((np.arange(len(row)), -row))[:k])
            expect = np.full(k, -1, np.int32)
            expect[: full.size] = full
            assert np.array_equal(idx[b].numpy(), expect), (rank, b)
        q.put(("ok", rank))
    except Exception as e:  # reported to the parent
        q.put(("fail", f"{rank}: {type(e).__name__}: {e}"))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_gloo_ranks_merge_to_the_global_top_k():
    g = np.random.default_rng(3)
    # rows with ties across the shard boundary, a short row, and k > a shard
    rows = [g.standard_normal(300).astype(np.float32),
            np.round(g.standard_normal(257) * 4).astype(np.float32),
            g.standard_normal(40).astype(np.float32),
            g.standard_normal(90).astype(np.float32)]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, rows, 64, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
    assert all(r[0] == "ok" for r in res), res
