"""Pins of the oracle's paged-cache map (oracle/paged.py)."""

import numpy as np
import pytest

from dsa_inputs import custom_workload, make_inputs
from dsa_inputs.paged import paged_layout
from oracle import paged


def test_hand_worked_rows():
    # page size 64; sequence 0 owns pages 3 then 0, sequence 1 owns page 1
    table = [[3, 0], [1, -1]]
    assert paged.pool_row(table, 64, 0, 0) == 192
    assert paged.pool_row(table, 64, 0, 63) == 255
    assert paged.pool_row(table, 64, 0, 64) == 0
    assert paged.pool_row(table, 64, 0, 70) == 6
    assert paged.pool_row(table, 64, 1, 5) == 69
    with pytest.raises(IndexError):
        paged.pool_row(table, 64, 1, 64)


def test_identity_table_is_the_flat_cache():
    pool = np.arange(6 * 128 * 3).reshape(6 * 128, 3)
    table = np.array([[0, 1, 2], [3, 4, 5]])
    for b in range(2):
        got = paged.logical_view(pool, table, 128, b, 300)
        assert np.array_equal(got, pool[b * 384:b * 384 + 300])


def test_generator_layout_round_trips_through_the_oracle_map():
    # the input generator scatters pages in a seeded random order; the oracle's
    # own map must bring every sequence back unchanged
    x = make_inputs(custom_workload("pg", [200, 64, 129, 1], [1, 1, 2, 1], k_sel=16, n_heads=16), seed=2)
    for page in (64, 128):
        pc = paged_layout(x, page, seed=5)
        assert pc.num_pages * page == pc.k8.shape[0]
        for b in range(x.batch.num_seqs):
            k0, kv = int(x.batch.kv_start[b]), int(x.batch.kv_len[b])
            assert np.array_equal(paged.logical_view(pc.k8, pc.block_table, page, b, kv), x.k8[k0:k0 + kv])
            assert np.array_equal(paged.logical_view(pc.k_scale, pc.block_table, page, b, kv),
                                  x.k_scale[k0:k0 + kv])
            assert np.array_equal(paged.logical_view(pc.latent, pc.block_table, page, b, kv),
                                  x.latent[k0:k0 + kv])
        # the pages really are scattered: the table is not the sequential assignment
        used = pc.block_table[pc.block_table >= 0]
        assert not np.array_equal(np.sort(used), used)
