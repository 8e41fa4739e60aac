"""The multi-GPU path of bench.py on CPU: two ranks over gloo.

Every rank runs its own replica of the workload (no data-path collective); the
only collectives are the barrier and the max-over-ranks reduction of the elapsed
times, from which rank 0 reports the whole-job rate.  These tests run that
aggregation in two gloo processes, and check that the reference arm does no
work on ranks other than 0.
"""

import os
import socket

import pytest
import torch
import torch.distributed as td
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, times, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    td.init_process_group("gloo", rank=rank, world_size=world)
    try:
        td.barrier()
        slow = bench.slowest_rank(times[rank], td, "cpu")
        rate = bench.whole_job_rate(world, 4096, 5, slow)
        out.put((rank, slow, rate))
        td.barrier()
    finally:
        td.destroy_process_group()


def test_two_ranks_report_the_slowest_rank_and_the_whole_job_rate():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    times = [0.021, 0.025]
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, times, out)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(out.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slow, rate in res:
        assert slow == pytest.approx(0.025)                  # every rank sees the max
        assert rate == pytest.approx(2 * 4096 * 5 / 0.025)   # all ranks' tokens / the slowest time


def test_single_process_keeps_its_own_time():
    assert bench.slowest_rank(0.5, None, "cpu") == 0.5
    assert bench.whole_job_rate(1, 10, 2, 0.5) == pytest.approx(40.0)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    class A:
        workload, steps, warmup, ref_rows = "tiny_prefill_512", 1, 1, 1
    assert bench.run_reference(A(), 2, 1) == 0
    assert capsys.readouterr().out == ""
