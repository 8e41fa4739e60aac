"""The device error path, exercised without faulting or hanging the GPU.

A test-only host flag (DSA_TEST_SKIP_ARRIVAL) makes CTA (0,0,0) of the
(non-clustered) indexer kernel withhold one plain thread arrival -- its
epilogue's release of an accumulator buffer, a barrier that no TMA, bulk copy
or tensor-core operation completes.  With a short wait budget
(DSA_WAIT_BUDGET_CYCLES) the MMA warp's bounded wait for that buffer runs out,
the roles that depend on it time out in turn, every load and MMA already
issued is waited for before the CTA leaves, and the host reads
DSA_ERR_DEVICE_TIMEOUT from the workspace.  The next call, without the flag,
must succeed and give the normal scores.
"""

import numpy as np
import pytest
import torch

import long_context_sparse_lightning_b200 as dsa
from dsa_inputs import make_inputs
from tests.parity import GpuRun

pytestmark = pytest.mark.gpu


def test_withheld_arrival_times_out_and_the_next_call_succeeds(monkeypatch):
    x = make_inputs("tiny_prefill_512")
    g = GpuRun(x)
    ref = g.scores().cpu().numpy()
    monkeypatch.setenv("DSA_WAIT_BUDGET_CYCLES", "20000000")     # ~10 ms per bounded wait
    monkeypatch.setenv("DSA_TEST_SKIP_ARRIVAL", "0")
    s = torch.full((x.batch.total_q, g.ld), float("nan"), dtype=torch.float32, device="cuda")
    ws = dsa.workspace(dsa.OP_INDEXER, g.batch)
    dsa.indexer_scores(g.batch, g.t["q8"], g.t["q_scale"], g.t["w"], g.t["k8"], g.t["k_scale"], s, ws)
    with pytest.raises(dsa.DSAError) as e:
        dsa.check_device_error(ws)
    assert e.value.status == 5                                   # DSA_ERR_DEVICE_TIMEOUT
    assert e.value.site in (110, 111, 122, 123, 130)             # indexer wait sites
    # the error word was read and cleared; the context is still usable
    dsa.check_device_error(ws)
    monkeypatch.delenv("DSA_TEST_SKIP_ARRIVAL")
    monkeypatch.delenv("DSA_WAIT_BUDGET_CYCLES")
    again = g.scores().cpu().numpy()
    for r in range(x.batch.total_q):
        t = int(x.batch.q_pos[r])
        assert np.array_equal(again[r, : t + 1], ref[r, : t + 1])
