"""bench.py's host arithmetic without a GPU: the per-stage roofline entries and
the prep line (bytes per unit x units / measured time against the HBM peak)."""

import pytest

import bench

PK = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1400.0, "source": "test"}


def test_prep_bytes_per_unit():
    w = bench.prep_work(10)
    assert w["quantize_q"]["bytes"] == 10 * 64 * (256 + 128 + 4)      # 64 head vectors per query row
    assert w["cache_write"]["bytes"] == 10 * (256 + 132 + 2 * 1152)   # key in, codes + scale out, latent in + out


def test_prep_line_is_an_hbm_roofline():
    line = bench.prep_line({"quantize_q": 1e-5, "cache_write": 2e-6}, 4096, PK)
    q = line["quantize_q"]
    assert q["bound"] == "hbm" and q["unit"] == "GB/s" and q["peak"] == PK["hbm_gbs"]
    assert q["achieved"] == pytest.approx(4096 * 64 * 388 / 1e-5 / 1e9)
    assert q["frac"] == pytest.approx(q["achieved"] / PK["hbm_gbs"])
    assert q["ideal_us"] == pytest.approx(4096 * 64 * 388 / (PK["hbm_gbs"] * 1e9) * 1e6)
    assert line["cache_write"]["us"] == pytest.approx(2.0)


def test_prep_line_passes_errors_through():
    assert bench.prep_line(None, 4, PK) is None
    err = {"error": "DSAError: x"}
    assert bench.prep_line(err, 4, PK) is err


def test_tensor_bound_stage_uses_the_sustained_peak():
    e = bench.roofline_entry("sparse_mla", {"flops": 2.0e12, "bytes": 1.0e6, "peak": "bf16"}, 2.0e-3, PK)
    assert e["bound"] == "tensor" and e["peak"] == 1400.0
    assert e["achieved"] == pytest.approx(1000.0)
    f = bench.roofline_entry("indexer", {"flops": 2.0e12, "bytes": 1.0e6, "peak": "fp8"}, 1.0e-3, PK)
    assert f["peak"] == 2800.0 and f["frac"] == pytest.approx(2000.0 / 2800.0)
