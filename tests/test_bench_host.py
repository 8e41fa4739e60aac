"""bench.py's host arithmetic without a GPU: the per-stage roofline entries and
the prep line (bytes per unit x units / measured time against the HBM peak)."""

import pytest

import bench

PK = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "fp8_tflops": 2900.0, "source": "test"}


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


def test_tensor_bound_stage_uses_the_burst_peak_of_its_type():
    # stages are timed on their own, so the burst GEMM rate is the denominator;
    # the FP8 indexer is measured against the FP8 peak, the MLA against bf16
    e = bench.roofline_entry("sparse_mla", {"flops": 2.0e12, "bytes": 1.0e6, "peak": "bf16"}, 2.0e-3, PK)
    assert e["bound"] == "tensor" and e["peak"] == 1500.0
    assert e["achieved"] == pytest.approx(1000.0)
    assert e["frac"] == pytest.approx(1000.0 / 1500.0)
    f = bench.roofline_entry("indexer", {"flops": 2.0e12, "bytes": 1.0e6, "peak": "fp8"}, 1.0e-3, PK)
    assert f["peak"] == 2900.0 and f["frac"] == pytest.approx(2000.0 / 2900.0)


def test_bandwidth_bound_stage_takes_the_slower_roof():
    # 1 GFLOP of FP8 work and 60 MB: 0.34 us of tensor time, 10 us of HBM time
    e = bench.roofline_entry("indexer", {"flops": 1.0e9, "bytes": 6.0e7, "peak": "fp8"}, 2.0e-5, PK)
    assert e["bound"] == "hbm" and e["unit"] == "GB/s"
    assert e["ideal_us"] == pytest.approx(10.0)
    assert e["frac"] == pytest.approx(0.5)


def test_peaks_default_fp8_to_twice_bf16():
    pk = bench.peaks()
    assert pk["fp8_tflops"] == pytest.approx(2.0 * pk["bf16_tflops"])
    assert "bf16_tflops_sustained" not in pk
