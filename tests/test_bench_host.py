"""The benchmark's host arithmetic, without a GPU: the algorithmic work it
divides by (bytes and FLOPs per stage, from the workload's lengths), the
roofline fields built from it, the whole-job rate, and the clock summary
parsed from nvidia-smi samples."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.join(os.path.dirname(__file__), ".."))
import bench  # noqa: E402
from sparse_mla_attention_indexer_b200 import synth  # noqa: E402


@pytest.fixture
def cheap_pools(monkeypatch):
    monkeypatch.setattr(synth, "_fill_latent",
                        lambda seed, name, num_pages: np.zeros(num_pages * synth.LATENT_PAGE, np.uint8))
    monkeypatch.setattr(synth, "_fill_index",
                        lambda seed, name, num_pages: np.zeros(num_pages * synth.INDEX_PAGE, np.uint8))


def test_layer_units_from_the_lengths(cheap_pools):
    # request 0: one query over 300 tokens; request 1: three causal queries
    # ending at 5,000 tokens, so they see 4,998, 4,999 and 5,000 positions
    wl = synth.make_workload("units", [300, 5000], [1, 3], 16, topk=2048,
                             layers=(("rope", 64, True, None), ("nope", 0, True, None), ("shared", 64, False, 1)))
    gathered = 300 + 3 * 2048
    n_sum = 300 + 4998 + 4999 + 5000
    u = bench.layer_units(wl, 0)
    assert u["gathered"] == gathered
    assert u["mla_bytes"] == gathered * 656
    assert u["mla_flops"] == gathered * 2 * 16 * (576 + 512)
    assert u["indexer_bytes"] == 5300 * 132 + n_sum * 4 + 4 * (64 * 128 + 4 + 64 * 4)
    assert u["indexer_flops"] == n_sum * 2 * 64 * 128
    assert u["topk_bytes"] == n_sum * 4
    nope = bench.layer_units(wl, 1)
    assert nope["mla_bytes"] == gathered * 528 and nope["mla_flops"] == gathered * 2 * 16 * 1024
    shared = bench.layer_units(wl, 2)
    assert "indexer_bytes" not in shared and shared["mla_bytes"] == u["mla_bytes"]


PK = dict(hbm_gbs=1000.0, bf16_tflops=100.0, fp8_tflops=200.0, source="test")


def test_rooflines_take_the_slower_of_bytes_and_flops():
    # 1 MB at 1,000 GB/s = 1 us; 1 GFLOP at 100 TFLOP/s = 10 us: tensor-bound
    r = bench.mla_roofline(dict(mla_bytes=10**6, mla_flops=10**9), 0.02, PK, traffic=123)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(50.0) and r["frac"] == pytest.approx(0.5)
    assert r["roofline_us"] == pytest.approx(10.0) and r["measured_us"] == pytest.approx(20.0)
    assert r["gbs"] == pytest.approx(50.0) and r["frac_of_fp8_peak"] == pytest.approx(0.25)
    assert r["traffic"] == 123
    # 100 MB = 100 us at HBM; 1 GFLOP of FP8 at 200 TFLOP/s = 5 us: HBM-bound
    r = bench.indexer_roofline(dict(indexer_bytes=10**8, indexer_flops=10**9), 0.2, PK)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    assert r["achieved"] == pytest.approx(500.0) and r["frac"] == pytest.approx(0.5)
    assert r["frac_of_8000_gbs"] == pytest.approx(500.0 / 8000.0)
    assert r["roofline_us"] == pytest.approx(100.0) and r["traffic"] is None


def test_whole_job_rate_is_every_ranks_units_over_the_slowest_rank():
    assert bench.whole_job_rate(1, 32, 0.08) == pytest.approx(400_000.0)
    assert bench.whole_job_rate(4, 32, 0.1) == pytest.approx(1_280_000.0)


def test_peaks_fall_back_without_the_measured_file(monkeypatch, tmp_path):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    pk = bench.peaks()
    assert pk["source"] == "fallback" and pk["hbm_gbs"] == bench.FALLBACK_HBM_GBS
    assert pk["fp8_tflops"] == 2 * pk["bf16_tflops"]
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6500.0, "bf16_tflops": 1600.0}')
    pk = bench.peaks()
    assert (pk["source"], pk["hbm_gbs"], pk["fp8_tflops"]) == ("measured", 6500.0, 3200.0)


def test_clock_summary_reads_the_samples(tmp_path):
    s = bench.ClockSampler(0)
    s.proc = object()   # as if nvidia-smi had run
    f = tmp_path / "clocks.csv"
    f.write_text("0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
                 "0, 1950, 1965, 980.2, 0x4, Not Active, Not Active, Not Active, Active\n"
                 "0, 1965, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n")
    s.file = open(f)
    out = s.summary()
    assert out["sm_mhz"] == 1965.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 3
