"""Host logic of bench.py, on CPU: the roofline of a scan launch (HBM- or tensor-bound by
the workload's intensity against the peaks' ridge), whole-job throughput, and the DRAM
traffic taken from the committed ncu summary only while it matches the kernel sources."""
import json

import pytest

import bench
from mla_attention_decode_paged_b200 import workloads as W


def _wl(name, **kw):
    return W.make_workload(name, **kw)


def test_bound_follows_the_intensity_against_the_ridge(monkeypatch):
    peaks = {"hbm_gbs": 6527.8, "bf16_tflops": 1642.8}
    monkeypatch.setattr(bench, "load_peaks", lambda: (dict(peaks), "measured"))
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)  # FLOP per byte
    m64 = _wl("agent_spec", B=1, seq=("fixed", 640))        # 1.889 * 64 = 121 FLOP/B < ridge
    m256 = _wl("long_m256", B=1, seq=("fixed", 640))        # 1.889 * 256 = 484 FLOP/B > ridge
    assert m64.flops() / m64.kv_bytes() < ridge < m256.flops() / m256.kv_bytes()
    roof, nominal, t_roof = bench.roofline_of(m64, 1e-6, None)
    assert roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["achieved"] == pytest.approx(m64.kv_bytes() / 1e-6 / 1e9)
    assert roof["frac"] == pytest.approx(roof["achieved"] / peaks["hbm_gbs"])
    assert t_roof == pytest.approx(m64.kv_bytes() / (peaks["hbm_gbs"] * 1e9))
    roof, _, t_roof = bench.roofline_of(m256, 1e-6, 123)
    assert roof["bound"] == "tensor" and roof["unit"] == "TFLOP/s" and roof["traffic"] == 123
    assert roof["achieved"] == pytest.approx(m256.flops() / 1e-6 / 1e12)
    assert t_roof == pytest.approx(m256.flops() / (peaks["bf16_tflops"] * 1e12))


def test_algorithmic_units_are_the_cache_bytes_and_1088_flops_per_token_row():
    wl = _wl("fp8_batch", B=3, seq_lens=[100, 64, 1])
    tokens = 165
    assert wl.kv_bytes() == tokens * 576 * 1                       # e4m3: one byte per value
    assert wl.flops() == 2 * wl.spec.M * tokens * (576 + 512)
    wl = _wl("agent_spec", B=2, seq_lens=[65, 7])
    assert wl.kv_bytes() == 72 * 576 * 2


def test_whole_job_throughput_counts_every_rank():
    assert bench.job_gbs(1e9, 4, 10, 100.0) == pytest.approx(1e9 * 4 * 10 / 0.1 / 1e9)


def test_traffic_is_used_only_for_the_kernel_sources_it_was_taken_on(tmp_path, monkeypatch):
    prof = tmp_path / "profiles"
    prof.mkdir()
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_hash", lambda: "abc")
    (prof / "ncu_traffic.json").write_text(json.dumps({"agent_spec": {"kernel_hash": "abc",
                                                                       "dram_bytes_per_launch": 42},
                                                        "tiny": {"kernel_hash": "old", "dram_bytes_per_launch": 7}}))
    assert bench.ncu_traffic("agent_spec") == 42
    assert bench.ncu_traffic("tiny") is None          # taken on other sources
    assert bench.ncu_traffic("long_m256") is None     # never taken
