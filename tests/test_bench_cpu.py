"""Host-side logic of bench.py: the schedule a workload's expert GEMMs run
on, the validity rule of the recorded DRAM traffic, and the algorithmic
work counts the roofline divides by."""
import json

import numpy as np
import pytest

import bench
import synth


@pytest.mark.parametrize("name,T,decode", [("mixtral_bf16", None, False), ("gptoss_bf16", None, False),
                                           ("deepseek_bf16", None, False), ("decode_bf16", 1, True),
                                           ("decode_bf16", 64, True), ("tiny_f32", None, False)])
def test_schedule_of_each_workload(name, T, decode):
    cfg = synth.workload(name) if T is None else synth.workload(name, T=T)
    assert bench.uses_decode_schedule(cfg) == decode


def test_traffic_record_applies_only_to_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    rec = tmp_path / "dram_traffic.json"
    good = bench.gemm_sources_sha256("tc")
    rec.write_text(json.dumps({"mixtral_bf16": {"bytes_per_step": 3.2e9, "gemm_sources_sha256": good},
                               "gptoss_bf16": {"bytes_per_step": 7.2e9, "gemm_sources_sha256": "0" * 64}}))
    monkeypatch.setattr(bench, "TRAFFIC_FILE", rec)
    assert bench.recorded_traffic("mixtral_bf16", "tc") == 3.2e9
    assert bench.recorded_traffic("mixtral_bf16", "decode") is None    # another schedule's sources
    assert bench.recorded_traffic("gptoss_bf16", "tc") is None         # taken on other sources
    assert bench.recorded_traffic("deepseek_bf16", "tc") is None       # no record
    monkeypatch.setattr(bench, "TRAFFIC_FILE", tmp_path / "missing.json")
    assert bench.recorded_traffic("mixtral_bf16", "tc") is None


def test_schedules_digest_different_sources():
    assert bench.gemm_sources_sha256("tc") != bench.gemm_sources_sha256("decode")
    assert "grouped_gemm_tc.cu" in bench.GEMM_SOURCES["tc"]
    assert "grouped_gemm_swap.cu" in bench.GEMM_SOURCES["decode"]


def test_layer_flops_and_bytes():
    # Mixtral-shaped: 2*T*d*E router FLOPs, 6*d*f per routed row, no shared expert
    cfg = synth.workload("mixtral_bf16")
    counts = np.array([512] * 8)
    fl = bench.layer_flops(cfg, counts)
    assert fl["router"] == 2.0 * 2048 * 4096 * 8
    assert fl["experts"] == 6.0 * 4096 * 14336 * 4096
    assert fl["shared"] == 0 and fl["total"] == fl["router"] + fl["experts"]
    by = bench.layer_bytes(cfg, counts)
    assert by["touched"] == 8
    assert by["weights"] == 8 * 3 * 4096 * 14336 * 2 + 8 * 4096 * 2
    # a GELU expert has two matrices; an idle expert's weights are not read
    g = cfg.replace(act=1)
    counts2 = np.array([1024] * 4 + [0] * 4)
    assert bench.layer_flops(g, counts2)["experts"] == 4.0 * 4096 * 14336 * 4096
    assert bench.layer_bytes(g, counts2)["touched"] == 4


def test_launches_per_step():
    assert bench.launches_per_step(synth.workload("mixtral_bf16")) == 8
    assert bench.launches_per_step(synth.workload("decode_bf16", T=1)) == 6
    assert bench.launches_per_step(synth.workload("deepseek_bf16")) == 10
    # 8-bit: gather-quantise in place of the gather, h re-quantised between the
    # routed GEMMs, the shared expert's x and h quantised
    assert bench.launches_per_step(synth.workload("mixtral_bf16", e4m3=True)) == 9
    assert bench.launches_per_step(synth.workload("deepseek_bf16", e4m3=True)) == 13
