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
    assert bench.launches_per_step(synth.workload("mixtral_bf16")) == 6   # 4096 assignments, 8 experts: one-block sort
    assert bench.launches_per_step(synth.workload("decode_bf16", T=1)) == 6
    assert bench.launches_per_step(synth.workload("deepseek_bf16")) == 10
    assert bench.launches_per_step(synth.workload("tiny_f32")) == 6   # one-block sort, gather, 2 GEMMs
    # 8-bit: gather-quantise in place of the gather, h re-quantised between the
    # routed GEMMs, the shared expert's x and h quantised
    assert bench.launches_per_step(synth.workload("mixtral_bf16", e4m3=True)) == 7
    assert bench.launches_per_step(synth.workload("deepseek_bf16", e4m3=True)) == 13
    assert bench.launches_per_step(synth.workload("gptoss_bf16")) == 8    # 32768 assignments: count / scan / scatter


def test_workload_keys_and_selection():
    assert bench.workload_key("decode_bf16", {"T": 4}) == "decode_bf16[T=4]"
    assert bench.workload_key("decode_bf16", {"T": 16, "zipf_s": 1.2}) == "decode_bf16[T=16,zipf=1.2]"
    assert bench.workload_key("gptoss_bf16", {"e4m3": True}) == "gptoss_bf16[e4m3]"
    keys = [bench.workload_key(n, ov) for n, ov in bench.parse_workloads("all", "mixtral_bf16")]
    assert len(keys) == len(set(keys)) == len(bench.EXTRA_WORKLOADS)
    assert {"gptoss_bf16", "deepseek_bf16", "tiny_f32", "decode_bf16[T=1]", "decode_bf16[T=64,zipf=1.2]",
            "mixtral_bf16[e4m3]"} <= set(keys)
    assert bench.parse_workloads("none", "mixtral_bf16") == []
    assert [bench.workload_key(n, ov) for n, ov in bench.parse_workloads("decode_bf16[T=4],tiny_f32", "x")] == \
        ["decode_bf16[T=4]", "tiny_f32"]


def test_l2_flush_only_for_inputs_that_fit_in_l2():
    assert bench.needs_l2_flush(synth.workload("tiny_f32"))
    for name in ("mixtral_bf16", "gptoss_bf16", "deepseek_bf16"):
        assert not bench.needs_l2_flush(synth.workload(name))
    assert not bench.needs_l2_flush(synth.workload("decode_bf16", T=1))


def test_oracle_sample_is_the_batch_or_a_fixed_subset():
    assert bench.oracle_sample_tokens(synth.workload("mixtral_bf16")) == 2048
    assert bench.oracle_sample_tokens(synth.workload("tiny_f32")) == 256
    assert bench.oracle_sample_tokens(synth.workload("gptoss_bf16")) == 1024
    assert bench.oracle_sample_tokens(synth.workload("decode_bf16", T=4)) == 4


def test_roofline_of_follows_from_its_numbers():
    cfg = synth.workload("mixtral_bf16")
    counts = np.array([512] * 8)
    stage = {"routed_ffn": 1.0, "shared_ffn": 0.0}
    pk = ({"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback")
    r = bench.roofline_of(cfg, counts, stage, pk)
    flops = 6.0 * 4096 * 14336 * 4096
    assert r["bound"] == "tensor" and r["achieved"] == pytest.approx(flops / 1e-3 / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / 1590.0)
    dec = synth.workload("decode_bf16", T=1)
    r = bench.roofline_of(dec, np.array([1, 1, 0, 0, 0, 0, 0, 0]), {"routed_ffn": 0.1, "shared_ffn": 0.0}, pk)
    assert r["bound"] == "hbm"
    assert r["achieved"] == pytest.approx(2 * 3 * 4096 * 14336 * 2 / 1e-4 / 1e9)
    tiny = bench.roofline_of(synth.workload("tiny_f32"), np.array([64] * 8), stage, pk)
    assert tiny["bound"] == "alu"


def test_gemm_time_is_its_share_of_the_traced_step_applied_to_the_timed_step():
    stage = {"routed_ffn": 1.5, "shared_ffn": 0.5, "step": 2.5}
    g, share = bench.gemm_ms_in_step(stage, 2.0)
    assert share == pytest.approx(0.8) and g == pytest.approx(1.6) and g <= 2.0
    cfg = synth.workload("mixtral_bf16")
    pk = ({"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback")
    r = bench.roofline_of(cfg, np.array([512] * 8), stage, pk, 2.0)
    assert r["stage_ms"] == pytest.approx(1.6) and r["share_of_step"] == pytest.approx(0.8)
    assert r["achieved"] == pytest.approx(6.0 * 4096 * 14336 * 4096 / 1.6e-3 / 1e12)
