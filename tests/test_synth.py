"""The seeded input generator: host and device implementations agree bit for bit."""
import math

import numpy as np
import pytest
import torch

import synth


def test_numpy_and_torch_cpu_are_bit_identical():
    a = synth.normal_f32(1001, 2, 5_000_000_000, 1 << 18, 1 / 64)
    b = synth.normal_torch(1001, 2, 5_000_000_000, 1 << 18, 1 / 64, "f32", "cpu", chunk=1 << 16).numpy()
    assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    bits = synth.f32_to_bf16_bits(a)
    tb = synth.normal_torch(1001, 2, 5_000_000_000, 1 << 18, 1 / 64, "bf16", "cpu")
    assert np.array_equal(bits, tb.view(torch.int16).numpy().view(np.uint16))


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5, 3.0e-39], dtype=np.float32)
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert synth.bf16_bits_to_f32(ours)[1] == 1.0            # tie rounds to even
    assert synth.bf16_bits_to_f32(ours)[2] == 1.0 + 2 ** -6  # tie rounds up to even


def test_moments_and_support():
    v = synth.normal_f32(7, 0, 0, 1 << 20).astype(np.float64)
    assert abs(v.mean()) < 5e-3
    assert abs(v.var() - 1.0) < 5e-3
    assert np.max(np.abs(v)) <= 2 * math.sqrt(3.0)
    # excess kurtosis of the 4-term Irwin-Hall sum is -0.3
    k = np.mean(v ** 4) / v.var() ** 2 - 3.0
    assert abs(k + 0.3) < 0.02


def test_slices_regenerate_the_whole():
    cfg = synth.workload("tiny_f32")
    whole = synth.host_tensor(cfg, "w_gate_up")
    part = synth.host_tensor(cfg, "w_gate_up", start=3 * 1024 * 256 + 17, count=999)
    assert np.array_equal(whole[3 * 1024 * 256 + 17: 3 * 1024 * 256 + 17 + 999], part)
    st = synth.host_storage(cfg, "w_gate_up")
    assert st.shape == (8, 1024, 256) and st.dtype == np.float32
    assert np.array_equal(st.reshape(-1).astype(np.float64), whole)


def test_streams_and_seeds_differ():
    a = synth.normal_f32(1, 0, 0, 64)
    assert not np.array_equal(a, synth.normal_f32(1, 1, 0, 64))
    assert not np.array_equal(a, synth.normal_f32(2, 0, 0, 64))


@pytest.mark.parametrize("name", ["deepseek_bf16", "decode_bf16"])
def test_zipf_bias_shares(name):
    cfg = synth.workload(name)
    if cfg.zipf_s == 0:
        cfg = cfg.replace(zipf_s=synth.DECODE_ZIPF_S)
    b = synth.zipf_bias(cfg).astype(np.float64)
    E = cfg.n_experts
    p = np.exp(b) / E                        # shares the bias encodes
    assert abs(p.sum() - 1.0) < 1e-5
    ranks = np.argsort(np.argsort(-p)) + 1   # 1 = most popular
    expect = ranks.astype(np.float64) ** -cfg.zipf_s
    expect /= expect.sum()
    assert np.allclose(p, expect, rtol=1e-5)
    assert synth.zipf_bias(synth.workload("mixtral_bf16")) is None
