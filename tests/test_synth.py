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


def test_moments_support_and_quantiles_are_standard_normal():
    v = synth.normal_f32(7, 0, 0, 1 << 22).astype(np.float64)
    n = len(v)
    assert abs(v.mean()) < 4.0 / math.sqrt(n)
    assert abs(v.var() - 1.0) < 5.0 * math.sqrt(2.0 / n)
    assert np.max(np.abs(v)) <= 6.2
    k = np.mean(v ** 4) / v.var() ** 2 - 3.0          # excess kurtosis of a normal is 0
    assert abs(k) < 0.02
    # tail probabilities of N(0,1): P(z < -1.96) = 0.025, P(z < -3) = 0.00135, P(z > 4) = 3.2e-5
    for z, p in ((-1.959963984540054, 0.025), (-3.0, 0.0013498980316301), (-4.0, 3.167124183311998e-05)):
        got = np.mean(v < z)
        assert abs(got - p) < 5.0 * math.sqrt(p * (1 - p) / n) + 1e-6, (z, got, p)


def test_quantile_table_edges_are_normal_quantiles():
    q = synth.quantile_table()
    m = 1 << synth.QUANTILE_BITS
    assert len(q) == m + 1 and np.all(np.diff(q) > 0)
    assert q[m // 2] == 0.0
    assert abs(q[int(0.975 * m)] - 1.959963984540054) < 1e-5   # Phi^-1(0.975)
    assert np.allclose(q[1:m][::-1], -q[1:m], rtol=0, atol=1e-9)


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
