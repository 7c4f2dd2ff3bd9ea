"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (one moe_forward call on the whole batch).

Routing (ids, weights) and per-expert counts are checked on every token; layer
outputs on every token for the decode sweep and on sampled tokens for the
large layers (the oracle evaluates tokens one by one, in float64, under forced
routing with the GPU's ids).  Tolerances as in test_gpu_parity.py.
"""
import numpy as np
import pytest
import torch

import synth
from tests import moe_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("name,n_sample", [("mixtral_bf16", 256), ("gptoss_bf16", 256), ("deepseek_bf16", 256)])
def test_full_size_layer(name, n_sample):
    """Sampled tokens cover every expert's last partial tile, the hot expert's
    block boundaries and random tokens (moe_harness.coverage_tokens)."""
    cfg = synth.workload(name)
    inp = H.make_inputs(cfg)
    H.spot_check_device_inputs(inp)
    out = H.run_forward(inp)
    st = H.check_forward(inp, out, n_sample=n_sample)
    print(name, st)
    del inp, out
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", synth.DECODE_T)
@pytest.mark.parametrize("skew", ["uniform", "zipf"])
def test_decode_sweep(T, skew):
    cfg = synth.workload("decode_bf16", T=T, zipf_s=synth.DECODE_ZIPF_S if skew == "zipf" else 0.0)
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    st = H.check_forward(inp, out)
    print(cfg.name, T, skew, st)
    del inp, out
    torch.cuda.empty_cache()


def test_full_size_repeat_is_bitwise_identical():
    cfg = synth.workload("gptoss_bf16")
    inp = H.make_inputs(cfg)
    a = H.run_forward(inp)
    b = H.run_forward(inp)
    assert torch.equal(a["y"].view(torch.int16), b["y"].view(torch.int16))
    assert torch.equal(a["ids"], b["ids"]) and torch.equal(a["counts"], b["counts"])
    assert np.all(a["counts"].cpu().numpy() >= 0)


@pytest.mark.parametrize("name,n_sample", [("gptoss_bf16", 128), ("mixtral_bf16", 128), ("deepseek_bf16", 64)])
def test_full_size_layer_with_8bit_experts(name, n_sample):
    """The full-size layer with E4M3 expert weights, in the launch configuration
    the benchmark times with --e4m3; sampled tokens against the oracle's own
    quantisation of the same bf16 values."""
    cfg = synth.workload(name, e4m3=True)
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    st = H.check_forward(inp, out, n_sample=n_sample)
    print(name, "e4m3", st)
    del inp, out
    torch.cuda.empty_cache()


def test_full_size_layer_with_capacity_factor():
    """Mixtral-shaped layer with a capacity factor of 1.0 under Zipf(1.2)-skewed
    routing: the hot experts drop their late tokens (first come, first served)."""
    cfg = synth.workload("mixtral_bf16", zipf_s=1.2, capacity_factor=1.0)
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    st = H.check_forward(inp, out, n_sample=128)
    assert st["dropped"] > 0
    print("capacity", st)


@pytest.mark.parametrize("skew", ["uniform", "zipf"])
def test_decode_experts_touched_over_draws_against_the_closed_form(skew):
    """"Mixture of experts: how MoE works and what it costs", "How batching
    changes the mixture of experts math": with uniform routing a batch of T
    tokens is expected to touch E (1 - (1 - k/E)^T) experts, 8 (1 - 0.75^T) =
    2 / 5.47 / 7.92 / 8.00 at the decode sizes; skewed routing touches fewer
    (the page calls the closed form an upper bound).  The GPU router runs once
    per seeded batch, 1000 batches per size; its expert ids must equal the
    oracle's outside near ties, and the mean count must sit within a
    statistical bound of the closed form (uniform) or below it (Zipf(1.2))."""
    draws = 1000
    base = synth.workload("decode_bf16", zipf_s=synth.DECODE_ZIPF_S if skew == "zipf" else 0.0)
    E, k, d = base.n_experts, base.top_k, base.d_model
    wr_host = synth.host_tensor(base, "w_router").reshape(E, d)
    w_router = H.host_to_device(synth.host_storage(base, "w_router"), base)
    bias_np = synth.zipf_bias(base)
    bias = torch.from_numpy(bias_np).cuda() if bias_np is not None else None
    for T in synth.DECODE_T:
        cfg = base.replace(T=T)
        c = H.moe_cfg(cfg)
        ws = torch.empty(H.moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
        x_all = synth.device_tensor(cfg.replace(T=draws * T, seed=cfg.seed + 500009), "x", "cuda")
        # one output row per draw, padded so that every draw's outputs start on 16 bytes (the ABI's alignment)
        width = -(-T * k // 4) * 4
        ids = torch.empty(draws, width, dtype=torch.int32, device="cuda")
        w = torch.empty(draws, width, dtype=torch.float32, device="cuda")
        for i in range(draws):
            H.moe.moe_router_topk(c, x_all[i * T:(i + 1) * T], w_router, bias, ids[i], w[i], ws)
        torch.cuda.synchronize()
        gpu_ids = ids[:, :T * k].reshape(draws * T, k).cpu().numpy().astype(np.int64)
        w = w[:, :T * k].reshape(draws * T, k)
        r = H.oracle.route(H.device_to_host_f64(x_all), wr_host,
                           bias_np.astype(np.float64) if bias_np is not None else None, k, cfg.gating,
                           cfg.bias_select_only)
        H.check_routing(cfg, gpu_ids, w.cpu().numpy().astype(np.float64), r, draws * T)
        touched = np.array([len(np.unique(gpu_ids[i * T:(i + 1) * T])) for i in range(draws)], dtype=np.float64)
        mean, se = touched.mean(), touched.std() / np.sqrt(draws)
        closed = H.oracle.occupancy_closed_form(k, E, T) * E
        print(skew, T, "mean", mean, "closed", closed, "se", se)
        if T == 1:
            assert np.all(touched == k)          # one token always touches exactly k experts
        elif skew == "uniform":
            assert abs(mean - closed) <= 4 * se + 0.02, (T, mean, closed)
        else:
            assert mean <= closed + 4 * se, (T, mean, closed)
            if T in (4, 16):
                assert mean < closed - 0.1, (T, mean, closed)
        del x_all
        torch.cuda.empty_cache()
