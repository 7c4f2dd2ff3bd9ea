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


@pytest.mark.parametrize("name,n_sample", [("mixtral_bf16", 48), ("gptoss_bf16", 32), ("deepseek_bf16", 16)])
def test_full_size_layer(name, n_sample):
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


@pytest.mark.parametrize("name,n_sample", [("gptoss_bf16", 16), ("mixtral_bf16", 24)])
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
    st = H.check_forward(inp, out, n_sample=32)
    assert st["dropped"] > 0
    print("capacity", st)
