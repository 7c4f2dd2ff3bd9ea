"""Bounded device waits: a wait limit that is certain to expire makes the
tensor-core GEMMs give up, drain their own copies, free their tensor memory
and report MOE_ERR_TIMEOUT through the status word -- no trap, no hang -- and
the next call on the same context runs normally."""
import pytest
import torch

import synth
import top_routing_expert_gemm_b200 as moe
from tests import moe_harness as H

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("cfg", [
    # large batch: token-rows-as-M GEMMs; long reductions (d = f = 4096) outlast a 1 ns limit
    synth.LayerConfig("timeout", 1024, 4096, 8, 2, 4096, "bf16", synth.SOFTMAX_TOPK, seed=21),
    # decode schedule (split reductions, partial tiles and counters)
    synth.LayerConfig("timeout_decode", 4, 4096, 64, 2, 4096, "bf16", synth.SOFTMAX_TOPK, seed=22),
    # tensor-core router (64 experts, more than 64 tokens) ahead of the decode schedule
    synth.LayerConfig("timeout_router_tc", 256, 4096, 64, 2, 2048, "bf16", synth.SOFTMAX_TOPK, seed=24),
    # 8-bit experts with a shared expert
    synth.LayerConfig("timeout_e4m3", 512, 4096, 8, 2, 2048, "bf16", synth.SOFTMAX_TOPK, n_shared=1,
                      d_ff_shared=2048, e4m3=True, seed=23),
], ids=lambda c: c.name)
def test_expired_wait_limit_reports_timeout_and_context_survives(cfg):
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp, wait_limit_ns=1)
    assert out["status"] == moe.MOE_ERR_TIMEOUT
    good = H.run_forward(inp)
    assert good["status"] == 0
    H.check_forward(inp, good)
