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


def test_injected_launch_failure_launches_nothing_and_the_next_call_runs(monkeypatch):
    """MOE_FAULT=launch (a host-side hook; nothing is injected on the device):
    every launching entry point reports MOE_ERR_CUDA, its outputs keep their
    canary values and the workspace status word is untouched; with the
    variable cleared the same call runs and matches the oracle."""
    cfg = synth.workload("tiny_f32").replace(T=64, seed=31)
    inp = H.make_inputs(cfg)
    c = H.moe_cfg(cfg)
    dev = inp.dev
    T, k, E, d = cfg.T, cfg.top_k, cfg.n_experts, cfg.d_model
    ws = torch.full((moe.moe_workspace_bytes(c),), 0x5A, dtype=torch.uint8, device="cuda")
    y = torch.full((T, d), 7.0, dtype=torch.float32, device="cuda")
    ids = torch.full((T, k), -9, dtype=torch.int32, device="cuda")
    w = torch.full((T, k), 3.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), -9, dtype=torch.int32, device="cuda")
    offsets = torch.full((E + 1,), -9, dtype=torch.int32, device="cuda")
    perm = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    row_of = torch.full((T * k,), -9, dtype=torch.int32, device="cuda")
    x_perm = torch.full((T * k, d), 5.0, dtype=torch.float32, device="cuda")
    canaries = [t.clone() for t in (ws, y, ids, w, counts, offsets, perm, row_of, x_perm)]
    ids_in = torch.zeros(T, k, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    calls = {
        "moe_forward": lambda: moe.moe_forward(c, dev["x"], dev["w_router"], None, dev["w_gate_up"], dev["w_down"],
                                               None, None, y, ids, w, counts, ws),
        "moe_router_topk": lambda: moe.moe_router_topk(c, dev["x"], dev["w_router"], None, ids, w, ws),
        "moe_permute": lambda: moe.moe_permute(c, ids_in, dev["x"], counts, offsets, perm, row_of, x_perm, ws),
        "moe_permute_noalloc": lambda: moe.moe_permute_noalloc(c, ids_in, dev["x"], counts, offsets, perm, row_of,
                                                               x_perm),
        "moe_grouped_ffn": lambda: moe.moe_grouped_ffn(c, x_perm, offsets, dev["w_gate_up"], dev["w_down"], x_perm,
                                                       ws),
        "moe_combine": lambda: moe.moe_combine(c, x_perm, row_of, w, None, y),
    }
    monkeypatch.setenv("MOE_FAULT", "launch")
    for name, call in calls.items():
        with pytest.raises(moe.MoeError) as e:
            call()
        assert e.value.status == 4, name
    torch.cuda.synchronize()
    for before, after in zip(canaries, (ws, y, ids, w, counts, offsets, perm, row_of, x_perm)):
        assert torch.equal(before, after)
    monkeypatch.delenv("MOE_FAULT")
    good = H.run_forward(inp)
    assert good["status"] == 0
    H.check_forward(inp, good)
