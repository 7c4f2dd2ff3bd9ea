"""GPU parity: every C-ABI call against the CPU oracle on seeded inputs.

Tolerances (written here, not derived at run time):
  * expert ids, counts, offsets, perm, row_of, x_perm: bit-exact (ids outside
    the near-tie set; a token whose k-th / (k+1)-th selection-key gap is under
    1e-3 may flip, and flipped tokens must stay under 0.1% of T);
  * routing weights: |w - w_ref| <= 2e-5 (fp32 softmax/sigmoid on fp32 logits);
  * layer outputs: max|y - y_ref| / max|y_ref| <= 1e-4 (fp32), 2e-2 (bf16).
"""
import numpy as np
import pytest
import torch

import oracle
import synth
import top_routing_expert_gemm_b200 as moe
from tests import moe_harness as H

pytestmark = pytest.mark.gpu

SMALL = {
    # ragged token counts, several tiles, empty experts, every gating rule
    "mixtral_like": synth.LayerConfig("mixtral_like", 300, 512, 8, 2, 640, "bf16", synth.SOFTMAX_TOPK, seed=11),
    "gptoss_like": synth.LayerConfig("gptoss_like", 517, 320, 128, 4, 320, "bf16", synth.SOFTMAX_TOPK, seed=12),
    "deepseek_like": synth.LayerConfig("deepseek_like", 257, 512, 64, 8, 256, "bf16", synth.SIGMOID_TOPK_RENORM,
                                       n_shared=1, d_ff_shared=384, zipf_s=1.0, bias_select_only=1, seed=13),
    "allrenorm_bf16": synth.LayerConfig("allrenorm_bf16", 129, 256, 16, 3, 200, "bf16",
                                        synth.SOFTMAX_ALL_RENORM, zipf_s=1.2, seed=14),
    "f32_sigmoid_shared": synth.LayerConfig("f32_sigmoid_shared", 190, 264, 12, 3, 136, "f32",
                                            synth.SIGMOID_TOPK_RENORM, n_shared=1, d_ff_shared=96, zipf_s=0.8,
                                            seed=15),
    "k_equals_E": synth.LayerConfig("k_equals_E", 64, 256, 4, 4, 256, "bf16", synth.SOFTMAX_ALL_RENORM, seed=16),
    "single_expert": synth.LayerConfig("single_expert", 200, 256, 1, 1, 384, "bf16", synth.SOFTMAX_TOPK, seed=17),
    "one_token": synth.LayerConfig("one_token", 1, 512, 8, 2, 512, "bf16", synth.SOFTMAX_TOPK, seed=18),
    # softmax weights kept without renormalisation; k = 1 is the raw top-1 probability
    "norenorm_top1": synth.LayerConfig("norenorm_top1", 300, 256, 8, 1, 256, "bf16", synth.SOFTMAX_ALL_NO_RENORM,
                                       seed=22),
    "norenorm_f32_k3": synth.LayerConfig("norenorm_f32_k3", 150, 136, 6, 3, 72, "f32", synth.SOFTMAX_ALL_NO_RENORM,
                                         zipf_s=0.7, seed=23),
    "norenorm_tc_router": synth.LayerConfig("norenorm_tc_router", 270, 256, 64, 2, 128, "bf16",
                                            synth.SOFTMAX_ALL_NO_RENORM, seed=24),
    # capacity factor with token dropping (Zipf-skewed routing so that some experts overflow)
    "capacity_1_0": synth.LayerConfig("capacity_1_0", 333, 256, 8, 2, 384, "bf16", synth.SOFTMAX_TOPK,
                                      zipf_s=1.2, capacity_factor=1.0, seed=25),
    "capacity_f32_0_5": synth.LayerConfig("capacity_f32_0_5", 200, 128, 4, 2, 96, "f32", synth.SOFTMAX_ALL_RENORM,
                                          zipf_s=1.0, capacity_factor=0.5, seed=26),
    "capacity_shared": synth.LayerConfig("capacity_shared", 257, 512, 64, 8, 256, "bf16", synth.SIGMOID_TOPK_RENORM,
                                         n_shared=1, d_ff_shared=384, zipf_s=1.0, bias_select_only=1,
                                         capacity_factor=1.25, seed=27),
    # two-matrix GELU experts
    "gelu_bf16": synth.LayerConfig("gelu_bf16", 300, 256, 8, 2, 320, "bf16", synth.SOFTMAX_ALL_RENORM, act=1,
                                   seed=28),
    "gelu_decode_bf16": synth.LayerConfig("gelu_decode_bf16", 20, 512, 16, 2, 384, "bf16", synth.SOFTMAX_TOPK,
                                          act=1, seed=29),
    "gelu_f32_shared": synth.LayerConfig("gelu_f32_shared", 140, 128, 6, 2, 200, "f32", synth.SOFTMAX_ALL_RENORM,
                                         n_shared=1, d_ff_shared=136, act=1, seed=30),
    "gelu_capacity_shared": synth.LayerConfig("gelu_capacity_shared", 200, 256, 16, 4, 192, "bf16",
                                              synth.SOFTMAX_ALL_NO_RENORM, n_shared=1, d_ff_shared=256, act=1,
                                              zipf_s=1.0, capacity_factor=0.8, seed=31),
    # 8-bit (E4M3) experts: large-batch and decode schedules, shared expert, GELU
    "e4m3_mixtral_like": synth.LayerConfig("e4m3_mixtral_like", 300, 512, 8, 2, 640, "bf16", synth.SOFTMAX_TOPK,
                                           e4m3=True, seed=32),
    "e4m3_decode": synth.LayerConfig("e4m3_decode", 5, 1024, 8, 2, 1536, "bf16", synth.SOFTMAX_TOPK, e4m3=True,
                                     seed=33),
    "e4m3_deepseek_like": synth.LayerConfig("e4m3_deepseek_like", 257, 512, 64, 8, 256, "bf16",
                                            synth.SIGMOID_TOPK_RENORM, n_shared=1, d_ff_shared=384, zipf_s=1.0,
                                            bias_select_only=1, e4m3=True, seed=34),
    "e4m3_gelu": synth.LayerConfig("e4m3_gelu", 200, 256, 16, 2, 320, "bf16", synth.SOFTMAX_ALL_RENORM, act=1,
                                   e4m3=True, seed=35),
    # decode-sized layers whose shared expert also runs on the decode kernel:
    # the shared GEMM-1 reuses the unit counters the routed GEMM-2 left at zero
    "decode_shared": synth.LayerConfig("decode_shared", 24, 512, 16, 4, 256, "bf16", synth.SIGMOID_TOPK_RENORM,
                                       n_shared=1, d_ff_shared=384, zipf_s=1.0, bias_select_only=1, seed=36),
    "e4m3_decode_shared": synth.LayerConfig("e4m3_decode_shared", 9, 1024, 8, 2, 768, "bf16", synth.SOFTMAX_TOPK,
                                            n_shared=1, d_ff_shared=512, e4m3=True, seed=37),
}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    moe.lib()


# ------------------------------------------------------------------ whole layer, small
def test_tiny_f32_layer_full_parity():
    cfg = synth.workload("tiny_f32")
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    st = H.check_forward(inp, out)
    assert st["mismatched"] == 0


@pytest.mark.parametrize("name", list(SMALL))
def test_small_layers_full_parity(name):
    cfg = SMALL[name]
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    H.check_forward(inp, out)


@pytest.mark.parametrize("name", ["deepseek_like", "decode_shared"])
def test_forward_is_deterministic(name):
    inp = H.make_inputs(SMALL[name])
    a = H.run_forward(inp)
    b = H.run_forward(inp)
    assert torch.equal(a["y"].view(torch.int16), b["y"].view(torch.int16))
    assert torch.equal(a["ids"], b["ids"]) and torch.equal(a["w"], b["w"])


def test_huge_bias_sends_every_token_to_one_expert():
    cfg = synth.LayerConfig("forced", 700, 256, 8, 2, 256, "bf16", synth.SOFTMAX_TOPK, seed=19)
    inp = H.make_inputs(cfg)
    b = np.zeros(8, np.float32)
    b[5] = 1e4
    inp.bias = b
    inp.dev["bias"] = torch.from_numpy(b).cuda()
    out = H.run_forward(inp)
    assert np.all(out["ids"].cpu().numpy()[:, 0] == 5)
    assert int(out["counts"][5]) == 700
    H.check_forward(inp, out)


def test_zero_tokens_is_a_no_op():
    cfg = SMALL["mixtral_like"]
    c = H.moe_cfg(cfg, T=0)
    inp = H.make_inputs(cfg)
    ws = torch.empty(max(256, moe.moe_workspace_bytes(c)), dtype=torch.uint8, device="cuda")
    counts = torch.full((8,), 7, dtype=torch.int32, device="cuda")
    y = torch.empty(0, cfg.d_model, dtype=torch.bfloat16, device="cuda")
    moe.moe_forward(c, inp.dev["x"], inp.dev["w_router"], None, inp.dev["w_gate_up"], inp.dev["w_down"], None, None,
                    y, None, None, counts, ws)
    torch.cuda.synchronize()
    assert torch.all(counts == 0)


# ------------------------------------------------------------------ single entry points
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("gating", [0, 1, 2, 3])
@pytest.mark.parametrize("E,k", [(8, 2), (64, 6), (256, 8)])
@pytest.mark.parametrize("T", [333, 17])  # a warp per token / a block per token (decode-sized batches)
def test_router_topk(dtype, gating, E, k, T):
    cfg = synth.LayerConfig("r", T, 264, E, k, 8, dtype, gating, zipf_s=1.1, bias_select_only=1, seed=E + k + T)
    inp = H.make_inputs(cfg)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    ids = torch.empty(cfg.T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(cfg.T, k, dtype=torch.float32, device="cuda")
    moe.moe_router_topk(c, inp.dev["x"], inp.dev["w_router"], inp.dev["bias"], ids, w, ws)
    torch.cuda.synchronize()
    x = synth.host_tensor(cfg, "x").reshape(cfg.T, cfg.d_model)
    wr = synth.host_tensor(cfg, "w_router").reshape(E, cfg.d_model)
    r = oracle.route(x, wr, inp.bias.astype(np.float64), k, gating, cfg.bias_select_only)
    H.check_routing(cfg, ids.cpu().numpy().astype(np.int64), w.cpu().numpy().astype(np.float64), r, cfg.T)



# The tensor-core router at model-like widths (d = 1024, 2048), ragged last
# tile; repeated calls agree bitwise.
@pytest.mark.parametrize("gating", [0, 1, 2, 3])
@pytest.mark.parametrize("E,k", [(64, 6), (256, 8), (144, 16)])
@pytest.mark.parametrize("T,d", [(333, 1024), (1000, 2048)])
def test_router_topk_long_rows(gating, E, k, T, d):
    cfg = synth.LayerConfig("rs", T, d, E, k, 8, "bf16", gating, zipf_s=1.1, bias_select_only=1, seed=E + d + T)
    inp = H.make_inputs(cfg)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    out = []
    for _ in range(2):
        ids = torch.empty(cfg.T, k, dtype=torch.int32, device="cuda")
        w = torch.empty(cfg.T, k, dtype=torch.float32, device="cuda")
        moe.moe_router_topk(c, inp.dev["x"], inp.dev["w_router"], inp.dev["bias"], ids, w, ws)
        torch.cuda.synchronize()
        out.append((ids, w))
    assert torch.equal(out[0][0], out[1][0]) and torch.equal(out[0][1], out[1][1])
    x = synth.host_tensor(cfg, "x").reshape(cfg.T, cfg.d_model)
    wr = synth.host_tensor(cfg, "w_router").reshape(E, cfg.d_model)
    r = oracle.route(x, wr, inp.bias.astype(np.float64), k, gating, cfg.bias_select_only)
    ids, w = out[0]
    H.check_routing(cfg, ids.cpu().numpy().astype(np.int64), w.cpu().numpy().astype(np.float64), r, cfg.T)

@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (1000, 8, 2), (4099, 256, 8), (2048, 1024, 16), (333, 5, 5),
                                   (1024, 64, 8), (1025, 64, 8)])
@pytest.mark.parametrize("skew", ["uniform", "one_expert", "half_empty"])
@pytest.mark.parametrize("cf", [0.0, 1.0, 0.3])
def test_permute_bit_exact(T, E, k, skew, cf):
    rng = np.random.default_rng(T + E + k)
    if skew == "uniform":
        keys = rng.random((T, E))
    elif skew == "one_expert":
        keys = rng.random((T, E))
        keys[:, E // 2] += 10.0
    else:
        keys = rng.random((T, E))
        keys[:, : (E + 1) // 2] += 10.0
    ids = np.argsort(-keys, axis=1, kind="stable")[:, :k].astype(np.int32)
    d = 136
    x = rng.standard_normal((T, d)).astype(np.float32)
    cfg = synth.LayerConfig("p", T, d, E, k, 8, "f32", 0, capacity_factor=cf)
    c = H.moe_cfg(cfg)
    cap = H.capacity_of(cfg)
    assert moe.moe_expert_capacity(c) == (T * k if cap is None else min(cap, T))
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    dids = torch.from_numpy(ids).cuda()
    dx = torch.from_numpy(x).cuda()
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * k, d, dtype=torch.float32, device="cuda")
    moe.moe_permute(c, dids, dx, counts, offsets, perm, row_of, x_perm, ws)
    assert moe.moe_device_status(ws) == 0
    rc, ro, rp, rr = oracle.dispatch(ids.astype(np.int64), E, cap)
    n_kept = int(ro[-1])
    assert np.array_equal(counts.cpu().numpy(), rc)
    assert np.array_equal(offsets.cpu().numpy(), ro)
    assert np.array_equal(perm.cpu().numpy()[:n_kept], rp)
    assert np.array_equal(row_of.cpu().numpy(), rr)
    assert np.array_equal(x_perm.cpu().numpy()[:n_kept], x[rp // k])


def test_permute_flags_out_of_range_ids():
    T, E, k, d = 100, 8, 2, 16
    ids = np.zeros((T, k), np.int32)
    ids[:, 1] = 1
    ids[7, 1] = 9  # out of range
    cfg = synth.LayerConfig("p", T, d, E, k, 8, "f32", 0)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * k, d, dtype=torch.float32, device="cuda")
    x = torch.zeros(T, d, device="cuda")
    moe.moe_permute(c, torch.from_numpy(ids).cuda(), x, counts, offsets, perm, row_of, x_perm, ws)
    assert moe.moe_device_status(ws) == moe.MOE_ERR_BAD_EXPERT_ID
    assert int(offsets[E]) == T * k - 1
    assert int(row_of[7 * k + 1]) == -1


def _ragged_offsets(sizes):
    return np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("sizes,d,f", [
    ([0, 1, 127, 129, 300, 0, 256], 256, 384),   # several m-tiles, ragged tails, empty groups
    ([5, 0, 140], 264, 200),                     # partial n-tiles in both GEMMs
    ([1000], 512, 1024),                          # one big group
    ([3] * 40, 128, 136),                         # many tiny groups
    ([70, 0, 1, 64, 65], 4096, 640),              # decode schedule: 2-chunk groups, split reductions
    ([1, 1], 4096, 14336),                        # decode schedule: one token per expert
    ([3, 0, 40, 1], 1024, 1536),                  # decode schedule: units cut across several CTAs
    ([2100, 17, 0, 256, 257], 256, 192),          # 256-token chunks, a 9-chunk group, N = 16 remainders
    ([300, 0, 129, 128], 448, 448),               # five-stage ring of N = 224 in both GEMMs (448 = 4 x 112 = 2 x 224)
])
def test_grouped_ffn_against_dense_experts(dtype, sizes, d, f):
    rng = np.random.default_rng(sum(sizes) + d + f)
    G = len(sizes)
    rows = int(sum(sizes))
    offs = _ragged_offsets(sizes)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    a = torch.from_numpy(rng.standard_normal((rows, d)).astype(np.float32)).to(tdt).cuda()
    wgu = torch.from_numpy((rng.standard_normal((G, 2 * f, d)) / np.sqrt(d)).astype(np.float32)).to(tdt).cuda()
    wd = torch.from_numpy((rng.standard_normal((G, d, f)) / np.sqrt(f)).astype(np.float32)).to(tdt).cuda()
    y = torch.full((rows, d), float("nan"), dtype=tdt, device="cuda")
    # the call's T*k must equal the row count: use k = 1, T = rows
    cfg = synth.LayerConfig("g", rows, d, G, 1, f, dtype, 0)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    moe.moe_grouped_ffn(c, a, torch.from_numpy(offs).cuda(), wgu, wd, y, ws)
    assert moe.moe_device_status(ws) == 0
    A = H.device_to_host_f64(a)
    WGU = H.device_to_host_f64(wgu)
    WD = H.device_to_host_f64(wd)
    ref = np.zeros((rows, d))
    for g in range(G):
        r0, r1 = offs[g], offs[g + 1]
        if r1 > r0:
            ref[r0:r1] = oracle.swiglu_expert(A[r0:r1], WGU[g, :f], WGU[g, f:], WD[g])
    got = H.device_to_host_f64(y)
    assert not np.any(np.isnan(got))
    assert H.rel_err(got, ref) <= H.TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("sizes,d,f", [
    ([0, 1, 127, 129, 300, 0, 256], 256, 384),   # large-batch schedule
    ([3, 0, 40, 1], 1024, 1536),                  # decode schedule, units cut across CTAs
    ([600, 17], 264, 200),                        # partial weight blocks, N = 32 remainder
])
def test_grouped_ffn_gelu_against_dense_experts(dtype, sizes, d, f):
    """Two-matrix experts: y = GELU(a Wu^T) Wd^T per group."""
    rng = np.random.default_rng(sum(sizes) + d + f + 1)
    G = len(sizes)
    rows = int(sum(sizes))
    offs = _ragged_offsets(sizes)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    a = torch.from_numpy(rng.standard_normal((rows, d)).astype(np.float32)).to(tdt).cuda()
    wu = torch.from_numpy((rng.standard_normal((G, f, d)) / np.sqrt(d)).astype(np.float32)).to(tdt).cuda()
    wd = torch.from_numpy((rng.standard_normal((G, d, f)) / np.sqrt(f)).astype(np.float32)).to(tdt).cuda()
    y = torch.full((rows, d), float("nan"), dtype=tdt, device="cuda")
    cfg = synth.LayerConfig("g", rows, d, G, 1, f, dtype, 0, act=1)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    moe.moe_grouped_ffn(c, a, torch.from_numpy(offs).cuda(), wu, wd, y, ws)
    assert moe.moe_device_status(ws) == 0
    A = H.device_to_host_f64(a)
    WU = H.device_to_host_f64(wu)
    WD = H.device_to_host_f64(wd)
    ref = np.zeros((rows, d))
    for g in range(G):
        r0, r1 = offs[g], offs[g + 1]
        if r1 > r0:
            ref[r0:r1] = oracle.gelu_expert(A[r0:r1], WU[g], WD[g])
    got = H.device_to_host_f64(y)
    assert not np.any(np.isnan(got))
    assert H.rel_err(got, ref) <= H.TOL[dtype]


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("shared", [False, True])
def test_combine(dtype, shared):
    rng = np.random.default_rng(3)
    T, k, d = 257, 3, 264
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    yp = torch.from_numpy(rng.standard_normal((T * k, d)).astype(np.float32)).to(tdt).cuda()
    row_of = rng.permutation(T * k).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    ys = torch.from_numpy(rng.standard_normal((T, d)).astype(np.float32)).to(tdt).cuda() if shared else None
    y = torch.empty(T, d, dtype=tdt, device="cuda")
    cfg = synth.LayerConfig("c", T, d, 8, k, 8, dtype, 0)
    moe.moe_combine(H.moe_cfg(cfg), yp, torch.from_numpy(row_of).cuda(), torch.from_numpy(w).cuda(), ys, y)
    torch.cuda.synchronize()
    ref = H.oracle.combine(H.device_to_host_f64(yp), row_of, w.astype(np.float64),
                           H.device_to_host_f64(ys) if shared else None)
    assert H.rel_err(H.device_to_host_f64(y), ref) <= (1e-6 if dtype == "f32" else 8e-3)


# ------------------------------------------------------------------ router penalties
@pytest.mark.parametrize("dtype,E,k,d,T", [("bf16", 8, 2, 512, 700), ("bf16", 256, 8, 1024, 333),
                                           ("f32", 12, 3, 264, 190), ("bf16", 64, 1, 256, 1)])
def test_router_aux_losses(dtype, E, k, d, T):
    """Balance loss (without alpha) and z-loss from the bias-free logits, against
    the oracle on the same stored inputs and the GPU's own routed-slot counts.
    Relative tolerance 1e-4: fp32 logits and fp32 sums in a fixed order."""
    cfg = synth.LayerConfig("aux", T, d, E, k, 8, dtype, synth.SOFTMAX_TOPK, zipf_s=1.1, seed=E + T)
    inp = H.make_inputs(cfg)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_router_topk(c, inp.dev["x"], inp.dev["w_router"], inp.dev["bias"], ids, w, ws)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * k, d, dtype=H.torch_dtype(cfg), device="cuda")
    moe.moe_permute(c, ids, inp.dev["x"], counts, offsets, perm, row_of, x_perm, ws)
    out = torch.full((4,), float("nan"), dtype=torch.float32, device="cuda")
    moe.moe_router_aux_losses(c, inp.dev["x"], inp.dev["w_router"], counts, out, ws)
    assert moe.moe_device_status(ws) == 0
    x = synth.host_tensor(cfg, "x").reshape(T, d)
    wr = synth.host_tensor(cfg, "w_router").reshape(E, d)
    logits = oracle.router_logits(x, wr)
    cnt = counts.cpu().numpy()
    ref = (oracle.balance_loss(logits, cnt), oracle.router_z_loss(logits))
    got = out.cpu().numpy()
    assert abs(got[0] - ref[0]) <= 1e-4 * abs(ref[0]), (got, ref)
    assert abs(got[1] - ref[1]) <= 1e-4 * abs(ref[1]), (got, ref)
    assert np.isnan(got[2]) and np.isnan(got[3])  # nothing written past out[1]


# ------------------------------------------------------------------ 8-bit experts
# row lengths: rows shorter than one unrolled step, and unrolled steps with
# and without a ragged tail of 16-byte vectors
@pytest.mark.parametrize("cols", [272, 1040, 2880, 4096, 7168, 7184, 14336])
def test_quantize_e4m3_matches_the_oracle_bit_for_bit(cols):
    """Codes and scales of moe_quantize_e4m3 equal the oracle's per-row E4M3
    quantisation of the same bf16 values (the rounding decisions are taken
    in float32 on both sides): values exactly, scales exactly."""
    rng = np.random.default_rng(40 + cols)
    rows = 70
    w = rng.standard_normal((rows, cols)).astype(np.float32)
    w[3] = 0.0
    w[5] *= 1e-4
    w[6] *= 3e3
    w[7, 11] = 1e6  # one outlier dominates its row's scale
    wt = torch.from_numpy(w).to(torch.bfloat16).cuda()
    blob = H.e4m3_blob(wt)
    assert blob.numel() == moe.moe_e4m3_weight_bytes(rows, cols) == (rows * cols + 255) // 256 * 256 + 4 * rows
    codes = blob[: rows * cols].cpu().numpy().reshape(rows, cols)
    off = (rows * cols + 255) // 256 * 256
    scales = blob[off: off + 4 * rows].cpu().numpy().view(np.float32).astype(np.float64)
    table = np.array([oracle.e4m3_decode(c) for c in range(256)])
    q_ref, s_ref = oracle.quantize_rows_e4m3(H.device_to_host_f64(wt))
    assert np.array_equal(scales, s_ref)
    assert np.array_equal(table[codes], q_ref)


@pytest.mark.parametrize("act", [0, 1])
@pytest.mark.parametrize("sizes,d,f", [
    ([0, 1, 127, 129, 300, 0, 256], 256, 384),   # large-batch schedule
    ([3, 0, 40, 1], 1024, 1536),                  # decode schedule, units cut across CTAs
    ([600, 17], 272, 208),                        # partial weight blocks
    ([300, 129], 480, 480),                       # partial last tile of 128 and of 256 output columns
])
def test_grouped_ffn_e4m3_against_the_oracle(act, sizes, d, f):
    """8-bit experts through moe_grouped_ffn: weights quantised on the GPU,
    activations and h inside the call; the oracle quantises the same bf16
    values itself (e4m3_expert).  Tolerance: the bf16 one."""
    rng = np.random.default_rng(sum(sizes) + d + f + act)
    G = len(sizes)
    rows = int(sum(sizes))
    offs = _ragged_offsets(sizes)
    m = 2 if act == 0 else 1
    a = torch.from_numpy(rng.standard_normal((rows, d)).astype(np.float32)).to(torch.bfloat16).cuda()
    wgu = torch.from_numpy((rng.standard_normal((G, m * f, d)) / np.sqrt(d)).astype(np.float32)).to(torch.bfloat16)
    wd = torch.from_numpy((rng.standard_normal((G, d, f)) / np.sqrt(f)).astype(np.float32)).to(torch.bfloat16)
    wgu, wd = wgu.cuda(), wd.cuda()
    y = torch.full((rows, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    cfg = synth.LayerConfig("g", rows, d, G, 1, f, "bf16", 0, act=act, e4m3=True)
    c = H.moe_cfg(cfg)
    ws = torch.zeros(moe.moe_workspace_bytes(c), dtype=torch.uint8, device="cuda")
    moe.moe_grouped_ffn(c, a, torch.from_numpy(offs).cuda(), H.e4m3_blob(wgu), H.e4m3_blob(wd), y, ws)
    assert moe.moe_device_status(ws) == 0
    A = H.device_to_host_f64(a)
    WGU = H.device_to_host_f64(wgu)
    WD = H.device_to_host_f64(wd)
    ref = np.zeros((rows, d))
    for g in range(G):
        r0, r1 = offs[g], offs[g + 1]
        if r1 > r0:
            wts = (WGU[g, :f], WGU[g, f:], WD[g]) if act == 0 else (WGU[g], WD[g])
            ref[r0:r1] = oracle.e4m3_expert(A[r0:r1], wts, act)
    got = H.device_to_host_f64(y)
    assert not np.any(np.isnan(got))
    assert H.rel_err(got, ref) <= H.TOL["bf16"]


def _stage_by_stage(inp):
    """moe_router_topk -> moe_permute (bf16 x_perm) -> moe_grouped_ffn -> moe_combine."""
    cfg, dev = inp.cfg, inp.dev
    c = H.moe_cfg(cfg)
    T, k, E, d = cfg.T, cfg.top_k, cfg.n_experts, cfg.d_model
    i32 = dict(dtype=torch.int32, device="cuda")
    ws = torch.empty(max(256, moe.moe_workspace_bytes(c)), dtype=torch.uint8, device="cuda")
    ids, w = torch.empty(T, k, **i32), torch.empty(T, k, dtype=torch.float32, device="cuda")
    moe.moe_router_topk(c, dev["x"], dev["w_router"], dev["bias"], ids, w, ws)
    counts, offsets = torch.empty(E, **i32), torch.empty(E + 1, **i32)
    perm, row_of = torch.empty(T * k, **i32), torch.empty(T * k, **i32)
    x_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_permute(c, ids, dev["x"], counts, offsets, perm, row_of, x_perm, ws)
    y_perm = torch.empty(T * k, d, dtype=torch.bfloat16, device="cuda")
    q = "_q" if cfg.e4m3 else ""
    moe.moe_grouped_ffn(c, x_perm, offsets, dev["w_gate_up" + q], dev["w_down" + q], y_perm, ws)
    y = torch.empty(T, d, dtype=torch.bfloat16, device="cuda")
    moe.moe_combine(c, y_perm, row_of, w, None, y)
    torch.cuda.synchronize()
    return y


@pytest.mark.parametrize("cfg", [
    SMALL["e4m3_mixtral_like"],                                   # token-rows-as-M GEMMs
    SMALL["e4m3_decode"],                                         # decode schedule
    SMALL["e4m3_gelu"],
    synth.LayerConfig("e4m3_cap", 333, 2880, 16, 4, 640, "bf16", synth.SOFTMAX_TOPK,
                      zipf_s=1.2, capacity_factor=0.8, e4m3=True, seed=41),  # dropped slots
], ids=lambda c: c.name)
def test_forward_e4m3_equals_the_stage_calls(cfg):
    """With 8-bit experts moe_forward quantises the dispatched rows straight
    from x (no bf16 copy); the stage-by-stage path quantises the gathered bf16
    copy inside moe_grouped_ffn.  Same codes, same GEMMs: the outputs are
    bitwise equal."""
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    assert out["status"] == 0
    y = _stage_by_stage(inp)
    assert torch.equal(out["y"].view(torch.int16), y.view(torch.int16))


@pytest.mark.parametrize("cfg", [
    SMALL["mixtral_like"],
    SMALL["gptoss_like"],                                         # many experts, half-height tail tiles
    SMALL["gelu_bf16"],
    SMALL["capacity_1_0"],                                        # dropped slots
    synth.LayerConfig("hot_expert", 3000, 256, 8, 2, 384, "bf16", synth.SOFTMAX_TOPK, zipf_s=2.0, seed=42),
], ids=lambda c: c.name)
def test_forward_bf16_equals_the_stage_calls(cfg):
    """Large bf16 batches: moe_forward (chained launches) and the four stage
    calls run the same kernels on the same operands in the same order, so
    the outputs are bitwise equal -- including skewed routing with a hot
    expert, half-height tail tiles and dropped slots."""
    inp = H.make_inputs(cfg)
    out = H.run_forward(inp)
    assert out["status"] == 0
    y = _stage_by_stage(inp)
    assert torch.equal(out["y"].view(torch.int16), y.view(torch.int16))


@pytest.mark.parametrize("cfg", [
    SMALL["mixtral_like"],
    SMALL["deepseek_like"],                                       # shared expert: six stages all non-empty
    synth.LayerConfig("decode_traced", 4, 512, 8, 2, 1024, "bf16", synth.SOFTMAX_TOPK, seed=43),
], ids=lambda c: c.name)
def test_forward_traced_equals_forward_and_records_its_stages(cfg):
    """moe_forward_traced runs the same launches as moe_forward with six
    events recorded between them: bitwise the same outputs, every event
    recorded on the launching stream, in order, and the stage times add up to
    the step's."""
    inp = H.make_inputs(cfg)
    ref = H.run_forward(inp)
    assert ref["status"] == 0
    c = H.moe_cfg(cfg)
    dev = inp.dev
    T, k, E, d = cfg.T, cfg.top_k, cfg.n_experts, cfg.d_model
    y = torch.empty(T, d, dtype=H.torch_dtype(cfg), device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(256, moe.moe_workspace_bytes(c)), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.Stream()                                  # not the current stream
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(6)]
    moe.moe_forward_traced(c, dev["x"], dev["w_router"], dev["bias"], dev["w_gate_up"], dev["w_down"],
                           dev.get("ws_gate_up"), dev.get("ws_down"), y, ids, w, counts, ws, stream=stream,
                           stage_events=evs)
    assert moe.moe_device_status(ws, stream=stream) == 0
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref["y"].view(torch.int16))
    assert torch.equal(ids, ref["ids"]) and torch.equal(w, ref["w"]) and torch.equal(counts, ref["counts"])
    assert all(e.query() for e in evs)
    stages = [evs[j].elapsed_time(evs[j + 1]) for j in range(5)]
    assert all(s >= 0.0 for s in stages)
    assert abs(sum(stages) - evs[0].elapsed_time(evs[5])) <= 1e-3 + 1e-3 * evs[0].elapsed_time(evs[5])
    # None entries are skipped
    moe.moe_forward_traced(c, dev["x"], dev["w_router"], dev["bias"], dev["w_gate_up"], dev["w_down"],
                           dev.get("ws_gate_up"), dev.get("ws_down"), y, ids, w, counts, ws, stream=stream,
                           stage_events=[evs[0], None, None, None, None, evs[5]])
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref["y"].view(torch.int16))
