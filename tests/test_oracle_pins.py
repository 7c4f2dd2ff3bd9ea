"""Pins for the CPU oracle: what the pages and plain mathematics fix.

None of these re-types the oracle's own formula: each compares it with a
closed form, a value the pages print (``tests/golden``), brute force on tiny
inputs written independently here, or a special case that reduces to a
dense FFN.  Each test names the mistake it would catch.
"""
import itertools
import json
import math
import pathlib

import numpy as np
import pytest

import oracle

GOLDEN = pathlib.Path(__file__).parent / "golden"
MODES = (oracle.SOFTMAX_ALL_RENORM, oracle.SOFTMAX_TOPK, oracle.SIGMOID_TOPK_RENORM)


def _rand(rng, *shape, scale=1.0):
    return rng.standard_normal(shape) * scale


def _layer(rng, T=9, d=6, E=5, f=4):
    x = _rand(rng, T, d)
    wr = _rand(rng, E, d, scale=0.7)
    wgu = _rand(rng, E, 2 * f, d, scale=0.5)
    wd = _rand(rng, E, d, f, scale=0.5)
    return x, wr, wgu, wd


def _experts(wgu, wd):
    f = wd.shape[2]
    return lambda e: (wgu[e, :f], wgu[e, f:], wd[e])


# ------------------------------------------------------------------ pure-Python references
def _dot(a, b):
    return math.fsum(p * q for p, q in zip(a, b))


def _swiglu_loops(xv, wg, wu, wd):
    """Dense SwiGLU FFN of one token with explicit loops (independent of numpy @)."""
    f = len(wg)
    h = []
    for j in range(f):
        g = _dot(xv, wg[j])
        u = _dot(xv, wu[j])
        h.append(g / (1.0 + math.exp(-g)) * u)
    return [_dot(h, wd[i]) for i in range(len(wd))]


# ------------------------------------------------------------------ scores and weights
@pytest.mark.parametrize("E", [1, 2, 8, 256])
def test_softmax_sums_to_one(E):
    rng = np.random.default_rng(E)
    p = oracle.softmax(_rand(rng, 64, E, scale=4.0), axis=1)
    assert np.all(p > 0)
    assert np.max(np.abs(p.sum(axis=1) - 1.0)) <= 1e-12


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("E,k", [(8, 1), (8, 2), (128, 4), (256, 8), (6, 6)])
def test_routing_weights_sum_to_one_and_positive(mode, E, k):
    rng = np.random.default_rng(10 * E + k)
    x = _rand(rng, 50, 16)
    wr = _rand(rng, E, 16, scale=0.5)
    bias = _rand(rng, E, scale=0.3)
    r = oracle.route(x, wr, bias, k, mode, bias_select_only=1)
    assert np.all(r.w > 0)
    assert np.max(np.abs(r.w.sum(axis=1) - 1.0)) <= 1e-12


def test_k1_renormalised_weight_is_one():
    """[SEV] "Why top-1 routing cannot renormalise": with k=1 the weight is exactly 1."""
    rng = np.random.default_rng(1)
    x = _rand(rng, 40, 12)
    wr = _rand(rng, 8, 12)
    for mode in MODES:
        r = oracle.route(x, wr, None, 1, mode)
        assert np.all(r.w == 1.0)


def test_softmax_before_and_after_topk_agree():
    """[SEV] "Softmax before or after the top-k step": renormalised full
    softmax equals softmax over the kept logits: the common denominator
    cancels.  The page measured a difference under 1e-7 on 512 tokens in
    float32; in float64 only rounding remains."""
    rng = np.random.default_rng(2)
    x = _rand(rng, 512, 64)
    wr = _rand(rng, 8, 64, scale=0.125)
    a = oracle.route(x, wr, None, 2, oracle.SOFTMAX_ALL_RENORM)
    b = oracle.route(x, wr, None, 2, oracle.SOFTMAX_TOPK)
    assert np.array_equal(a.ids, b.ids)
    assert np.max(np.abs(a.w - b.w)) <= 1e-12


def test_topk_matches_brute_force_sort_and_repeated_argmax():
    """Selection vs a pure-Python sort of (key desc, index asc) pairs and k rounds of argmax.
    Catches an ascending sort, a wrong tie rule or a dropped slot."""
    rng = np.random.default_rng(3)
    key = np.round(_rand(rng, 200, 10), 1)   # coarse values force many exact ties
    for k in (1, 2, 3, 10):
        ids = oracle.topk_select(key, k)
        for t in range(key.shape[0]):
            brute = [e for _, e in sorted((-key[t, e], e) for e in range(10))][:k]
            assert ids[t].tolist() == brute
            rest = list(range(10))
            picks = []
            for _ in range(k):
                best = rest[0]
                for e in rest[1:]:
                    if key[t, e] > key[t, best]:
                        best = e
                picks.append(best)
                rest.remove(best)
            assert ids[t].tolist() == picks


def test_topk_gap_brute_force():
    rng = np.random.default_rng(4)
    key = _rand(rng, 30, 7)
    gap = oracle.topk_gap(key, 3)
    for t in range(30):
        s = sorted(key[t].tolist(), reverse=True)
        assert gap[t] == pytest.approx(s[2] - s[3], abs=0)
    assert np.all(np.isinf(oracle.topk_gap(key, 7)))


def test_softmax_topk_is_shift_invariant_sigmoid_is_not():
    """Softmax weights ignore a constant added to every logit; sigmoid weights do not
    (catches a sigmoid rule that silently used softmax, or the reverse)."""
    rng = np.random.default_rng(5)
    x = _rand(rng, 20, 8)
    wr = _rand(rng, 6, 8)
    shift = np.full(6, 0.75)
    for mode in (oracle.SOFTMAX_ALL_RENORM, oracle.SOFTMAX_TOPK):
        a = oracle.route(x, wr, None, 3, mode)
        b = oracle.route(x, wr, shift, 3, mode)
        assert np.array_equal(a.ids, b.ids)
        assert np.allclose(a.w, b.w, rtol=0, atol=1e-14)
    a = oracle.route(x, wr, None, 3, oracle.SIGMOID_TOPK_RENORM)
    b = oracle.route(x, wr, shift, 3, oracle.SIGMOID_TOPK_RENORM, bias_select_only=0)
    assert np.array_equal(a.ids, b.ids)
    assert np.max(np.abs(a.w - b.w)) > 1e-3


def test_sigmoid_bias_steers_selection_only():
    """[AFD] "Why load balancing is the hard part of MoE": the bias shifts routing
    without distorting the gate values used for output."""
    rng = np.random.default_rng(6)
    x = _rand(rng, 64, 16)
    wr = _rand(rng, 16, 16, scale=0.25)
    bias = _rand(rng, 16, scale=2.0)
    r = oracle.route(x, wr, bias, 4, oracle.SIGMOID_TOPK_RENORM, bias_select_only=1)
    # hand computation of the weights from the unbiased logits on the chosen ids
    for t in range(64):
        g = [1.0 / (1.0 + math.exp(-_dot(x[t], wr[e]))) for e in r.ids[t]]
        assert r.w[t].tolist() == pytest.approx([v / sum(g) for v in g], rel=1e-13)
    # and the selection did follow the biased key
    keys = x @ wr.T + bias
    assert np.array_equal(r.ids, oracle.topk_select(keys, 4))


def test_huge_bias_forces_an_expert_and_zero_bias_is_no_bias():
    rng = np.random.default_rng(7)
    x = _rand(rng, 33, 8)
    wr = _rand(rng, 5, 8)
    bias = np.zeros(5)
    bias[3] = 1e6
    for mode in MODES:
        r = oracle.route(x, wr, bias, 2, mode, bias_select_only=1)
        assert np.all(r.ids[:, 0] == 3)
        a = oracle.route(x, wr, None, 2, mode)
        b = oracle.route(x, wr, np.zeros(5), 2, mode)
        assert np.array_equal(a.ids, b.ids) and np.array_equal(a.w, b.w)


# ------------------------------------------------------------------ dispatch
@pytest.mark.parametrize("T,E,k", [(1, 1, 1), (17, 4, 2), (100, 8, 2), (64, 256, 8), (5, 6, 6)])
def test_dispatch_is_a_stable_grouping(T, E, k):
    rng = np.random.default_rng(T * 31 + E)
    key = _rand(rng, T, E)
    ids = oracle.topk_select(key, k)
    counts, offsets, perm, row_of = oracle.dispatch(ids, E)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[E] == T * k
    assert np.array_equal(np.diff(offsets), counts)
    assert np.array_equal(np.sort(perm), np.arange(T * k))          # bijection
    assert np.array_equal(row_of[perm], np.arange(T * k))           # inverse
    # brute force: rows are the (expert, token, slot) triples in lexicographic order
    triples = sorted((int(ids[t, s]), t, s) for t in range(T) for s in range(k))
    assert perm.tolist() == [t * k + s for _, t, s in triples]
    for e in range(E):
        assert counts[e] == sum(1 for tr in triples if tr[0] == e)


def test_toy_run_tokens_per_expert_sum():
    """[SEV] build: the tokens-per-expert list adds up to 512 tokens x 2 picks."""
    g = json.loads((GOLDEN / "param_counts.json").read_text())["toy_layer"]
    rng = np.random.default_rng(0)
    x = _rand(rng, g["tokens"], g["d_model"])
    wr = _rand(rng, g["n_experts"], g["d_model"], scale=0.125)
    r = oracle.route(x, wr, None, g["top_k"], oracle.SOFTMAX_ALL_RENORM)
    counts, *_ = oracle.dispatch(r.ids, g["n_experts"])
    assert int(counts.sum()) == g["tokens_per_expert_sum"]


# ------------------------------------------------------------------ expert FFN and layer
def test_swiglu_closed_form_fixes_gate_up_order():
    """d = f = 1: y = Wd * SiLU(Wg x) * (Wu x) = -1.5 * SiLU(1) * 6.
    Swapping gate and up would give -1.5 * SiLU(6) * 1 instead."""
    y = oracle.swiglu_expert(np.array([[2.0]]), np.array([[0.5]]), np.array([[3.0]]), np.array([[-1.5]]))
    silu1 = 1.0 / (1.0 + math.exp(-1.0))
    assert y[0, 0] == pytest.approx(-9.0 * silu1, rel=1e-15)
    assert abs(y[0, 0] - (-1.5 * 6.0 / (1.0 + math.exp(-6.0)))) > 1.0


def test_silu_and_sigmoid_special_values():
    assert oracle.silu(np.array([0.0]))[0] == 0.0
    assert oracle.sigmoid(np.array([0.0]))[0] == 0.5
    assert oracle.silu(np.array([40.0]))[0] == pytest.approx(40.0, rel=1e-15)
    assert abs(oracle.silu(np.array([-800.0]))[0]) == 0.0
    assert oracle.silu(np.array([1.0]))[0] == pytest.approx(0.7310585786300049, rel=1e-15)


def test_single_expert_layer_is_a_dense_ffn():
    """E = 1, k = 1 (k = E with one expert): the layer is the dense SwiGLU FFN."""
    rng = np.random.default_rng(8)
    x, wr, wgu, wd = _layer(rng, T=7, d=5, E=1, f=3)
    for mode in MODES:
        y, r, _ = oracle.moe_layer(x, wr, None, 1, mode, _experts(wgu, wd), 1)
        for t in range(7):
            ref = _swiglu_loops(x[t], wgu[0, :3], wgu[0, 3:], wd[0])
            assert y[t].tolist() == pytest.approx(ref, rel=1e-12, abs=1e-13)


def _dense_with_zero_weights(x, wr, bias, k, mode, wgu, wd, bias_select_only=0):
    """[SEV] build: "a slow version that runs every expert with zero weights for
    unpicked ones" -- written here with loops over tokens and all experts."""
    T, d = x.shape
    E = wr.shape[0]
    f = wd.shape[2]
    y = np.zeros_like(x)
    for t in range(T):
        logits = [_dot(x[t], wr[e]) for e in range(E)]
        key = [logits[e] + (0.0 if bias is None else bias[e]) for e in range(E)]
        chosen = [e for _, e in sorted((-key[e], e) for e in range(E))][:k]
        if mode == oracle.SOFTMAX_ALL_RENORM:
            m = max(key)
            p = [math.exp(v - m) for v in key]
            z = sum(p)
            p = [v / z for v in p]
            s = sum(p[e] for e in chosen)
            weight = {e: p[e] / s for e in chosen}
        elif mode == oracle.SOFTMAX_TOPK:
            m = max(key[e] for e in chosen)
            ex = {e: math.exp(key[e] - m) for e in chosen}
            s = sum(ex.values())
            weight = {e: ex[e] / s for e in chosen}
        else:
            sc = logits if bias_select_only else key
            g = {e: 1.0 / (1.0 + math.exp(-sc[e])) for e in chosen}
            s = sum(g.values())
            weight = {e: g[e] / s for e in chosen}
        for e in range(E):
            out = _swiglu_loops(x[t], wgu[e, :f], wgu[e, f:], wd[e])
            w = weight.get(e, 0.0)
            for i in range(d):
                y[t, i] += w * out[i]
    return y


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("k", [1, 2, 5])
def test_expert_loop_equals_dense_with_zero_weights(mode, k):
    """[SEV]: the per-expert loop and the dense zero-weight form match.  With
    k = E = 5 this is also the k = E reduction to sum_e p_e FFN_e(x)."""
    rng = np.random.default_rng(100 + 10 * mode + k)
    x, wr, wgu, wd = _layer(rng, T=6, d=5, E=5, f=3)
    bias = _rand(rng, 5, scale=0.2)
    y, _, _ = oracle.moe_layer(x, wr, bias, k, mode, _experts(wgu, wd), 5, bias_select_only=1,
                               decision_dtype=None)
    ref = _dense_with_zero_weights(x, wr, bias, k, mode, wgu, wd, bias_select_only=1)
    assert np.max(np.abs(y - ref)) <= 1e-12 * max(1.0, np.max(np.abs(ref)))


def test_shared_expert_adds_its_dense_ffn():
    rng = np.random.default_rng(9)
    x, wr, wgu, wd = _layer(rng)
    sg, su, sd = _rand(rng, 4, 6), _rand(rng, 4, 6), _rand(rng, 6, 4)
    y0, _, _ = oracle.moe_layer(x, wr, None, 2, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 5)
    y1, _, _ = oracle.moe_layer(x, wr, None, 2, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 5,
                                shared_weights=[(sg, su, sd)])
    for t in range(x.shape[0]):
        assert (y1[t] - y0[t]).tolist() == pytest.approx(_swiglu_loops(x[t], sg, su, sd), rel=1e-12, abs=1e-13)


def test_forced_routing_reproduces_free_routing():
    rng = np.random.default_rng(11)
    x, wr, wgu, wd = _layer(rng)
    for mode in MODES:
        y, r, w = oracle.moe_layer(x, wr, None, 2, mode, _experts(wgu, wd), 5)
        y2, r2, w2 = oracle.moe_layer(x, wr, None, 2, mode, _experts(wgu, wd), 5, ids=r.ids)
        assert r2 is None and np.array_equal(y, y2) and np.array_equal(w, w2)


def test_token_subsets_are_independent():
    """Token-choice routing is per token, so any subset of tokens gives the same rows."""
    rng = np.random.default_rng(12)
    x, wr, wgu, wd = _layer(rng, T=20)
    y, _, _ = oracle.moe_layer(x, wr, None, 2, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 5)
    sub = [3, 7, 19]
    ys, _, _ = oracle.moe_layer(x[sub], wr, None, 2, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 5)
    assert np.max(np.abs(ys - y[sub])) <= 1e-12 * np.max(np.abs(y))


# ------------------------------------------------------------------ occupancy
def test_occupancy_closed_form_reproduces_printed_table():
    g = json.loads((GOLDEN / "occupancy_table.json").read_text())
    for name, row in g["rows"].items():
        for b, pct in zip(g["batches"], row["percent"]):
            got = 100.0 * oracle.occupancy_closed_form(row["k"], row["experts"], b)
            assert round(got, 1) == pct, (name, b, got)
    wt = g["weights_read_table"]
    for b, pct in zip(wt["batches"], wt["percent"]):
        assert round(100.0 * oracle.occupancy_closed_form(wt["k"], wt["experts"], b), 1) == pct


@pytest.mark.parametrize("k,E,B,draws", [(2, 8, 8, 1_000_000), (2, 8, 4, 1_000_000), (8, 256, 16, 40_000)])
def test_occupancy_monte_carlo_within_page_tolerance(k, E, B, draws):
    g = json.loads((GOLDEN / "occupancy_table.json").read_text())
    tol = g["monte_carlo_tolerance_pp"]
    mc = oracle.occupancy_monte_carlo(k, E, B, draws, seed=B)
    cf = oracle.occupancy_closed_form(k, E, B)
    assert abs(100.0 * (mc - cf)) < tol


# ------------------------------------------------------------------ parameter accounting
def test_parameter_counts_reproduce_the_pages():
    g = json.loads((GOLDEN / "param_counts.json").read_text())
    toy = g["toy_layer"]
    args = (toy["d_model"], toy["d_ff"])
    assert oracle.expert_params(*args, toy["n_matrices"]) == toy["params_per_expert"]
    assert oracle.moe_layer_params(*args, toy["n_experts"], toy["n_matrices"]) == toy["total_params"]
    assert oracle.active_params(*args, toy["n_experts"], toy["top_k"], toy["n_matrices"]) == \
        toy["active_params_per_token"]
    ge = g["gated_expert"]
    assert round(oracle.expert_params(ge["d_model"], ge["d_ff"], ge["n_matrices"]) / 1e6, 1) == \
        ge["params_millions_rounded_1"]
    rs = g["router_size"]
    assert oracle.moe_layer_params(rs["d_model"], 0, rs["n_experts"], 3) == rs["router_weights"]
    ds = g["deepseek_v3_expert"]
    per = oracle.expert_params(ds["d_model"], ds["d_ff"], ds["n_matrices"])
    assert round(per / 1e6) == ds["params_per_expert_millions_rounded_0"]
    assert round(per * ds["layers"] * ds["experts_per_layer"] / 1e9, 1) == ds["all_expert_params_billions_rounded_1"]


def test_brute_force_exhaustive_tiny_routing():
    """Every key ordering of 4 experts (with ties), all k: the selected set is
    the k largest and ties resolve to the lower index."""
    vals = [0.0, 1.0, 1.0, 2.0]
    for keyrow in set(itertools.permutations(vals)):
        key = np.array([keyrow])
        for k in range(1, 5):
            ids = oracle.topk_select(key, k)[0].tolist()
            ranked = sorted(range(4), key=lambda e: (-keyrow[e], e))
            assert ids == ranked[:k]


# ------------------------------------------------------------------ routing without renormalisation
def test_no_renorm_top1_weight_is_the_raw_router_probability():
    """[SEV] "Why top-1 routing cannot renormalise": with k = 1 the chosen expert
    is scaled by its raw router probability.  Reference: a pure-Python softmax
    of each row, its largest entry.  Catches a renormalisation (weight 1) or a
    softmax over the kept score only."""
    rng = np.random.default_rng(41)
    x = _rand(rng, 30, 10)
    wr = _rand(rng, 6, 10, scale=0.8)
    r = oracle.route(x, wr, None, 1, oracle.SOFTMAX_ALL_NO_RENORM, decision_dtype=None)
    for t in range(30):
        l = [_dot(x[t], wr[e]) for e in range(6)]
        m = max(l)
        z = math.fsum(math.exp(v - m) for v in l)
        assert abs(r.w[t, 0] - max(math.exp(v - m) / z for v in l)) <= 1e-14
        assert r.w[t, 0] < 1.0


@pytest.mark.parametrize("k", [1, 2, 3, 6])
def test_no_renorm_weights_are_the_unscaled_renorm_weights(k):
    """[TOK] keeps the softmax probabilities as they are; [SEV] divides them by
    their sum.  So the no-renormalisation weights, divided by their sum, are the
    renormalised ones; their sum is at most 1 and exactly 1 at k = E."""
    rng = np.random.default_rng(50 + k)
    x = _rand(rng, 40, 8)
    wr = _rand(rng, 6, 8)
    bias = _rand(rng, 6, scale=0.5)
    a = oracle.route(x, wr, bias, k, oracle.SOFTMAX_ALL_NO_RENORM)
    b = oracle.route(x, wr, bias, k, oracle.SOFTMAX_ALL_RENORM)
    assert np.array_equal(a.ids, b.ids)
    s = a.w.sum(axis=1)
    assert np.max(np.abs(a.w / s[:, None] - b.w)) <= 1e-14
    assert np.all(s <= 1.0 + 1e-15)
    if k == 6:
        assert np.max(np.abs(s - 1.0)) <= 1e-14
    else:
        assert np.all(s < 1.0)


# ------------------------------------------------------------------ capacity factor and token dropping
def test_capacity_reproduces_the_page_cases():
    """[SEV] capacity script on the page's printed tokens-per-expert line."""
    g = json.loads((GOLDEN / "capacity_and_balance.json").read_text())
    run = g["toy_run_counts"]
    counts = np.array(run["tokens_per_expert"])
    assert counts.sum() == run["tokens"] * run["top_k"]
    for c in g["capacity_cases"]["cases"]:
        cap = oracle.expert_capacity(run["tokens"], run["top_k"], run["n_experts"], c["factor"])
        assert cap == c["capacity"]
        assert oracle.dropped_slots(counts, cap) == c["dropped"]


def test_capacity_rounds_up_not_down():
    """ceil, not floor or round: 10 tokens x 1 / 3 experts x 1.0 = 3.33 -> 4."""
    assert oracle.expert_capacity(10, 1, 3, 1.0) == 4
    assert oracle.expert_capacity(9, 1, 3, 1.0) == 3
    assert oracle.expert_capacity(8, 2, 8, 1.5) == 3


@pytest.mark.parametrize("T,E,k,cap", [(40, 4, 2, 13), (57, 8, 3, 9), (25, 5, 5, 25), (30, 3, 1, 4), (12, 6, 2, 0)])
def test_capacity_dispatch_keeps_the_first_arrivals(T, E, k, cap):
    """Brute force: per expert, list its (token, slot) assignments in token
    order and keep the first ``cap``.  Catches keeping the last arrivals,
    ranking by slot instead of token, or offsets built from the raw counts."""
    rng = np.random.default_rng(T * 100 + cap)
    ids = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int64)
    counts, offsets, perm, row_of = oracle.dispatch(ids, E, cap)
    kept_rows = []
    for e in range(E):
        mine = [t * k + s for t in range(T) for s in range(k) if ids[t, s] == e]
        assert counts[e] == len(mine)
        kept_rows += mine[:cap]
        for i in mine[cap:]:
            assert row_of[i] == -1
    assert list(perm) == kept_rows
    assert offsets[-1] == len(kept_rows) == T * k - oracle.dropped_slots(counts, cap)
    for r, i in enumerate(perm):
        assert row_of[i] == r


def test_capacity_layer_drops_expert_updates_and_keeps_other_weights():
    """A dropped slot adds nothing; the token's other slots keep their weights
    ([SEV]: a skipped token simply gets no expert update in that layer).
    Reference: per-token loops over the kept slots."""
    rng = np.random.default_rng(7)
    x, wr, wgu, wd = _layer(rng, T=12, d=5, E=3, f=4)
    k, cap = 2, 5
    y, r, w = oracle.moe_layer(x, wr, None, k, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 3, capacity=cap)
    _, _, _, row_of = oracle.dispatch(r.ids, 3, cap)
    f = wd.shape[2]
    for t in range(12):
        ref = [0.0] * 5
        for s in range(k):
            if row_of[t * k + s] < 0:
                continue
            e = int(r.ids[t, s])
            o = _swiglu_loops(list(x[t]), wgu[e, :f].tolist(), wgu[e, f:].tolist(), wd[e].tolist())
            ref = [a + w[t, s] * b for a, b in zip(ref, o)]
        assert np.max(np.abs(y[t] - np.array(ref))) <= 1e-12
    assert np.any(row_of < 0)  # the case does drop something


def test_capacity_at_or_above_the_batch_is_dropless():
    rng = np.random.default_rng(8)
    x, wr, wgu, wd = _layer(rng, T=20, d=6, E=4, f=3)
    a, *_ = oracle.moe_layer(x, wr, None, 2, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 4)
    b, *_ = oracle.moe_layer(x, wr, None, 2, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 4, capacity=20)
    assert np.array_equal(a, b)


# ------------------------------------------------------------------ two-matrix GELU expert
def test_gelu_special_values():
    """GELU(z) = z * Phi(z): Phi(1) = 0.841344746068543 (normal table), GELU(0) = 0,
    GELU(z) - GELU(-z) = z, GELU(z) -> z for large z and -> 0 for very negative z.
    Catches the tanh approximation (GELU(1) = 0.841192) or a missing 1/2."""
    g = oracle.gelu(np.array([1.0, 0.0, 2.5, -2.5, 30.0, -30.0]))
    assert abs(g[0] - 0.8413447460685429) <= 1e-15
    assert g[1] == 0.0
    assert abs((g[2] - g[3]) - 2.5) <= 1e-15
    assert g[4] == 30.0 and abs(g[5]) < 1e-150


def test_gelu_single_expert_layer_is_the_pages_two_matrix_ffn():
    """E = 1, k = 1: the layer is [SEV]'s Expert, down(GELU(up(x))), written here
    with loops and math.erf."""
    rng = np.random.default_rng(9)
    T, d, f = 7, 5, 6
    x = _rand(rng, T, d)
    wup = _rand(rng, f, d, scale=0.6)
    wdn = _rand(rng, d, f, scale=0.6)
    y, _, _ = oracle.moe_layer(x, _rand(rng, 1, d), None, 1, oracle.SOFTMAX_TOPK, lambda e: (wup, wdn), 1,
                               act=oracle.ACT_GELU)
    for t in range(T):
        h = []
        for j in range(f):
            z = _dot(x[t], wup[j])
            h.append(0.5 * z * (1.0 + math.erf(z / math.sqrt(2.0))))
        ref = [_dot(h, wdn[i]) for i in range(d)]
        assert np.max(np.abs(y[t] - np.array(ref))) <= 1e-12


# ------------------------------------------------------------------ router penalties
def test_balance_loss_page_bounds():
    """[SEV]: N * sum f_i P_i is 1 for an even split and N (8.0) when every
    token goes to one expert with top-1 and certainty."""
    g = json.loads((GOLDEN / "capacity_and_balance.json").read_text())["balance_loss_bounds"]
    even = oracle.balance_loss(np.zeros((64, 8)), np.full(8, 16))
    assert abs(even - g["even"]) <= 1e-15
    peaked = np.full((64, 8), -1000.0)
    peaked[:, 3] = 0.0
    counts = np.zeros(8)
    counts[3] = 64
    assert abs(oracle.balance_loss(peaked, counts) - g["all_to_one_top1_n8"]) <= 1e-12


def test_balance_loss_brute_force():
    """Loops: f_i from the slot counts, P_i the mean of each token's softmax row."""
    rng = np.random.default_rng(12)
    l = _rand(rng, 20, 5, scale=2.0)
    counts = np.array([7, 0, 13, 9, 11])
    tot = 0.0
    for i in range(5):
        p_i = math.fsum(math.exp(l[t, i]) / math.fsum(math.exp(v) for v in l[t]) for t in range(20)) / 20
        tot += counts[i] / counts.sum() * p_i
    assert abs(oracle.balance_loss(l, counts) - 5 * tot) <= 1e-14


def test_router_z_loss_closed_forms():
    """Equal logits c: log-sum-exp = c + ln E, so the loss is (c + ln E)^2;
    a shift by c does not leave it unchanged (unlike softmax)."""
    assert abs(oracle.router_z_loss(np.zeros((9, 8))) - math.log(8) ** 2) <= 1e-14
    assert abs(oracle.router_z_loss(np.full((3, 4), 2.0)) - (2.0 + math.log(4)) ** 2) <= 1e-13
    l = np.array([[0.0, math.log(3.0)], [1.0, 1.0]])
    ref = (math.log(1 + 3) ** 2 + (1 + math.log(2)) ** 2) / 2
    assert abs(oracle.router_z_loss(l) - ref) <= 1e-14


# ------------------------------------------------------------------ FP8 E4M3 quantisation
def _e4m3_table():
    """All finite E4M3 values from the bit layout (sign, 4-bit exponent with
    bias 7, 3-bit mantissa, subnormals at exponent 0, NaN at S.1111.111)."""
    vals = []
    for code in range(256):
        v = oracle.e4m3_decode(code)
        if not math.isnan(v):
            vals.append(v)
    return np.array(sorted(set(vals)))


def test_e4m3_decode_landmarks():
    """448 largest finite, 2^-9 smallest subnormal, 2^-6 smallest normal, 1.0 = 0x38."""
    assert oracle.e4m3_decode(0x7E) == 448.0 and math.isnan(oracle.e4m3_decode(0x7F))
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9 and oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x38) == 1.0 and oracle.e4m3_decode(0xB8) == -1.0
    assert len(_e4m3_table()) == 253  # 254 finite codes, +0 and -0 equal


def test_e4m3_round_is_nearest_representable_ties_to_even():
    """Brute force against the decoded table: every value maps to its nearest
    representable neighbour, midpoints to the one with an even mantissa, the
    table onto itself, and anything beyond 448 saturates."""
    table = _e4m3_table()
    assert np.array_equal(oracle.e4m3_round(table), table)
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(4000) * 10.0, rng.standard_normal(2000) * 0.01,
                        (table[1:] + table[:-1]) / 2])       # every midpoint
    got = oracle.e4m3_round(v)
    for x, g in zip(v, got):
        d = np.abs(table - x)
        near = table[d == d.min()]
        if x > 448.0 or x < -448.0:
            assert g == np.sign(x) * 448.0
        elif len(near) == 1:
            assert g == near[0], x
        else:  # a tie: the even mantissa (its code has bit 0 clear)
            even = [t for t in near if int(round(abs(t) / _ulp(abs(t)))) % 2 == 0]
            assert g == even[0], (x, near)


def _ulp(a: float) -> float:
    if a < 2.0 ** -6:
        return 2.0 ** -9
    return 2.0 ** (math.floor(math.log2(a)) - 3)


def test_quantize_rows_reconstructs_within_half_a_step():
    """x ~ q * s with |x - q s| <= half an E4M3 step of x / s; the row's largest
    magnitude maps to exactly 448; a zero row gets scale 1."""
    rng = np.random.default_rng(5)
    x = rng.standard_normal((20, 300)).astype(np.float32)
    x[3] = 0.0
    q, s = oracle.quantize_rows_e4m3(x)
    assert s[3] == 1.0 and np.all(q[3] == 0.0)
    for r in range(20):
        if r == 3:
            continue
        assert np.max(np.abs(q[r])) == 448.0
        y = x[r].astype(np.float64) / s[r]
        for a, b in zip(y, q[r]):
            assert abs(a - b) <= 0.5 * _ulp(abs(a)) * (1 + 1e-6) + 1e-12


def test_round_bf16_is_nearest_of_the_two_neighbours():
    """Brute force: the bf16 result is the closer of the two bf16 values around
    the float32 value (ties to the one whose last mantissa bit is 0)."""
    rng = np.random.default_rng(11)
    v = np.concatenate([rng.standard_normal(3000), np.array([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -2.5])])
    got = oracle.round_bf16(v)
    for x, g in zip(v.astype(np.float32).astype(np.float64), got):
        m, e = math.frexp(abs(x))            # |x| = m 2^e, m in [0.5, 1)
        step = 2.0 ** (e - 8)                # bf16 keeps 8 significant bits
        lo = math.floor(abs(x) / step) * step
        hi = lo + step
        if abs(x) - lo < hi - abs(x):
            want = lo
        elif abs(x) - lo > hi - abs(x):
            want = hi
        else:
            want = lo if int(lo / step) % 2 == 0 else hi
        assert g == math.copysign(want, x), (x, g, want)


def _e4m3_layer_inputs(rng, n=6, d=40, f=24):
    x = rng.standard_normal((n, d))
    wg = rng.standard_normal((f, d)) / np.sqrt(d)
    wu = rng.standard_normal((f, d)) / np.sqrt(d)
    wd = rng.standard_normal((d, f)) / np.sqrt(f)
    return x, (wg, wu, wd)


def test_e4m3_expert_scales_are_per_token_and_per_output_channel():
    """Changing one token row leaves the other rows' outputs bit-identical (no
    per-tensor activation scale); scaling one down-projection row by 2^k
    scales exactly that output column by 2^k (its codes are unchanged, only
    its scale moves) and leaves the others bit-identical (no per-input-column
    weight scale)."""
    rng = np.random.default_rng(21)
    x, (wg, wu, wd) = _e4m3_layer_inputs(rng)
    base = oracle.e4m3_expert(x, (wg, wu, wd), oracle.ACT_SWIGLU)
    x2 = x.copy()
    x2[2] *= 37.0
    y2 = oracle.e4m3_expert(x2, (wg, wu, wd), oracle.ACT_SWIGLU)
    assert np.array_equal(np.delete(y2, 2, axis=0), np.delete(base, 2, axis=0))
    wd2 = wd.copy()
    wd2[5] *= 8.0
    y3 = oracle.e4m3_expert(x, (wg, wu, wd2), oracle.ACT_SWIGLU)
    assert np.array_equal(y3[:, 5], 8.0 * base[:, 5])
    assert np.array_equal(np.delete(y3, 5, axis=1), np.delete(base, 5, axis=1))


@pytest.mark.parametrize("act", [0, 1])
def test_e4m3_expert_stays_close_to_the_float_expert(act):
    """Each quantised operand is within half an E4M3 step (2^-4 relative) of the
    float one, so the expert output stays within a few percent of the float
    expert; a wrong scale (e.g. s instead of 1/s) would be off by orders."""
    rng = np.random.default_rng(30 + act)
    x, (wg, wu, wd) = _e4m3_layer_inputs(rng, n=16, d=256, f=128)
    if act == 0:
        ref = oracle.swiglu_expert(x, wg, wu, wd)
        got = oracle.e4m3_expert(x, (wg, wu, wd), act)
    else:
        ref = oracle.gelu_expert(x, wu, wd)
        got = oracle.e4m3_expert(x, (wu, wd), act)
    err = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    assert 1e-4 < err < 0.08


# ------------------------------------------------------------------ combine
def test_combine_of_dispatched_rows_equals_the_per_token_sum():
    """oracle.combine against the pages' per-token definition written with
    plain loops here: each token adds weight x its expert's output for that
    token (the rows sit wherever the dispatch put them), plus the shared
    output.  Catches a transposed (t, s) index, a dropped slot that still adds,
    or a missing shared term."""
    rng = np.random.default_rng(11)
    T, k, d, E = 13, 3, 5, 6
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    w = rng.random((T, k))
    _, _, perm, row_of = oracle.dispatch(ids, E, capacity=2)   # some slots dropped
    y_rows = _rand(rng, len(perm), d)
    ys = _rand(rng, T, d)
    got = oracle.combine(y_rows, row_of, w, ys)
    for t in range(T):
        want = list(ys[t])
        for s in range(k):
            r = int(row_of[t * k + s])
            if r < 0:
                continue
            assert perm[r] == t * k + s
            for j in range(d):
                want[j] += w[t, s] * y_rows[r, j]
        assert np.allclose(got[t], want, rtol=0, atol=1e-12)
    assert np.any(row_of < 0)


def test_combine_of_expert_rows_reproduces_the_layer():
    """Dispatching a small layer, running each expert on its rows and
    combining gives the per-expert-loop layer output (both fp64)."""
    rng = np.random.default_rng(12)
    x, wr, wgu, wd = _layer(rng, T=11, d=6, E=5, f=4)
    k = 2
    y, r, w = oracle.moe_layer(x, wr, None, k, oracle.SOFTMAX_TOPK, _experts(wgu, wd), 5)
    _, _, perm, row_of = oracle.dispatch(r.ids, 5)
    f = wd.shape[2]
    y_rows = np.stack([oracle.swiglu_expert(x[p // k][None], wgu[r.ids[p // k, p % k], :f],
                                            wgu[r.ids[p // k, p % k], f:], wd[r.ids[p // k, p % k]])[0]
                       for p in perm])
    assert np.allclose(oracle.combine(y_rows, row_of, w), y, rtol=0, atol=1e-12)


# ------------------------------------------------------------------ 8-bit expert, independent evaluation
def _e4m3_values_from_bits():
    """Every finite E4M3 value, built here from the format's bit layout
    (sign, four exponent bits with bias 7, three mantissa bits, exponent 0
    subnormal, S.1111.111 reserved for NaN), with its code."""
    out = []
    for code in range(256):
        e, m = (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue
        mag = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        out.append((-mag if code & 0x80 else mag, code))
    return out


_E4M3 = _e4m3_values_from_bits()


def _nearest_e4m3(y: float) -> float:
    """Exhaustive nearest E4M3 value; a tie goes to the even code (mantissa
    LSB 0); beyond the largest value saturate."""
    best = min(_E4M3, key=lambda vc: (abs(vc[0] - y), vc[1] & 1, vc[1]))
    return best[0]


def _bf16_round(v: float) -> float:
    import struct
    f = struct.unpack("<f", struct.pack("<f", v))[0]            # to float32, nearest even
    b = struct.unpack("<I", struct.pack("<f", f))[0]
    lo = b & 0xFFFF
    b >>= 16
    if lo > 0x8000 or (lo == 0x8000 and (b & 1)):
        b += 1
    return struct.unpack("<f", struct.pack("<I", (b & 0xFFFF) << 16))[0]


def _quant_rows_python(rows):
    """Per-row absolute-max quantisation written out: the scale and the
    division in float32 (the precision the method decides in), then the
    exhaustive nearest code; returns the dequantised rows."""
    out = []
    for row in rows:
        r32 = [float(np.float32(v)) for v in row]
        amax = max(abs(v) for v in r32)
        s = float(np.float32(amax) / np.float32(448.0)) if amax > 0 else 1.0
        out.append([_nearest_e4m3(float(np.float32(v) / np.float32(s))) * s for v in r32])
    return out


def _e4m3_swiglu_python(x, wg, wu, wd):
    xd, gd, ud, dd = (_quant_rows_python(m) for m in (x, wg, wu, wd))
    out = []
    for xv in xd:
        h = []
        for j in range(len(gd)):
            g = math.fsum(a * b for a, b in zip(xv, gd[j]))
            u = math.fsum(a * b for a, b in zip(xv, ud[j]))
            h.append(_bf16_round(g / (1.0 + math.exp(-g)) * u))
        hd = _quant_rows_python([h])[0]
        out.append([math.fsum(a * b for a, b in zip(hd, dd[i])) for i in range(len(dd))])
    return np.array(out)


def test_e4m3_expert_equals_a_pure_python_evaluation_of_the_scheme():
    """oracle.e4m3_expert against the 8-bit scheme written out independently:
    an E4M3 table from the format's bit layout, exhaustive nearest-value
    rounding, per-row float32 scales, exact sums, h stored as bf16 and
    re-quantised per row.  Catches a scale applied on the wrong side, a
    missing bf16 rounding of h, a per-column instead of per-row scale, or a
    wrong tie rule."""
    rng = np.random.default_rng(21)
    n, d, f = 3, 16, 8
    x = rng.standard_normal((n, d)).astype(np.float32).astype(np.float64)
    wg = (rng.standard_normal((f, d)) / 4).astype(np.float32).astype(np.float64)
    wu = (rng.standard_normal((f, d)) / 4).astype(np.float32).astype(np.float64)
    wd = (rng.standard_normal((d, f)) / 3).astype(np.float32).astype(np.float64)
    got = oracle.e4m3_expert(x, (wg, wu, wd), oracle.ACT_SWIGLU)
    want = _e4m3_swiglu_python(x.tolist(), wg.tolist(), wu.tolist(), wd.tolist())
    assert np.allclose(got, want, rtol=1e-9, atol=1e-12)
    # and it is not the float expert: quantisation moves the output
    assert not np.allclose(got, oracle.swiglu_expert(x, wg, wu, wd), rtol=1e-4)
