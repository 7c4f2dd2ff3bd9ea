"""Plain, slow, obviously correct CPU statement of the sparse MoE layer forward.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path imports, calls or
links this module: the CUDA library under ``top_routing_expert_gemm_b200``
must never fall back to it.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg use it.  It shares no code with
the CUDA path; the only common dependency is the seeded input generator
(``synth``), which holds none of the layer's arithmetic.

Everything is float64 numpy.  Stored inputs (float32 or bfloat16 values) are
upcast exactly, then the layer is evaluated with no intermediate rounding.
Library primitives used as single steps: ``@`` (matrix product), ``np.exp``,
``np.argsort(kind="stable")``.

Sources (page title, then section):

* [TOK] "Mixture of Experts (MoE): routing, expert parallelism, and memory"
  (docs.tokios.com) -- "How does MoE routing work", "Shared experts".
* [TUR] "Mixture of Experts: why a model with 671 billion parameters uses only
  37" (turinginstitut.cz) -- "The router: how a token chooses experts" (the
  pseudo-PyTorch MoE layer), "How many experts to pick and how to score them:
  top-k, softmax, sigmoid", "The problem learned routing brings: load
  balancing", "Shared expert and fine-grained experts".
* [AFD] "Mixture of experts: how MoE works and what it costs"
  (aifordevs.org) -- "What mixture of experts means in an LLM", "Why load
  balancing is the hard part of MoE", "How batching changes the mixture of
  experts math" (occupancy closed form and its table), "Loaded versus active
  parameters in open-weight MoE models".
* [SEV] "Mixture of Experts Explained: Routers, Active Parameters and VRAM"
  (sevydevy.in) -- the five router steps (Score, Normalise, Keep the top k,
  Renormalise, Run and combine), the runnable top-k MoE build, "Softmax
  before or after the top-k step", "Why top-1 routing cannot renormalise".

Readings where the pages are silent (each also listed in the design notes):

* SwiGLU expert.  [SEV] only says "a gated feed-forward block with three
  matrices".  Read as ``o = (SiLU(x Wg^T) * (x Wu^T)) Wd^T`` with
  ``SiLU(z) = z / (1 + e^-z)``; in the stacked ``w_gate_up[e]`` of shape
  ``[2f, d]`` the first f rows are Wg, the next f rows Wu.
* Selection compares ``kappa = logit + bias`` (logit units).  Softmax and
  sigmoid are strictly increasing, so the selected set is the one the
  probabilities give in exact arithmetic; ties go to the lower expert index
  and slots are ordered by descending kappa.
* The top-k decision is taken in float32 (``decision_dtype``), the
  precision the CUDA kernels compare in, because the pages fix none.
* Bias: softmax rules add it to the logits (it moves both selection and
  weights); the sigmoid rule with ``bias_select_only`` uses it for
  selection only ([AFD] "Why load balancing...": the bias shifts routing
  without distorting the gate values used for output).
* The output is the MoE sublayer alone (no residual), dropless, and shared
  experts enter with weight 1.

Parity is pinned by ``tests/test_oracle_pins.py`` against closed forms, the
pages' printed numbers and brute force; see each function's docstring.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Sequence

import numpy as np

SOFTMAX_ALL_RENORM = 0
SOFTMAX_TOPK = 1
SIGMOID_TOPK_RENORM = 2

__all__ = [
    "SOFTMAX_ALL_RENORM", "SOFTMAX_TOPK", "SIGMOID_TOPK_RENORM",
    "router_logits", "selection_key", "topk_select", "topk_gap", "softmax", "sigmoid",
    "gate_weights", "Routing", "route", "dispatch", "silu", "swiglu_expert", "moe_layer",
    "occupancy_closed_form", "occupancy_monte_carlo", "expert_params", "moe_layer_params",
    "active_params",
]


# ---------------------------------------------------------------- router
def router_logits(x: np.ndarray, w_router: np.ndarray) -> np.ndarray:
    """Step "Score" of [SEV] and [TUR] "The router": one linear layer without
    bias, ``l[t, e] = sum_i x[t, i] * W_r[e, i]``  (x: [T, d], W_r: [E, d])."""
    return np.asarray(x, dtype=np.float64) @ np.asarray(w_router, dtype=np.float64).T


def selection_key(logits: np.ndarray, bias: np.ndarray | None) -> np.ndarray:
    """kappa = logits + per-expert bias ([TUR] load balancing: a small bias is
    added to each expert's score).  ``bias=None`` means zero bias."""
    if bias is None:
        return np.array(logits, dtype=np.float64, copy=True)
    return logits + np.asarray(bias, dtype=np.float64)[None, :]


def topk_select(key: np.ndarray, k: int) -> np.ndarray:
    """Step "Keep the top k" of [SEV]: per row the k largest keys, slots in
    descending key order, equal keys resolved towards the lower index.
    A stable ascending sort of ``-key`` gives exactly that order."""
    order = np.argsort(-key, axis=1, kind="stable")
    return order[:, :k].astype(np.int64)


def topk_gap(key: np.ndarray, k: int) -> np.ndarray:
    """``key_(k) - key_(k+1)`` per row (the margin by which the k-th expert
    beat the first excluded one); ``inf`` when k equals the expert count."""
    E = key.shape[1]
    if k >= E:
        return np.full(key.shape[0], np.inf)
    s = -np.sort(-key, axis=1)
    return s[:, k - 1] - s[:, k]


def softmax(v: np.ndarray, axis: int = -1) -> np.ndarray:
    """exp(v - max) / sum exp(v - max): positive, sums to 1 ([SEV] step "Normalise")."""
    m = np.max(v, axis=axis, keepdims=True)
    e = np.exp(v - m)
    return e / np.sum(e, axis=axis, keepdims=True)


def sigmoid(v: np.ndarray) -> np.ndarray:
    """1 / (1 + e^-v), an independent score in (0, 1) per expert ([TUR] sigmoid gating)."""
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-v))


def gate_weights(logits: np.ndarray, bias: np.ndarray | None, ids: np.ndarray, gating: int,
                 bias_select_only: int = 0) -> np.ndarray:
    """Routing weights of the selected experts, ``w[t, s]`` for ``ids[t, s]``.

    * SOFTMAX_ALL_RENORM -- [SEV] steps 2-4: softmax over all E experts of
      kappa, keep the selected probabilities, divide by their sum.
    * SOFTMAX_TOPK -- [TUR] pseudo-PyTorch layer and [AFD] (Mixtral: "a
      softmax over those two scores"): softmax over the k selected kappas.
    * SIGMOID_TOPK_RENORM -- [TUR] sigmoid gating: g = sigmoid(score) per
      expert, only the selected set is normalised.  With
      ``bias_select_only`` the score is the raw logit (bias steers selection
      only), else kappa.
    """
    T, k = ids.shape
    key = selection_key(logits, bias)
    rows = np.arange(T)[:, None]
    if gating == SOFTMAX_ALL_RENORM:
        p = softmax(key, axis=1)
        sel = p[rows, ids]
        return sel / sel.sum(axis=1, keepdims=True)
    if gating == SOFTMAX_TOPK:
        sel = key[rows, ids]
        return softmax(sel, axis=1)
    if gating == SIGMOID_TOPK_RENORM:
        score = logits if bias_select_only else key
        g = sigmoid(score)[rows, ids]
        return g / g.sum(axis=1, keepdims=True)
    raise ValueError(f"unknown gating rule {gating}")


@dataclasses.dataclass
class Routing:
    ids: np.ndarray        # [T, k] int64, slots in descending key order
    w: np.ndarray          # [T, k] float64 routing weights
    logits: np.ndarray     # [T, E] float64
    key: np.ndarray        # [T, E] float64 selection key (logits + bias)
    gap: np.ndarray        # [T] float64 key_(k) - key_(k+1)


def route(x: np.ndarray, w_router: np.ndarray, bias: np.ndarray | None, k: int, gating: int,
          bias_select_only: int = 0, decision_dtype=np.float32) -> Routing:
    """Router logits, top-k selection and gate weights for every token.

    The selection key is rounded to ``decision_dtype`` before the top-k
    comparison (float32: the precision the kernels decide in; ``None`` keeps
    float64).  The near-tie gap is measured on the float64 key.
    """
    logits = router_logits(x, w_router)
    key = selection_key(logits, bias)
    dkey = key if decision_dtype is None else key.astype(decision_dtype).astype(np.float64)
    ids = topk_select(dkey, k)
    w = gate_weights(logits, bias, ids, gating, bias_select_only)
    return Routing(ids=ids, w=w, logits=logits, key=key, gap=topk_gap(key, k))


# ---------------------------------------------------------------- dispatch
def dispatch(ids: np.ndarray, n_experts: int):
    """Group the T*k (token, slot) assignments by expert, dropless.

    [TUR] "How data centres handle it": tokens are grouped by their assigned
    expert; [TUR] "Capacity factor": dropless means each expert gets exactly
    as many rows as the router assigned to it.  A plain counting sort over
    the assignments in order i = t*k + s gives, per expert in ascending
    order, its assignments in ascending token order:

    counts[e]   number of rows of expert e          ([SEV] tokens per expert)
    offsets     exclusive scan of counts, offsets[E] = T*k
    perm[row]   = t*k + s, the assignment stored at that row
    row_of[i]   = row of assignment i (inverse of perm)
    """
    T, k = ids.shape
    flat = ids.reshape(-1)
    counts = np.zeros(n_experts, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    for e in range(n_experts):
        offsets[e + 1] = offsets[e] + counts[e]
    cursor = offsets[:-1].copy()
    perm = np.empty(T * k, dtype=np.int64)
    row_of = np.empty(T * k, dtype=np.int64)
    for i, e in enumerate(flat):
        r = cursor[e]
        cursor[e] += 1
        perm[r] = i
        row_of[i] = r
    return counts, offsets, perm, row_of


# ---------------------------------------------------------------- experts
def silu(z: np.ndarray) -> np.ndarray:
    """SiLU(z) = z / (1 + e^-z) (the "Swish" gate of a SwiGLU block)."""
    with np.errstate(over="ignore"):
        return z / (1.0 + np.exp(-z))


def swiglu_expert(xr: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """Gated three-matrix expert FFN ([SEV]: "a gated feed-forward block with
    three matrices"), read as ``(SiLU(x Wg^T) * (x Wu^T)) Wd^T``.

    xr [n, d], w_gate/w_up [f, d], w_down [d, f]  ->  [n, d]."""
    g = xr @ w_gate.T
    u = xr @ w_up.T
    return (silu(g) * u) @ w_down.T


ExpertWeights = Callable[[int], tuple[np.ndarray, np.ndarray, np.ndarray]]


def moe_layer(x: np.ndarray, w_router: np.ndarray | None, bias: np.ndarray | None, k: int, gating: int,
              expert_weights: ExpertWeights, n_experts: int,
              shared_weights: Sequence[tuple[np.ndarray, np.ndarray, np.ndarray]] = (),
              bias_select_only: int = 0, ids: np.ndarray | None = None,
              decision_dtype=np.float32) -> tuple[np.ndarray, Routing | None, np.ndarray]:
    """Sparse MoE sublayer output for the tokens ``x`` [T, d].

    Router -> top-k -> per-expert loop -> weighted sum, as in [TUR]'s
    pseudo-PyTorch layer and [SEV]'s runnable build: every expert computes
    only over the rows the router assigned to it, and adds its output scaled
    by that row's routing weight.  Shared experts ([TOK] "Shared experts";
    [TUR] "Shared expert and fine-grained experts") see every token, weight 1.

    ``expert_weights(e)`` returns float64 ``(W_gate [f,d], W_up [f,d], W_down [d,f])``.

    Forced routing: when ``ids`` is given the selection is taken from it and
    only the gate weights and expert outputs are recomputed (``w_router``
    still supplies the logits the weights need).

    Returns ``(y, routing, w)``; ``routing`` is None under forced routing.
    """
    x = np.asarray(x, dtype=np.float64)
    T = x.shape[0]
    if ids is None:
        r = route(x, w_router, bias, k, gating, bias_select_only, decision_dtype)
        ids_, w = r.ids, r.w
    else:
        r = None
        ids_ = np.asarray(ids, dtype=np.int64)
        w = gate_weights(router_logits(x, w_router), bias, ids_, gating, bias_select_only)
    y = np.zeros_like(x)
    for e in range(n_experts):
        rows, slots = np.nonzero(ids_ == e)
        if rows.size == 0:
            continue
        wg, wu, wd = expert_weights(e)
        y[rows] += w[rows, slots][:, None] * swiglu_expert(x[rows], wg, wu, wd)
    for wg, wu, wd in shared_weights:
        y += swiglu_expert(x, wg, wu, wd)
    return y, r, w


# ---------------------------------------------------------------- occupancy
def occupancy_closed_form(k: int, n_experts: int, batch: int) -> float:
    """[AFD] "How batching changes the mixture of experts math": with uniform
    routing each expert is missed by one token with probability 1 - k/E, so
    the expected share touched by at least one of B tokens is 1 - (1-k/E)^B."""
    return 1.0 - (1.0 - k / n_experts) ** batch


def occupancy_monte_carlo(k: int, n_experts: int, batch: int, draws: int, seed: int = 0,
                          chunk: int = 4096) -> float:
    """Mean share of experts touched when each of ``batch`` tokens routes to
    the top k of E independent uniform random scores, i.e. a uniformly random
    k-subset ([AFD]: the Monte Carlo cross-check with random top-k routing)."""
    rng = np.random.default_rng(seed)
    touched = 0
    done = 0
    while done < draws:
        n = min(chunk, draws - done)
        scores = rng.random((n, batch, n_experts))
        picks = np.argsort(-scores, axis=2)[:, :, :k]           # [n, B, k]
        used = np.zeros((n, n_experts), dtype=bool)
        for b in range(batch):
            np.put_along_axis(used, picks[:, b, :], True, axis=1)
        touched += int(used.sum())
        done += n
    return touched / (draws * n_experts)


# ---------------------------------------------------------------- parameter accounting
def expert_params(d_model: int, d_ff: int, n_matrices: int) -> int:
    """Weights of one expert: n_matrices matrices of d_model x d_ff, no biases
    ([SEV] "Check the numbers by hand"; three for the gated block)."""
    return n_matrices * d_model * d_ff


def moe_layer_params(d_model: int, d_ff: int, n_experts: int, n_matrices: int, n_shared: int = 0,
                     d_ff_shared: int = 0) -> int:
    """All weights of one MoE layer: E routed experts, shared experts and the
    E x d router ([SEV]: eight experts plus a 64 x 8 router)."""
    return (n_experts * expert_params(d_model, d_ff, n_matrices)
            + n_shared * expert_params(d_model, d_ff_shared, n_matrices)
            + n_experts * d_model)


def active_params(d_model: int, d_ff: int, n_experts: int, k: int, n_matrices: int, n_shared: int = 0,
                  d_ff_shared: int = 0) -> int:
    """Weights one token touches: the router, its k experts and the shared ones."""
    return (n_experts * d_model + k * expert_params(d_model, d_ff, n_matrices)
            + n_shared * expert_params(d_model, d_ff_shared, n_matrices))

