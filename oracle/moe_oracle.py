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
``np.log``, ``scipy.special.erf``, ``np.argsort(kind="stable")``.

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
* The output is the MoE sublayer alone (no residual), dropless unless a
  capacity is given, and shared experts enter with weight 1.
* Capacity: ceil(T*k/E * factor) rows per expert ([SEV]'s script counts
  routing slots); an expert keeps its first arrivals in token order (the
  pages say only that the tokens past the capacity go without that expert); a dropped
  slot adds nothing and the token's other weights are not rescaled.
* Balance loss and z-loss are computed from the bias-free router logits
  (the pages define them on the router's own output) and returned without
  their loss weights (alpha = 0.01, 0.001 on the pages); the balance loss
  counts routing slots before any capacity cut, and the z-loss is the mean
  over tokens of the squared log-sum-exp.
* Two-matrix expert: [SEV]'s build, ``GELU(x W_up^T) W_down^T`` with the exact
  (erf) GELU, its library default.

Parity is pinned by ``tests/test_oracle_pins.py`` against closed forms, the
pages' printed numbers and brute force; see each function's docstring.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Sequence

import numpy as np

SOFTMAX_ALL_RENORM = 0
SOFTMAX_TOPK = 1
SIGMOID_TOPK_RENORM = 2
SOFTMAX_ALL_NO_RENORM = 3

ACT_SWIGLU = 0   # gated expert, three matrices (w_gate_up [2f, d], w_down [d, f])
ACT_GELU = 1     # plain expert, two matrices (w_up [f, d], w_down [d, f])

__all__ = [
    "SOFTMAX_ALL_RENORM", "SOFTMAX_TOPK", "SIGMOID_TOPK_RENORM", "SOFTMAX_ALL_NO_RENORM",
    "ACT_SWIGLU", "ACT_GELU", "gelu", "gelu_expert", "expert_capacity", "dropped_slots",
    "balance_loss", "router_z_loss", "logsumexp", "E4M3_MAX", "e4m3_round", "e4m3_decode",
    "quantize_rows_e4m3", "round_bf16", "e4m3_expert",
    "router_logits", "selection_key", "topk_select", "topk_gap", "softmax", "sigmoid",
    "gate_weights", "Routing", "route", "dispatch", "silu", "swiglu_expert", "moe_layer",
    "combine", "occupancy_closed_form", "occupancy_monte_carlo", "expert_params", "moe_layer_params",
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
    * SOFTMAX_ALL_NO_RENORM -- [TOK] "How does MoE routing work": softmax over
      all E, the selected experts' outputs combined with those probabilities
      as they are (no renormalisation); with k = 1 this is [SEV] "Why top-1
      routing cannot renormalise": the chosen expert scaled by the raw router
      probability.
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
    if gating == SOFTMAX_ALL_NO_RENORM:
        return softmax(key, axis=1)[rows, ids]
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
def expert_capacity(T: int, k: int, n_experts: int, capacity_factor: float) -> int:
    """Most rows one expert takes in a batch: tokens per expert times the
    capacity factor, rounded up ([TUR] "Capacity factor: when tokens don't
    fit"; [SEV] counts routing slots, T*k/E, for top-k and rounds up).
    Evaluated as ceil(((T*k)/E)*cf) in float64."""
    return int(math.ceil(float(T * k) / float(n_experts) * float(capacity_factor)))


def dropped_slots(counts: np.ndarray, capacity: int) -> int:
    """Routing slots beyond the capacity, summed over experts ([SEV])."""
    return int(sum(max(int(c) - capacity, 0) for c in counts))


def dispatch(ids: np.ndarray, n_experts: int, capacity: int | None = None):
    """Group the T*k (token, slot) assignments by expert.

    [TUR] "How data centres handle it": tokens are grouped by their assigned
    expert; [TUR] "Capacity factor": dropless means each expert gets exactly
    as many rows as the router assigned to it.  A plain counting sort over
    the assignments in order i = t*k + s gives, per expert in ascending
    order, its assignments in ascending token order:

    counts[e]   number of assignments routed to expert e ([SEV] tokens per
                expert: the router's demand, before any capacity cut)
    offsets     exclusive scan of the rows each expert keeps, offsets[E] =
                rows kept (T*k when dropless)
    perm[row]   = t*k + s, the assignment stored at that row
    row_of[i]   = row of assignment i (inverse of perm), -1 when dropped

    With a ``capacity`` C an expert keeps its first C assignments in that
    order and the rest skip it ([SEV]: the tokens over an expert's capacity
    are not processed by it); ``perm`` then has ``offsets[E]`` entries.
    """
    T, k = ids.shape
    flat = ids.reshape(-1)
    counts = np.zeros(n_experts, dtype=np.int64)
    for e in flat:
        counts[e] += 1
    kept = counts if capacity is None else np.minimum(counts, capacity)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    for e in range(n_experts):
        offsets[e + 1] = offsets[e] + kept[e]
    seen = np.zeros(n_experts, dtype=np.int64)
    perm = np.empty(int(offsets[n_experts]), dtype=np.int64)
    row_of = np.full(T * k, -1, dtype=np.int64)
    for i, e in enumerate(flat):
        rank = seen[e]
        seen[e] += 1
        if rank < kept[e]:
            r = offsets[e] + rank
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


def gelu(z: np.ndarray) -> np.ndarray:
    """GELU(z) = z * Phi(z) = z/2 * (1 + erf(z / sqrt 2)), the exact form
    ([SEV]'s runnable build applies ``F.gelu`` between its two matrices)."""
    from scipy.special import erf

    z = np.asarray(z, dtype=np.float64)
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def gelu_expert(xr: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """Two-matrix expert of [SEV]'s build: ``GELU(x W_up^T) W_down^T``.

    xr [n, d], w_up [f, d], w_down [d, f]  ->  [n, d]."""
    return gelu(xr @ w_up.T) @ w_down.T


ExpertWeights = Callable[[int], tuple[np.ndarray, np.ndarray, np.ndarray]]


def moe_layer(x: np.ndarray, w_router: np.ndarray | None, bias: np.ndarray | None, k: int, gating: int,
              expert_weights: ExpertWeights, n_experts: int,
              shared_weights: Sequence[tuple[np.ndarray, np.ndarray, np.ndarray]] = (),
              bias_select_only: int = 0, ids: np.ndarray | None = None,
              decision_dtype=np.float32, act: int = ACT_SWIGLU,
              capacity: int | None = None,
              keep: np.ndarray | None = None,
              e4m3: bool = False) -> tuple[np.ndarray, Routing | None, np.ndarray]:
    """Sparse MoE sublayer output for the tokens ``x`` [T, d].

    Router -> top-k -> per-expert loop -> weighted sum, as in [TUR]'s
    pseudo-PyTorch layer and [SEV]'s runnable build: every expert computes
    only over the rows the router assigned to it, and adds its output scaled
    by that row's routing weight.  Shared experts ([TOK] "Shared experts";
    [TUR] "Shared expert and fine-grained experts") see every token, weight 1.

    ``expert_weights(e)`` returns float64 ``(W_gate [f,d], W_up [f,d], W_down [d,f])``
    for ``act = ACT_SWIGLU`` and ``(W_up [f,d], W_down [d,f])`` for ``ACT_GELU``
    (the same for ``shared_weights``).

    ``capacity``: when given, each expert processes only its first
    ``capacity`` assignments in token order (:func:`dispatch`); a dropped
    assignment adds nothing to its token's output and the other weights are
    left as they are ([SEV]: a skipped token gets no expert update in that
    layer; the residual connection that carries it lies outside this sublayer).
    ``keep`` ([T, k] bool) gives the kept slots directly, for evaluating a
    subset of a batch whose drops were decided over the whole batch.

    ``e4m3``: experts run with 8-bit weights and activations
    (:func:`e4m3_expert`).

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
    if keep is None:
        keep = np.ones(ids_.shape, dtype=bool)
        if capacity is not None:
            _, _, _, row_of = dispatch(ids_, n_experts, capacity)
            keep = (row_of >= 0).reshape(ids_.shape)

    def ffn(xr, wts):
        if e4m3:
            return e4m3_expert(xr, wts, act)
        return swiglu_expert(xr, *wts) if act == ACT_SWIGLU else gelu_expert(xr, *wts)

    y = np.zeros_like(x)
    for e in range(n_experts):
        rows, slots = np.nonzero((ids_ == e) & keep)
        if rows.size == 0:
            continue
        y[rows] += w[rows, slots][:, None] * ffn(x[rows], expert_weights(e))
    for wts in shared_weights:
        y += ffn(x, wts)
    return y, r, w


def combine(y_rows: np.ndarray, row_of: np.ndarray, w: np.ndarray,
            y_shared: np.ndarray | None = None) -> np.ndarray:
    """The weighted sum that ends the layer, from the dispatched expert rows.

    [SEV] router step "Run and combine" and [TUR]'s per-expert loop: token
    t's output is the sum over its k slots of the routing weight times the
    output its expert produced for it, ``y[t] = sum_s w[t,s] * y_rows[row]``
    with ``row = row_of[t*k + s]`` (the dispatch row of that assignment);
    a dropped slot (``row = -1``) adds nothing; a shared expert's output
    ``y_shared[t]`` is added with weight 1 ([TOK] "Shared experts").
    """
    w = np.asarray(w, dtype=np.float64)
    T, k = w.shape
    rows = np.asarray(row_of, dtype=np.int64).reshape(T, k)
    y = np.zeros((T, y_rows.shape[1]), dtype=np.float64)
    for s in range(k):
        kept = rows[:, s] >= 0
        y[kept] += w[kept, s][:, None] * np.asarray(y_rows, dtype=np.float64)[rows[kept, s]]
    if y_shared is not None:
        y += y_shared
    return y


# ---------------------------------------------------------------- 8-bit experts
E4M3_MAX = 448.0


def e4m3_decode(code: int) -> float:
    """Value of an FP8 E4M3 code (1 sign bit, 4 exponent bits with bias 7,
    3 mantissa bits; exponent 0 is subnormal; S.1111.111 is NaN, so the
    largest finite value is 1.75 * 2^8 = 448)."""
    sgn = -1.0 if code & 0x80 else 1.0
    ex = (code >> 3) & 0xF
    man = code & 0x7
    if ex == 0xF and man == 0x7:
        return float("nan")
    if ex == 0:
        return sgn * man / 8.0 * 2.0 ** -6
    return sgn * (1.0 + man / 8.0) * 2.0 ** (ex - 7)


def e4m3_round(v) -> np.ndarray:
    """Nearest FP8 E4M3 value (ties to even), saturating at +-448, as float64.

    Normal binades [2^e, 2^(e+1)) for e in -6..8 hold 8 values spaced
    2^(e-3); below 2^-6 the subnormals are spaced 2^-9.  ``np.rint`` rounds
    half to even; scaling by a power of two is exact."""
    a = np.abs(np.asarray(v, dtype=np.float64))
    _, ex = np.frexp(np.where(a > 0, a, 1.0))   # a = m * 2^ex, m in [0.5, 1)
    e = np.clip(ex - 1, -6, 8)
    step = np.ldexp(1.0, e - 3)
    q = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(q, np.asarray(v, dtype=np.float64))


def quantize_rows_e4m3(x: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    """Per-row FP8 E4M3 quantisation with a float32 scale: ``s = max|x| / 448``
    (1 for an all-zero row), ``q = e4m3(float32(x / s))``, so that x ~ q * s.
    The pages name 8-bit experts without a scheme; this per-row absolute-max
    scaling is the plainest one.  The decisions are taken in float32, the
    precision of the kernels (x is exact in float32: bf16 or fp32 storage).
    Returns (q as float64 values, s as float64)."""
    x32 = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x32), axis=1)
    s = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    q = e4m3_round((x32 / s[:, None]).astype(np.float32))
    return q, s.astype(np.float64)


def round_bf16(v: np.ndarray) -> np.ndarray:
    """float64 -> float32 -> bfloat16, each step to nearest with ties to even
    (how a kernel stores an fp32 result as bf16), returned as float64."""
    f = np.ascontiguousarray(np.asarray(v, dtype=np.float64).astype(np.float32))
    b = f.view(np.uint32).astype(np.uint64)
    b = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
    return b.astype(np.uint32).view(np.float32).astype(np.float64)


def e4m3_expert(xr: np.ndarray, weights, act: int) -> np.ndarray:
    """One expert with 8-bit weights and activations.

    The pages name 8-bit and 4-bit experts ([TUR] "How data centres handle
    it", [AFD] "What mixture of experts costs in memory") but fix no scheme;
    the plainest one is used: every weight row (output channel) and every
    token row of the expert's input is quantised to FP8 E4M3 with its own
    scale (:func:`quantize_rows_e4m3`), the products are exact and summed
    without rounding, the hidden activation h is stored as bf16 (the
    kernels' storage) and quantised per token row the same way before the
    down projection.  xr [n, d] (the stored bf16 values); weights as in
    :func:`moe_layer`."""
    def deq(m):
        q, s = quantize_rows_e4m3(m)
        return q * s[:, None]

    xd = deq(xr)
    if act == ACT_SWIGLU:
        wg, wu, wd = weights
        h = silu(xd @ deq(wg).T) * (xd @ deq(wu).T)
    else:
        wu, wd = weights
        h = gelu(xd @ deq(wu).T)
    return deq(round_bf16(h)) @ deq(wd).T


# ---------------------------------------------------------------- router penalties
def logsumexp(v: np.ndarray, axis: int = -1) -> np.ndarray:
    """log sum exp(v) = max + log sum exp(v - max)."""
    m = np.max(v, axis=axis)
    return m + np.log(np.sum(np.exp(v - np.expand_dims(m, axis)), axis=axis))


def balance_loss(logits: np.ndarray, counts: np.ndarray) -> float:
    """Load-balancing penalty of [SEV] (the top-1 routing paper's, extended to
    top-k by counting routing slots), without its alpha:
    ``N * sum_i f_i * P_i`` with f_i = share of the routed slots sent to
    expert i and P_i = mean over tokens of the router's softmax probability
    of expert i (softmax of the bias-free router logits).  Equals 1 for an
    even split and N when every token goes to one expert with certainty."""
    n = logits.shape[1]
    c = np.asarray(counts, dtype=np.float64)
    f = c / c.sum()
    P = softmax(logits, axis=1).mean(axis=0)
    return float(n * np.sum(f * P))


def router_z_loss(logits: np.ndarray) -> float:
    """Router z-loss ([TUR] "Router z-loss", [SEV]): the square of the
    log-sum-exp of each token's router logits, averaged over tokens
    (without the loss weight)."""
    return float(np.mean(logsumexp(logits, axis=1) ** 2))


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

