"""Seeded synthetic inputs for the sparse MoE layer forward.

This module only *produces* numbers: token activations, router and expert
weights and an optional per-expert routing bias.  It holds none of the
layer's arithmetic (no routing, no expert FFN, no combine), so both the CUDA
path and the CPU oracle may draw their inputs from it.

Generator
---------
Every tensor is a pure function of ``(seed, stream, flat element index)``:

* a 32-bit counter hash U built from the MurmurHash3 ``fmix32`` finaliser,
  applied twice (low word of the index, then high word);
* a standard normal value by the inverse-CDF method: U picks one of 2**20
  equal-probability cells (its top 20 bits) and a point inside it (its low 12
  bits, offset by half a step); the value interpolates linearly between the
  normal quantiles at the cell's edges, ``Phi^-1(j / 2**20)``, taken from a
  table computed once in float64 (the two outermost edges are clamped at
  ``Phi^-1(2**-33)``, about -6.1 and +6.1);
* ``value = float32(z * std)`` with ``std = 1/sqrt(fan_in)`` for weights and
  1 for activations, then rounded to bfloat16 (round-to-nearest-even) for the
  bf16 workloads.

Only integer operations, a table lookup and correctly rounded IEEE-754
binary64 ``+ - * /`` (each a separate operation, no fused multiply-add)
appear per element, so the numpy (host) and torch (device) implementations
below return bit-identical values; any element can be regenerated on its
own, which lets the oracle rebuild exactly the slices it needs.

Streams: x=0, router=1, routed gate/up=2, routed down=3, shared gate/up=4,
shared down=5, routing-bias permutation=6.  Seed = 1000 + workload index.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

MASK32 = 0xFFFFFFFF

STREAM_X = 0
STREAM_ROUTER = 1
STREAM_GATE_UP = 2
STREAM_DOWN = 3
STREAM_SHARED_GATE_UP = 4
STREAM_SHARED_DOWN = 5
STREAM_BIAS_PERM = 6

# gating rules, numbered as in include/moe.h
SOFTMAX_ALL_RENORM = 0
SOFTMAX_TOPK = 1
SIGMOID_TOPK_RENORM = 2
SOFTMAX_ALL_NO_RENORM = 3


# --------------------------------------------------------------------------
# counter hash, written once against an "array namespace" so numpy arrays and
# torch tensors (CPU or CUDA) run the very same integer operations
# --------------------------------------------------------------------------
def _fmix32_py(h: int) -> int:
    h &= MASK32
    h ^= h >> 16
    h = (h * 0x85EBCA6B) & MASK32
    h ^= h >> 13
    h = (h * 0xC2B2AE35) & MASK32
    h ^= h >> 16
    return h


def _mul32(a, m: int):
    """(a * m) mod 2**32 for 0 <= a < 2**32, never forming a product >= 2**49."""
    lo = m & 0xFFFF
    hi = m >> 16
    return (a * lo + (((a * hi) & 0xFFFF) << 16)) & MASK32


def _fmix32(h):
    h = h ^ (h >> 16)
    h = _mul32(h, 0x85EBCA6B)
    h = h ^ (h >> 13)
    h = _mul32(h, 0xC2B2AE35)
    h = h ^ (h >> 16)
    return h


def _lane_keys(seed: int, stream: int, lane: int) -> tuple[int, int]:
    k1 = _fmix32_py(_fmix32_py(seed * 0x9E3779B9 + 0x7F4A7C15) ^ (stream * 2 + lane + 1))
    k2 = _fmix32_py(k1 ^ 0x68E31DA4)
    return k1, k2


def _hash_lane(idx, seed: int, stream: int, lane: int):
    """32-bit hash of the int64 element indices ``idx`` (numpy or torch)."""
    k1, k2 = _lane_keys(seed, stream, lane)
    lo = idx & MASK32
    hi = idx >> 32
    h = _fmix32(lo ^ k1)
    h = _fmix32(h ^ ((hi + k2) & MASK32))
    return h


QUANTILE_BITS = 20          # 2**20 equal-probability cells
FRAC_BITS = 32 - QUANTILE_BITS
_TABLE = {}


def quantile_table() -> np.ndarray:
    """Normal quantiles at the 2**20 + 1 cell edges j / 2**20 (float64); the
    infinite outer edges are clamped at Phi^-1(2**-33) and its negative."""
    if "host" not in _TABLE:
        from scipy.special import ndtri

        m = 1 << QUANTILE_BITS
        q = ndtri(np.arange(m + 1, dtype=np.float64) / m)
        q[0] = ndtri(2.0 ** -33)
        q[m] = -q[0]
        _TABLE["host"] = q
    return _TABLE["host"]


def _device_table(device):
    import torch

    key = str(device)
    if key not in _TABLE:
        _TABLE[key] = torch.from_numpy(quantile_table()).to(device)
    return _TABLE[key]


def _cell_and_fraction(idx, seed: int, stream: int):
    """Cell index (top 20 bits of the hash) and the point inside the cell,
    ((low 12 bits) + 0.5) / 2**12 as an exact binary64 fraction."""
    u = _hash_lane(idx, seed, stream, 0)
    return u >> FRAC_BITS, u & ((1 << FRAC_BITS) - 1)


# --------------------------------------------------------------------------
# host (numpy) side
# --------------------------------------------------------------------------
def normal_f32(seed: int, stream: int, start: int, count: int, std: float = 1.0) -> np.ndarray:
    """float32 values of elements [start, start+count) of one stream (numpy)."""
    idx = np.arange(start, start + count, dtype=np.int64)
    j, lo = _cell_and_fraction(idx, seed, stream)
    q = quantile_table()
    q0, q1 = q[j], q[j + 1]
    f = (lo.astype(np.float64) + 0.5) / float(1 << FRAC_BITS)
    z = q0 + f * (q1 - q0)
    if std != 1.0:
        z = z * np.float64(std)
    return z.astype(np.float32)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    b = (b + 0x7FFF + ((b >> 16) & 1)) >> 16
    return b.astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def stored_values(seed: int, stream: int, start: int, count: int, std: float, dtype: str) -> np.ndarray:
    """The exact values a device tensor of ``dtype`` holds, as float64."""
    v = normal_f32(seed, stream, start, count, std)
    if dtype == "bf16":
        v = bf16_bits_to_f32(f32_to_bf16_bits(v))
    return v.astype(np.float64)


# --------------------------------------------------------------------------
# device (torch) side; torch is imported lazily so the oracle never needs it
# --------------------------------------------------------------------------
def normal_torch(seed: int, stream: int, start: int, count: int, std: float, dtype: str, device,
                 out=None, chunk: int = 1 << 25):
    """Same values as :func:`normal_f32` (then bf16-rounded if asked), built with torch ops."""
    import torch

    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    if out is None:
        out = torch.empty(count, dtype=tdt, device=device)
    flat = out.view(-1)
    for c0 in range(0, count, chunk):
        n = min(chunk, count - c0)
        idx = torch.arange(start + c0, start + c0 + n, dtype=torch.int64, device=device)
        j, lo = _cell_and_fraction(idx, seed, stream)
        del idx
        q = _device_table(device)
        q0, q1 = q[j], q[j + 1]
        del j
        f = (lo.to(torch.float64) + 0.5) / float(1 << FRAC_BITS)
        del lo
        d = q1 - q0
        del q1
        z = q0 + f * d
        del q0, d, f
        if std != 1.0:
            z = z * std
        flat[c0:c0 + n] = z.to(torch.float32).to(tdt)
        del z
    return out


# --------------------------------------------------------------------------
# workloads
# --------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shape and routing of one sparse MoE layer workload."""

    name: str
    T: int                 # tokens
    d_model: int
    n_experts: int         # routed experts E
    top_k: int
    d_ff: int
    dtype: str             # "f32" or "bf16": x, weights and y
    gating: int            # SOFTMAX_ALL_RENORM / SOFTMAX_TOPK / SIGMOID_TOPK_RENORM
    n_shared: int = 0
    d_ff_shared: int = 0
    zipf_s: float = 0.0    # 0: no routing bias; >0: Zipf(s) logit bias per expert
    bias_select_only: int = 0
    seed: int = 1000
    act: int = 0           # 0: SwiGLU expert (gate+up rows), 1: GELU expert (up rows only)
    capacity_factor: float = 0.0  # 0: dropless
    e4m3: bool = False     # expert weights run as FP8 E4M3 (quantised from the generated bf16 values)

    def replace(self, **kw) -> "LayerConfig":
        return dataclasses.replace(self, **kw)


def workload(name: str, **overrides) -> LayerConfig:
    base = WORKLOADS[name]
    return base.replace(**overrides) if overrides else base


WORKLOADS: dict[str, LayerConfig] = {
    # tiny fp32 layer: softmax over all E, keep top-2, renormalise
    "tiny_f32": LayerConfig("tiny_f32", 256, 256, 8, 2, 512, "f32", SOFTMAX_ALL_RENORM, seed=1000),
    # Mixtral-shaped: top-2 logits, softmax over the two
    "mixtral_bf16": LayerConfig("mixtral_bf16", 2048, 4096, 8, 2, 14336, "bf16", SOFTMAX_TOPK, seed=1001),
    # decode sweep at the Mixtral shape (T set per case), uniform or Zipf(1.2)-skewed
    "decode_bf16": LayerConfig("decode_bf16", 1, 4096, 8, 2, 14336, "bf16", SOFTMAX_TOPK, seed=1002),
    # gpt-oss-120b-shaped: 128 experts, top-4 logits, softmax over the four
    "gptoss_bf16": LayerConfig("gptoss_bf16", 8192, 2880, 128, 4, 2880, "bf16", SOFTMAX_TOPK, seed=1003),
    # DeepSeek-V3-shaped: 256 routed + 1 shared, sigmoid scores renormalised over the 8
    "deepseek_bf16": LayerConfig("deepseek_bf16", 8192, 7168, 256, 8, 2048, "bf16", SIGMOID_TOPK_RENORM,
                                 n_shared=1, d_ff_shared=2048, zipf_s=1.0, bias_select_only=1, seed=1004),
}

DECODE_T = (1, 4, 16, 64)
DECODE_ZIPF_S = 1.2


# element counts and standard deviations of every input tensor
def tensor_specs(cfg: LayerConfig) -> dict[str, tuple[tuple[int, ...], int, float]]:
    """``w_gate_up`` holds 2f rows per expert (gate, then up) for the SwiGLU
    expert and f rows (up only) for the GELU expert."""
    d, E, f = cfg.d_model, cfg.n_experts, cfg.d_ff
    m = 2 if cfg.act == 0 else 1
    specs = {
        "x": ((cfg.T, d), STREAM_X, 1.0),
        "w_router": ((E, d), STREAM_ROUTER, 1.0 / math.sqrt(d)),
        "w_gate_up": ((E, m * f, d), STREAM_GATE_UP, 1.0 / math.sqrt(d)),
        "w_down": ((E, d, f), STREAM_DOWN, 1.0 / math.sqrt(f)),
    }
    if cfg.n_shared:
        fs = cfg.d_ff_shared
        specs["ws_gate_up"] = ((cfg.n_shared, m * fs, d), STREAM_SHARED_GATE_UP, 1.0 / math.sqrt(d))
        specs["ws_down"] = ((cfg.n_shared, d, fs), STREAM_SHARED_DOWN, 1.0 / math.sqrt(fs))
    return specs


def host_tensor(cfg: LayerConfig, name: str, start: int = 0, count: int | None = None) -> np.ndarray:
    """Exact stored values (float64) of elements [start, start+count) of one input tensor."""
    shape, stream, std = tensor_specs(cfg)[name]
    n = int(np.prod(shape))
    if count is None:
        count = n - start
    return stored_values(cfg.seed, stream, start, count, std, cfg.dtype)


def host_storage(cfg: LayerConfig, name: str) -> np.ndarray:
    """A whole input tensor as the host-side storage the device receives:
    float32 array, or uint16 bfloat16 bits."""
    shape, stream, std = tensor_specs(cfg)[name]
    v = normal_f32(cfg.seed, stream, 0, int(np.prod(shape)), std).reshape(shape)
    return f32_to_bf16_bits(v) if cfg.dtype == "bf16" else v


def device_tensor(cfg: LayerConfig, name: str, device):
    """A whole input tensor generated directly in device memory with torch ops."""
    shape, stream, std = tensor_specs(cfg)[name]
    n = int(np.prod(shape))
    return normal_torch(cfg.seed, stream, 0, n, std, cfg.dtype, device).view(shape)


def uniform_u32(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    idx = np.arange(start, start + count, dtype=np.int64)
    return _hash_lane(idx, seed, stream, 0).astype(np.uint64)


def zipf_bias(cfg: LayerConfig) -> np.ndarray | None:
    """Per-expert logit bias that skews token-choice routing towards a Zipf(s) load.

    Ranks are a seeded Fisher-Yates permutation of 1..E; expert e gets the
    share p_e = r_e^-s / sum_j r_j^-s and the bias ln(E p_e), so uniform
    logits would route in proportion to p.  Returned as float32 (the values
    both sides use).  ``None`` when the workload has no bias.
    """
    if cfg.zipf_s <= 0.0:
        return None
    E = cfg.n_experts
    perm = list(range(E))
    draws = uniform_u32(cfg.seed, STREAM_BIAS_PERM, 0, E)
    for i in range(E - 1, 0, -1):
        j = int(draws[i]) % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    ranks = np.array(perm, dtype=np.float64) + 1.0
    p = ranks ** (-cfg.zipf_s)
    p /= p.sum()
    return np.log(E * p).astype(np.float32)
