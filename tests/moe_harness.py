"""Shared helpers of the GPU parity tests: seeded inputs on the device, calls
through the C ABI, and comparison with the CPU oracle.

Inputs come only from ``synth``.  The oracle sees the exact stored values:
for small workloads regenerated on the host, for full-size ones copied back
bit for bit from the generator's device tensors (and spot-checked against the
host generator).  Nothing the CUDA path computes is ever fed to the oracle
except the expert ids under "forced routing", which is how near-tie tokens
are scored.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

import oracle
import synth
import top_routing_expert_gemm_b200 as moe

NEAR_TIE = 1e-3          # logit-unit gap under which a top-k decision may flip
MISMATCH_CAP = 1e-3      # mismatched tokens must stay below 0.1% of T
TOL = {"f32": 1e-4, "bf16": 2e-2}


def torch_dtype(cfg):
    return torch.bfloat16 if cfg.dtype == "bf16" else torch.float32


def moe_cfg(cfg: synth.LayerConfig, T: int | None = None, wait_limit_ns: int = 0) -> moe.MoeConfig:
    return moe.make_config(cfg.T if T is None else T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff,
                           moe.MOE_BF16 if cfg.dtype == "bf16" else moe.MOE_F32, cfg.gating,
                           cfg.n_shared, cfg.d_ff_shared, cfg.bias_select_only, wait_limit_ns,
                           expert_act=cfg.act, capacity_factor=cfg.capacity_factor,
                           weight_format=moe.MOE_W_E4M3 if cfg.e4m3 else moe.MOE_W_NATIVE)


def e4m3_blob(w: torch.Tensor) -> torch.Tensor:
    """The library's E4M3 blob of a bf16 weight tensor [..., rows, cols] (made on the GPU)."""
    cols = w.shape[-1]
    rows = w.numel() // cols
    blob = torch.empty(moe.moe_e4m3_weight_bytes(rows, cols), dtype=torch.uint8, device=w.device)
    moe.moe_quantize_e4m3(w, rows, cols, blob)
    return blob


def capacity_of(cfg: synth.LayerConfig) -> int | None:
    """The oracle's capacity for the workload (the factor as the float32 the ABI carries)."""
    if cfg.capacity_factor == 0:
        return None
    return oracle.expert_capacity(cfg.T, cfg.top_k, cfg.n_experts, float(np.float32(cfg.capacity_factor)))


def host_to_device(arr: np.ndarray, cfg, device="cuda") -> torch.Tensor:
    if cfg.dtype == "bf16":
        return torch.from_numpy(arr.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(arr).to(device)


def device_to_host_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 values of a device tensor (bf16 copied as raw bits)."""
    if t.dtype == torch.bfloat16:
        bits = t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        return synth.bf16_bits_to_f32(bits).astype(np.float64)
    return t.float().cpu().numpy().astype(np.float64)


@dataclasses.dataclass
class Inputs:
    cfg: synth.LayerConfig
    dev: dict            # name -> device tensor
    bias: np.ndarray | None
    on_host: bool        # True when generated on the host (small workloads)


def make_inputs(cfg: synth.LayerConfig, device="cuda", host_limit: int = 1 << 24) -> Inputs:
    specs = synth.tensor_specs(cfg)
    n_elems = sum(int(np.prod(s[0])) for s in specs.values())
    on_host = n_elems <= host_limit
    dev = {}
    for name in specs:
        if on_host:
            dev[name] = host_to_device(synth.host_storage(cfg, name), cfg, device)
        else:
            dev[name] = synth.device_tensor(cfg, name, device)
    bias = synth.zipf_bias(cfg)
    dev["bias"] = torch.from_numpy(bias).to(device) if bias is not None else None
    if cfg.e4m3:  # the kernels read the 8-bit blobs; the oracle quantises the bf16 values itself
        for name in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
            if name in dev:
                dev[name + "_q"] = e4m3_blob(dev[name])
    return Inputs(cfg, dev, bias, on_host)


def spot_check_device_inputs(inp: Inputs, n: int = 4096, seed: int = 0) -> None:
    """Device-generated inputs equal the host generator on random elements."""
    rng = np.random.default_rng(seed)
    for name, (shape, _s, _std) in synth.tensor_specs(inp.cfg).items():
        total = int(np.prod(shape))
        start = int(rng.integers(0, max(1, total - n)))
        cnt = min(n, total - start)
        host = synth.host_tensor(inp.cfg, name, start, cnt)
        devv = device_to_host_f64(inp.dev[name].reshape(-1)[start:start + cnt])
        assert np.array_equal(host, devv), f"device generator differs from host for {name}"


class OracleWeights:
    """float64 expert weights for the oracle, fetched per expert on demand."""

    def __init__(self, inp: Inputs):
        self.inp = inp
        self.cfg = inp.cfg
        self._cache = {}

    def routed(self, e: int):
        if e in self._cache:
            return self._cache[e]
        f = self.cfg.d_ff
        m = 2 if self.cfg.act == oracle.ACT_SWIGLU else 1
        if self.inp.on_host:
            d = self.cfg.d_model
            gu = synth.host_tensor(self.cfg, "w_gate_up", e * m * f * d, m * f * d).reshape(m * f, d)
            wd = synth.host_tensor(self.cfg, "w_down", e * d * f, d * f).reshape(d, f)
        else:
            gu = device_to_host_f64(self.inp.dev["w_gate_up"][e])
            wd = device_to_host_f64(self.inp.dev["w_down"][e])
        w = (gu[:f], gu[f:], wd) if m == 2 else (gu, wd)
        if self.inp.on_host:  # full-size experts are refetched rather than held in host memory
            self._cache[e] = w
        return w

    def shared(self):
        out = []
        m = 2 if self.cfg.act == oracle.ACT_SWIGLU else 1
        for s in range(self.cfg.n_shared):
            fs, d = self.cfg.d_ff_shared, self.cfg.d_model
            if self.inp.on_host:
                gu = synth.host_tensor(self.cfg, "ws_gate_up", s * m * fs * d, m * fs * d).reshape(m * fs, d)
                wd = synth.host_tensor(self.cfg, "ws_down", s * d * fs, d * fs).reshape(d, fs)
            else:
                gu = device_to_host_f64(self.inp.dev["ws_gate_up"][s])
                wd = device_to_host_f64(self.inp.dev["ws_down"][s])
            out.append((gu[:fs], gu[fs:], wd) if m == 2 else (gu, wd))
        return out

    def w_router(self) -> np.ndarray:
        return synth.host_tensor(self.cfg, "w_router").reshape(self.cfg.n_experts, self.cfg.d_model)


def run_forward(inp: Inputs, wait_limit_ns: int = 0):
    cfg = inp.cfg
    c = moe_cfg(cfg, wait_limit_ns=wait_limit_ns)
    dev = inp.dev
    T, k, E, d = cfg.T, cfg.top_k, cfg.n_experts, cfg.d_model
    y = torch.empty(T, d, dtype=torch_dtype(cfg), device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    ws = torch.empty(max(256, moe.moe_workspace_bytes(c)), dtype=torch.uint8, device="cuda")
    q = "_q" if cfg.e4m3 else ""
    moe.moe_forward(c, dev["x"], dev["w_router"], dev["bias"], dev["w_gate_up" + q], dev["w_down" + q],
                    dev.get("ws_gate_up" + q), dev.get("ws_down" + q), y, ids, w, counts, ws)
    st = moe.moe_device_status(ws)
    torch.cuda.synchronize()
    return dict(y=y, ids=ids, w=w, counts=counts, ws=ws, status=st)


def check_routing(cfg, gpu_ids: np.ndarray, gpu_w: np.ndarray, r: oracle.Routing, T_total: int):
    """ids bit-exact outside the near-tie set; mismatches < 0.1% of T; weights close where ids agree."""
    k = cfg.top_k
    s = -np.sort(-r.key, axis=1)
    gaps = s[:, :-1] - s[:, 1:] if s.shape[1] > 1 else np.full((s.shape[0], 1), np.inf)
    boundary = r.gap < NEAR_TIE
    order = np.any(gaps[:, :max(0, k - 1)] < NEAR_TIE, axis=1) if k > 1 else np.zeros(len(r.gap), bool)
    near = boundary | order
    mism = np.any(gpu_ids != r.ids, axis=1)
    assert not np.any(mism & ~near), f"{int(np.sum(mism & ~near))} tokens differ outside the near-tie set"
    assert np.sum(mism) < max(1.0, MISMATCH_CAP * T_total) or np.sum(mism) == 0, \
        f"{int(np.sum(mism))} mismatched tokens of {T_total}"
    ok = ~mism
    if np.any(ok):
        assert np.max(np.abs(gpu_w[ok] - r.w[ok])) <= 2e-5
    return dict(near_tie=int(np.sum(near)), boundary_near_tie=int(np.sum(boundary)), mismatched=int(np.sum(mism)))


def rel_err(y: np.ndarray, y_ref: np.ndarray) -> float:
    den = np.max(np.abs(y_ref))
    return float(np.max(np.abs(y - y_ref)) / den) if den > 0 else float(np.max(np.abs(y)))


def sample_tokens(T: int, n: int, seed: int = 0) -> np.ndarray:
    if n >= T:
        return np.arange(T)
    rng = np.random.default_rng(seed)
    mid = rng.choice(np.arange(1, T - 1), size=n - 2, replace=False)
    return np.sort(np.concatenate([[0, T - 1], mid]))


TILE_ROWS = 128          # token rows per tile of the large-batch expert GEMMs
BLOCK_ROWS = 16 * 128    # rows of one block of a hot expert's walk (16 m-tiles)


def coverage_tokens(offsets: np.ndarray, perm: np.ndarray, k: int, T: int, n_min: int,
                    seed: int = 0) -> np.ndarray:
    """Tokens whose rows reach the parts of the grouped GEMMs that only full
    sizes exercise: every expert's last row and the first row of its last
    (partial) 128-row tile, the rows on both sides of every 2048-row block
    boundary of the hottest expert, the first and last dispatched rows (the
    experts after the persistent grid's first wave are among "every expert");
    then random tokens up to ``n_min``.  ``offsets``/``perm`` are the dispatch
    of the routing under test."""
    want = set()
    E = len(offsets) - 1
    n = np.diff(offsets)
    for e in range(E):
        if n[e] <= 0:
            continue
        lo, hi = int(offsets[e]), int(offsets[e + 1])
        want.add(int(perm[hi - 1]) // k)
        want.add(int(perm[lo + ((hi - lo - 1) // TILE_ROWS) * TILE_ROWS]) // k)
    hot = int(np.argmax(n))
    for b in range(BLOCK_ROWS, int(n[hot]), BLOCK_ROWS):
        for r in (b - 1, b):
            want.add(int(perm[offsets[hot] + r]) // k)
    if offsets[-1] > 0:
        want.add(int(perm[0]) // k)
        want.add(int(perm[offsets[-1] - 1]) // k)
    rng = np.random.default_rng(seed)
    rest = np.setdiff1d(np.arange(T), np.fromiter(want, dtype=np.int64))
    extra = max(0, n_min - len(want))
    if extra and len(rest):
        want |= set(rng.choice(rest, size=min(extra, len(rest)), replace=False).tolist())
    return np.array(sorted(want), dtype=np.int64)


def check_forward(inp: Inputs, out: dict, n_sample: int | None = None) -> dict:
    """Parity of one moe_forward call against the oracle.

    Routing and dispatch counts on every token; layer outputs on every token,
    or on ``n_sample`` sampled tokens for full-size layers, under forced
    routing with the GPU's ids (so a near-tie flip is scored on the experts the
    GPU actually used)."""
    cfg = inp.cfg
    T, k, E = cfg.T, cfg.top_k, cfg.n_experts
    ow = OracleWeights(inp)
    if inp.on_host:
        x_all = synth.host_tensor(cfg, "x").reshape(T, cfg.d_model)
    else:
        x_all = device_to_host_f64(inp.dev["x"])
    wr = ow.w_router()
    bias = inp.bias.astype(np.float64) if inp.bias is not None else None
    gpu_ids = out["ids"].cpu().numpy().astype(np.int64)
    gpu_w = out["w"].cpu().numpy().astype(np.float64)
    r = oracle.route(x_all, wr, bias, k, cfg.gating, cfg.bias_select_only)
    stats = check_routing(cfg, gpu_ids, gpu_w, r, T)
    cap = capacity_of(cfg)
    counts, offsets, perm, row_of = oracle.dispatch(gpu_ids, E, cap)
    assert np.array_equal(out["counts"].cpu().numpy(), counts)
    keep = (row_of >= 0).reshape(T, k)  # slots the capacity keeps, decided over the whole batch
    tokens = np.arange(T) if n_sample is None else coverage_tokens(offsets, perm, k, T, n_sample)
    y_ref, _, _ = oracle.moe_layer(x_all[tokens], wr, bias, k, cfg.gating, ow.routed, E,
                                   shared_weights=ow.shared(), bias_select_only=cfg.bias_select_only,
                                   ids=gpu_ids[tokens], act=cfg.act, keep=keep[tokens], e4m3=cfg.e4m3)
    y = device_to_host_f64(out["y"][torch.from_numpy(tokens).cuda()])
    err = rel_err(y, y_ref)
    assert err <= TOL[cfg.dtype], f"relative error {err:.3e} > {TOL[cfg.dtype]}"
    assert out["status"] == 0
    stats.update(rel_err=err, tokens_checked=len(tokens),
                 experts_touched=int(np.sum(counts > 0)), dropped=int(np.sum(~keep)))
    return stats
