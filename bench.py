"""Benchmark of the sparse MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--T T] [--workloads all|none|NAME,...]

One step = one full pass of the layer (router + top-k, dispatch, grouped SwiGLU
experts, combine) over one batch of T synthetic tokens already resident in HBM.
Headline workload: the Mixtral-shaped bf16 layer (T=2048, d=4096, E=8, k=2,
f=14336).  Inputs are larger than L2 (2.8 GB of expert weights per step), so L2
is not flushed between steps (decode-sized steps flush it, see below).  With
N>1 (torchrun) every rank runs an independent replica on its own T tokens (weak
scaling, no data-path collective); the step time is the max over ranks.

Rank 0 prints one JSON line.  ``value`` is tokens/s over all ranks; the line
also carries active TFLOP/s, the per-stage split of the step, the roofline of
the grouped expert GEMMs (their time measured inside traced moe_forward steps),
an end-to-end number through host buffers, SM clocks sampled during the timed
region and the CPU oracle's throughput.  ``workloads`` holds the same device
measurements for every other configuration (gpt-oss, DeepSeek, the decode
sweep with experts touched against the closed form, the fp32 layer, 8-bit
experts), taken in the same run.  ``--impl reference`` times the CPU oracle
itself on the same workload and sample.
"""
from __future__ import annotations

import argparse
import json
import os
import pathlib
import statistics
import sys
import time

import numpy as np

ROOT = pathlib.Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

import synth  # noqa: E402

METRIC = "MoE-layer tokens/s (active TFLOP/s and roofline fraction alongside)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# the sources of the expert GEMMs of each schedule (token-rows-as-M kernel for
# large batches, swapped-operand kernel for the decode regime)
GEMM_SOURCES = {
    "tc": ("grouped_gemm_tc.cu", "tc_primitives.cuh", "common.cuh", "kernels.cuh"),
    "decode": ("grouped_gemm_swap.cu", "tc_primitives.cuh", "pdl.cuh", "common.cuh", "kernels.cuh"),
}
TRAFFIC_FILE = ROOT / "profiles" / "dram_traffic.json"


def gemm_sources_sha256(schedule: str) -> str:
    """Digest of the expert-GEMM kernel sources of a schedule: a DRAM-traffic
    record taken with ncu applies only while this matches."""
    import hashlib

    h = hashlib.sha256()
    for name in GEMM_SOURCES[schedule]:
        h.update((ROOT / "top_routing_expert_gemm_b200" / "csrc" / name).read_bytes())
    return h.hexdigest()


def recorded_traffic(workload: str, schedule: str):
    """DRAM bytes (read + write) per step of the expert GEMMs from the committed
    ncu record, or None when there is none or the kernels changed since."""
    if not TRAFFIC_FILE.exists():
        return None
    rec = json.loads(TRAFFIC_FILE.read_text()).get(workload)
    if not rec or rec.get("gemm_sources_sha256") != gemm_sources_sha256(schedule):
        return None
    return rec.get("bytes_per_step")


def uses_decode_schedule(cfg) -> bool:
    """The library's choice for the routed experts: the decode schedule when
    the expected tokens per touched expert (uniform routing) is at most 64."""
    rows = cfg.T * cfg.top_k
    touched = max(1.0, cfg.n_experts * (1.0 - (1.0 - 1.0 / cfg.n_experts) ** rows))
    return cfg.dtype == "bf16" and rows / touched <= 64


def max_over_ranks(v: float, world: int, device: str = "cuda") -> float:
    """The slowest rank's value (every rank takes part; NCCL on GPUs, gloo on CPU)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(tokens_per_rank: int, world: int, ms_max: float) -> float:
    """Tokens/s of the whole job: every replica processed its own batch in at
    most ``ms_max`` milliseconds (weak scaling)."""
    return world * tokens_per_rank / (ms_max / 1000.0)


def launches_per_step(cfg) -> int:
    """Kernels of ours one moe_forward step launches: router, dispatch (one
    block-wide kernel for at most 1024 assignments, or at most 8192 over at
    most 64 experts, else count / scan / scatter) and the row gather (with
    8-bit experts the gather-quantise), two expert GEMMs for the routed
    experts (8-bit: with the re-quantisation of h between them) and for each
    shared expert (8-bit: after quantising x, and with the re-quantisation of
    h), and the combine."""
    n = cfg.T * cfg.top_k
    dispatch = 2 if n <= 1024 or (n <= 8192 and cfg.n_experts <= 64) else 4
    routed = 2 + (1 if cfg.e4m3 else 0)
    shared = cfg.n_shared * (2 + (2 if cfg.e4m3 else 0))
    return 1 + dispatch + routed + shared + 1


def peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def layer_flops(cfg: synth.LayerConfig, counts: np.ndarray) -> dict:
    """Algorithmic FLOPs of one step, split by stage (rows = measured tokens per expert)."""
    rows = float(np.sum(counts))
    mats = 3 if cfg.act == 0 else 2  # SwiGLU: gate, up, down; GELU: up, down
    router = 2.0 * cfg.T * cfg.d_model * cfg.n_experts
    experts = 2.0 * mats * cfg.d_model * cfg.d_ff * rows
    shared = 2.0 * mats * cfg.d_model * cfg.d_ff_shared * cfg.n_shared * cfg.T
    return dict(router=router, experts=experts, shared=shared, total=router + experts + shared)


def layer_bytes(cfg: synth.LayerConfig, counts: np.ndarray) -> dict:
    """Algorithmic HBM bytes of one step: x, router, touched experts, shared experts, y.
    8-bit experts: one byte per weight plus one fp32 scale per weight row."""
    b = 2 if cfg.dtype == "bf16" else 4
    touched = int(np.sum(counts > 0))
    d, f, fs = cfg.d_model, cfg.d_ff, cfg.d_ff_shared
    mats = 3 if cfg.act == 0 else 2
    if cfg.e4m3:
        per_expert = mats * d * f + 4 * ((mats - 1) * f + d)
        per_shared = mats * d * fs + 4 * ((mats - 1) * fs + d)
    else:
        per_expert, per_shared = mats * d * f * b, mats * d * fs * b
    weights = touched * per_expert + cfg.n_shared * per_shared + cfg.n_experts * d * b
    act = 2 * cfg.T * d * b
    return dict(weights=weights, activations=act, total=weights + act, touched=touched)


class ClockSampler:
    """SM clock and clock-event reasons sampled through NVML every few
    milliseconds while the timed region runs (read-only queries)."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap",
               "hw_power_brake_slowdown": "nvmlClocksEventReasonHwPowerBrakeSlowdown"}

    def __init__(self, gpu_index: int, period_s: float = 0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = None
        self._thread = None
        self.error = None

    def _run(self):
        import pynvml
        h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
        while not self._stop.is_set():
            try:
                self.samples.append((pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM),
                                     pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except pynvml.NVMLError as e:  # pragma: no cover - driver dependent
                self.error = str(e)
                return
            self._stop.wait(self.period)

    def __enter__(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - no NVML
            self.error = str(e)
            return self
        self._stop = threading.Event()
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()
        return self

    def __exit__(self, *exc):
        if self._thread is not None:
            self._stop.set()
            self._thread.join(timeout=2)

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "error": self.error}
        import pynvml
        mhz = [m for m, _ in self.samples]
        seen = 0
        for _, r in self.samples:
            seen |= r
        reasons = sorted(n for n, attr in self.REASONS.items() if seen & getattr(pynvml, attr))
        return {"sm_mhz": statistics.median(mhz), "sm_min_mhz": min(mhz), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(self.samples)}


def config_dict(cfg: synth.LayerConfig, world: int) -> dict:
    return {"workload": cfg.name, "T": cfg.T, "d_model": cfg.d_model, "n_experts": cfg.n_experts,
            "top_k": cfg.top_k, "d_ff": cfg.d_ff, "n_shared": cfg.n_shared, "d_ff_shared": cfg.d_ff_shared,
            "gating": cfg.gating, "zipf_s": cfg.zipf_s,
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "weights": "e4m3 (per-row fp32 scales)" if cfg.e4m3 else cfg.dtype,
            "l2": "not flushed: inputs larger than L2 (expert weights %.2f GB)" % (
                (3 if cfg.act == 0 else 2) * cfg.n_experts * cfg.d_model * cfg.d_ff
                * (1 if cfg.e4m3 else 2 if cfg.dtype == "bf16" else 4) / 1e9)}


def _bits_to_f64(t) -> np.ndarray:
    """Exact float64 copy of a device tensor (bf16 moved as raw bits)."""
    import torch

    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f32(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)).astype(
            np.float64)
    return t.float().cpu().numpy().astype(np.float64)


class OracleInputs:
    """The workload's stored inputs as float64 host arrays, the form the oracle reads.

    Expert weights are upcast once up front when they fit in ``prefetch_gb``
    of host memory (the oracle then runs on resident inputs, like the GPU);
    otherwise each oracle call upcasts the experts it touches and that time is
    part of the measurement."""

    def __init__(self, cfg: synth.LayerConfig, dev: dict, n_tokens: int, prefetch_gb: float = 16.0):
        self.cfg = cfg
        self.dev = dev
        self.n = min(n_tokens, cfg.T)
        self.x = _bits_to_f64(dev["x"][: self.n])
        self.wr = _bits_to_f64(dev["w_router"])
        b = synth.zipf_bias(cfg)
        self.bias = b.astype(np.float64) if b is not None else None
        fs = cfg.d_ff_shared
        self.shared = []
        for s in range(cfg.n_shared):
            gu = _bits_to_f64(dev["ws_gate_up"][s])
            dn = _bits_to_f64(dev["ws_down"][s])
            self.shared.append((gu[:fs], gu[fs:], dn) if cfg.act == 0 else (gu, dn))
        per_expert_gb = 3 * cfg.d_model * cfg.d_ff * 8 / 1e9
        self.prefetched = per_expert_gb * cfg.n_experts <= prefetch_gb
        self.cache = {e: self._fetch(e) for e in range(cfg.n_experts)} if self.prefetched else None

    def _fetch(self, e: int):
        f = self.cfg.d_ff
        gu = _bits_to_f64(self.dev["w_gate_up"][e])
        dn = _bits_to_f64(self.dev["w_down"][e])
        return (gu[:f], gu[f:], dn) if self.cfg.act == 0 else (gu, dn)

    def expert(self, e: int):
        return self.cache[e] if self.cache is not None else self._fetch(e)

    def describe(self) -> str:
        return (f"first {self.n} of {self.cfg.T} tokens of the same layer, float64 numpy; expert weights "
                + ("upcast to float64 before timing" if self.prefetched else "upcast inside each timed call"))


def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        return max([i.get("num_threads", 1) for i in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        return os.cpu_count() or 1


def time_oracle(oi: OracleInputs) -> float:
    """Seconds for one call of the CPU oracle on the prepared sample."""
    import oracle

    cfg = oi.cfg
    t0 = time.perf_counter()
    oracle.moe_layer(oi.x, oi.wr, oi.bias, cfg.top_k, cfg.gating, oi.expert, cfg.n_experts,
                     shared_weights=oi.shared, bias_select_only=cfg.bias_select_only, act=cfg.act, e4m3=cfg.e4m3)
    return time.perf_counter() - t0


ORACLE_FULL_BATCH_MAX = 2048  # the oracle runs on the whole batch up to this many tokens
ORACLE_SUBSET = 1024          # else on the first 1024 tokens, throughput extrapolated to the batch


def oracle_sample_tokens(cfg: synth.LayerConfig) -> int:
    """Tokens the CPU oracle runs on, the same in the bench line's cpu_baseline
    and in --impl reference: the whole batch when it has at most 2048 tokens
    (the oracle then takes seconds), else a fixed 1024-token subset, whose
    throughput stands for the batch's because token-choice routing and the
    expert FFNs are per token."""
    return cfg.T if cfg.T <= ORACLE_FULL_BATCH_MAX else ORACLE_SUBSET


def sample_label(oi: "OracleInputs") -> str:
    kind = "full batch" if oi.n == oi.cfg.T else "extrapolated from a fixed subset"
    return f"{kind}: {oi.describe()}"


def cpu_baseline(cfg: synth.LayerConfig, dev: dict, n_tokens: int, calls: int = 2) -> dict:
    """The CPU oracle, as it stands, on the fixed sample of the workload
    (mean over ``calls`` timed calls after one untimed one)."""
    oi = OracleInputs(cfg, dev, n_tokens)
    time_oracle(oi)
    dt = statistics.mean(time_oracle(oi) for _ in range(calls))
    return {"value": oi.n / dt, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": sample_label(oi), "seconds": dt}


def run_reference(args, cfg) -> None:
    """--impl reference: the CPU oracle timed on the host cores (rank 0 only)."""
    import torch

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev_name = "cuda" if torch.cuda.is_available() else "cpu"
    dev = {name: synth.device_tensor(cfg, name, dev_name) for name in synth.tensor_specs(cfg)}
    oi = OracleInputs(cfg, dev, args.ref_tokens if args.ref_tokens else oracle_sample_tokens(cfg))
    times = []
    for i in range(args.warmup + args.steps):
        dt = time_oracle(oi)
        if i >= args.warmup:
            times.append(dt)
    n = oi.n
    ms = 1000.0 * sum(times) / len(times)
    val = n / (ms / 1000.0)
    r = {"cores": cpu_cores(), "sample": sample_label(oi)}
    line = {
        "impl": "reference", "metric": METRIC, "value": val, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": dict(config_dict(cfg, args.gpus), oracle_tokens_per_step=n),
        "cpu_baseline": {"value": val, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": val, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------
# device measurement of one workload
# ----------------------------------------------------------------------------
# the configurations measured besides the headline, in the same run
EXTRA_WORKLOADS = (
    ("gptoss_bf16", {}),
    ("deepseek_bf16", {}),
    *[("decode_bf16", {"T": t}) for t in synth.DECODE_T],
    *[("decode_bf16", {"T": t, "zipf_s": synth.DECODE_ZIPF_S}) for t in synth.DECODE_T],
    ("tiny_f32", {}),
    ("mixtral_bf16", {"e4m3": True}),
    ("gptoss_bf16", {"e4m3": True}),
    ("deepseek_bf16", {"e4m3": True}),
)
L2_BYTES = 126 * 1024 * 1024
STAGES = ("router_topk", "dispatch", "routed_ffn", "shared_ffn", "combine")
FP32_CORE_FLOP_PER_CLK_PER_SM = 256  # 128 fp32 lanes x 2 (fused multiply-add)
DECODE_DRAWS = 1000


def workload_key(name: str, ov: dict) -> str:
    parts = [f"T={ov['T']}"] if "T" in ov else []
    if ov.get("zipf_s"):
        parts.append(f"zipf={ov['zipf_s']}")
    if ov.get("e4m3"):
        parts.append("e4m3")
    return name + (f"[{','.join(parts)}]" if parts else "")


def weight_bytes_total(cfg: synth.LayerConfig) -> int:
    mats = 3 if cfg.act == 0 else 2
    b = 1 if cfg.e4m3 else 2 if cfg.dtype == "bf16" else 4
    return mats * cfg.d_model * (cfg.n_experts * cfg.d_ff + cfg.n_shared * cfg.d_ff_shared) * b


def needs_l2_flush(cfg: synth.LayerConfig) -> bool:
    """Steps whose inputs fit in L2 get it flushed between timed steps."""
    return weight_bytes_total(cfg) < 2 * L2_BYTES


class Layer:
    """Device inputs, outputs and workspace of one workload, and its step."""

    def __init__(self, cfg: synth.LayerConfig, rank: int = 0):
        import torch

        import top_routing_expert_gemm_b200 as moe

        self.moe, self.cfg = moe, cfg
        dev = {}
        for name in synth.tensor_specs(cfg):
            dev[name] = synth.device_tensor(cfg if name != "x" else cfg.replace(seed=cfg.seed + 7919 * rank),
                                            name, "cuda")
        b = synth.zipf_bias(cfg)
        self.bias = torch.from_numpy(b).cuda() if b is not None else None
        wfmt = moe.MOE_W_E4M3 if cfg.e4m3 else moe.MOE_W_NATIVE
        if cfg.e4m3:  # the expert weights as the library's 8-bit blobs, quantised on the GPU
            for name in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
                if name in dev:
                    src = dev[name]
                    rows = src.numel() // src.shape[-1]
                    blob = torch.empty(moe.moe_e4m3_weight_bytes(rows, src.shape[-1]), dtype=torch.uint8,
                                       device="cuda")
                    moe.moe_quantize_e4m3(src, rows, src.shape[-1], blob)
                    dev[name + "_q"] = blob  # the bf16 values stay for the CPU oracle, which quantises them itself
        self.dev = dev
        self.q = "_q" if cfg.e4m3 else ""
        self.c = moe.make_config(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff,
                                 moe.MOE_BF16 if cfg.dtype == "bf16" else moe.MOE_F32, cfg.gating, cfg.n_shared,
                                 cfg.d_ff_shared, cfg.bias_select_only, expert_act=cfg.act, weight_format=wfmt)
        self.tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
        T, d, k, E = cfg.T, cfg.d_model, cfg.top_k, cfg.n_experts
        self.ws_bytes = moe.moe_workspace_bytes(self.c)
        self.ws = torch.empty(self.ws_bytes, dtype=torch.uint8, device="cuda")
        self.y = torch.empty(T, d, dtype=self.tdt, device="cuda")
        self.ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
        self.w = torch.empty(T, k, dtype=torch.float32, device="cuda")
        self.counts = torch.empty(E, dtype=torch.int32, device="cuda")

    def args(self, x=None, y=None):
        d, q = self.dev, self.q
        return (self.c, d["x"] if x is None else x, d["w_router"], self.bias, d["w_gate_up" + q], d["w_down" + q],
                d.get("ws_gate_up" + q), d.get("ws_down" + q), self.y if y is None else y, self.ids, self.w,
                self.counts, self.ws, self.ws_bytes)

    def step(self, stream, x=None, y=None):
        self.moe.moe_forward(*self.args(x, y), stream)

    def traced(self, stream, events):
        self.moe.moe_forward_traced(*self.args(), stream, events)


def time_steps(layer: Layer, steps: int, warmup: int, world: int, local: int, flush_buf=None) -> tuple:
    """Device time per step (max over ranks) of `steps` moe_forward steps, and
    the SM clocks sampled meanwhile.  Without a flush buffer the steps run back
    to back between two events; with one, L2 is overwritten before every step
    and each step is timed on its own."""
    import torch

    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        layer.step(stream)
    torch.cuda.synchronize()
    st = layer.moe.moe_device_status(layer.ws, layer.ws_bytes, stream)
    if st != 0:
        raise RuntimeError(f"{layer.cfg.name}: device status {st} after warm-up")
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        if flush_buf is None:
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(steps):
                layer.step(stream)
            e1.record(stream)
            torch.cuda.synchronize()
            ms = e0.elapsed_time(e1) / steps
        else:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for a, b in evs:
                flush_buf.zero_()
                a.record(stream)
                layer.step(stream)
                b.record(stream)
            torch.cuda.synchronize()
            ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        barrier(world)
    return max_over_ranks(ms, world), clk.summary()


def traced_stages(layer: Layer, steps: int, flush_buf=None) -> dict:
    """Per-stage device time of moe_forward_traced steps, mean over `steps`:
    the stage markers are recorded by the library on the launching stream
    between its launches."""
    import torch

    stream = torch.cuda.current_stream()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(steps)]
    for e in evs:
        if flush_buf is not None:
            flush_buf.zero_()
        layer.traced(stream, e)
    torch.cuda.synchronize()
    out = {n: statistics.mean(e[j].elapsed_time(e[j + 1]) for e in evs) for j, n in enumerate(STAGES)}
    out["step"] = statistics.mean(e[0].elapsed_time(e[5]) for e in evs)
    return out


def gemm_ms_in_step(stage: dict, ms_per_step: float) -> tuple[float, float]:
    """Device time of the expert GEMMs inside a timed step: their share of the
    traced steps (stage markers recorded between the launches) applied to the
    timed step, so it can never exceed the step it belongs to; and the share."""
    share = (stage["routed_ffn"] + stage["shared_ffn"]) / stage["step"]
    return share * ms_per_step, share


def roofline_of(cfg: synth.LayerConfig, counts: np.ndarray, stage: dict, peaks_: tuple,
                ms_per_step: float | None = None) -> dict:
    """Roofline of the grouped expert GEMMs (routed + shared): tensor-bound
    large batches, HBM-bound decode-sized ones, the fp32 layer on the CUDA
    cores.  Their time is their share of the traced steps applied to the timed
    step (without a timed step: the traced stage time itself)."""
    pk, pk_kind = peaks_
    fl = layer_flops(cfg, counts)
    by = layer_bytes(cfg, counts)
    if ms_per_step is None:
        g_ms, share = stage["routed_ffn"] + stage["shared_ffn"], None
    else:
        g_ms, share = gemm_ms_in_step(stage, ms_per_step)
    if cfg.dtype != "bf16":
        # fp32 CUDA cores: 148 SMs x 128 lanes x 2 FLOP per clock at the max SM clock
        peak = 148 * FP32_CORE_FLOP_PER_CLK_PER_SM * 1.965e9 / 1e12
        ach = (fl["experts"] + fl["shared"]) / (g_ms / 1e3) / 1e12
        return {"bound": "alu", "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": ach / peak,
                "traffic": None, "stage_ms": g_ms, "share_of_step": share,
                "kernel": "grouped_gemm_f32_kernel (CUDA cores): the two expert GEMM launches",
                "peak_source": "derived: 148 SMs x 128 fp32 lanes x 2 FLOP x 1.965 GHz"}
    if uses_decode_schedule(cfg):
        gbs = (by["weights"] - cfg.n_experts * cfg.d_model * 2) / (g_ms / 1e3) / 1e9
        r = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s", "frac": gbs / pk["hbm_gbs"],
             "kernel": "grouped_gemm_swap_kernel, decode schedule (weight rows as M, reductions split evenly over "
                       "the CTAs): the GEMM-1 and GEMM-2 launches", "peak_source": pk_kind}
    else:
        mult = 2.0 if cfg.e4m3 else 1.0  # 8-bit: the bf16 peak x 2, the nominal dense fp8 / bf16 ratio
        tpk = pk["bf16_tflops"] * mult
        ach = (fl["experts"] + fl["shared"]) / (g_ms / 1e3) / 1e12
        r = {"bound": "tensor", "achieved": ach, "peak": tpk, "unit": "TFLOP/s", "frac": ach / tpk,
             "frac_of_sustained": ach / (pk.get("bf16_tflops_sustained", pk["bf16_tflops"]) * mult),
             "kernel": "grouped_gemm_tc_kernel (token rows as M): the GEMM-1 and GEMM-2 launches",
             "peak_source": pk_kind + (" bf16 x 2 (nominal fp8/bf16 dense ratio)" if cfg.e4m3 else "")}
    if cfg.n_shared:
        r["kernel"] += " of the routed and the shared experts"
    r["traffic"] = recorded_traffic(cfg.name, "decode" if uses_decode_schedule(cfg) else "tc")
    r["stage_ms"] = g_ms
    r["share_of_step"] = share
    return r


def decode_occupancy(layer: Layer, draws: int = DECODE_DRAWS) -> dict:
    """Experts touched by a decode batch of T tokens, mean over `draws` seeded
    batches routed by the GPU router (moe_router_topk, one call per batch),
    next to the uniform-routing closed form E * (1 - (1 - k/E)^T)."""
    import torch

    cfg, moe = layer.cfg, layer.moe
    T, k, E = cfg.T, cfg.top_k, cfg.n_experts
    x_all = synth.device_tensor(cfg.replace(T=draws * T, seed=cfg.seed + 500009), "x", "cuda")
    width = -(-T * k // 4) * 4  # every draw's outputs start on 16 bytes, as the ABI requires
    ids = torch.empty(draws, width, dtype=torch.int32, device="cuda")
    w = torch.empty(draws, width, dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream()
    for i in range(draws):
        moe.moe_router_topk(layer.c, x_all[i * T:(i + 1) * T], layer.dev["w_router"], layer.bias, ids[i], w[i],
                            layer.ws, layer.ws_bytes, stream)
    hit = torch.zeros(draws, E, dtype=torch.int32, device="cuda")
    hit.scatter_(1, ids[:, :T * k].long(), 1)
    touched = hit.sum(1).double().cpu().numpy()
    closed = E * (1.0 - (1.0 - k / E) ** T)
    return {"draws": draws, "mean": float(touched.mean()), "std_of_mean": float(touched.std() / np.sqrt(draws)),
            "closed_form": closed, "routing": "zipf %.1f" % cfg.zipf_s if cfg.zipf_s else "uniform"}


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def measure_workload(cfg: synth.LayerConfig, steps: int, warmup: int, world: int, rank: int, local: int,
                     peaks_: tuple, flush_buf=None) -> tuple[dict, "Layer"]:
    """The device measurements of one workload (no host copies)."""
    layer = Layer(cfg, rank)
    fb = flush_buf if needs_l2_flush(cfg) else None
    ms, clocks = time_steps(layer, steps, warmup, world, local, fb)
    stage = traced_stages(layer, steps, fb)
    counts = layer.counts.cpu().numpy()
    fl = layer_flops(cfg, counts)
    rec = {
        "ms_per_step": ms,
        "tokens_per_s": replica_throughput(cfg.T, world, ms),
        "active_tflops": world * fl["total"] / (ms / 1000.0) / 1e12,
        "stage_ms": {n: stage[n] for n in STAGES},
        "traced_step_ms": stage["step"],
        "roofline": roofline_of(cfg, counts, stage, peaks_, ms),
        "experts_touched": int(np.sum(counts > 0)),
        "clocks": clocks,
        "l2": "flushed before every step (inputs fit in L2)" if fb is not None else
              "not flushed: inputs larger than L2 (weights %.2f GB)" % (weight_bytes_total(cfg) / 1e9),
        "gpu_launches": steps * launches_per_step(cfg),
    }
    if cfg.name.startswith("decode_bf16") and rank == 0:
        rec["experts_touched_over_draws"] = decode_occupancy(layer)
    return rec, layer


def e2e_throughput(layer: Layer, steps: int, warmup: int, world: int) -> dict:
    """The same step through moe_forward with the input copied in from pinned
    host memory and the output copied back, every step.  Serving-style double
    buffering: step i's input copy runs on an input stream and its output copy
    on an output stream, so they overlap the layer of the neighbouring steps;
    every step's two copies lie inside the timed region (it starts before the
    first input copy and ends after the last output copy)."""
    import torch

    cfg, dev, y = layer.cfg, layer.dev, layer.y
    T, d = cfg.T, cfg.d_model
    stream = torch.cuda.current_stream()
    x_host = torch.empty(T, d, dtype=layer.tdt, pin_memory=True)
    x_host.copy_(dev["x"].cpu())
    y_host = [torch.empty(T, d, dtype=layer.tdt, pin_memory=True) for _ in range(2)]
    x_in = [torch.empty_like(dev["x"]) for _ in range(2)]
    y_out = [torch.empty_like(y) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = {name: [torch.cuda.Event() for _ in range(2)] for name in ("h2d", "done", "d2h")}
    used = [False, False]

    def e2e_step(i):
        b = i % 2
        if used[b]:
            s_in.wait_event(ev["done"][b])     # x_in[b] consumed by step i - 2
            stream.wait_event(ev["d2h"][b])    # y_out[b] copied out by step i - 2
        with torch.cuda.stream(s_in):
            x_in[b].copy_(x_host, non_blocking=True)
            ev["h2d"][b].record(s_in)
        stream.wait_event(ev["h2d"][b])
        layer.step(stream, x=x_in[b], y=y_out[b])
        ev["done"][b].record(stream)
        s_out.wait_event(ev["done"][b])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(y_out[b], non_blocking=True)
            ev["d2h"][b].record(s_out)
        used[b] = True

    for i in range(warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    layer.step(stream)  # the device-resident step's output, for the comparison below
    torch.cuda.synchronize()
    used[0] = used[1] = False
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(steps):
        e2e_step(i)
    for b in range(2):
        if used[b]:
            stream.wait_event(ev["d2h"][b])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / steps, world)
    # the last step's output, read back on the host, is the device-resident step's
    same = bool(torch.equal(y_host[(steps - 1) % 2].view(torch.uint8), y.cpu().view(torch.uint8)))
    return {"value": replica_throughput(T, world, e2e_ms), "unit": "tokens/s",
            "h2d_bytes_per_step": T * d * x_host.element_size(),
            "d2h_bytes_per_step": T * d * y_host[0].element_size(),
            "copies": "pinned host <-> device every step on their own streams, double-buffered against the layer",
            "output_matches_device_step": same}


def parse_workloads(spec: str, headline: str) -> list:
    if spec == "none":
        return []
    if spec == "all":
        return list(EXTRA_WORKLOADS)
    want = set(spec.split(","))
    return [(n, ov) for n, ov in EXTRA_WORKLOADS if workload_key(n, ov) in want or n in want]


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="mixtral_bf16", choices=sorted(synth.WORKLOADS))
    ap.add_argument("--T", type=int, default=None, help="override the token count (decode sweep)")
    ap.add_argument("--zipf", type=float, default=None, help="override the Zipf routing-bias exponent")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=INT",
                    help="override a shape field of the workload (d_model, d_ff, n_experts, top_k), e.g. for a "
                         "small profiling case")
    ap.add_argument("--workloads", default=None,
                    help="other configurations measured in the same run: all (default for the unmodified "
                         "headline workload), none, or a comma list of names / keys such as decode_bf16[T=4]")
    ap.add_argument("--cpu-tokens", type=int, default=0,
                    help="tokens of the CPU-oracle sample (0: the whole batch up to 2048 tokens, else 1024)")
    ap.add_argument("--ref-tokens", type=int, default=0, help="tokens per step of --impl reference (0: as above)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e4m3", action="store_true",
                    help="run the experts with 8-bit (FP8 E4M3) weights, quantised on the GPU from the bf16 ones")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    cfg = synth.workload(args.workload)
    if args.T is not None:
        cfg = cfg.replace(T=args.T)
    if args.zipf is not None:
        cfg = cfg.replace(zipf_s=args.zipf)
    for kv in args.set:
        field, val = kv.split("=", 1)
        if field not in ("d_model", "d_ff", "n_experts", "top_k", "d_ff_shared"):
            ap.error(f"--set: unknown field {field}")
        cfg = cfg.replace(**{field: int(val)})
    if args.e4m3:
        if cfg.dtype != "bf16":
            ap.error("--e4m3 needs a bf16 workload")
        cfg = cfg.replace(e4m3=True)
    modified = bool(args.set or args.T is not None or args.zipf is not None or args.e4m3)
    if modified:
        cfg = cfg.replace(name=f"{cfg.name}[T={cfg.T},d={cfg.d_model},f={cfg.d_ff},E={cfg.n_experts},"
                               f"k={cfg.top_k},zipf={cfg.zipf_s}" + (",e4m3]" if cfg.e4m3 else "]"))
    spec = args.workloads if args.workloads is not None else (
        "all" if not modified and args.workload == "mixtral_bf16" else "none")

    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)
    pk = peaks()
    flush_buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")

    # ---- the headline workload: device steps, traced stages, end to end
    rec, layer = measure_workload(cfg, args.steps, args.warmup, world, rank, local, pk, flush_buf)
    e2e = e2e_throughput(layer, args.steps, args.warmup, world)
    line = {
        "metric": METRIC,
        "value": rec["tokens_per_s"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": rec["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if cfg.e4m3 else cfg.dtype,
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": dict(config_dict(cfg, world), l2=rec["l2"]),
        "active_tflops": rec["active_tflops"],
        "stage_ms": rec["stage_ms"],
        "traced_step_ms": rec["traced_step_ms"],
        "roofline": rec["roofline"],
        "experts_touched": rec["experts_touched"],
        "clocks": rec["clocks"],
        "e2e": e2e,
        "gpu_launches": rec["gpu_launches"],
    }
    if "experts_touched_over_draws" in rec:
        line["experts_touched_over_draws"] = rec["experts_touched_over_draws"]
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n = args.cpu_tokens if args.cpu_tokens else oracle_sample_tokens(cfg)
        line["cpu_baseline"] = {k2: v for k2, v in cpu_baseline(cfg, layer.dev, n).items() if k2 != "seconds"}
    del layer
    torch.cuda.empty_cache()

    # ---- every other configuration, device steps and traced stages
    extra = {}
    for name, ov in parse_workloads(spec, cfg.name):
        wcfg = synth.workload(name, **ov)
        wcfg = wcfg.replace(name=workload_key(name, ov))  # the key its DRAM-traffic record is stored under
        r, lay = measure_workload(wcfg, args.steps, args.warmup, world, rank, local, pk, flush_buf)
        extra[workload_key(name, ov)] = r
        del lay
        torch.cuda.empty_cache()
    if extra:
        line["workloads"] = extra
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
