"""Benchmark of the sparse MoE layer forward on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload mixtral_bf16|gptoss_bf16|deepseek_bf16|decode_bf16|tiny_f32] [--T T]

One step = one full pass of the layer (router + top-k, dispatch, grouped SwiGLU
experts, combine) over one batch of T synthetic tokens already resident in HBM.
Default workload: the Mixtral-shaped bf16 layer (T=2048, d=4096, E=8, k=2,
f=14336).  Inputs are larger than L2 (2.8 GB of expert weights per step), so L2
is not flushed between steps.  With N>1 (torchrun) every rank runs an
independent replica on its own T tokens (weak scaling, no data-path
collective); the step time is the max over ranks.

Rank 0 prints one JSON line.  ``value`` is tokens/s over all ranks; the line
also carries active TFLOP/s, the per-stage split, the roofline of the grouped
expert GEMMs, an end-to-end number through host buffers, SM clocks sampled
during the timed region and the CPU oracle's throughput on a bounded sample.
``--impl reference`` times the CPU oracle itself on the same workload.
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
    block-wide kernel for at most 1024 assignments, else count / scan /
    scatter) and the row gather (with 8-bit experts the gather-quantise), two
    expert GEMMs for the routed experts (8-bit: with the re-quantisation of h
    between them) and for each shared expert (8-bit: after quantising x, and
    with the re-quantisation of h), and the combine."""
    dispatch = 2 if cfg.T * cfg.top_k <= 1024 else 4
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


def cpu_baseline(cfg: synth.LayerConfig, dev: dict, n_tokens: int) -> dict:
    """The CPU oracle, as it stands, on a bounded sample of the workload."""
    oi = OracleInputs(cfg, dev, n_tokens)
    dt = time_oracle(oi)
    return {"value": oi.n / dt, "unit": "tokens/s", "cores": cpu_cores(), "kind": "oracle",
            "sample": oi.describe(), "seconds": dt}


def run_reference(args, cfg) -> None:
    """--impl reference: the CPU oracle timed on the host cores (rank 0 only)."""
    import torch

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev_name = "cuda" if torch.cuda.is_available() else "cpu"
    dev = {name: synth.device_tensor(cfg, name, dev_name) for name in synth.tensor_specs(cfg)}
    oi = OracleInputs(cfg, dev, args.ref_tokens)
    times = []
    for i in range(args.warmup + args.steps):
        dt = time_oracle(oi)
        if i >= args.warmup:
            times.append(dt)
    n = oi.n
    ms = 1000.0 * sum(times) / len(times)
    val = n / (ms / 1000.0)
    r = {"cores": cpu_cores(), "sample": oi.describe()}
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
    ap.add_argument("--cpu-tokens", type=int, default=128, help="tokens in the CPU-oracle baseline sample")
    ap.add_argument("--ref-tokens", type=int, default=32, help="tokens per step of --impl reference")
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
    if args.set or args.T is not None or args.zipf is not None or args.e4m3:
        cfg = cfg.replace(name=f"{cfg.name}[T={cfg.T},d={cfg.d_model},f={cfg.d_ff},E={cfg.n_experts},"
                               f"k={cfg.top_k},zipf={cfg.zipf_s}" + (",e4m3]" if cfg.e4m3 else "]"))

    if args.impl == "reference":
        run_reference(args, cfg)
        return

    import torch
    import torch.distributed as dist

    import top_routing_expert_gemm_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if world != args.gpus and rank == 0:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE {world}", file=sys.stderr)

    # ---- inputs, generated in HBM (each rank its own token batch: seed + rank)
    dev = {}
    for name in synth.tensor_specs(cfg):
        dev[name] = synth.device_tensor(cfg if name != "x" else cfg.replace(seed=cfg.seed + 7919 * rank),
                                        name, "cuda")
    bias_np = synth.zipf_bias(cfg)
    bias = torch.from_numpy(bias_np).cuda() if bias_np is not None else None
    wfmt = moe.MOE_W_E4M3 if cfg.e4m3 else moe.MOE_W_NATIVE
    if cfg.e4m3:  # the expert weights as the library's 8-bit blobs, quantised on the GPU
        for name in ("w_gate_up", "w_down", "ws_gate_up", "ws_down"):
            if name in dev:
                src = dev[name]
                rows = src.numel() // src.shape[-1]
                blob = torch.empty(moe.moe_e4m3_weight_bytes(rows, src.shape[-1]), dtype=torch.uint8, device="cuda")
                moe.moe_quantize_e4m3(src, rows, src.shape[-1], blob)
                dev[name + "_q"] = blob  # the bf16 values stay for the CPU oracle, which quantises them itself
    c = moe.make_config(cfg.T, cfg.d_model, cfg.n_experts, cfg.top_k, cfg.d_ff,
                        moe.MOE_BF16 if cfg.dtype == "bf16" else moe.MOE_F32, cfg.gating, cfg.n_shared,
                        cfg.d_ff_shared, cfg.bias_select_only, expert_act=cfg.act, weight_format=wfmt)
    tdt = torch.bfloat16 if cfg.dtype == "bf16" else torch.float32
    T, d, k, E = cfg.T, cfg.d_model, cfg.top_k, cfg.n_experts
    ws_bytes = moe.moe_workspace_bytes(c)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    y = torch.empty(T, d, dtype=tdt, device="cuda")
    ids = torch.empty(T, k, dtype=torch.int32, device="cuda")
    w = torch.empty(T, k, dtype=torch.float32, device="cuda")
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    stream = torch.cuda.current_stream()

    q = "_q" if cfg.e4m3 else ""  # the expert weights the kernels read

    def step():
        moe.moe_forward(c, dev["x"], dev["w_router"], bias, dev["w_gate_up" + q], dev["w_down" + q],
                        dev.get("ws_gate_up" + q), dev.get("ws_down" + q), y, ids, w, counts, ws, ws_bytes, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st = moe.moe_device_status(ws, ws_bytes, stream)
    if st != 0:
        raise RuntimeError(f"device status {st} after warm-up")
    counts_np = counts.cpu().numpy()

    # ---- timed region: K full steps through moe_forward
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        barrier()
        torch.cuda.synchronize()
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world)
    clocks = clk.summary()

    # ---- same step as its four C-ABI stages, events between them (per-stage split, roofline)
    ids2, w2 = torch.empty_like(ids), torch.empty_like(w)
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    counts2 = torch.empty_like(counts)
    perm = torch.empty(T * k, dtype=torch.int32, device="cuda")
    row_of = torch.empty(T * k, dtype=torch.int32, device="cuda")
    x_perm = torch.empty(T * k, d, dtype=tdt, device="cuda")
    y_perm = torch.empty(T * k, d, dtype=tdt, device="cuda")
    stage_names = ["router_topk", "permute", "grouped_ffn"] + (["shared_ffn"] if cfg.n_shared else []) + ["combine"]
    if cfg.n_shared:
        # the always-on expert as one group over all T tokens
        c_s = moe.make_config(T, d, 1, 1, cfg.d_ff_shared, c.dtype, cfg.gating, expert_act=cfg.act,
                              weight_format=wfmt)
        ws_s_bytes = moe.moe_workspace_bytes(c_s)
        ws_s = torch.zeros(ws_s_bytes, dtype=torch.uint8, device="cuda")
        off_s = torch.tensor([0, T], dtype=torch.int32, device="cuda")
        y_sh = torch.empty(T, d, dtype=tdt, device="cuda")
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(stage_names) + 1)] for _ in range(args.steps)]

    def staged(e=None):
        j = 0

        def mark():
            nonlocal j
            if e is not None:
                e[j].record(stream)
            j += 1

        mark()
        moe.moe_router_topk(c, dev["x"], dev["w_router"], bias, ids2, w2, ws, ws_bytes, stream)
        mark()
        moe.moe_permute(c, ids2, dev["x"], counts2, offsets, perm, row_of, x_perm, ws, ws_bytes, stream)
        mark()
        moe.moe_grouped_ffn(c, x_perm, offsets, dev["w_gate_up" + q], dev["w_down" + q], y_perm, ws, ws_bytes, stream)
        mark()
        if cfg.n_shared:
            moe.moe_grouped_ffn(c_s, dev["x"], off_s, dev["ws_gate_up" + q], dev["ws_down" + q], y_sh, ws_s,
                                ws_s_bytes, stream)
            mark()
        moe.moe_combine(c, y_perm, row_of, w2, y_sh if cfg.n_shared else None, y, stream)
        mark()

    for _ in range(args.warmup):
        staged()
    torch.cuda.synchronize()
    for i in range(args.steps):
        staged(evs[i])
    torch.cuda.synchronize()
    stage_ms = {n: statistics.mean(evs[i][j].elapsed_time(evs[i][j + 1]) for i in range(args.steps))
                for j, n in enumerate(stage_names)}

    # ---- end to end: pinned host x in, host y out, every step, through
    # moe_forward.  Serving-style double buffering: step i's input copy runs
    # on an input stream and its output copy on an output stream, so they
    # overlap the layer of the neighbouring steps; every step's two copies lie
    # inside the timed region (it starts before the first input copy and ends
    # after the last output copy).
    x_host = torch.empty(T, d, dtype=tdt, pin_memory=True)
    x_host.copy_(dev["x"].cpu())
    y_host = [torch.empty(T, d, dtype=tdt, pin_memory=True) for _ in range(2)]
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
        moe.moe_forward(c, x_in[b], dev["w_router"], bias, dev["w_gate_up" + q], dev["w_down" + q],
                        dev.get("ws_gate_up" + q), dev.get("ws_down" + q), y_out[b], ids, w, counts, ws, ws_bytes,
                        stream)
        ev["done"][b].record(stream)
        s_out.wait_event(ev["done"][b])
        with torch.cuda.stream(s_out):
            y_host[b].copy_(y_out[b], non_blocking=True)
            ev["d2h"][b].record(s_out)
        used[b] = True

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    used[0] = used[1] = False
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    s_in.wait_event(e0)
    s_out.wait_event(e0)
    for i in range(args.steps):
        e2e_step(i)
    for b in range(2):
        if used[b]:
            stream.wait_event(ev["d2h"][b])
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    # the last step's output, read back on the host, is the device-resident step's
    e2e_same = bool(torch.equal(y_host[(args.steps - 1) % 2].view(torch.uint8), y.cpu().view(torch.uint8)))

    pk, pk_kind = peaks()
    fl = layer_flops(cfg, counts_np)
    by = layer_bytes(cfg, counts_np)
    tokens_per_s = replica_throughput(T, world, ms)
    active_tflops = world * fl["total"] / (ms / 1000.0) / 1e12
    # dominant kernel: the grouped expert GEMMs (tcgen05), timed as the moe_grouped_ffn stage
    g_ms = stage_ms["grouped_ffn"] + stage_ms.get("shared_ffn", 0.0)
    gemm_tflops = (fl["experts"] + fl["shared"]) / (g_ms / 1000.0) / 1e12
    decode = cfg.T <= 64
    if decode:
        gbs = by["weights"] / (g_ms / 1000.0) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / pk["hbm_gbs"], "traffic": None}
    else:
        # 8-bit experts: the measured bf16 peak x 2, the nominal dense fp8 / bf16 ratio (4.5 / 2.25 PFLOP/s)
        tpk = pk["bf16_tflops"] * (2.0 if cfg.e4m3 else 1.0)
        roof = {"bound": "tensor", "achieved": gemm_tflops, "peak": tpk, "unit": "TFLOP/s",
                "frac": gemm_tflops / tpk, "traffic": None}
    if cfg.dtype != "bf16":
        kname = "grouped_gemm_f32_kernel (CUDA cores)"
    elif uses_decode_schedule(cfg):
        kname = "grouped_gemm_swap_kernel, decode schedule (weight rows as M, reductions split evenly over the CTAs)"
    else:
        kname = "grouped_gemm_tc_kernel (token rows as M)"
    roof["kernel"] = (kname + ": the GEMM-1 and GEMM-2 launches of moe_grouped_ffn"
                      + (" (routed and shared experts)" if cfg.n_shared else ""))
    roof["traffic"] = recorded_traffic(cfg.name, "decode" if uses_decode_schedule(cfg) else "tc")
    roof["peak_source"] = pk_kind + (" bf16 x 2 (nominal fp8/bf16 dense ratio)" if cfg.e4m3 and not decode else "")
    line = {
        "metric": METRIC,
        "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if cfg.e4m3 else cfg.dtype,
        "data": "synthetic (seeded counter-based generator; random-init weights)",
        "config": config_dict(cfg, world),
        "active_tflops": active_tflops,
        "stage_ms": stage_ms,
        "roofline": roof,
        "experts_touched": by["touched"],
        "clocks": clocks,
        "e2e": {"value": replica_throughput(T, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": T * d * x_host.element_size(),
                "d2h_bytes_per_step": T * d * y_host[0].element_size(),
                "copies": "pinned host <-> device every step on their own streams, double-buffered against the layer",
                "output_matches_device_step": e2e_same},
        "gpu_launches": args.steps * launches_per_step(cfg),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k2: v for k2, v in cpu_baseline(cfg, dev, args.cpu_tokens).items() if k2 != "seconds"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
