"""Python binding of the sm_100a sparse MoE layer library (``libmoe_b200.so``).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  The functions carry the C ABI's names (see ``include/moe.h``) and
take torch tensors (device memory) or raw integer addresses.  A missing or
unloadable library raises immediately -- there is no fallback path.
"""
from __future__ import annotations

import ctypes
import pathlib

__all__ = [
    "MoeError", "MoeConfig", "lib", "make_config", "moe_workspace_bytes", "moe_status_string",
    "moe_router_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward", "moe_device_status",
    "moe_permute_noalloc", "moe_expert_capacity", "moe_router_aux_losses", "moe_e4m3_weight_bytes",
    "moe_quantize_e4m3", "moe_forward_traced", "MOE_W_NATIVE", "MOE_W_E4M3",
    "MOE_F32", "MOE_BF16", "MOE_SOFTMAX_ALL_RENORM", "MOE_SOFTMAX_TOPK", "MOE_SIGMOID_TOPK_RENORM",
    "MOE_SOFTMAX_ALL_NO_RENORM", "MOE_ACT_SWIGLU", "MOE_ACT_GELU",
    "EXPORTED_SYMBOLS", "LIB_PATH",
]

LIB_PATH = pathlib.Path(__file__).resolve().parent / "libmoe_b200.so"

MOE_OK = 0
MOE_ERR_TIMEOUT = 5
MOE_ERR_BAD_EXPERT_ID = 6
MOE_F32, MOE_BF16 = 0, 1
MOE_SOFTMAX_ALL_RENORM, MOE_SOFTMAX_TOPK, MOE_SIGMOID_TOPK_RENORM, MOE_SOFTMAX_ALL_NO_RENORM = 0, 1, 2, 3
MOE_ACT_SWIGLU, MOE_ACT_GELU = 0, 1
MOE_W_NATIVE, MOE_W_E4M3 = 0, 1

EXPORTED_SYMBOLS = (
    "moe_workspace_bytes", "moe_status_string", "moe_router_topk", "moe_permute", "moe_grouped_ffn",
    "moe_combine", "moe_forward", "moe_device_status", "moe_permute_noalloc", "moe_expert_capacity",
    "moe_router_aux_losses", "moe_e4m3_weight_bytes", "moe_quantize_e4m3", "moe_forward_traced",
)


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {moe_status_string(status)} (status {status})")


class MoeConfig(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int64),
        ("d_model", ctypes.c_int32),
        ("n_experts", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("d_ff", ctypes.c_int32),
        ("n_shared", ctypes.c_int32),
        ("d_ff_shared", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("gating", ctypes.c_int32),
        ("bias_select_only", ctypes.c_int32),
        ("expert_act", ctypes.c_int32),
        ("wait_limit_ns", ctypes.c_int64),
        ("capacity_factor", ctypes.c_float),
        ("weight_format", ctypes.c_int32),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m top_routing_expert_gemm_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        vp, sz, i32 = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
        cfgp = ctypes.POINTER(MoeConfig)
        L.moe_workspace_bytes.argtypes = [cfgp]
        L.moe_workspace_bytes.restype = sz
        L.moe_status_string.argtypes = [i32]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_router_topk.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_permute.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_grouped_ffn.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_combine.argtypes = [cfgp, vp, vp, vp, vp, vp, vp]
        L.moe_forward.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_forward_traced.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp,
                                         ctypes.POINTER(vp)]
        L.moe_device_status.argtypes = [vp, sz, vp]
        L.moe_permute_noalloc.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, vp]
        L.moe_expert_capacity.argtypes = [cfgp]
        L.moe_router_aux_losses.argtypes = [cfgp, vp, vp, vp, vp, vp, sz, vp]
        L.moe_e4m3_weight_bytes.argtypes = [ctypes.c_int64, ctypes.c_int64]
        L.moe_quantize_e4m3.argtypes = [vp, ctypes.c_int64, ctypes.c_int32, vp, vp]
        for name in EXPORTED_SYMBOLS[2:]:
            getattr(L, name).restype = i32
        L.moe_expert_capacity.restype = ctypes.c_int64
        L.moe_e4m3_weight_bytes.restype = sz
        _lib = L
    return _lib


def make_config(T: int, d_model: int, n_experts: int, top_k: int, d_ff: int, dtype: int, gating: int,
                n_shared: int = 0, d_ff_shared: int = 0, bias_select_only: int = 0,
                wait_limit_ns: int = 0, expert_act: int = MOE_ACT_SWIGLU,
                capacity_factor: float = 0.0, weight_format: int = MOE_W_NATIVE) -> MoeConfig:
    return MoeConfig(T, d_model, n_experts, top_k, d_ff, n_shared, d_ff_shared, dtype, gating,
                     bias_select_only, expert_act, wait_limit_ns, capacity_factor, weight_format)


def _p(v) -> int | None:
    """Device address of a tensor / integer / None."""
    if v is None:
        return None
    if isinstance(v, int):
        return v
    return v.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str) -> None:
    if status != MOE_OK:
        raise MoeError(status, where)


def moe_status_string(status: int) -> str:
    return lib().moe_status_string(int(status)).decode()


def moe_workspace_bytes(cfg: MoeConfig) -> int:
    return int(lib().moe_workspace_bytes(ctypes.byref(cfg)))


def moe_expert_capacity(cfg: MoeConfig) -> int:
    """Rows each expert keeps (T*k when dropless); -1 for an invalid config."""
    return int(lib().moe_expert_capacity(ctypes.byref(cfg)))


def moe_router_topk(cfg, x, w_router, logit_bias, topk_ids, topk_w, ws, ws_bytes=None, stream=None) -> None:
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check(lib().moe_router_topk(ctypes.byref(cfg), _p(x), _p(w_router), _p(logit_bias), _p(topk_ids),
                                 _p(topk_w), _p(ws), nb, _stream(stream)), "moe_router_topk")


def moe_e4m3_weight_bytes(rows: int, cols: int) -> int:
    return int(lib().moe_e4m3_weight_bytes(rows, cols))


def moe_quantize_e4m3(src, rows: int, cols: int, blob, stream=None) -> None:
    """bf16 [rows, cols] -> E4M3 blob (codes, then one fp32 scale per row)."""
    _check(lib().moe_quantize_e4m3(_p(src), rows, cols, _p(blob), _stream(stream)), "moe_quantize_e4m3")


def moe_router_aux_losses(cfg, x, w_router, counts, out, ws, ws_bytes=None, stream=None) -> None:
    """out[0] = balance loss (without alpha), out[1] = router z-loss (without its weight)."""
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check(lib().moe_router_aux_losses(ctypes.byref(cfg), _p(x), _p(w_router), _p(counts), _p(out), _p(ws), nb,
                                       _stream(stream)), "moe_router_aux_losses")


def moe_permute(cfg, topk_ids, x, counts, offsets, perm, row_of, x_perm, ws, ws_bytes=None, stream=None) -> None:
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check(lib().moe_permute(ctypes.byref(cfg), _p(topk_ids), _p(x), _p(counts), _p(offsets), _p(perm),
                             _p(row_of), _p(x_perm), _p(ws), nb, _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg, topk_ids, x, counts, offsets, perm, row_of, x_perm, stream=None) -> None:
    """moe_permute without a workspace (its scratch is a fixed array inside the library)."""
    _check(lib().moe_permute_noalloc(ctypes.byref(cfg), _p(topk_ids), _p(x), _p(counts), _p(offsets), _p(perm),
                                     _p(row_of), _p(x_perm), _stream(stream)), "moe_permute_noalloc")


def moe_grouped_ffn(cfg, x_perm, offsets, w_gate_up, w_down, y_perm, ws, ws_bytes=None, stream=None) -> None:
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check(lib().moe_grouped_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(w_gate_up), _p(w_down),
                                 _p(y_perm), _p(ws), nb, _stream(stream)), "moe_grouped_ffn")


def moe_combine(cfg, y_perm, row_of, topk_w, y_shared, y, stream=None) -> None:
    _check(lib().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(row_of), _p(topk_w), _p(y_shared), _p(y),
                             _stream(stream)), "moe_combine")


def moe_forward(cfg, x, w_router, logit_bias, w_gate_up, w_down, ws_gate_up, ws_down, y,
                opt_topk_ids=None, opt_topk_w=None, opt_counts=None, ws=None, ws_bytes=None, stream=None) -> None:
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    _check(lib().moe_forward(ctypes.byref(cfg), _p(x), _p(w_router), _p(logit_bias), _p(w_gate_up), _p(w_down),
                             _p(ws_gate_up), _p(ws_down), _p(y), _p(opt_topk_ids), _p(opt_topk_w),
                             _p(opt_counts), _p(ws), nb, _stream(stream)), "moe_forward")


def moe_forward_traced(cfg, x, w_router, logit_bias, w_gate_up, w_down, ws_gate_up, ws_down, y,
                       opt_topk_ids=None, opt_topk_w=None, opt_counts=None, ws=None, ws_bytes=None, stream=None,
                       stage_events=None) -> None:
    """moe_forward with six stage markers: ``stage_events`` is a sequence of six
    torch.cuda.Event (or None entries) recorded at the stage boundaries."""
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    arr = None
    if stage_events is not None:
        if len(stage_events) != 6:
            raise ValueError("stage_events needs six entries")
        handles = []
        for ev in stage_events:
            if ev is None:
                handles.append(None)
                continue
            if not ev.cuda_event:  # torch creates its events on the first record
                ev.record(torch_stream(stream))
            handles.append(ev.cuda_event)
        arr = (ctypes.c_void_p * 6)(*handles)
    _check(lib().moe_forward_traced(ctypes.byref(cfg), _p(x), _p(w_router), _p(logit_bias), _p(w_gate_up),
                                    _p(w_down), _p(ws_gate_up), _p(ws_down), _p(y), _p(opt_topk_ids),
                                    _p(opt_topk_w), _p(opt_counts), _p(ws), nb, _stream(stream), arr),
           "moe_forward_traced")


def torch_stream(stream):
    """The torch stream object for the ``stream`` argument of the calls above."""
    import torch
    if stream is None:
        return torch.cuda.current_stream()
    if isinstance(stream, int):
        return torch.cuda.ExternalStream(stream)
    return stream


def moe_device_status(ws, ws_bytes=None, stream=None) -> int:
    """Synchronise ``stream`` and return the workspace status word as a moe_status code."""
    nb = ws_bytes if ws_bytes is not None else ws.numel() * ws.element_size()
    return int(lib().moe_device_status(_p(ws), nb, _stream(stream)))
