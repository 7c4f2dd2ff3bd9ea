"""Host-side checks of the C ABI that need no GPU: the library builds, loads,
exports every entry point include/moe.h declares, and rejects bad arguments
before launching anything."""
import ctypes
import pathlib
import re

import pytest

import top_routing_expert_gemm_b200 as moe
from top_routing_expert_gemm_b200 import build

ROOT = pathlib.Path(__file__).resolve().parents[1]


@pytest.fixture(scope="module")
def L():
    build.build()
    return moe.lib()


def _declared():
    names = set()
    for h in (ROOT / "include").glob("*.h"):
        txt = re.sub(r"/\*.*?\*/", "", h.read_text(), flags=re.S)
        names |= set(re.findall(r"\b(moe_[a-z0-9_]+)\s*\(", txt))
    return names


def test_every_declared_symbol_is_exported(L):
    declared = _declared()
    assert declared, "no declarations parsed"
    assert declared <= set(moe.EXPORTED_SYMBOLS) | declared
    for name in declared:
        assert hasattr(L, name), name
        assert ctypes.cast(getattr(L, name), ctypes.c_void_p).value


def test_binding_covers_the_header():
    assert _declared() == set(moe.EXPORTED_SYMBOLS)


def test_status_strings(L):
    assert moe.moe_status_string(0) == "ok"
    assert "workspace" in moe.moe_status_string(3)
    assert moe.moe_status_string(99) == "unknown status"


def _cfg(**kw):
    base = dict(T=64, d_model=256, n_experts=8, top_k=2, d_ff=512, dtype=moe.MOE_BF16, gating=1)
    base.update(kw)
    return moe.make_config(**base)


def test_workspace_bytes_valid_and_invalid(L):
    n = moe.moe_workspace_bytes(_cfg())
    # at least x_perm + h + y_perm for 128 rows
    assert n >= 2 * (128 * 256 * 2) + 128 * 512 * 2
    assert n % 256 == 0
    assert moe.moe_workspace_bytes(_cfg(top_k=9)) == 0          # k > E
    assert moe.moe_workspace_bytes(_cfg(d_model=250)) == 0      # not a multiple of 8
    assert moe.moe_workspace_bytes(_cfg(n_experts=2048, top_k=2)) == 0
    assert moe.moe_workspace_bytes(_cfg(gating=7)) == 0
    big = moe.moe_workspace_bytes(_cfg(n_shared=1, d_ff_shared=512))
    assert big > n


def _call_forward(L, cfg, ws_bytes=1 << 20, ptr=256):
    # fake, aligned, never-dereferenced addresses: every call below must fail its host checks
    p = ctypes.c_void_p(ptr)
    return L.moe_forward(ctypes.byref(cfg), p, p, None, p, p, None, None, p, None, None, None, p, ws_bytes, None)


def test_host_checks_reject_before_launch(L):
    assert _call_forward(L, _cfg(top_k=0)) == 1                     # invalid
    assert _call_forward(L, _cfg(n_experts=2000)) == 2              # beyond the build's limits
    assert _call_forward(L, _cfg(top_k=17, n_experts=32)) == 2      # beyond the build's limits
    assert _call_forward(L, _cfg(), ws_bytes=16) == 3               # workspace too small
    assert _call_forward(L, _cfg(), ptr=258) == 1                   # misaligned pointers
    assert _call_forward(L, _cfg(n_shared=1, d_ff_shared=512), ws_bytes=1 << 30) == 1  # shared weights missing
    cfg = _cfg()
    assert L.moe_forward(ctypes.byref(cfg), None, None, None, None, None, None, None, None, None, None, None,
                         ctypes.c_void_p(256), 1 << 30, None) == 1  # null tensors
    assert L.moe_router_topk(None, None, None, None, None, None, None, 0, None) == 1


def test_config_struct_layout():
    assert ctypes.sizeof(moe.MoeConfig) == 64
    assert moe.MoeConfig.expert_act.offset == 44
    assert moe.MoeConfig.wait_limit_ns.offset == 48
    assert moe.MoeConfig.capacity_factor.offset == 56
    assert moe.MoeConfig.weight_format.offset == 60


def test_expert_capacity_host_arithmetic(L):
    """ceil(T*k/E * factor) on the host, T*k when dropless, capped at T."""
    assert moe.moe_expert_capacity(_cfg(T=512, top_k=2, n_experts=8, capacity_factor=1.25)) == 160
    assert moe.moe_expert_capacity(_cfg(T=512, top_k=2, n_experts=8, capacity_factor=1.0)) == 128
    assert moe.moe_expert_capacity(_cfg(T=10, top_k=1, n_experts=3, d_ff=8, capacity_factor=1.0)) == 4
    assert moe.moe_expert_capacity(_cfg(T=64, top_k=2)) == 128
    assert moe.moe_expert_capacity(_cfg(T=64, top_k=2, capacity_factor=100.0)) == 64
    assert moe.moe_expert_capacity(_cfg(capacity_factor=-1.0)) == -1
    assert moe.moe_expert_capacity(_cfg(capacity_factor=float("nan"))) == -1
    assert moe.moe_expert_capacity(_cfg(expert_act=2)) == -1
    assert moe.moe_expert_capacity(_cfg(gating=4)) == -1


def _fake(addr=256):
    return ctypes.c_void_p(addr)


def _launching_calls(L, cfg, ws_bytes=1 << 30):
    """Every entry point that launches work, with valid shapes and fake aligned addresses."""
    p, c = _fake(), ctypes.byref(cfg)
    return {
        "moe_router_topk": lambda: L.moe_router_topk(c, p, p, None, p, p, p, ws_bytes, None),
        "moe_permute": lambda: L.moe_permute(c, p, p, p, p, p, p, p, p, ws_bytes, None),
        "moe_grouped_ffn": lambda: L.moe_grouped_ffn(c, p, p, p, p, p, p, ws_bytes, None),
        "moe_combine": lambda: L.moe_combine(c, p, p, p, None, p, None),
        "moe_forward": lambda: L.moe_forward(c, p, p, None, p, p, None, None, p, None, None, None, p, ws_bytes,
                                             None),
        "moe_permute_noalloc": lambda: L.moe_permute_noalloc(c, p, p, p, p, p, p, p, None),
        "moe_router_aux_losses": lambda: L.moe_router_aux_losses(c, p, p, p, p, p, ws_bytes, None),
        "moe_quantize_e4m3": lambda: L.moe_quantize_e4m3(p, 64, 256, p, None),
    }


def test_injected_launch_failure_reports_cuda_error_after_host_checks(L, monkeypatch):
    """MOE_FAULT=launch: each launching entry point answers MOE_ERR_CUDA once its
    host-side checks pass (the hook sits before the first CUDA call of the
    call, so nothing is launched; the GPU tests check that no output changes)."""
    monkeypatch.setenv("MOE_FAULT", "launch")
    for name, call in _launching_calls(L, _cfg()).items():
        assert call() == 4, name
    # host-side checks still come first: the injected failure never masks them
    bad = _launching_calls(L, _cfg(top_k=0))
    for name in ("moe_router_topk", "moe_permute", "moe_grouped_ffn", "moe_combine", "moe_forward",
                 "moe_permute_noalloc", "moe_router_aux_losses"):
        assert bad[name]() == 1, name
    assert _launching_calls(L, _cfg(), ws_bytes=16)["moe_forward"]() == 3
    assert _launching_calls(L, _cfg(n_experts=2048))["moe_permute_noalloc"]() == 2
    assert L.moe_quantize_e4m3(_fake(), 64, 250, _fake(), None) == 1
    # any other value of the variable injects nothing
    monkeypatch.setenv("MOE_FAULT", "none")
    assert _launching_calls(L, _cfg(top_k=0))["moe_forward"]() == 1


def test_noalloc_dispatch_reports_the_same_config_status_as_moe_permute(L):
    for cfg, want in ((_cfg(n_experts=2048), 2), (_cfg(top_k=17, n_experts=32), 2), (_cfg(top_k=0), 1),
                      (_cfg(d_model=250), 1), (_cfg(n_shared=2, d_ff_shared=512), 2)):
        got = L.moe_permute_noalloc(ctypes.byref(cfg), _fake(), _fake(), _fake(), _fake(), _fake(), _fake(),
                                    _fake(), None)
        ref = L.moe_permute(ctypes.byref(cfg), _fake(), _fake(), _fake(), _fake(), _fake(), _fake(), _fake(),
                            _fake(), 1 << 30, None)
        assert got == ref == want, (cfg.n_experts, cfg.top_k, got, ref)
