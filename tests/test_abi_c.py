"""The C ABI from C: tests/abi_host_client.c includes include/moe.h as C99
(no C++), links the built library and calls its host-side entry points;
tests/abi_device_client.c (GPU) runs one layer through moe_forward with device
memory from the CUDA runtime's C API."""
import pathlib
import shutil
import subprocess

import numpy as np
import pytest

import oracle
import synth
from top_routing_expert_gemm_b200 import build
import top_routing_expert_gemm_b200 as moe

ROOT = pathlib.Path(__file__).resolve().parents[1]


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_client_builds_links_and_runs(tmp_path):
    build.build()
    lib_dir = moe.LIB_PATH.parent
    exe = tmp_path / "abi_host_client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", str(ROOT / "include"),
                    str(ROOT / "tests" / "abi_host_client.c"), "-o", str(exe), f"-L{lib_dir}", "-lmoe_b200",
                    f"-Wl,-rpath,{lib_dir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"


CUDA = pathlib.Path("/usr/local/cuda")


@pytest.mark.gpu
@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_client_runs_a_layer_on_the_gpu(tmp_path):
    build.build()
    lib_dir = moe.LIB_PATH.parent
    exe = tmp_path / "abi_device_client"
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", str(ROOT / "include"),
                    "-I", str(CUDA / "include"), str(ROOT / "tests" / "abi_device_client.c"), "-o", str(exe),
                    f"-L{lib_dir}", "-lmoe_b200", f"-L{CUDA / 'lib64'}", "-lcudart", "-lm",
                    f"-Wl,-rpath,{lib_dir}", f"-Wl,-rpath,{CUDA / 'lib64'}"], check=True)
    dump = tmp_path / "y_ids.bin"
    out = subprocess.run([str(exe), str(dump)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
    _compare_with_the_oracle(dump)


# The C client's layer and its inputs: splitmix64 draws (the published
# generator: state += 0x9E3779B97F4A7C15, then the two xor-shift-multiply
# rounds and a final xor-shift), scaled to [-1, 1) and by a per-tensor scale
# in float, rounded to bf16 (nearest even) -- regenerated here from that
# definition, in the order the client draws them.
C_T, C_D, C_E, C_K, C_F = 300, 512, 8, 2, 640


def _splitmix64_uniform(seed: int, n: int) -> tuple[np.ndarray, int]:
    with np.errstate(over="ignore"):
        i = np.arange(1, n + 1, dtype=np.uint64)
        z = np.uint64(seed) + i * np.uint64(0x9E3779B97F4A7C15)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    u = ((z >> np.uint64(11)).astype(np.float64) / 9007199254740992.0 * 2.0 - 1.0).astype(np.float32)
    end = (seed + n * 0x9E3779B97F4A7C15) % (1 << 64)
    return u, end


def _client_inputs():
    seed = 7
    out = []
    for n, scale in ((C_T * C_D, 1.0), (C_E * C_D, 0.05), (C_E * 2 * C_F * C_D, 0.05), (C_E * C_D * C_F, 0.05)):
        u, seed = _splitmix64_uniform(seed, n)
        v = (u * np.float32(scale)).astype(np.float32)
        out.append(synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(v)).astype(np.float64))
    x, wr, wgu, wd = out
    return (x.reshape(C_T, C_D), wr.reshape(C_E, C_D), wgu.reshape(C_E, 2 * C_F, C_D), wd.reshape(C_E, C_D, C_F))


def _compare_with_the_oracle(dump):
    raw = dump.read_bytes()
    y_bits = np.frombuffer(raw[:C_T * C_D * 2], dtype=np.uint16)
    ids = np.frombuffer(raw[C_T * C_D * 2:], dtype=np.int32).reshape(C_T, C_K).astype(np.int64)
    y = synth.bf16_bits_to_f32(y_bits).astype(np.float64).reshape(C_T, C_D)
    x, wr, wgu, wd = _client_inputs()
    r = oracle.route(x, wr, None, C_K, oracle.SOFTMAX_TOPK)
    flipped = np.any(r.ids != ids, axis=1)
    assert not np.any(flipped & (r.gap >= 1e-3))            # ids agree outside near ties
    y_ref, _, _ = oracle.moe_layer(x, wr, None, C_K, oracle.SOFTMAX_TOPK,
                                   lambda e: (wgu[e, :C_F], wgu[e, C_F:], wd[e]), C_E, ids=ids)
    err = float(np.max(np.abs(y - y_ref)) / np.max(np.abs(y_ref)))
    assert err <= 2e-2, err


def test_splitmix64_reference_values():
    """The generator above against splitmix64's published first outputs for
    seed 0 (0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, ...)."""
    with np.errstate(over="ignore"):
        z = np.uint64(0) + np.arange(1, 3, dtype=np.uint64) * np.uint64(0x9E3779B97F4A7C15)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        z = z ^ (z >> np.uint64(31))
    assert [int(v) for v in z] == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4]
