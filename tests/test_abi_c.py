"""The C ABI from C: tests/abi_host_client.c includes include/moe.h as C99
(no C++), links the built library and calls its host-side entry points;
tests/abi_device_client.c (GPU) runs one layer through moe_forward with device
memory from the CUDA runtime's C API."""
import pathlib
import shutil
import subprocess

import pytest

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
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "ok"
