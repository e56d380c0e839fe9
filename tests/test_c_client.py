"""The C ABI from plain C: compile tests/c/abi_host_calls.c with gcc against include/etp.h, link
libetp.so, run the host-only calls (no GPU needed)."""
import os
import shutil
import subprocess

import pytest

import equivariant_mlip_tensor_edge_b200 as etp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("gcc") is None, reason="no C compiler")
def test_plain_c_client(tmp_path):
    lib = etp.LIB_PATH
    assert os.path.exists(lib)
    exe = tmp_path / "abi_host_calls"
    cuda_lib = "/usr/local/cuda/lib64"
    cmd = ["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"),
           os.path.join(ROOT, "tests", "c", "abi_host_calls.c"), lib, "-o", str(exe),
           f"-Wl,-rpath,{os.path.dirname(lib)}", f"-Wl,-rpath,{cuda_lib}"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, run.stdout + run.stderr
    assert "ok uniform" in run.stdout and "ok general" in run.stdout and "ok errors" in run.stdout
