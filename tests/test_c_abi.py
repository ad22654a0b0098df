"""The C ABI used from a plain C program (tests/c_abi_example.c): compiled with
gcc against include/fp8amax.h, linked with libfp8amax.so, the CUDA runtime and
the oracle's C library; on a B200 it must run and print its success line."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    from fp8_tensor_scaled_b200 import build as lib_build
    from oracle import build as oracle_build
    lib = lib_build.build()
    olib = oracle_build.build()
    exe = str(tmp_path / "c_abi_example")
    cmd = ["gcc", "-O2", "-std=c11", os.path.join(ROOT, "tests", "c_abi_example.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-o", exe, lib, olib, "-L", os.path.join(CUDA, "lib64"), "-lcudart", "-lm",
           "-Wl,-rpath," + os.path.dirname(lib) + ":" + os.path.dirname(olib) + ":"
           + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True)
    return exe


@pytest.mark.skipif(shutil.which("gcc") is None, reason="needs gcc")
def test_c_program_compiles_and_links(tmp_path):
    assert os.path.exists(_build(tmp_path))


@pytest.mark.gpu
def test_c_program_runs(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr + r.stdout
    assert "C ABI example ok" in r.stdout
