"""libuw driven from a plain C program on the GPU (no Python between the
caller and the library): tests/c_caller/uw_c_caller.c is compiled with gcc
against include/uw.h, linked with libuw.so and the CUDA runtime, and run.
It encodes, binds, decodes (bit-exact) and runs a fused stream-K matmul that
must equal the plain-BF16 kernel bit for bit."""
import os
import shutil
import subprocess

import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PKG = os.path.join(ROOT, "decode_gemm_exponent_b200")
CUDA_HOME = os.environ.get("CUDA_HOME", "/usr/local/cuda")

pytestmark = pytest.mark.gpu


def test_c_caller_decode_and_matmul(tmp_path):
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    lib = os.path.join(PKG, "libuw.so")
    assert os.path.exists(lib), "build libuw.so first"
    cc = shutil.which("gcc") or shutil.which("cc")
    assert cc, "no C compiler"
    exe = str(tmp_path / "uw_c_caller")
    subprocess.check_call([cc, "-std=c99", "-O1", "-Wall", "-Werror",
                           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA_HOME, "include"),
                           os.path.join(ROOT, "tests", "c_caller", "uw_c_caller.c"), "-o", exe,
                           "-L", PKG, "-luw", "-L", os.path.join(CUDA_HOME, "lib64"), "-lcudart",
                           "-Wl,-rpath," + PKG + ":" + os.path.join(CUDA_HOME, "lib64")])
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "c caller ok" in r.stdout
