"""The C ABI from plain C (a forward and a two-block ring step checked against
a closed form on the GPU): tests/host/abi_c_probe.c is compiled with gcc
against include/lca.h and liblca.so (no Python, no torch in the client).
The CPU part checks status strings and synchronous argument errors; the GPU
part runs a causal forward whose answer is a closed form (zero keys: each
output row is the running mean of v, lse_i = ln(i + 1))."""

import os
import shutil
import subprocess

import pytest

from long_context_exact_attention_b200 import lca

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "host", "abi_c_probe.c")
BIN = os.path.join(HERE, "host", "abi_c_probe.bin")
CUDA = "/usr/local/cuda"


def cuda_root():
    nvcc = shutil.which("nvcc")
    return os.path.dirname(os.path.dirname(nvcc)) if nvcc else CUDA


@pytest.fixture(scope="module")
def probe():
    lib = lca.lib()  # builds nothing; liblca.so must exist
    libdir = os.path.dirname(lca.LIB_PATH)
    cr = cuda_root()
    cudalib = next(p for p in (os.path.join(cr, "lib64"), os.path.join(cr, "targets",
                               "x86_64-linux", "lib")) if os.path.isdir(p))
    if not os.path.exists(BIN) or os.path.getmtime(BIN) < max(
            os.path.getmtime(SRC), os.path.getmtime(lca.LIB_PATH),
            os.path.getmtime(os.path.join(ROOT, "include", "lca.h"))):
        subprocess.run(["gcc", "-std=c11", "-O2", "-Wall", "-Werror", "-o", BIN, SRC,
                        "-I", os.path.join(ROOT, "include"), "-I", os.path.join(cr, "include"),
                        "-L", libdir, "-llca", "-L", cudalib, "-lcudart", "-lm",
                        f"-Wl,-rpath,{libdir}", f"-Wl,-rpath,{cudalib}"], check=True)
    del lib
    return BIN


def test_c_client_cpu(probe):
    r = subprocess.run([probe, "cpu"], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "ok" in r.stdout


@pytest.mark.gpu
def test_c_client_gpu_closed_form(probe):
    r = subprocess.run([probe, "gpu"], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stdout + r.stderr
    assert "ok" in r.stdout
