"""The C ABI on its own: a plain C program (tests/c_abi_roundtrip.c) built
against include/rans_b200.h and librans_b200.so, with no Python or PyTorch in
the process, codes and decodes on the GPU."""
import os
import subprocess

import pytest

from rans_entropy_coding_b200 import build as rbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(tmp_path):
    lib = rbuild.build()
    exe = str(tmp_path / "c_abi_roundtrip")
    cmd = ["gcc", "-O2", "-std=c99", "-Wall", "-Wextra",
           os.path.join(ROOT, "tests", "c_abi_roundtrip.c"), "-o", exe,
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           os.path.abspath(lib), "-L", os.path.join(CUDA, "lib64"), "-lcudart",
           "-Wl,-rpath," + os.path.dirname(os.path.abspath(lib)),
           "-Wl,-rpath," + os.path.join(CUDA, "lib64")]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_client_compiles(tmp_path):
    """Builds without a GPU: the header is plain C."""
    assert os.path.exists(_compile(tmp_path))


@pytest.mark.gpu
def test_c_client_round_trip(tmp_path):
    exe = _compile(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.startswith("ok ")
