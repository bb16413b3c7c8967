"""The C ABI used from plain C (no Python objects, no PyTorch): a program
linked against the library and the CUDA runtime compiles here; on a GPU it
runs one fp32 forward (CUDA-core kernels) and one bf16 forward + backward
(tensor-core kernels) and checks them against the CPU oracle."""
import os
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _build(tmp_path):
    from lsh_attention_02_b200 import build
    from oracle import oracle
    lib = build.build()
    olib = oracle.build()
    exe = str(tmp_path / "abi_forward")
    cmd = ["gcc", "-std=c99", "-O1", "-Wall", "-Werror", os.path.join(ROOT, "tests", "c_abi", "abi_forward.c"),
           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
           "-L", os.path.dirname(lib), "-L", os.path.dirname(olib), "-L", os.path.join(CUDA, "lib64"),
           "-Wl,-rpath," + os.path.dirname(lib), "-Wl,-rpath," + os.path.dirname(olib),
           "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
           "-l:" + os.path.basename(lib), "-l:" + os.path.basename(olib), "-lcudart", "-lm", "-o", exe]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return exe


def test_c_program_links_against_the_library(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([exe, "--compile-check"], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr


@pytest.mark.gpu
def test_c_program_forward_matches_oracle(tmp_path):
    exe = _build(tmp_path)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip().endswith("ok")
