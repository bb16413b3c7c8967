"""Builds liblsh_attn.so (the C-ABI CUDA library) in-tree with nvcc for sm_100a."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "csrc")
ROOT = os.path.dirname(HERE)
LIB = os.path.join(HERE, "liblsh_attn.so")
SOURCES = ["api.cu", "simt.cu", "sort.cu", "hash_tc.cu", "attn_fwd_tc.cu", "fused_fwd_tc.cu", "attn_bwd_tc.cu",
           "selftest.cu", "rotations.cu", "revblock.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]


def nvcc() -> str:
    cand = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "bin", "nvcc")
    return cand if os.path.exists(cand) else "nvcc"


def sources() -> list[str]:
    return [os.path.join(CSRC, s) for s in SOURCES]


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = sources() + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] + [os.path.join(ROOT, "include", "lsh_attn.h")]
    return any(os.path.getmtime(p) > t for p in deps)


def build(force: bool = False, verbose: bool = False, phase_trace: bool = False) -> str:
    """Compiles the library; phase_trace=True builds liblsh_attn_trace.so with the
    per-phase timestamp points compiled in (a tuning build, never the default)."""
    lib = LIB.replace(".so", "_trace.so") if phase_trace else LIB
    if not force and not phase_trace and not _stale():
        return LIB
    tmp = lib + f".tmp{os.getpid()}"
    cmd = [nvcc(), *ARCH, *FLAGS, *(["-DLSH_PHASE_TRACE"] if phase_trace else []), "-o", tmp, *sources()]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.check_call(cmd)
    os.replace(tmp, lib)
    return lib


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, verbose=True, phase_trace="--phase-trace" in sys.argv))
