"""Build libregen_attn.so in-tree with nvcc for sm_100a.

    python -m dit_attention_b200.build [--verbose]

The library links the CUDA runtime statically and exports only the regen_*
symbols declared in include/regen_attn.h.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
LIB = os.path.join(PKG, "libregen_attn.so")
SOURCES = ["regen_attn.cu"]
HEADERS = ["ctx_cache.h", "ptx.cuh", "attn_fwd.cuh", "attn_bwd.cuh", "attn_fp8.cuh", "proj_gemm.cuh", "rope3d.cuh", "lse_merge.cuh"]
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS + ["exports.map"]]
    deps.append(os.path.join(ROOT, "include", "regen_attn.h"))
    deps.append(os.path.abspath(__file__))
    return any(os.path.getmtime(d) > t for d in deps)


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = [
        NVCC, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
        "-shared", "-Xcompiler", "-fPIC,-fvisibility=hidden", "-cudart", "static",
        "-I", os.path.join(ROOT, "include"), "-I", CSRC,
        "-Xlinker", "--version-script=" + os.path.join(CSRC, "exports.map"),
        "-o", tmp,
    ] + [os.path.join(CSRC, f) for f in SOURCES]
    if verbose:
        cmd.insert(1, "-Xptxas=-v")
    res = subprocess.run(cmd, capture_output=True, text=True)
    if verbose or res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
    if res.returncode != 0:
        raise RuntimeError("nvcc failed building libregen_attn.so")
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force=True, verbose="--verbose" in sys.argv)
    print(LIB)
