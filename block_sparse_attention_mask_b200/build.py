"""Build libvsa.so (the CUDA kernels + C ABI) in-tree with nvcc for sm_100a.

Usage: python -m block_sparse_attention_mask_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
from typing import List

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libvsa.so")
SOURCES = ["vsa_plan.cu", "vsa_permute.cu", "vsa_attn.cu", "vsa_route.cu", "vsa_ulysses.cu", "vsa_pipeline.cu", "vsa_api.cu", "vsa_noalloc.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = os.environ.get("NVCC") or shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    return cand


def _inputs() -> List[str]:
    files = [os.path.join(CSRC, s) for s in SOURCES]
    files += [os.path.join(CSRC, f) for f in sorted(os.listdir(CSRC)) if f.endswith((".h", ".cuh"))]
    files += [os.path.join(INCLUDE, "vsa.h")]
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def build(force: bool = False, verbose: bool = False, extra: List[str] | None = None) -> str:
    if not force and up_to_date():
        return LIB
    objdir = os.path.join(HERE, "_build")
    os.makedirs(objdir, exist_ok=True)
    flags = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC,-O2", "-I", INCLUDE, "-I", CSRC,
             "--expt-relaxed-constexpr"] + ARCH + (extra or [])
    if verbose:
        flags += ["-Xptxas", "-v"]
    objs = [os.path.join(objdir, src.replace(".cu", ".o")) for src in SOURCES]
    cmds = [[nvcc(), "-c", os.path.join(CSRC, src), "-o", obj] + flags for src, obj in zip(SOURCES, objs)]
    # translation units compile in parallel
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max(1, min(len(cmds), os.cpu_count() or 1))) as ex:
        for _ in ex.map(subprocess.check_call, cmds):
            pass
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.check_call([nvcc(), "-shared", "-o", tmp] + objs + ARCH + ["-cudart", "static"])
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
