"""Builds the CUDA library in-tree: gated_delta_rule_147_b200/libgdr.so (sm_100a).

Each source compiles to its own object (in parallel, under _build/), then one
link step makes the shared library.

Usage: python -m gated_delta_rule_147_b200.build [--force] [--verbose]
"""
from __future__ import annotations

import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
OBJDIR = os.path.join(ROOT, "_build")
SOURCES = ["api.cu", "decode.cu", "recurrent.cu", "chunk_sm100.cu", "chunk_erasefree_sm100.cu",
           "chunk_bwd.cu", "chunk_bwd_tc_sm100.cu", "chunk_bwd_grad_sm100.cu",
           "chunk_twopass_sm100.cu", "chunk_twopass256_sm100.cu", "chunk_twopass_general_sm100.cu", "selftest.cu",
           "static_scratch.cu"]
HEADERS = ["common.cuh", "chunk_common.cuh", "rcp_seed.h"]
LIB = os.path.join(HERE, "libgdr.so")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
COMPILE_FLAGS = [*ARCH, "-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC",
                 "--expt-relaxed-constexpr"]


def _nvcc() -> str:
    for cand in (os.environ.get("NVCC"), "/usr/local/cuda/bin/nvcc", "nvcc"):
        if cand and (os.path.isabs(cand) and os.path.exists(cand) or not os.path.isabs(cand)):
            return cand
    return "nvcc"


def _deps():
    deps = [os.path.join(CSRC, f) for f in SOURCES + HEADERS]
    deps.append(os.path.join(ROOT, "include", "gdr.h"))
    return deps


def _stale() -> bool:
    if not os.path.exists(LIB):
        return True
    t = os.path.getmtime(LIB)
    return any(os.path.getmtime(d) > t for d in _deps())


def _obj(src: str) -> str:
    return os.path.join(OBJDIR, os.path.splitext(src)[0] + ".o")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and not _stale():
        return LIB
    os.makedirs(OBJDIR, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include")]
    # a header change rebuilds every object; otherwise only sources newer than their object
    hdr_t = max(os.path.getmtime(d) for d in _deps() if not d.endswith(".cu"))

    def compile_one(src: str):
        obj = _obj(src)
        path = os.path.join(CSRC, src)
        if not force and os.path.exists(obj) and os.path.getmtime(obj) > max(os.path.getmtime(path), hdr_t):
            return
        cmd = [_nvcc(), *COMPILE_FLAGS, *inc, "-c", "-o", obj, path]
        if verbose:
            cmd.insert(1, "-Xptxas=-v")
            print(" ".join(cmd), flush=True)
        subprocess.run(cmd, check=True)

    with ThreadPoolExecutor(max_workers=min(len(SOURCES), os.cpu_count() or 4)) as ex:
        for f in [ex.submit(compile_one, s) for s in SOURCES]:
            f.result()
    link = [_nvcc(), *ARCH, "-shared", "-Xcompiler", "-fPIC", "-o", LIB, *[_obj(s) for s in SOURCES]]
    subprocess.run(link, check=True)
    return LIB


if __name__ == "__main__":
    build(force="--force" in sys.argv, verbose="--verbose" in sys.argv)
    print(LIB)
