"""Build libpagedkv.so in place with nvcc for sm_100a.

Each source compiles to its own object (in parallel) under ``_build/``; the
objects are then linked into one shared library.

Usage: python -m paged_kv_cache_383_b200.build_lib [--verbose] [--ptxas]
"""
from __future__ import annotations

import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(HERE, "libpagedkv.so")
OBJ_DIR = os.path.join(HERE, "_build")

SOURCES = ["status.cpp", "block_manager.cpp", "cache_ops.cu", "decode.cu",
           "prefill.cu", "probe.cu", "swap.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
# No --split-compile: splitting a translation unit's device code into
# partitions compiled in parallel made the generated code differ from build to
# build, and the prefill kernel's speed with it (up to 8 %).
FLAGS = ["-O3", "-lineinfo", "-std=c++17", "-Xcompiler", "-fPIC,-O3,-Wall"]


def nvcc() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"),
                 "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def _compile(src: str, ptxas_verbose: bool, verbose: bool) -> str:
    obj = os.path.join(OBJ_DIR, os.path.basename(src) + ".o")
    cmd = [nvcc(), *ARCH, *FLAGS, "-I", INCLUDE, "-I", CSRC, "-c", src,
           "-o", obj + ".tmp"]
    if ptxas_verbose:
        cmd.insert(1, "-Xptxas=-v")
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError(f"nvcc failed on {src}:\n" + res.stdout +
                           res.stderr)
    if verbose or ptxas_verbose:
        sys.stdout.write(res.stdout + res.stderr)
    os.replace(obj + ".tmp", obj)
    return obj


def build(verbose: bool = False, ptxas_verbose: bool = False) -> str:
    """Compile every source into one shared library; returns its path."""
    srcs = [os.path.join(CSRC, s) for s in SOURCES]
    newest = max(os.path.getmtime(p) for p in
                 srcs + [os.path.join(CSRC, f) for f in os.listdir(CSRC)] +
                 [os.path.join(INCLUDE, "pagedkv.h"), __file__])
    if (os.path.exists(LIB) and os.path.getmtime(LIB) >= newest
            and not ptxas_verbose):
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    workers = max(1, min(len(srcs), os.cpu_count() or 1))
    with cf.ThreadPoolExecutor(workers) as pool:
        objs = list(pool.map(lambda s: _compile(s, ptxas_verbose, verbose),
                             srcs))
    cmd = [nvcc(), *ARCH, "-shared", "-o", LIB + ".tmp", *objs]
    if verbose:
        print(" ".join(cmd), flush=True)
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("nvcc link failed:\n" + res.stdout + res.stderr)
    os.replace(LIB + ".tmp", LIB)
    return LIB


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv,
                ptxas_verbose="--ptxas" in sys.argv))
