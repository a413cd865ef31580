"""Builds libpsa.so in-tree from csrc/ with nvcc for sm_100a.

    python -m shared_prefix_attention_b200.build [--verbose-ptxas] [--debug]

Objects go to shared_prefix_attention_b200/_build/ (git-ignored); the
shared library lands next to this file so it travels with the tree.  With
--debug the same sources are compiled with PSA_DEBUG=1 into _build_debug/
and libpsa_debug.so (device-side bounds checks that report PSA_ERR_BOUNDS).
"""
from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(HERE, "csrc")
BUILD = os.path.join(HERE, "_build")
LIB = os.path.join(HERE, "libpsa.so")
BUILD_DEBUG = os.path.join(HERE, "_build_debug")
LIB_DEBUG = os.path.join(HERE, "libpsa_debug.so")
INCLUDE = os.path.join(ROOT, "include")


def nvcc_path() -> str:
    for cand in (os.environ.get("NVCC"), shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def common_flags(ptxas_verbose: bool = False, debug: bool = False) -> list[str]:
    flags = ["-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo", "-O3", "-std=c++17",
             "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden",
             "--expt-relaxed-constexpr", "-I", INCLUDE, "-I", CSRC]
    if debug:
        flags += ["-DPSA_DEBUG=1"]
    if ptxas_verbose:
        flags += ["-Xptxas", "-v"]
    return flags


def sources() -> list[str]:
    return sorted(os.path.join(CSRC, f) for f in os.listdir(CSRC)
                  if f.endswith((".cu", ".cpp")))


def build(ptxas_verbose: bool = False, force: bool = False, debug: bool = False) -> str:
    """Compile libpsa.so, or with ``debug`` libpsa_debug.so: the same sources
    with PSA_DEBUG=1, whose kernels check the indices they take from caller
    data and report PSA_ERR_BOUNDS instead of following a bad one."""
    build_dir = BUILD_DEBUG if debug else BUILD
    lib_path = LIB_DEBUG if debug else LIB
    os.makedirs(build_dir, exist_ok=True)
    nvcc = nvcc_path()
    headers = [os.path.join(CSRC, f) for f in os.listdir(CSRC) if f.endswith((".h", ".cuh"))]
    headers.append(os.path.join(INCLUDE, "psa.h"))
    newest_header = max(os.path.getmtime(h) for h in headers)
    objs = []
    for src in sources():
        obj = os.path.join(build_dir, os.path.basename(src) + ".o")
        objs.append(obj)
        if (not force and os.path.exists(obj)
                and os.path.getmtime(obj) >= max(os.path.getmtime(src), newest_header)):
            continue
        lang = ["-x", "cu"] if src.endswith(".cu") else ["-x", "c++"]
        cmd = [nvcc] + common_flags(ptxas_verbose, debug) + lang + ["-c", src, "-o", obj]
        subprocess.run(cmd, check=True)
    if force or not os.path.exists(lib_path) or os.path.getmtime(lib_path) < max(
            os.path.getmtime(o) for o in objs):
        cmd = [nvcc, "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o",
               lib_path] + objs + ["-lcudart"]
        subprocess.run(cmd, check=True)
    return lib_path


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose-ptxas", action="store_true")
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--debug", action="store_true",
                    help="build libpsa_debug.so (device-side bounds checks)")
    args = ap.parse_args()
    print(build(args.verbose_ptxas, args.force, args.debug))
    sys.exit(0)
