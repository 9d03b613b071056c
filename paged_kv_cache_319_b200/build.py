"""Builds libkvp.so in place (sm_100a) with nvcc.

Usage: ``python -m paged_kv_cache_319_b200.build [--force] [--verbose]``.
The library lands next to this file so the package loads it from the source
tree; intermediate output (the ptxas report) goes to ``_build/``.
"""

from __future__ import annotations

import argparse
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
INCLUDE = os.path.join(ROOT, "include")
LIB = os.path.join(PKG, "libkvp.so")
BUILD_DIR = os.path.join(PKG, "_build")

SOURCES = [
    os.path.join(CSRC, "host", "block_pool.cpp"),
    os.path.join(CSRC, "host", "group_plan.cpp"),
    os.path.join(CSRC, "host", "vcache.cpp"),
    os.path.join(CSRC, "kvp_device.cu"),
]


def _inputs():
    files = list(SOURCES)
    for d in (CSRC, INCLUDE):
        for dp, _, fs in os.walk(d):
            files += [os.path.join(dp, f) for f in fs if f.endswith((".h", ".cuh", ".cu", ".cpp"))]
    files.append(os.path.abspath(__file__))
    return files


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(f) <= t for f in _inputs())


def nvcc() -> str:
    for cand in (shutil.which("nvcc"), "/usr/local/cuda/bin/nvcc"):
        if cand and os.path.exists(cand):
            return cand
    raise RuntimeError("nvcc not found")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and up_to_date():
        return LIB
    os.makedirs(BUILD_DIR, exist_ok=True)
    tmp = LIB + ".tmp"
    cmd = [
        nvcc(), "-std=c++17", "-O3", "-lineinfo", "-DNDEBUG",
        "-gencode", "arch=compute_100a,code=sm_100a",
        "-Xcompiler", "-fPIC,-O3,-fvisibility=hidden",
        "-Xptxas", "-v",
        "-I", INCLUDE, "-I", CSRC,
        "-shared", "-o", tmp,
    ] + SOURCES
    res = subprocess.run(cmd, capture_output=True, text=True)
    with open(os.path.join(BUILD_DIR, "nvcc.log"), "w") as f:
        f.write(" ".join(cmd) + "\n\n" + res.stdout + res.stderr)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed; see " + os.path.join(BUILD_DIR, "nvcc.log"))
    os.replace(tmp, LIB)
    if verbose:
        sys.stdout.write(res.stdout + res.stderr)
    return LIB


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    args = ap.parse_args()
    print(build(force=args.force, verbose=args.verbose))


if __name__ == "__main__":
    main()
