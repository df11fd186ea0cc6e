"""Builds the in-tree CUDA library ``int4_quant_b200/libarnq.so`` for sm_100a.

    python -m int4_quant_b200.build [--force] [--verbose]

nvcc cross-compiles on a machine without a GPU.  The library is linked with
the static CUDA runtime, so it loads (and its host-side argument checks run)
on a machine with no driver; kernels need a B200.
"""
from __future__ import annotations

import argparse
import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
SRC_DIR = os.path.join(PKG, "csrc")
SOURCES = [os.path.join(SRC_DIR, f) for f in ["arnq_api.cu"] + [
    f"arnq_k_{dt}_{q}{cl}.cu" for dt in ("bf16", "fp16") for q in ("int8", "int4")
    for cl in ("", "_cl")]]
DEPS = SOURCES + [os.path.join(SRC_DIR, "arnq_kernels.cuh"), os.path.join(SRC_DIR, "arnq_table.h"),
                  os.path.join(ROOT, "include", "arnq.h")]
LIB = os.path.join(PKG, "libarnq.so")
OBJ_DIR = os.path.join(ROOT, "_build")

NVCC_FLAGS = [
    "-O3", "-std=c++17", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
    "-Xcompiler", "-fPIC", "-Xcompiler", "-fvisibility=hidden", "--expt-relaxed-constexpr",
]


def nvcc() -> str:
    for c in (os.environ.get("CUDA_HOME", ""), "/usr/local/cuda"):
        p = os.path.join(c, "bin", "nvcc") if c else ""
        if p and os.path.exists(p):
            return p
    return "nvcc"


def up_to_date() -> bool:
    if not os.path.exists(LIB):
        return False
    t = os.path.getmtime(LIB)
    return all(os.path.getmtime(d) <= t for d in DEPS)


def build(force: bool = False, verbose: bool = False) -> str:
    """Compiles every translation unit in parallel, then links the library."""
    if not force and up_to_date():
        return LIB
    os.makedirs(OBJ_DIR, exist_ok=True)
    inc = ["-I", os.path.join(ROOT, "include")]
    procs = []
    for src in SOURCES:
        obj = os.path.join(OBJ_DIR, os.path.basename(src) + ".o")
        cmd = [nvcc(), *NVCC_FLAGS, *(["-Xptxas=-v"] if verbose else []), *inc, "-c", "-o", obj,
               src]
        procs.append((obj, subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT,
                                            text=True)))
    objs, failed = [], False
    for obj, p in procs:
        out, _ = p.communicate()
        if p.returncode != 0 or verbose:
            sys.stderr.write(out)
        failed |= p.returncode != 0
        objs.append(obj)
    if failed:
        raise RuntimeError("nvcc failed compiling libarnq")
    link = [nvcc(), "-shared", "-cudart", "static", "-gencode", "arch=compute_100a,code=sm_100a",
            "-o", LIB, *objs]
    res = subprocess.run(link, capture_output=True, text=True)
    if res.returncode != 0:
        sys.stderr.write(res.stdout + res.stderr)
        raise RuntimeError("nvcc failed linking libarnq.so")
    return LIB


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--force", action="store_true")
    ap.add_argument("--verbose", action="store_true")
    a = ap.parse_args()
    print(build(force=a.force, verbose=a.verbose))
