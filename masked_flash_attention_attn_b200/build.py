"""Build the in-tree shared library ``libattn_b200.so`` for sm_100a with nvcc.

    python -m masked_flash_attention_attn_b200.build [--verbose]

Objects go to ``_build/`` at the repository root; the library lands next to this file.
``-Xptxas -v`` output (registers, spills, shared memory) is printed with --verbose.
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
import os
import shutil
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libattn_b200.so")
SOURCES = ["attn_plan.cpp", "attn_custom.cu", "attn_fwd.cu", "attn_bwd.cu"]
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]


def nvcc() -> str:
    cand = shutil.which("nvcc") or "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(cand):
        raise RuntimeError("nvcc not found: the CUDA toolkit is required to build libattn_b200.so")
    return cand


def _compile(src: str, verbose: bool, defines=()) -> str:
    obj = os.path.join(BUILD, src + "".join("." + d for d in defines) + ".o")
    cmd = [nvcc(), "-c", os.path.join(CSRC, src), "-o", obj, "-O3", "-std=c++17", "-lineinfo",
           "-Xcompiler", "-fPIC", "-I", os.path.join(ROOT, "include"), "-I", CSRC, *ARCH,
           *[f"-D{d}" for d in defines]]
    if src.endswith(".cu"):
        cmd += ["-Xptxas", "-v"] if verbose else []
    else:
        cmd += ["-x", "cu"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    if verbose and (r.stdout or r.stderr):
        print(f"== {src}\n{r.stdout}{r.stderr}", file=sys.stderr)
    return obj


def build(verbose: bool = False, defines=(), out: str = LIB) -> str:
    """Compile and link; ``defines`` are extra NAME=VALUE macros, ``out`` the library path."""
    os.makedirs(BUILD, exist_ok=True)
    with cf.ThreadPoolExecutor(len(SOURCES)) as ex:
        objs = list(ex.map(lambda s: _compile(s, verbose, tuple(defines)), SOURCES))
    tmp = out + ".tmp"
    cmd = [nvcc(), "-shared", "-o", tmp, *objs, *ARCH, "-lcudart_static", "-ldl", "-lpthread", "-lrt"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"link failed:\n{r.stdout}\n{r.stderr}")
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    ap = argparse.ArgumentParser()
    ap.add_argument("--verbose", action="store_true")
    ap.add_argument("-D", dest="defines", action="append", default=[], help="extra macro NAME=VALUE")
    ap.add_argument("--out", default=LIB)
    a = ap.parse_args()
    print(build(a.verbose, a.defines, a.out))
