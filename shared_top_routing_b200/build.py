"""Builds libsa.so (the C ABI in include/sa.h) in-tree with nvcc for sm_100a,
and its debug variant libsa_debug.so (compiled with SA_DEBUG: gathered row
indices and workspace canaries checked on the device, see sa.h).

    python -m shared_top_routing_b200.build [--verbose] [--debug]

Objects go to ``_build/`` (``_build/debug/``) at the repository root; the
shared libraries are written next to this file, where the binding loads them.
"""
from __future__ import annotations

import os
import subprocess
import sys

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
CSRC = os.path.join(PKG, "csrc")
BUILD = os.path.join(ROOT, "_build")
LIB = os.path.join(PKG, "libsa.so")
LIB_DEBUG = os.path.join(PKG, "libsa_debug.so")
NVCC = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
ARCH = ["-gencode", "arch=compute_100a,code=sm_100a"]
FLAGS = ["-O3", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-Xcompiler", "-O2",
         "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include")]
SOURCES = ["abi.cu", "attn.cu", "index_topk.cu", "index_tc.cu", "index_fp8.cu", "noalloc.cu", "selftest.cu"]


def _run(cmd, verbose):
    if verbose:
        print(" ".join(cmd), flush=True)
    return subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.STDOUT, text=True)


def build(verbose: bool = False, extra_flags: list[str] | None = None, debug: bool = False) -> str:
    out_dir = os.path.join(BUILD, "debug") if debug else BUILD
    os.makedirs(out_dir, exist_ok=True)
    extra = list(extra_flags or []) + (["-DSA_DEBUG"] if debug else [])
    procs = []
    objs = []
    for src in SOURCES:
        obj = os.path.join(out_dir, src.replace(".cu", ".o"))
        objs.append(obj)
        cmd = [NVCC, *ARCH, *FLAGS, *extra, "-c", os.path.join(CSRC, src), "-o", obj]
        procs.append((src, _run(cmd, verbose)))
    failed = []
    for src, p in procs:
        out, _ = p.communicate()
        if verbose and out:
            print(out)
        if p.returncode != 0:
            failed.append((src, out))
    if failed:
        msg = "\n".join(f"--- {s}\n{o}" for s, o in failed)
        raise RuntimeError(f"nvcc failed:\n{msg}")
    lib = LIB_DEBUG if debug else LIB
    cmd = [NVCC, *ARCH, "-shared", "-o", lib, *objs, "-lcudart"]
    p = _run(cmd, verbose)
    out, _ = p.communicate()
    if p.returncode != 0:
        raise RuntimeError(f"link failed:\n{out}")
    return lib


if __name__ == "__main__":
    print(build(verbose="--verbose" in sys.argv, debug="--debug" in sys.argv))
