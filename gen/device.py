"""ctypes binding of the device generator ``libsagen.so`` (see gen/device.cu).

Fills caller-owned torch CUDA tensors (dtype bfloat16 or int16/uint16 views)
on the current stream.  Built by ``__graft_entry__.build()``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsagen.so")
_lib = None


def _load():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"device generator not built: {LIB_PATH} is missing")
        lib = ctypes.CDLL(LIB_PATH)
        lib.sagen_fill_int_bf16.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_uint,
                                            ctypes.c_uint, ctypes.c_longlong, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_void_p]
        lib.sagen_fill_int_bf16.restype = ctypes.c_int
        lib.sagen_fill_normal_bf16.argtypes = [ctypes.c_void_p, ctypes.c_longlong, ctypes.c_uint,
                                               ctypes.c_uint, ctypes.c_longlong, ctypes.c_void_p]
        lib.sagen_fill_normal_bf16.restype = ctypes.c_int
        _lib = lib
    return _lib


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def fill_int(t, seed: int, tid: int, start: int = 0, lo: int = -4, hi: int = 4):
    """Fill a contiguous 2-byte CUDA tensor with integer values as bf16 bits."""
    assert t.is_cuda and t.is_contiguous() and t.element_size() == 2
    rc = _load().sagen_fill_int_bf16(ctypes.c_void_p(t.data_ptr()), t.numel(), seed, tid,
                                     start, lo, hi, _stream())
    if rc != 0:
        raise RuntimeError(f"sagen_fill_int_bf16 failed: cuda error {rc}")
    return t


def fill_normal(t, seed: int, tid: int, start: int = 0):
    """Fill a contiguous 2-byte CUDA tensor with Irwin-Hall normals as bf16 bits."""
    assert t.is_cuda and t.is_contiguous() and t.element_size() == 2
    rc = _load().sagen_fill_normal_bf16(ctypes.c_void_p(t.data_ptr()), t.numel(), seed, tid,
                                        start, _stream())
    if rc != 0:
        raise RuntimeError(f"sagen_fill_normal_bf16 failed: cuda error {rc}")
    return t


def build(verbose: bool = False) -> str:
    """Compile gen/device.cu into gen/libsagen.so (nvcc, sm_100a)."""
    import subprocess
    nvcc = os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc")
    cmd = [nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", os.path.join(_HERE, "device.cu"), "-o", LIB_PATH]
    if verbose:
        print(" ".join(cmd), flush=True)
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for gen/device.cu:\n{r.stdout}\n{r.stderr}")
    return LIB_PATH
