"""Seeded synthetic inputs shared by the CPU oracle and the GPU path.

This package only draws inputs (activations, router and expert weights,
q4_0-packed experts).  It holds none of the MoE layer's arithmetic.  The host
generator (``synth.c``) and the device generator (``synth_cuda.cu``) are
bit-identical; see ``synth.h`` for the definition.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
HOST_SO = os.path.join(_HERE, "_synth_host.so")
CUDA_SO = os.path.join(_HERE, "_synth_cuda.so")

DT_F32, DT_BF16, DT_F16 = 0, 1, 2
_NP_OF = {DT_F32: np.float32, DT_BF16: np.uint16, DT_F16: np.uint16}


def _stale(target: str, sources: list[str]) -> bool:
    if not os.path.exists(target):
        return True
    t = os.path.getmtime(target)
    return any(os.path.getmtime(s) > t for s in sources)


def build_host(force: bool = False) -> str:
    srcs = [os.path.join(_HERE, "synth.c"), os.path.join(_HERE, "synth.h")]
    if force or _stale(HOST_SO, srcs):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
             srcs[0], "-o", HOST_SO + ".tmp", "-lm"])
        os.replace(HOST_SO + ".tmp", HOST_SO)
    return HOST_SO


def build_cuda(force: bool = False) -> str:
    srcs = [os.path.join(_HERE, "synth_cuda.cu"), os.path.join(_HERE, "synth.h")]
    if force or _stale(CUDA_SO, srcs):
        subprocess.check_call(
            ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
             "-Xcompiler", "-fPIC", "-shared", srcs[0], "-o", CUDA_SO + ".tmp"])
        os.replace(CUDA_SO + ".tmp", CUDA_SO)
    return CUDA_SO


_host = None
_cuda = None


def host_lib():
    global _host
    if _host is None:
        lib = ctypes.CDLL(build_host())
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.synth_host_normal.argtypes = [u64, u64, u64, u64, ctypes.c_float, ctypes.c_int, vp]
        lib.synth_host_rmsnorm_rows.argtypes = [u64, u64, i64, i64, i64, ctypes.c_int, vp]
        lib.synth_host_q4.argtypes = [u64, u64, i64, i64, i64, vp, vp]
        for f in (lib.synth_host_normal, lib.synth_host_rmsnorm_rows, lib.synth_host_q4):
            f.restype = None
        _host = lib
    return _host


def cuda_lib():
    global _cuda
    if _cuda is None:
        lib = ctypes.CDLL(build_cuda())
        u64, i64, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_void_p
        lib.synth_dev_normal.argtypes = [u64, u64, u64, u64, ctypes.c_float, ctypes.c_int, vp, vp]
        lib.synth_dev_rmsnorm_rows.argtypes = [u64, u64, i64, i64, i64, ctypes.c_int, vp, vp]
        lib.synth_dev_q4.argtypes = [u64, u64, i64, i64, i64, vp, vp, vp]
        for f in (lib.synth_dev_normal, lib.synth_dev_rmsnorm_rows, lib.synth_dev_q4):
            f.restype = ctypes.c_int
        _cuda = lib
    return _cuda


# ---------------------------------------------------------------- host side
def normal(seed: int, tensor_id: int, shape, sigma: float, dtype: int, offset: int = 0):
    n = int(np.prod(shape))
    out = np.empty(n, dtype=_NP_OF[dtype])
    host_lib().synth_host_normal(seed, tensor_id, offset, n, np.float32(sigma), dtype,
                                 out.ctypes.data)
    return out.reshape(shape)


def rmsnorm_rows(seed: int, tensor_id: int, rows: int, cols: int, dtype: int, row0: int = 0):
    out = np.empty(rows * cols, dtype=_NP_OF[dtype])
    host_lib().synth_host_rmsnorm_rows(seed, tensor_id, row0, rows, cols, dtype, out.ctypes.data)
    return out.reshape(rows, cols)


def q4(seed: int, tensor_id: int, rows: int, cols: int, row0: int = 0):
    qs = np.empty(rows * cols // 2, dtype=np.uint8)
    sc = np.empty(rows * cols // 32, dtype=np.uint16)
    host_lib().synth_host_q4(seed, tensor_id, row0, rows, cols, qs.ctypes.data, sc.ctypes.data)
    return qs.reshape(rows, cols // 2), sc.reshape(rows, cols // 32)


# -------------------------------------------------------------- device side
def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"synthetic {what} failed with status {rc}")


def normal_dev(seed, tensor_id, n, sigma, dtype, out_ptr, stream=0, offset=0):
    _check(cuda_lib().synth_dev_normal(seed, tensor_id, offset, n, np.float32(sigma), dtype,
                                       out_ptr, stream), "normal")


def rmsnorm_rows_dev(seed, tensor_id, rows, cols, dtype, out_ptr, stream=0, row0=0):
    _check(cuda_lib().synth_dev_rmsnorm_rows(seed, tensor_id, row0, rows, cols, dtype, out_ptr,
                                             stream), "rmsnorm_rows")


def q4_dev(seed, tensor_id, rows, cols, qs_ptr, scales_ptr, stream=0, row0=0):
    _check(cuda_lib().synth_dev_q4(seed, tensor_id, row0, rows, cols, qs_ptr, scales_ptr, stream),
           "q4")
