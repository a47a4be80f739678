"""Seeded synthetic input generator (binding to ``csrc/synth.c``).

Random numbers only: this module holds none of the MoE layer's arithmetic.
Both the CPU oracle and the CUDA library consume the arrays it returns, so a
parity check always compares the two on identical bytes.  bf16 arrays are
returned as ``numpy.uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csrc", "synth.c")
_SO = os.path.join(_HERE, "_synth.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the generator with gcc (host code, OpenMP)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        lib.synth_normal_f32.argtypes = [u64, u64, i64, dbl, dbl, vp]
        lib.synth_normal_bf16.argtypes = [u64, u64, i64, dbl, dbl, vp]
        lib.synth_u64.argtypes = [u64, u64, i64, vp]
        lib.synth_f32_to_bf16.argtypes = [vp, i64, vp]
        for f in (lib.synth_normal_f32, lib.synth_normal_bf16, lib.synth_u64, lib.synth_f32_to_bf16):
            f.restype = None
        _lib = lib
    return _lib


def normal_f32(seed: int, stream: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.float32)
    _load().synth_normal_f32(seed, stream, out.size, mean, std, out.ctypes.data)
    return out


def normal_bf16(seed: int, stream: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    out = np.empty(shape, dtype=np.uint16)
    _load().synth_normal_bf16(seed, stream, out.size, mean, std, out.ctypes.data)
    return out


def u64(seed: int, stream: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().synth_u64(seed, stream, n, out.ctypes.data)
    return out


def f32_to_bf16(a: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a, dtype=np.float32)
    out = np.empty(a.shape, dtype=np.uint16)
    _load().synth_f32_to_bf16(a.ctypes.data, a.size, out.ctypes.data)
    return out


def bf16_to_f32(a: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(a, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)
