"""Seeded synthetic inputs shared by the oracle (in tests) and the CUDA path.

This module only draws numbers; it holds none of the layer's arithmetic.  The
generator (SplitMix64 keyed by (seed, stream, index), Box-Muller in double) is
written in ``synth.c`` and compiled with gcc/OpenMP on first use.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB = os.path.join(_HERE, "libqrx_synth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile synth.c into libqrx_synth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared",
                               "-ffp-contract=off", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.synth_normal_f32.argtypes = [u64, u64, i64, i64, dbl, dbl, vp]
            lib.synth_normal_bf16.argtypes = [u64, u64, i64, i64, dbl, dbl, vp]
            lib.synth_uniform_f64.argtypes = [u64, u64, i64, i64, vp]
            for f in (lib.synth_normal_f32, lib.synth_normal_bf16, lib.synth_uniform_f64):
                f.restype = None
            _lib = lib
    return _lib


def normal_f32(seed: int, stream: int, n: int, mean: float = 0.0, std: float = 1.0,
               offset: int = 0, out: np.ndarray | None = None) -> np.ndarray:
    """n f32 values mean + std * N(0,1), element i drawn at counter offset + i."""
    lib = _load()
    if out is None:
        out = np.empty(n, dtype=np.float32)
    assert out.dtype == np.float32 and out.flags.c_contiguous and out.size == n
    lib.synth_normal_f32(seed, stream, offset, n, mean, std, out.ctypes.data)
    return out


def normal_bf16(seed: int, stream: int, n: int, mean: float = 0.0, std: float = 1.0,
                offset: int = 0) -> np.ndarray:
    """The same draws as normal_f32, rounded to bf16; returned as uint16 bit patterns."""
    lib = _load()
    out = np.empty(n, dtype=np.uint16)
    lib.synth_normal_bf16(seed, stream, offset, n, mean, std, out.ctypes.data)
    return out


def uniform_f64(seed: int, stream: int, n: int, offset: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.float64)
    lib.synth_uniform_f64(seed, stream, offset, n, out.ctypes.data)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bf16 bit patterns (uint16) to f32 values exactly."""
    return (b.astype(np.uint32) << 16).view(np.float32)
