"""ctypes wrapper around the C input generator (see specgen.c for the exact
definition of every draw)."""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "specgen.c")
_LIB = os.path.join(_HERE, "libspecgen.so")
_lock = threading.Lock()
_lib = None


def build_generator(force: bool = False) -> str:
    """Compile specgen.c into libspecgen.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build_generator())
            u64, i64, f64 = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double
            vp = ctypes.c_void_p
            lib.sg_raw_u64.argtypes = [u64, u64, u64, i64, vp]
            lib.sg_uniform.argtypes = [u64, u64, u64, i64, vp]
            lib.sg_randint.argtypes = [u64, u64, u64, i64, i64, i64, vp]
            lib.sg_normal_f32.argtypes = [u64, u64, u64, i64, f64, vp]
            lib.sg_normal_bf16.argtypes = [u64, u64, u64, i64, f64, vp]
            lib.sg_normal_bf16_rows.argtypes = [u64, u64, u64, i64, i64, u64, f64, vp]
            lib.sg_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def fnv1a64(name: str) -> int:
    """64-bit FNV-1a hash of a UTF-8 name (Fowler, Noll, Vo): the stream id."""
    h = 0xCBF29CE484222325
    for byte in name.encode("utf-8"):
        h ^= byte
        h = (h * 0x100000001B3) & 0xFFFFFFFFFFFFFFFF
    return h


def _stream(stream) -> int:
    return fnv1a64(stream) if isinstance(stream, str) else int(stream)


def generator_threads() -> int:
    return int(_load().sg_num_threads())


def raw_u64(seed: int, stream, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _load().sg_raw_u64(seed, _stream(stream), offset, n, out.ctypes.data)
    return out


def uniform(seed: int, stream, offset: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.float64)
    _load().sg_uniform(seed, _stream(stream), offset, n, out.ctypes.data)
    return out


def randint(seed: int, stream, offset: int, n: int, lo: int, hi: int) -> np.ndarray:
    if hi <= lo:
        raise ValueError("randint needs hi > lo")
    out = np.empty(n, dtype=np.int64)
    _load().sg_randint(seed, _stream(stream), offset, n, lo, hi, out.ctypes.data)
    return out


def normal_f32(seed: int, stream, offset: int, n: int, scale: float = 1.0) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    _load().sg_normal_f32(seed, _stream(stream), offset, n, float(scale), out.ctypes.data)
    return out


def normal_bf16(seed: int, stream, offset: int, n: int, scale: float = 1.0, out=None) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, scale^2) draws at counters offset..offset+n-1."""
    if out is None:
        out = np.empty(n, dtype=np.uint16)
    assert out.dtype == np.uint16 and out.flags.c_contiguous and out.size == n
    _load().sg_normal_bf16(seed, _stream(stream), offset, n, float(scale), out.ctypes.data)
    return out


def normal_bf16_rows(seed: int, stream, offset: int, rows: int, cols: int, row_stride: int,
                     scale: float = 1.0) -> np.ndarray:
    """rows x cols block; row r starts at counter offset + r * row_stride."""
    out = np.empty((rows, cols), dtype=np.uint16)
    _load().sg_normal_bf16_rows(seed, _stream(stream), offset, rows, cols, row_stride, float(scale),
                                out.ctypes.data)
    return out
