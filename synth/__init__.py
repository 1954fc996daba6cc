"""Seeded synthetic inputs shared by the oracle and the CUDA path.

Holds only random-number generation and storage encoding (see ``synth.c``):
none of the DyT arithmetic lives here. ``workloads`` describes the five DyT
shapes and their value distributions.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_synth.so")
_SRC = os.path.join(_HERE, "synth.c")

DTYPE_CODES = {"f32": 0, "bf16": 1, "f16": 2, "f64": 3}
NP_STORAGE = {"f32": np.float32, "bf16": np.uint16, "f16": np.float16, "f64": np.float64}

# One Philox key stream per tensor.
STREAM_X, STREAM_DY, STREAM_GAMMA, STREAM_BETA = 1, 2, 3, 4

_lib = None


def build(force: bool = False) -> str:
    """Compile ``synth.c`` into ``_synth.so`` next to it (gcc, no GPU needed)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
             "-o", _SO, _SRC, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        lib.synth_normal.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_double,
                                     ctypes.c_double, ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int,
                                     ctypes.c_int]
        lib.synth_normal.restype = ctypes.c_int
        lib.synth_philox4x64_10.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        lib.synth_philox4x64_10.restype = None
        _lib = lib
    return _lib


def philox4x64_10(counter, key) -> np.ndarray:
    """One Philox4x64-10 block for a 4-word counter and 2-word key."""
    lib = _load()
    c = np.ascontiguousarray(counter, dtype=np.uint64)
    k = np.ascontiguousarray(key, dtype=np.uint64)
    out = np.zeros(4, dtype=np.uint64)
    lib.synth_philox4x64_10(c.ctypes.data, k.ctypes.data, out.ctypes.data)
    return out


def normal(n: int, dtype: str, mean: float, std: float, seed: int, stream: int,
           nonzero: bool = False, threads: int | None = None) -> np.ndarray:
    """``n`` samples of mean + std * N(0, 1), stored in ``dtype``.

    bf16 is returned as its raw uint16 bit patterns (numpy has no bf16).
    """
    lib = _load()
    out = np.empty(int(n), dtype=NP_STORAGE[dtype])
    if threads is None:
        threads = max(1, min(32, len(os.sched_getaffinity(0))))
    rc = lib.synth_normal(out.ctypes.data if n else None, int(n), DTYPE_CODES[dtype], float(mean),
                          float(std), int(seed), int(stream), int(bool(nonzero)), int(threads))
    if rc != 0:
        raise ValueError("synth_normal rejected its arguments")
    return out
