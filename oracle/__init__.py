"""CPU oracle for the fused DyT layer (binary64, plain loops).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this; the product path never does. The
arithmetic lives in ``dyt_oracle.c`` (see its header for the definitions and
the readings of the Liger-Kernel page); this module only marshals numpy
arrays into it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SO = os.path.join(_HERE, "_dyt_oracle.so")
_SRC = os.path.join(_HERE, "dyt_oracle.c")

DTYPE_CODES = {"f32": 0, "bf16": 1, "f16": 2, "f64": 3}
NP_STORAGE = {"f32": np.float32, "bf16": np.uint16, "f16": np.float16, "f64": np.float64}

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc: -O2, no fast-math, no FMA contraction."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", _SO, _SRC, "-lm"])
    return _SO


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_SO)
        vp, i64, i32, dp = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_void_p
        lib.dyt_oracle_forward.argtypes = [vp, i32, vp, i32, vp, i32, vp, i32, i64, i64, dp]
        lib.dyt_oracle_forward.restype = i32
        lib.dyt_oracle_backward.argtypes = [vp, vp, i32, vp, i32, vp, i32, i64, i64, dp, dp, dp, dp, dp, dp, dp]
        lib.dyt_oracle_backward.restype = i32
        lib.dyt_oracle_round.argtypes = [dp, i64, i32, vp]
        lib.dyt_oracle_round.restype = i32
        lib.dyt_oracle_round_scalar.argtypes = [ctypes.c_double, i32]
        lib.dyt_oracle_round_scalar.restype = ctypes.c_double
        lib.dyt_oracle_decode.argtypes = [vp, i64, i32, dp]
        lib.dyt_oracle_decode.restype = None
        _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data


def _as(a, dtype):
    a = np.ascontiguousarray(a)
    want = NP_STORAGE[dtype]
    if a.dtype != want:
        raise TypeError(f"expected {want} storage for {dtype}, got {a.dtype}")
    return a


def _pdtypes(p_dtype):
    """(alpha, gamma, beta) storage dtypes from one name or a 3-tuple of names."""
    return (p_dtype,) * 3 if isinstance(p_dtype, str) else tuple(p_dtype)


def forward(x, alpha, gamma, beta, M: int, N: int, x_dtype: str, p_dtype) -> np.ndarray:
    """y (binary64, M*N) of the DyT forward. p_dtype: one dtype for alpha, gamma and
    beta, or a tuple (alpha, gamma, beta) of dtypes."""
    lib = _load()
    ad, gd, bd = _pdtypes(p_dtype)
    x, alpha, gamma, beta = _as(x, x_dtype), _as(alpha, ad), _as(gamma, gd), _as(beta, bd)
    y = np.empty(M * N, dtype=np.float64)
    rc = lib.dyt_oracle_forward(_ptr(x), DTYPE_CODES[x_dtype], _ptr(alpha), DTYPE_CODES[ad], _ptr(gamma),
                                DTYPE_CODES[gd], _ptr(beta), DTYPE_CODES[bd], M, N, _ptr(y))
    if rc:
        raise ValueError("dyt_oracle_forward rejected its arguments")
    return y


def backward(x, dy, alpha, gamma, M: int, N: int, x_dtype: str, p_dtype, want_dx: bool = True):
    """dict with dx (binary64 M*N, or None), dgamma, dbeta (N), dalpha (float) and the
    magnitude of each sum (mag_dgamma, mag_dbeta, mag_dalpha). p_dtype as for forward."""
    lib = _load()
    ad, gd, _ = _pdtypes(p_dtype)
    x, dy, alpha, gamma = _as(x, x_dtype), _as(dy, x_dtype), _as(alpha, ad), _as(gamma, gd)
    dx = np.empty(M * N, dtype=np.float64) if want_dx else None
    dg, db = np.empty(N), np.empty(N)
    mg, mb = np.empty(N), np.empty(N)
    da, ma = np.empty(1), np.empty(1)
    rc = lib.dyt_oracle_backward(_ptr(x), _ptr(dy), DTYPE_CODES[x_dtype], _ptr(alpha), DTYPE_CODES[ad],
                                 _ptr(gamma), DTYPE_CODES[gd], M, N, _ptr(dx), _ptr(dg), _ptr(db), _ptr(da),
                                 _ptr(mg), _ptr(mb), _ptr(ma))
    if rc:
        raise ValueError("dyt_oracle_backward rejected its arguments")
    return {"dx": dx, "dgamma": dg, "dbeta": db, "dalpha": float(da[0]),
            "mag_dgamma": mg, "mag_dbeta": mb, "mag_dalpha": float(ma[0])}


def round_to(v, dtype: str) -> np.ndarray:
    """binary64 values rounded once (ties to even) into ``dtype`` storage."""
    lib = _load()
    v = np.ascontiguousarray(v, dtype=np.float64)
    out = np.empty(v.size, dtype=NP_STORAGE[dtype])
    rc = lib.dyt_oracle_round(_ptr(v), v.size, DTYPE_CODES[dtype], _ptr(out))
    if rc:
        raise ValueError("dyt_oracle_round rejected its arguments")
    return out.reshape(v.shape)


def round_scalar(v: float, dtype: str) -> float:
    return float(_load().dyt_oracle_round_scalar(float(v), DTYPE_CODES[dtype]))


def decode(a, dtype: str) -> np.ndarray:
    """Storage values decoded exactly to binary64."""
    lib = _load()
    a = _as(a, dtype)
    out = np.empty(a.size, dtype=np.float64)
    lib.dyt_oracle_decode(_ptr(a), a.size, DTYPE_CODES[dtype], _ptr(out))
    return out
