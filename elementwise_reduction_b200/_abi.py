"""ctypes binding of libdyt.so, the C ABI declared in include/dyt.h.

Argument marshalling only: every step of the DyT computation runs in the CUDA
kernels behind these calls. There is no CPU fallback; importing this module
fails if the library is missing.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdyt.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python elementwise_reduction_b200/build.py` "
        "(the DyT layer has no fallback implementation)")

lib = ctypes.CDLL(LIB_PATH)

DYT_F32, DYT_BF16, DYT_F16 = 0, 1, 2
STATUS = {0: "DYT_OK", 1: "DYT_ERR_INVALID_VALUE", 2: "DYT_ERR_UNSUPPORTED_DTYPE",
          3: "DYT_ERR_WORKSPACE_TOO_SMALL", 4: "DYT_ERR_CUDA"}

_vp, _i64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t


class LaunchInfo(ctypes.Structure):
    _fields_ = [("op", _i32), ("path", _i32), ("vec", _i32), ("block", _i32), ("grid", _i32),
                ("row_lanes", _i32), ("rows_per_step", _i32), ("col_chunks", _i32),
                ("row_groups", _i32), ("kernels", _i32), ("async_stages", _i32),
                ("pack_rows", _i32), ("workspace_bytes", _i64)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


lib.dyt_forward.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _vp]
lib.dyt_forward.restype = _i32
lib.dyt_backward_workspace_bytes.argtypes = [_i64, _i64, _i32, _i32]
lib.dyt_backward_workspace_bytes.restype = _sz
lib.dyt_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _vp, _sz, _vp]
lib.dyt_backward.restype = _i32
lib.dyt_forward_strided.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _vp]
lib.dyt_forward_strided.restype = _i32
lib.dyt_backward_strided.argtypes = [_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i32,
                                     _i32, _vp, _sz, _vp]
lib.dyt_backward_strided.restype = _i32
lib.dyt_forward_ex.argtypes = [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _i32, _vp]
lib.dyt_forward_ex.restype = _i32
lib.dyt_backward_ex.argtypes = [_vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i32,
                                _i32, _i32, _i32, _vp, _sz, _vp]
lib.dyt_backward_ex.restype = _i32
lib.dyt_status_string.argtypes = [_i32]
lib.dyt_status_string.restype = ctypes.c_char_p
lib.dyt_last_cuda_error.argtypes = []
lib.dyt_last_cuda_error.restype = _i32
lib.dyt_last_launch_info.argtypes = [ctypes.POINTER(LaunchInfo)]
lib.dyt_last_launch_info.restype = _i32
lib.dyt_plan_query.argtypes = [_i64, _i64, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(LaunchInfo)]
lib.dyt_plan_query.restype = _i32
lib.dyt_backward_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _vp]
lib.dyt_backward_noalloc.restype = _i32
NOALLOC_SCRATCH_BYTES = 32 * 1024 * 1024  # DYT_NOALLOC_SCRATCH_BYTES in include/dyt.h


class DytError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        msg = lib.dyt_status_string(status).decode()
        if status == 4:
            msg += f" (cudaError {lib.dyt_last_cuda_error()})"
        super().__init__(f"{what}: {msg}")


def _check(status: int, what: str) -> None:
    if status != 0:
        raise DytError(status, what)


def dyt_forward(x, alpha, gamma, beta, y, M, N, x_dtype, param_dtype, stream) -> int:
    """Raw C-ABI call: pointers as ints. Returns the status code."""
    return lib.dyt_forward(x, alpha, gamma, beta, y, M, N, x_dtype, param_dtype, stream)


def dyt_backward_workspace_bytes(M, N, x_dtype, param_dtype) -> int:
    return int(lib.dyt_backward_workspace_bytes(M, N, x_dtype, param_dtype))


def dyt_backward(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype, workspace,
                 workspace_bytes, stream) -> int:
    """Raw C-ABI call: pointers as ints (beta may be None). Returns the status code."""
    return lib.dyt_backward(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype,
                            workspace, workspace_bytes, stream)


def dyt_forward_strided(x, ldx, alpha, gamma, beta, y, ldy, M, N, x_dtype, param_dtype, stream) -> int:
    """Raw C-ABI call with row pitches (elements). Returns the status code."""
    return lib.dyt_forward_strided(x, ldx, alpha, gamma, beta, y, ldy, M, N, x_dtype, param_dtype, stream)


def dyt_backward_strided(x, ldx, dy, lddy, alpha, gamma, beta, dx, lddx, dgamma, dbeta, dalpha, M, N, x_dtype,
                         param_dtype, workspace, workspace_bytes, stream) -> int:
    """Raw C-ABI call with row pitches (elements). Returns the status code."""
    return lib.dyt_backward_strided(x, ldx, dy, lddy, alpha, gamma, beta, dx, lddx, dgamma, dbeta, dalpha, M, N,
                                    x_dtype, param_dtype, workspace, workspace_bytes, stream)


def dyt_forward_ex(x, ldx, alpha, gamma, beta, y, ldy, M, N, x_dtype, alpha_dtype, gamma_dtype, beta_dtype,
                   stream) -> int:
    """Raw C-ABI call with row pitches and one dtype per parameter. Returns the status code."""
    return lib.dyt_forward_ex(x, ldx, alpha, gamma, beta, y, ldy, M, N, x_dtype, alpha_dtype, gamma_dtype,
                              beta_dtype, stream)


def dyt_backward_ex(x, ldx, dy, lddy, alpha, gamma, beta, dx, lddx, dgamma, dbeta, dalpha, M, N, x_dtype,
                    alpha_dtype, gamma_dtype, beta_dtype, workspace, workspace_bytes, stream) -> int:
    """Raw C-ABI call with row pitches and one dtype per parameter (dalpha, dgamma and
    dbeta come back in alpha_dtype, gamma_dtype, beta_dtype). Returns the status code."""
    return lib.dyt_backward_ex(x, ldx, dy, lddy, alpha, gamma, beta, dx, lddx, dgamma, dbeta, dalpha, M, N, x_dtype,
                               alpha_dtype, gamma_dtype, beta_dtype, workspace, workspace_bytes, stream)


def dyt_backward_noalloc(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype,
                         stream) -> int:
    """Raw C-ABI call of the backward that uses the library's built-in scratch
    instead of a workspace (for callers that cannot allocate). Returns the status."""
    return lib.dyt_backward_noalloc(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, x_dtype,
                                    param_dtype, stream)


def dyt_status_string(status: int) -> str:
    return lib.dyt_status_string(status).decode()


def dyt_plan_query(M, N, x_dtype, param_dtype, backward, vectorized, sm_count, ctas_per_sm) -> dict:
    """The launch plan for a shape on a hypothetical device (host arithmetic only)."""
    info = LaunchInfo()
    _check(lib.dyt_plan_query(M, N, x_dtype, param_dtype, int(backward), int(vectorized), sm_count,
                              ctas_per_sm, ctypes.byref(info)), "dyt_plan_query")
    return info.as_dict()


def dyt_last_launch_info() -> dict:
    info = LaunchInfo()
    _check(lib.dyt_last_launch_info(ctypes.byref(info)), "dyt_last_launch_info")
    return info.as_dict()
