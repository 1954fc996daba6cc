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
                ("pack_rows", _i32), ("shifted", _i32), ("shift", _i32), ("workspace_bytes", _i64)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}


lib.dyt_forward.argtypes = [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i32, _i32, _vp]
lib.dyt_forward.restype = _i32
lib.dyt_backward_workspace_bytes.argtypes = [_i64, _i64, _i32, _i32]
lib.dyt_backward_workspace_bytes.restype = _sz
lib.dyt_backward_workspace_bytes_strided.argtypes = [_i64, _i64, _i64, _i64, _i64, _i32, _i32]
lib.dyt_backward_workspace_bytes_strided.restype = _sz
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
lib.dyt_plan_query.argtypes = [_i64, _i64, _i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(LaunchInfo)]
lib.dyt_plan_query.restype = _i32
class PartialsLayout(ctypes.Structure):
    """dyt_partials_layout: where a stage-1 launch left its binary64 partials."""
    _fields_ = [("bytes", _i64), ("off_dgamma", _i64), ("off_dbeta", _i64), ("off_dalpha", _i64),
                ("rows", ctypes.c_int32), ("dalpha_parts", ctypes.c_int32)]

    def as_dict(self) -> dict:
        return {name: getattr(self, name) for name, _ in self._fields_}

    @classmethod
    def from_dict(cls, d: dict) -> "PartialsLayout":
        return cls(**{name: d[name] for name, _ in cls._fields_})


class IpcHandle(ctypes.Structure):
    """dyt_ipc_handle: a CUDA IPC memory handle and a byte offset in its allocation."""
    _fields_ = [("bytes", ctypes.c_ubyte * 64), ("offset", _i64)]

    def to_bytes(self) -> bytes:
        return bytes(self.bytes) + int(self.offset).to_bytes(8, "little", signed=True)

    @classmethod
    def from_bytes(cls, b: bytes) -> "IpcHandle":
        h = cls()
        ctypes.memmove(h.bytes, b[:64], 64)
        h.offset = int.from_bytes(b[64:72], "little", signed=True)
        return h


MAX_RANKS = 8  # DYT_MAX_RANKS in include/dyt.h

lib.dyt_backward_partials.argtypes = [_vp, _i64, _vp, _i64, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _i32, _i32, _vp,
                                      _sz, ctypes.POINTER(PartialsLayout), _vp]
lib.dyt_backward_partials.restype = _i32
lib.dyt_partials_layout_query.argtypes = [_vp, _i64, _vp, _i64, _vp, _i64, _i64, _i64, _i32,
                                          ctypes.POINTER(PartialsLayout)]
lib.dyt_partials_layout_query.restype = _i32
lib.dyt_finalize_partials.argtypes = [ctypes.POINTER(_vp), ctypes.POINTER(PartialsLayout), _i32, _i64, _vp, _vp, _vp,
                                      _i32, _i32, _i32, _vp]
lib.dyt_finalize_partials.restype = _i32
lib.dyt_ipc_export.argtypes = [_vp, ctypes.POINTER(IpcHandle)]
lib.dyt_ipc_export.restype = _i32
lib.dyt_ipc_import.argtypes = [ctypes.POINTER(IpcHandle), ctypes.POINTER(_vp)]
lib.dyt_ipc_import.restype = _i32
lib.dyt_ipc_close.argtypes = [_vp, ctypes.POINTER(IpcHandle)]
lib.dyt_ipc_close.restype = _i32
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


def dyt_backward_workspace_bytes_strided(M, N, ldx, lddy, lddx, x_dtype, param_dtype) -> int:
    return int(lib.dyt_backward_workspace_bytes_strided(M, N, ldx, lddy, lddx, x_dtype, param_dtype))


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


def dyt_backward_partials(x, ldx, dy, lddy, alpha, gamma, dx, lddx, M, N, x_dtype, alpha_dtype, gamma_dtype,
                          workspace, workspace_bytes, stream):
    """Raw C-ABI call of stage 1. Returns (status, layout dict)."""
    lay = PartialsLayout()
    st = lib.dyt_backward_partials(x, ldx, dy, lddy, alpha, gamma, dx, lddx, M, N, x_dtype, alpha_dtype, gamma_dtype,
                                   workspace, workspace_bytes, ctypes.byref(lay), stream)
    return st, lay.as_dict()


def dyt_partials_layout_query(x, ldx, dy, lddy, dx, lddx, M, N, x_dtype) -> dict:
    """The partials layout stage 1 would report for these tensors (host arithmetic only)."""
    lay = PartialsLayout()
    _check(lib.dyt_partials_layout_query(x, ldx, dy, lddy, dx, lddx, M, N, x_dtype, ctypes.byref(lay)),
           "dyt_partials_layout_query")
    return lay.as_dict()


def dyt_finalize_partials(workspaces, layouts, N, dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype,
                          stream) -> int:
    """Raw C-ABI call: workspaces a list of device pointers (ints), layouts a list of dicts."""
    n = len(workspaces)
    ws = (_vp * max(1, n))(*workspaces)
    lays = (PartialsLayout * max(1, n))(*[PartialsLayout.from_dict(d) for d in layouts])
    return lib.dyt_finalize_partials(ws, lays, n, N, dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype,
                                     stream)


def dyt_ipc_export(ptr: int) -> bytes:
    """72 bytes: the CUDA IPC handle of ptr's allocation and ptr's offset in it."""
    h = IpcHandle()
    _check(lib.dyt_ipc_export(ptr, ctypes.byref(h)), "dyt_ipc_export")
    return h.to_bytes()


def dyt_ipc_import(handle: bytes) -> int:
    """A device pointer (int) to the exported bytes, readable from the current device."""
    h = IpcHandle.from_bytes(handle)
    p = _vp()
    _check(lib.dyt_ipc_import(ctypes.byref(h), ctypes.byref(p)), "dyt_ipc_import")
    return int(p.value)


def dyt_ipc_close(ptr: int, handle: bytes) -> None:
    h = IpcHandle.from_bytes(handle)
    _check(lib.dyt_ipc_close(ptr, ctypes.byref(h)), "dyt_ipc_close")


def dyt_status_string(status: int) -> str:
    return lib.dyt_status_string(status).decode()


def dyt_plan_query(M, N, x_dtype, param_dtype, backward, layout, sm_count, ctas_per_sm, shift=0) -> dict:
    """The launch plan for a shape on a hypothetical device (host arithmetic only).

    layout: 0 = rows that are not whole 16-byte vectors (one-element kernels),
    1 = contiguous and 16-byte aligned, 2 = contiguous with the output `shift`
    elements past a 16-byte boundary (the shifted kernels), 3 = strided rows of
    whole-vector pitches, every tensor `shift` elements past a boundary (the
    row frame, unless shift is 0 and N a multiple of the vector), 4 = as 3 with
    the inputs at other offsets."""
    info = LaunchInfo()
    _check(lib.dyt_plan_query(M, N, x_dtype, param_dtype, int(backward), int(layout), int(shift), sm_count,
                              ctas_per_sm, ctypes.byref(info)), "dyt_plan_query")
    return info.as_dict()


def dyt_last_launch_info() -> dict:
    info = LaunchInfo()
    _check(lib.dyt_last_launch_info(ctypes.byref(info)), "dyt_last_launch_info")
    return info.as_dict()
