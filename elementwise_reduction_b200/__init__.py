"""Fused Dynamic Tanh (DyT) forward/backward for NVIDIA B200 (sm_100a).

The computation lives in hand-written CUDA kernels behind a C ABI
(``include/dyt.h``, built into ``libdyt.so``). This package is a thin layer
over it: ctypes marshalling (``_abi``), tensor helpers that take PyTorch
tensors for their device memory and stream, and an autograd module. PyTorch
allocates memory and provides streams; it computes nothing here.

    y = gamma * tanh(alpha * x) + beta      (x: [..., N], alpha: [1], gamma/beta: [N])
"""
from __future__ import annotations

import torch

from . import _abi
from ._abi import (DYT_BF16, DYT_F16, DYT_F32, MAX_RANKS, DytError, dyt_backward, dyt_backward_ex,
                   dyt_backward_noalloc, dyt_backward_partials, dyt_backward_strided, dyt_backward_workspace_bytes,
                   dyt_finalize_partials, dyt_forward, dyt_forward_ex, dyt_forward_strided, dyt_ipc_close,
                   dyt_ipc_export, dyt_ipc_import, dyt_last_launch_info, dyt_partials_layout_query, dyt_plan_query,
                   dyt_status_string)

__all__ = ["forward", "backward", "workspace", "backward_partials", "partials_layout", "finalize_partials", "DyT",
           "DyTFunction", "dyt_forward", "dyt_backward", "dyt_forward_strided", "dyt_backward_strided",
           "dyt_forward_ex", "dyt_backward_ex", "dyt_backward_noalloc", "dyt_backward_partials",
           "dyt_partials_layout_query", "dyt_finalize_partials", "dyt_ipc_export", "dyt_ipc_import",
           "dyt_ipc_close", "row_pitch", "dyt_backward_workspace_bytes", "dyt_status_string",
           "dyt_last_launch_info", "dyt_plan_query", "DytError", "DTYPE_CODE", "DYT_F32", "DYT_BF16", "DYT_F16",
           "MAX_RANKS"]

DTYPE_CODE = {torch.float32: DYT_F32, torch.bfloat16: DYT_BF16, torch.float16: DYT_F16}


def _code(t: torch.Tensor, what: str) -> int:
    try:
        return DTYPE_CODE[t.dtype]
    except KeyError:
        raise TypeError(f"{what}: dtype {t.dtype} is not supported (float32, bfloat16, float16)") from None


def _cuda_contig(t: torch.Tensor, what: str) -> None:
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")


def row_pitch(t: torch.Tensor) -> int | None:
    """Elements between consecutive rows when t's leading dimensions collapse into
    one row index with a uniform pitch and its last dimension is dense; else None."""
    if t.dim() == 0:
        return None
    if t.dim() == 1:
        return t.shape[0] if t.shape[0] <= 1 or t.stride(0) == 1 else None
    if t.shape[-1] > 1 and t.stride(-1) != 1:
        return None
    ld = t.stride(-2)
    for i in range(t.dim() - 2):  # dimension i must step over whole blocks of dimension i + 1
        if t.shape[i] > 1 and t.stride(i) != t.shape[i + 1] * t.stride(i + 1):
            return None
    if t.numel() > t.shape[-1] and ld < t.shape[-1]:
        return None
    return max(ld, t.shape[-1])


def _rows(t: torch.Tensor, what: str) -> int:
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    ld = row_pitch(t)
    if ld is None:
        raise ValueError(f"{what}: rows must be dense and evenly spaced (stride 1 along the last dimension)")
    return ld


def _shape(x: torch.Tensor, gamma: torch.Tensor):
    N = gamma.numel()
    if x.dim() == 0 or x.shape[-1] != N:
        raise ValueError(f"x's last dimension {tuple(x.shape)} must equal gamma's length {N}")
    M = x.numel() // N if N else 0
    return M, N


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def forward(x: torch.Tensor, alpha: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor,
            out: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """y = gamma * tanh(alpha * x) + beta in x's dtype (one kernel launch). x and out
    may be row-strided views (dense rows, evenly spaced): no copy is made. alpha,
    gamma and beta may each have their own dtype."""
    for t, w in ((alpha, "alpha"), (gamma, "gamma"), (beta, "beta")):
        _cuda_contig(t, w)
    ldx = _rows(x, "x")
    M, N = _shape(x, gamma)
    y = torch.empty(x.shape, dtype=x.dtype, device=x.device) if out is None else out
    if y.shape != x.shape or y.dtype != x.dtype:
        raise ValueError("out must match x in shape and dtype")
    ldy = _rows(y, "out")
    with torch.cuda.device(x.device):
        st = dyt_forward_ex(x.data_ptr(), ldx, alpha.data_ptr(), gamma.data_ptr(), beta.data_ptr(), y.data_ptr(),
                            ldy, M, N, _code(x, "x"), _code(alpha, "alpha"), _code(gamma, "gamma"),
                            _code(beta, "beta"), _stream(x.device, stream))
    _abi._check(st, "dyt_forward")
    return y


def workspace(x: torch.Tensor, gamma: torch.Tensor, dy: torch.Tensor | None = None,
              dx: torch.Tensor | None = None) -> torch.Tensor:
    """A device workspace large enough for backward on x's shape and device;
    given dy (and dx), also for the phases their row pitches call for."""
    M, N = _shape(x, gamma)
    with torch.cuda.device(x.device):
        if dy is None:
            n = dyt_backward_workspace_bytes(M, N, _code(x, "x"), _code(gamma, "gamma"))
        else:
            ldx, lddy = _rows(x, "x"), _rows(dy, "dy")
            lddx = N if dx is None else _rows(dx, "dx")
            n = _abi.dyt_backward_workspace_bytes_strided(M, N, ldx, lddy, lddx, _code(x, "x"),
                                                          _code(gamma, "gamma"))
    return torch.empty(max(n, 16), dtype=torch.uint8, device=x.device)


def backward(x: torch.Tensor, dy: torch.Tensor, alpha: torch.Tensor, gamma: torch.Tensor,
             beta: torch.Tensor | None = None, dx: torch.Tensor | None = None, dgamma: torch.Tensor | None = None,
             dbeta: torch.Tensor | None = None, dalpha: torch.Tensor | None = None,
             ws: torch.Tensor | None = None, stream: torch.cuda.Stream | None = None):
    """(dx, dalpha, dgamma, dbeta): dx in x's dtype and each parameter gradient in
    its parameter's dtype (dbeta in beta's, or gamma's when beta is not given;
    beta's values are not read). x, dy and dx may be row-strided views (dense
    rows, evenly spaced)."""
    for t, w in ((alpha, "alpha"), (gamma, "gamma")):
        _cuda_contig(t, w)
    if beta is not None:
        _cuda_contig(beta, "beta")
    if dy.shape != x.shape or dy.dtype != x.dtype:
        raise ValueError("dy must match x in shape and dtype")
    ldx, lddy = _rows(x, "x"), _rows(dy, "dy")
    M, N = _shape(x, gamma)
    beta_like = gamma if beta is None else beta
    dx = torch.empty(x.shape, dtype=x.dtype, device=x.device) if dx is None else dx
    if dx.shape != x.shape or dx.dtype != x.dtype:
        raise ValueError("dx must match x in shape and dtype")
    lddx = _rows(dx, "dx")
    dgamma = torch.empty_like(gamma) if dgamma is None else dgamma
    dbeta = torch.empty_like(beta_like) if dbeta is None else dbeta
    dalpha = torch.empty(1, dtype=alpha.dtype, device=alpha.device) if dalpha is None else dalpha
    for t, like, w in ((dgamma, gamma, "dgamma"), (dbeta, beta_like, "dbeta"), (dalpha, alpha, "dalpha")):
        if t.dtype != like.dtype or t.numel() != like.numel():
            raise ValueError(f"{w} must match its parameter in size and dtype")
        _cuda_contig(t, w)
    ws = workspace(x, gamma, dy, dx) if ws is None else ws
    with torch.cuda.device(x.device):
        st = dyt_backward_ex(x.data_ptr(), ldx, dy.data_ptr(), lddy, alpha.data_ptr(), gamma.data_ptr(),
                             None if beta is None else beta.data_ptr(), dx.data_ptr(), lddx, dgamma.data_ptr(),
                             dbeta.data_ptr(), dalpha.data_ptr(), M, N, _code(x, "x"), _code(alpha, "alpha"),
                             _code(gamma, "gamma"), _code(beta_like, "beta"), ws.data_ptr(), ws.numel(),
                             _stream(x.device, stream))
    _abi._check(st, "dyt_backward")
    return dx, dalpha, dgamma, dbeta


def backward_partials(x: torch.Tensor, dy: torch.Tensor, alpha: torch.Tensor, gamma: torch.Tensor,
                      ws: torch.Tensor, dx: torch.Tensor | None = None,
                      stream: torch.cuda.Stream | None = None):
    """Stage 1 of the backward: (dx, layout). dx in x's dtype; the binary64 partial
    sums of the parameter gradients stay in ws, where `layout` (a dict) says."""
    for t, w in ((alpha, "alpha"), (gamma, "gamma")):
        _cuda_contig(t, w)
    if dy.shape != x.shape or dy.dtype != x.dtype:
        raise ValueError("dy must match x in shape and dtype")
    ldx, lddy = _rows(x, "x"), _rows(dy, "dy")
    M, N = _shape(x, gamma)
    dx = torch.empty(x.shape, dtype=x.dtype, device=x.device) if dx is None else dx
    if dx.shape != x.shape or dx.dtype != x.dtype:
        raise ValueError("dx must match x in shape and dtype")
    lddx = _rows(dx, "dx")
    with torch.cuda.device(x.device):
        st, layout = dyt_backward_partials(x.data_ptr(), ldx, dy.data_ptr(), lddy, alpha.data_ptr(), gamma.data_ptr(),
                                           dx.data_ptr(), lddx, M, N, _code(x, "x"), _code(alpha, "alpha"),
                                           _code(gamma, "gamma"), ws.data_ptr(), ws.numel(),
                                           _stream(x.device, stream))
    _abi._check(st, "dyt_backward_partials")
    return dx, layout


def partials_layout(x: torch.Tensor, dy: torch.Tensor, dx: torch.Tensor, N: int) -> dict:
    """The partials layout backward_partials reports for these tensors (no launch)."""
    M = x.numel() // N if N else 0
    with torch.cuda.device(x.device):
        return dyt_partials_layout_query(x.data_ptr(), _rows(x, "x"), dy.data_ptr(), _rows(dy, "dy"), dx.data_ptr(),
                                         _rows(dx, "dx"), M, N, _code(x, "x"))


def finalize_partials(workspaces, layouts, alpha: torch.Tensor, gamma: torch.Tensor,
                      beta: torch.Tensor | None = None, dgamma: torch.Tensor | None = None,
                      dbeta: torch.Tensor | None = None, dalpha: torch.Tensor | None = None,
                      stream: torch.cuda.Stream | None = None):
    """(dalpha, dgamma, dbeta) from the partials of several stage-1 launches:
    workspaces are device pointers (ints) the current device can read, one per
    rank, layouts their layouts, summed in that order and rounded once."""
    N = gamma.numel()
    beta_like = gamma if beta is None else beta
    dgamma = torch.empty_like(gamma) if dgamma is None else dgamma
    dbeta = torch.empty_like(beta_like) if dbeta is None else dbeta
    dalpha = torch.empty(1, dtype=alpha.dtype, device=alpha.device) if dalpha is None else dalpha
    with torch.cuda.device(gamma.device):
        st = dyt_finalize_partials(list(workspaces), list(layouts), N, dgamma.data_ptr(), dbeta.data_ptr(),
                                   dalpha.data_ptr(), _code(alpha, "alpha"), _code(gamma, "gamma"),
                                   _code(beta_like, "beta"), _stream(gamma.device, stream))
    _abi._check(st, "dyt_finalize_partials")
    return dalpha, dgamma, dbeta


class DyTFunction(torch.autograd.Function):
    """Autograd wrapper: t is recomputed in the backward, only x is saved."""

    @staticmethod
    def forward(ctx, x, alpha, gamma, beta):
        alpha, gamma, beta = (t.contiguous() for t in (alpha, gamma, beta))
        x = x if row_pitch(x) is not None else x.contiguous()
        ctx.save_for_backward(x, alpha, gamma, beta)
        return forward(x, alpha, gamma, beta)

    @staticmethod
    def backward(ctx, dy):
        x, alpha, gamma, beta = ctx.saved_tensors
        dy = dy if row_pitch(dy) is not None else dy.contiguous()
        dx, dalpha, dgamma, dbeta = backward(x, dy, alpha, gamma, beta)
        return dx, dalpha.reshape(alpha.shape), dgamma, dbeta


class DyT(torch.nn.Module):
    """DyT(x) = gamma * tanh(alpha * x) + beta over the last dimension.

    alpha is one scalar parameter; gamma and beta have one entry per channel.
    gamma and beta live in ``param_dtype``, alpha in ``alpha_dtype`` (default:
    ``param_dtype``); each gradient comes back in its parameter's dtype.
    """

    def __init__(self, num_features: int, alpha_init: float = 0.5, param_dtype=torch.float32,
                 device=None, alpha_dtype=None):
        super().__init__()
        alpha_dtype = param_dtype if alpha_dtype is None else alpha_dtype
        self.alpha = torch.nn.Parameter(torch.full((1,), alpha_init, dtype=alpha_dtype, device=device))
        self.gamma = torch.nn.Parameter(torch.ones(num_features, dtype=param_dtype, device=device))
        self.beta = torch.nn.Parameter(torch.zeros(num_features, dtype=param_dtype, device=device))

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        return DyTFunction.apply(x, self.alpha, self.gamma, self.beta)
