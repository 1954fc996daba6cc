"""The backward entry point that needs no caller-provided workspace.

dyt_backward_noalloc exists for callers that cannot allocate device memory
themselves (code inside a host application that owns all device memory through
its own pool, or loops that cannot afford cudaMalloc's implicit
synchronisation). It takes its scratch from a fixed array inside the library.
It runs the same kernels with the same launch plan as dyt_backward with a
workspace, so its results must be the same bits, call after call, even though
every call reuses the same array.

This file is collected last on purpose, so a run that stops at the first
failure has already run every other test.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from synth import workloads

pytestmark = pytest.mark.gpu

CODE = {"f32": 0, "bf16": 1, "f16": 2}
DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _tensor(a: np.ndarray, dtype: str) -> torch.Tensor:
    a = np.ascontiguousarray(a)
    t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) if dtype == "bf16" else torch.from_numpy(a)
    return t.cuda()


def _at(t: torch.Tensor, offset: int) -> torch.Tensor:
    """A copy of the flat tensor t starting `offset` elements past a 16-byte boundary."""
    buf = torch.empty(t.numel() + offset + 8, dtype=t.dtype, device=t.device)
    out = buf[offset:offset + t.numel()]
    out.copy_(t)
    return out


def _backward(inp, M, N, xd, pd, noalloc: bool, offset: int = 0):
    """One backward through the C ABI; returns the raw bytes of (dx, dgamma, dbeta, dalpha).
    offset: elements by which x, dy and dx start past a 16-byte boundary."""
    import elementwise_reduction_b200 as dyt
    from elementwise_reduction_b200 import _abi

    x, dy = _at(_tensor(inp["x"], xd), offset), _at(_tensor(inp["dy"], xd), offset)
    alpha, gamma = _tensor(inp["alpha"], pd), _tensor(inp["gamma"], pd)
    dx = _at(torch.full_like(x, float("nan")), offset)
    dg, db = torch.full_like(gamma, float("nan")), torch.full_like(gamma, float("nan"))
    da = torch.full((1,), float("nan"), dtype=gamma.dtype, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    if noalloc:
        st = _abi.dyt_backward_noalloc(x.data_ptr(), dy.data_ptr(), alpha.data_ptr(), gamma.data_ptr(), None,
                                       dx.data_ptr(), dg.data_ptr(), db.data_ptr(), da.data_ptr(), M, N,
                                       CODE[xd], CODE[pd], stream)
    else:
        ws = dyt.workspace(x.view(M, N), gamma)  # sized for any layout of this shape
        st = _abi.dyt_backward(x.data_ptr(), dy.data_ptr(), alpha.data_ptr(), gamma.data_ptr(), None,
                               dx.data_ptr(), dg.data_ptr(), db.data_ptr(), da.data_ptr(), M, N, CODE[xd],
                               CODE[pd], ws.data_ptr(), ws.numel(), stream)
    assert st == 0, _abi.dyt_status_string(st)
    torch.cuda.synchronize()
    return tuple(t.cpu().contiguous().view(torch.uint8).numpy() for t in (dx, dg, db, da))


CASES = [(65537, 32, "bf16", "f32"), (4096, 4096, "bf16", "f32"), (65537, 32, "bf16", "f32"),
         (3000, 100, "f32", "f32")]


def test_noalloc_backward_matches_workspace_backward_call_after_call():
    for M, N, xd, pd in CASES:  # consecutive calls share the library's scratch
        w = workloads.Workload("noalloc", M, N, xd, pd, alpha=0.7)
        inp = workloads.make_inputs(w)
        want = _backward(inp, M, N, xd, pd, noalloc=False)
        got = _backward(inp, M, N, xd, pd, noalloc=True)
        for name, g, r in zip(("dx", "dgamma", "dbeta", "dalpha"), got, want):
            assert np.array_equal(g, r), f"{name} differs from the workspace call ({M}x{N} {xd})"


def test_noalloc_backward_with_misaligned_tensors():
    # one element past a 16-byte boundary: the shifted kernels, same bits as
    # the workspace call on the same tensors
    from elementwise_reduction_b200 import _abi
    for M, N, xd in ((65537, 32, "bf16"), (3001, 255, "f32"), (2049, 4096, "bf16")):
        w = workloads.Workload("noalloc_off1", M, N, xd, "f32", alpha=0.7)
        inp = workloads.make_inputs(w)
        want = _backward(inp, M, N, xd, "f32", noalloc=False, offset=1)
        assert _abi.dyt_last_launch_info()["shifted"] == 1
        got = _backward(inp, M, N, xd, "f32", noalloc=True, offset=1)
        for name, g, r in zip(("dx", "dgamma", "dbeta", "dalpha"), got, want):
            assert np.array_equal(g, r), f"{name} differs from the workspace call ({M}x{N} {xd}, offset 1)"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import elementwise_reduction_b200 as dyt
    from elementwise_reduction_b200 import _abi

    # the narrowest power-of-two width whose scratch need, for 8 rows, exceeds the
    # array (wide rows need binary64 partials for every column)
    M, N = 8, 4096
    while dyt.dyt_backward_workspace_bytes(M, N, 1, 0) <= _abi.NOALLOC_SCRATCH_BYTES:
        N *= 2
    assert M * N * 2 < 1 << 30  # a small input all the same
    x = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    gamma = torch.ones(N, device="cuda")
    outs = [torch.empty(N, device="cuda") for _ in range(2)] + [torch.empty(1, device="cuda")]
    st = _abi.dyt_backward_noalloc(x.data_ptr(), x.data_ptr(), gamma.data_ptr(), gamma.data_ptr(), None,
                                   x.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(),
                                   M, N, 1, 0, torch.cuda.current_stream().cuda_stream)
    assert st == 3  # DYT_ERR_WORKSPACE_TOO_SMALL, nothing launched
