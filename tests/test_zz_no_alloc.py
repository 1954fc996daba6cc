"""The backward entry point that needs no caller-provided workspace.

dyt_backward_noalloc exists for callers that cannot allocate device memory
themselves (code inside a host application that owns all device memory through
its own pool, or loops that cannot afford cudaMalloc's implicit
synchronisation). It takes its scratch from a fixed array inside the library,
so its results must match those of dyt_backward with a workspace, call after
call, even though every call reuses the same array.

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


def _backward(inp, M, N, xd, pd, noalloc: bool):
    """One backward through the C ABI; returns (dx, dgamma, dbeta, dalpha) as float64 arrays."""
    import elementwise_reduction_b200 as dyt
    from elementwise_reduction_b200 import _abi

    x, dy = _tensor(inp["x"], xd), _tensor(inp["dy"], xd)
    alpha, gamma = _tensor(inp["alpha"], pd), _tensor(inp["gamma"], pd)
    dx = torch.full_like(x, float("nan"))
    dg, db = torch.full_like(gamma, float("nan")), torch.full_like(gamma, float("nan"))
    da = torch.full((1,), float("nan"), dtype=gamma.dtype, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    if noalloc:
        st = _abi.dyt_backward_noalloc(x.data_ptr(), dy.data_ptr(), alpha.data_ptr(), gamma.data_ptr(),
                                       dx.data_ptr(), dg.data_ptr(), db.data_ptr(), da.data_ptr(), M, N,
                                       CODE[xd], CODE[pd], stream)
    else:
        ws = dyt.workspace(x.view(M, N), gamma)
        st = _abi.dyt_backward(x.data_ptr(), dy.data_ptr(), alpha.data_ptr(), gamma.data_ptr(), dx.data_ptr(),
                               dg.data_ptr(), db.data_ptr(), da.data_ptr(), M, N, CODE[xd], CODE[pd],
                               ws.data_ptr(), ws.numel(), stream)
    assert st == 0, _abi.dyt_status_string(st)
    torch.cuda.synchronize()
    return tuple(t.double().cpu().numpy().ravel() for t in (dx, dg, db, da))


def _within_tolerance(a: np.ndarray, b: np.ndarray, dtype: str) -> None:
    """The parity tolerance of the test suite: binary32 |a - b| <= 2e-6 + 1e-5 |b|;
    16-bit values at most one unit in the last place apart."""
    assert np.array_equal(np.isnan(a), np.isnan(b))
    ok = ~np.isnan(b)
    a, b = a[ok], b[ok]
    if dtype == "f32":
        assert np.all(np.abs(a - b) <= 2e-6 + 1e-5 * np.abs(b))
    else:
        bits = lambda v: torch.from_numpy(v).to(DT[dtype]).view(torch.int16).numpy().astype(np.int64)
        order = lambda i: np.where(i < 0, -(i & 0x7FFF), i)
        assert np.all(np.abs(order(bits(a)) - order(bits(b))) <= 1)


CASES = [(65537, 32, "bf16", "f32"), (4096, 4096, "bf16", "f32"), (65537, 32, "bf16", "f32"),
         (3000, 100, "f32", "f32")]


def test_noalloc_backward_matches_workspace_backward_call_after_call():
    for M, N, xd, pd in CASES:  # consecutive calls share the library's scratch
        w = workloads.Workload("noalloc", M, N, xd, pd, alpha=0.7)
        inp = workloads.make_inputs(w)
        want = _backward(inp, M, N, xd, pd, noalloc=False)
        got = _backward(inp, M, N, xd, pd, noalloc=True)
        _within_tolerance(got[0], want[0], xd)
        for g, r in zip(got[1:], want[1:]):
            _within_tolerance(g, r, pd)


def test_noalloc_rejects_shapes_beyond_its_scratch():
    import elementwise_reduction_b200 as dyt
    from elementwise_reduction_b200 import _abi

    # the smallest row count (in steps of 1024) whose scratch need exceeds the array
    N, M = 65536, 1024
    while dyt.dyt_backward_workspace_bytes(M, N, 1, 0) <= _abi.NOALLOC_SCRATCH_BYTES:
        M += 1024
    assert M * N * 2 < 4 << 30  # a few GiB at most
    x = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
    gamma = torch.ones(N, device="cuda")
    outs = [torch.empty(N, device="cuda") for _ in range(2)] + [torch.empty(1, device="cuda")]
    st = _abi.dyt_backward_noalloc(x.data_ptr(), x.data_ptr(), gamma.data_ptr(), gamma.data_ptr(),
                                   x.data_ptr(), outs[0].data_ptr(), outs[1].data_ptr(), outs[2].data_ptr(),
                                   M, N, 1, 0, torch.cuda.current_stream().cuda_stream)
    assert st == 3  # DYT_ERR_WORKSPACE_TOO_SMALL, nothing launched
