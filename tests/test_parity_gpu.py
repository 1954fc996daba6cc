"""CUDA path vs the CPU oracle, through the C ABI, on seeded synthetic inputs.

Tolerances are those of tests/helpers.py. Shapes cover several tiles and a
ragged tail, both launch paths, every dtype pair, the edge cases of the
Liger-Kernel page ("fix(dyt): use a 1D grid and tile small-width rows":
65,537 rows, small and ragged widths, infinite alpha with padded rows, bf16
activations with fp32 parameters), parameters of three different dtypes, and
the full-size workloads, every element.
"""
from __future__ import annotations

import json
import os

import numpy as np
import pytest
import torch

import oracle
import synth
from synth import workloads
from tests import helpers as H

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.fail("GPU tests need a CUDA device")
    import elementwise_reduction_b200  # noqa: F401  (fails loudly if libdyt.so is missing)


def make(M, N, x_dtype="f32", p_dtype="f32", alpha=0.7, x_std=1.0, dy_std=1.0, seed=0, nonzero=False,
         gamma_std=0.1, beta_std=0.1):
    w = workloads.Workload("case", M, N, x_dtype, p_dtype, alpha=alpha, x_std=x_std, dy_std=dy_std,
                           gamma_std=gamma_std, beta_std=beta_std, nonzero=nonzero, seed=seed)
    return workloads.make_inputs(w)


def roundtrip(M, N, xd="f32", pd="f32", **kw):
    inp = make(M, N, xd, pd, **kw)
    out, info = H.run_cuda(inp, M, N, xd, pd)
    stats = H.compare_all(inp, out, M, N, xd, pd)
    return out, info, stats


# ---- shape sweep: both paths, tile boundaries, ragged tails ----------------------------------

NARROW = [1, 2, 3, 4, 7, 8, 9, 16, 17, 31, 32, 33, 63, 64, 100, 127, 128, 129, 255, 256]
WIDE = [257, 511, 512, 513, 1000, 1024, 2048, 4096, 4104, 8192, 8200, 16392]


@pytest.mark.parametrize("N", NARROW)
@pytest.mark.parametrize("xd,pd", [("f32", "f32"), ("bf16", "f32")])
def test_narrow_widths(N, xd, pd):
    M = 3000 + 7  # several groups and a ragged last step
    _, info, _ = roundtrip(M, N, xd, pd)
    assert info["bwd"]["path"] == 1 and info["fwd"]["path"] == 1


@pytest.mark.parametrize("N", WIDE)
@pytest.mark.parametrize("xd,pd", [("f32", "f32"), ("bf16", "f32"), ("f16", "f32")])
def test_wide_widths(N, xd, pd):
    M = 97
    roundtrip(M, N, xd, pd)


@pytest.mark.parametrize("xd,pd", [("f32", "bf16"), ("f32", "f16"), ("bf16", "bf16"), ("f16", "f16"),
                                   ("bf16", "f16"), ("f16", "bf16")])
@pytest.mark.parametrize("M,N", [(513, 64), (257, 17), (33, 4096), (5, 9000)])
def test_dtype_matrix(xd, pd, M, N):
    roundtrip(M, N, xd, pd)


@pytest.mark.parametrize("M", [1, 2, 3, 255, 256, 257, 1023, 1025])
def test_row_counts(M):
    roundtrip(M, 64, "bf16", "f32")
    roundtrip(M, 4096, "bf16", "f32")


# ---- edge cases from the page and the method ---------------------------------------------------

def test_page_row_count_crosses_grid_limit():
    facts = json.load(open(os.path.join(GOLDEN, "liger_dyt_page_facts.json")))
    M = facts["rows_case"]["value"]
    assert M > facts["grid_dim_limit"]["value"]
    for N, xd in ((32, "bf16"), (1, "f32"), (300, "f32")):
        _, info, _ = roundtrip(M, N, xd, "f32")
        assert info["bwd"]["grid"] <= 148 * 8  # 1D persistent grid


@pytest.mark.parametrize("N", [17, 100, 255, 1, 7, 300, 4100])
@pytest.mark.parametrize("xd", ["f32", "bf16"])
def test_infinite_alpha_with_padded_rows(N, xd):
    # Ragged row counts leave padded lanes in the last step; with alpha = +inf a
    # padded zero would give tanh(inf * 0) = NaN unless masked after the arithmetic.
    M = 1000 + 13
    inp = make(M, N, xd, "f32", alpha=float("inf"), nonzero=True)
    out, info = H.run_cuda(inp, M, N, xd, "f32")
    H.compare_all(inp, out, M, N, xd, "f32")
    dg = H.decode(out["dgamma"], "f32")
    db = H.decode(out["dbeta"], "f32")
    assert np.isfinite(dg).all() and np.isfinite(db).all()
    assert out["dalpha"] == 0.0
    assert np.isnan(H.decode(out["dx"], xd)).all()


def test_alpha_zero_gives_beta_and_zero_gradients():
    M, N = 777, 96
    for xd in ("f32", "bf16"):
        inp = make(M, N, xd, "f32", alpha=0.0)
        out, _ = H.run_cuda(inp, M, N, xd, "f32")
        y = H.decode(out["y"], xd).reshape(M, N)
        want = H.decode(oracle.round_to(inp["beta"].astype(np.float64), xd), xd)
        assert np.array_equal(y, np.broadcast_to(want, (M, N)))
        assert np.all(H.decode(out["dx"], xd) == 0.0)
        assert np.all(H.decode(out["dgamma"], "f32") == 0.0)
        H.compare_all(inp, out, M, N, xd, "f32")


def test_odd_symmetry_with_zero_beta():
    M, N = 300, 130
    inp = make(M, N, "f32", "f32", alpha=1.1)
    inp["beta"] = np.zeros(N, np.float32)
    out, _ = H.run_cuda(inp, M, N, "f32", "f32", bwd=False)
    neg = dict(inp, x=(-inp["x"]).astype(np.float32))
    outn, _ = H.run_cuda(neg, M, N, "f32", "f32", bwd=False)
    assert np.array_equal(outn["y"], -out["y"])


def test_dbeta_is_exact_for_integer_dy():
    M, N = 5000, 40
    inp = make(M, N, "f32", "f32")
    inp["dy"] = np.round(synth.normal(M * N, "f32", 0.0, 8.0, 1, 2)).astype(np.float32)
    out, _ = H.run_cuda(inp, M, N, "f32", "f32", fwd=False)
    want = inp["dy"].astype(np.int64).reshape(M, N).sum(0)
    assert np.array_equal(H.decode(out["dbeta"], "f32"), want.astype(np.float64))


def test_cancelling_outputs_are_correctly_rounded():
    # beta chosen so that gamma * tanh(alpha * x) + beta cancels for many x: each
    # column's beta is minus the value at one of its own entries.
    M, N = 4096, 64
    for xd in ("bf16", "f16"):
        inp = make(M, N, xd, "f32", alpha=0.9)
        X = H.decode(inp["x"], xd).reshape(M, N)
        g = inp["gamma"].astype(np.float64)
        inp["beta"] = (-g * np.tanh(0.9 * X[17])).astype(np.float32)
        out, _ = H.run_cuda(inp, M, N, xd, "f32", bwd=False)
        st = H.compare_all(inp, out, M, N, xd, "f32")
        assert st["y"]["max_ulp"] <= 1


def test_cancelling_outputs_in_the_f16_subnormal_range():
    # x ~ N(0, 1e-3) and beta ~ -tanh(x) of one row: y = gamma t + beta lands
    # around 1e-6, inside fp16's subnormal range (below 6.1e-5), where rounding
    # errors are absolute, and the cancellation threshold tau |beta| ~ 2e-6 is
    # itself subnormal.
    M, N = 4096, 64
    for pd in ("f32", "f16"):
        inp = make(M, N, "f16", pd, alpha=1.0, x_std=1e-3)
        X = H.decode(inp["x"], "f16").reshape(M, N)
        g = H.decode(inp["gamma"], pd)
        beta = -g * np.tanh(X[17])
        inp["beta"] = beta.astype(np.float32) if pd == "f32" else beta.astype(np.float16)
        out, _ = H.run_cuda(inp, M, N, "f16", pd, bwd=False)
        Y = np.abs(H.decode(out["y"], "f16"))
        assert ((Y > 0) & (Y < 6.1e-5)).sum() > 1000  # many subnormal outputs
        st = H.compare_all(inp, out, M, N, "f16", pd)
        assert st["y"]["max_ulp"] <= 1


def test_extreme_arguments():
    # Large |alpha x| (tanh saturates, 1 - t^2 underflows), tiny |alpha x|, and
    # special values in x.
    M, N = 64, 64
    inp = make(M, N, "f32", "f32", alpha=3.0, x_std=20.0)
    x = inp["x"]
    x[:8] = [0.0, -0.0, 1e-30, -1e-38, 1e-45, np.inf, -np.inf, np.nan]
    x[8:16] = [5.0, 10.0, 15.0, 20.0, 29.0, 30.0, 40.0, 50.0]
    out, _ = H.run_cuda(inp, M, N, "f32", "f32")
    H.compare_all(inp, out, M, N, "f32", "f32")


@pytest.mark.parametrize("xd", ["bf16", "f16", "f32"])
def test_saturated_arguments_keep_tiny_gradients(xd):
    # |alpha x| in (40, 52]: 1 - t^2 is below 2^-115 and reaches the binary32
    # subnormal range; dx = alpha gamma dy (1 - t^2) must still round correctly.
    M, N = 64, 128
    inp = make(M, N, xd, "f32", alpha=1.0)
    rng = np.random.default_rng(5)
    xs = rng.uniform(40.0, 52.0, M * N) * rng.choice([-1.0, 1.0], M * N)
    inp["x"] = oracle.round_to(xs, xd) if xd != "f32" else xs.astype(np.float32)
    inp["dy"] = oracle.round_to(rng.uniform(1e3, 1e4, M * N), xd) if xd != "f32" else \
        rng.uniform(1e3, 1e4, M * N).astype(np.float32)
    out, _ = H.run_cuda(inp, M, N, xd, "f32")
    H.compare_all(inp, out, M, N, xd, "f32")
    if xd != "f16":  # binary16 has no values this small: its dx is all zeros
        assert np.count_nonzero(H.decode(out["dx"], xd)) > M * N // 4


@pytest.mark.parametrize("xd", ["bf16", "f32"])
def test_subnormal_exponentials_scattered_in_ordinary_vectors(xd):
    # Mostly ordinary |alpha x|, with single elements at 44..51.9 (exp(-2|z|) a
    # nonzero binary32 subnormal), 53..80 (exp(-2|z|) rounds to 0) and +-inf,
    # spread so that most 16-byte vectors hold at most one of them.
    M, N = 512, 256
    inp = make(M, N, xd, "f32", alpha=1.0)
    rng = np.random.default_rng(11)
    X = H.decode(inp["x"], xd).astype(np.float64)
    idx = rng.permutation(M * N)
    win, far, inf = idx[:2000], idx[2000:3000], idx[3000:3100]
    X[win] = rng.uniform(44.0, 51.9, win.size) * rng.choice([-1.0, 1.0], win.size)
    X[far] = rng.uniform(53.0, 80.0, far.size) * rng.choice([-1.0, 1.0], far.size)
    X[inf] = np.inf * rng.choice([-1.0, 1.0], inf.size)
    inp["x"] = oracle.round_to(X, xd) if xd != "f32" else X.astype(np.float32)
    DY = H.decode(inp["dy"], xd).astype(np.float64)
    DY[win] = rng.uniform(1e3, 1e4, win.size)  # lifts dx above bf16's smallest subnormal
    inp["dy"] = oracle.round_to(DY, xd) if xd != "f32" else DY.astype(np.float32)
    out, _ = H.run_cuda(inp, M, N, xd, "f32")
    H.compare_all(inp, out, M, N, xd, "f32")
    dx = H.decode(out["dx"], xd)
    if xd == "bf16":  # the window's tiny gradients are kept, not flushed
        assert np.count_nonzero(dx[win]) > win.size // 2


def test_empty_shapes():
    import elementwise_reduction_b200 as dyt
    x = torch.empty(0, 7, device="cuda")
    g = torch.ones(7, device="cuda")
    a = torch.tensor([0.5], device="cuda")
    y = dyt.forward(x, a, g, g)
    assert y.shape == (0, 7)
    dg = torch.full((7,), 3.0, device="cuda")
    db = torch.full((7,), 3.0, device="cuda")
    da = torch.full((1,), 3.0, device="cuda")
    dyt.backward(x, x, a, g, dgamma=dg, dbeta=db, dalpha=da)
    torch.cuda.synchronize()
    assert (dg == 0).all() and (db == 0).all() and (da == 0).all()


# ---- layout: unaligned pointers, in-place, determinism ------------------------------------------

def _placed(src, M: int, N: int, offset: int, dtype, fill: float):
    """An M x N tensor `offset` elements past a 16-byte boundary, with guard
    elements of value `fill` on both sides (a fresh allocation starts on a
    512-byte boundary)."""
    buf = torch.full((M * N + offset + 24,), fill, dtype=dtype, device="cuda")
    m = buf[offset:offset + M * N].view(M, N)
    if src is not None:
        m.copy_(src.reshape(M, N))
    return buf, m


def _run_placed(inp, M, N, xd, pd, hx, hd, ho):
    """Forward and backward with x, dy at offsets hx, hd and y, dx at ho (elements)."""
    import elementwise_reduction_b200 as dyt
    t = H.gpu_inputs(inp, xd, pd)
    dt = t["x"].dtype
    _, x = _placed(t["x"], M, N, hx, dt, float("nan"))
    _, dy = _placed(t["dy"], M, N, hd, dt, float("nan"))
    ybuf, y = _placed(None, M, N, ho, dt, 7.0)
    dxbuf, dx = _placed(None, M, N, ho, dt, 7.0)
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=y)
    info_f = dyt.dyt_last_launch_info()
    _, da, dg, db = dyt.backward(x, dy, t["alpha"], t["gamma"], t["beta"], dx=dx)
    info_b = dyt.dyt_last_launch_info()
    torch.cuda.synchronize()
    for buf in (ybuf, dxbuf):  # nothing outside the outputs is written
        assert (buf[:ho] == 7).all() and (buf[ho + M * N:] == 7).all()
    ad, gd, bd = H.param_dtypes(pd)
    out = {"y": H.to_numpy(y, xd), "dx": H.to_numpy(dx, xd), "dgamma": H.to_numpy(dg, gd),
           "dbeta": H.to_numpy(db, bd), "dalpha": float(H.decode(H.to_numpy(da, ad), ad)[0])}
    return out, info_f, info_b


# Contiguous tensors off 16-byte boundaries take the shifted 16-byte kernels:
# each output vector whole, each input vector cut out of two aligned chunks
# (x and dy each at their own offset), the first and last vectors element by
# element. NaN guards around the inputs fail any read outside them; guards
# around the outputs any write outside them.
@pytest.mark.parametrize("xd", ["f32", "bf16", "f16"])
@pytest.mark.parametrize("M,N", [(1, 1), (3, 3), (7, 8), (33, 17), (129, 64), (65, 255), (9, 1001), (5, 4100),
                                 (2049, 32)])
@pytest.mark.parametrize("hx,hd,ho", [(1, 1, 1), (1, 0, 0), (0, 0, 1), (3, 5, 7), (7, 1, 2), (0, 7, 0), (2, 2, 6)])
def test_unaligned_tensors_take_the_shifted_kernels(xd, M, N, hx, hd, ho):
    vec = 4 if xd == "f32" else 8
    hx, hd, ho = hx % vec, hd % vec, ho % vec
    if hx == hd == ho == 0:
        pytest.skip("aligned")
    inp = make(M, N, xd, "f32")
    out, info_f, info_b = _run_placed(inp, M, N, xd, "f32", hx, hd, ho)
    # the forward sees x and y only
    for info, shifted in ((info_f, hx or ho), (info_b, True)):
        assert info["vec"] == vec and info["shifted"] == bool(shifted) and info["shift"] == (ho if shifted else 0)
        assert info["pack_rows"] == (vec if N % vec else 1)
    H.compare_all(inp, out, M, N, xd, "f32")
    # every element's arithmetic is the aligned kernels': the same bits
    ref, _ = H.run_cuda(inp, M, N, xd, "f32")
    assert np.array_equal(out["y"], ref["y"]) and np.array_equal(out["dx"], ref["dx"])


@pytest.mark.parametrize("xd,pd", [("bf16", ("bf16", "f32", "f16")), ("f16", "f16"), ("f32", "bf16")])
def test_shifted_kernels_with_parameter_dtypes(xd, pd):
    M, N = 1537, 100
    inp = make(M, N, xd, pd)
    out, info_f, info_b = _run_placed(inp, M, N, xd, pd, 3, 1, 1)
    assert info_f["shifted"] == info_b["shifted"] == 1
    H.compare_all(inp, out, M, N, xd, pd)


@pytest.mark.parametrize("N", [17, 1001])
def test_shifted_kernels_with_infinite_alpha(N):
    # the padded elements of the first and last vectors would give
    # tanh(inf * 0) = NaN if they entered a sum
    M = 4099
    inp = make(M, N, "f32", "f32", alpha=float("inf"), nonzero=True)
    out, _, info_b = _run_placed(inp, M, N, "f32", "f32", 1, 2, 3)
    assert info_b["shifted"] == 1
    stats = H.compare_all(inp, out, M, N, "f32", "f32")
    assert stats["dgamma"]["n_over_strict_elementwise"] == 0 and stats["dbeta"]["n_over_strict_elementwise"] == 0


def test_shifted_in_place():
    import elementwise_reduction_b200 as dyt
    M, N = 1001, 255
    inp = make(M, N, "bf16", "f32")
    ref, _ = H.run_cuda(inp, M, N, "bf16", "f32")
    t = H.gpu_inputs(inp, "bf16", "f32")
    _, x = _placed(t["x"], M, N, 3, torch.bfloat16, 0.0)
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=x)  # y over x
    assert dyt.dyt_last_launch_info()["shifted"] == 1
    assert np.array_equal(H.to_numpy(x, "bf16"), ref["y"])
    _, x = _placed(t["x"], M, N, 3, torch.bfloat16, 0.0)
    _, dy = _placed(t["dy"], M, N, 5, torch.bfloat16, 0.0)
    dyt.backward(x, dy, t["alpha"], t["gamma"], dx=dy)  # dx over dy
    assert np.array_equal(H.to_numpy(dy, "bf16"), ref["dx"])


# Ragged widths of aligned tensors are streamed in packs of 16 / size rows; the
# last pack may be short, down to a single row, and its one straddling vector
# is zero-filled and masked.
@pytest.mark.parametrize("M", [1, 2, 3, 5, 7, 8, 9, 13, 4099])
@pytest.mark.parametrize("N,xd", [(17, "f32"), (3, "f32"), (255, "bf16"), (1001, "f16"), (17, "bf16"),
                                  (4097, "f32")])
def test_ragged_widths_take_the_packed_path(M, N, xd):
    _, info, _ = roundtrip(M, N, xd, "f32")
    vec = 4 if xd == "f32" else 8
    for op in ("fwd", "bwd"):
        assert info[op]["pack_rows"] == vec and info[op]["vec"] == vec and info[op]["async_stages"] > 0


@pytest.mark.parametrize("N", [17, 1001])
def test_infinite_alpha_in_the_straddling_vector(N):
    # 4099 rows of 17 or 1001 fp32 columns end inside a 16-byte vector whose
    # zero-filled tail would give tanh(inf * 0) = NaN if it entered a sum.
    M = 4099
    inp = make(M, N, "f32", "f32", alpha=float("inf"), nonzero=True)
    out, info = H.run_cuda(inp, M, N, "f32", "f32")
    assert info["bwd"]["pack_rows"] == 4
    H.compare_all(inp, out, M, N, "f32", "f32")
    assert np.isfinite(H.decode(out["dgamma"], "f32")).all()
    assert np.isfinite(H.decode(out["dbeta"], "f32")).all()


@pytest.mark.parametrize("M,N", [(1000, 256), (1001, 255)])
def test_in_place_aliasing(M, N):
    import elementwise_reduction_b200 as dyt
    inp = make(M, N, "bf16", "f32")
    ref, _ = H.run_cuda(inp, M, N, "bf16", "f32")
    t = H.gpu_inputs(inp, "bf16", "f32")
    x = t["x"].view(M, N).clone()
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=x)  # y over x
    assert np.array_equal(H.to_numpy(x, "bf16"), ref["y"])
    x = t["x"].view(M, N)
    dy = t["dy"].view(M, N).clone()
    dyt.backward(x, dy, t["alpha"], t["gamma"], dx=dy)  # dx over dy
    assert np.array_equal(H.to_numpy(dy, "bf16"), ref["dx"])
    x2 = t["x"].view(M, N).clone()
    dyt.backward(x2, t["dy"].view(M, N), t["alpha"], t["gamma"], dx=x2)  # dx over x
    assert np.array_equal(H.to_numpy(x2, "bf16"), ref["dx"])


# ---- row-strided matrices: each tensor with its own leading dimension -----------------------------

def _phases(M: int, N: int, lds, size: int, backward: bool = False) -> int:
    # The library's phase count for these row pitches: a row's offset past a
    # 16-byte boundary repeats every 16 / (lowest set bit of pitch bytes mod 16)
    # rows; strided calls whose pitches are not all whole vectors run that many
    # phases of whole-vector pitch, when every phase moves at least 8 MiB
    # (forward) or 32 MiB (backward, 2 phases only) per tensor.
    def period(ld):
        r = (ld * size) % 16
        return 1 if r == 0 else 16 // (r & -r)
    k = max(period(ld) for ld in lds)
    if all(ld == N for ld in lds) or k == 1 or M < k:
        return 1
    smallest = (M - (k - 1) + k - 1) // k * N * size
    if smallest < ((32 if backward else 8) << 20) or (backward and k != 2):
        return 1
    return k


def _in_wider_rows(src: torch.Tensor, M: int, N: int, pitch: int, fill: float) -> tuple:
    buf = torch.full((M, pitch), fill, dtype=src.dtype, device="cuda")
    buf[:, :N] = src.view(M, N)
    return buf, buf[:, :N]


@pytest.mark.parametrize("N,pad,xd", [(64, 8, "bf16"), (64, 3, "bf16"), (100, 4, "f32"), (17, 3, "f32"),
                                      (4096, 64, "bf16"), (255, 1, "f32"), (8, 8, "f16"), (1000, 24, "f16")])
def test_strided_rows(N, pad, xd):
    import elementwise_reduction_b200 as dyt
    M = 3001
    inp = make(M, N, xd, "f32")
    t = H.gpu_inputs(inp, xd, "f32")
    _, x = _in_wider_rows(t["x"], M, N, N + pad, float("nan"))      # padding reaches no result
    _, dy = _in_wider_rows(t["dy"], M, N, N + 2 * pad, float("nan"))
    ybuf, y = _in_wider_rows(torch.zeros(M * N, dtype=x.dtype, device="cuda"), M, N, N + 3 * pad, 7.0)
    dxbuf, dx = _in_wider_rows(torch.zeros(M * N, dtype=x.dtype, device="cuda"), M, N, N + 4 * pad, 7.0)
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=y)
    info_f = dyt.dyt_last_launch_info()
    _, dalpha, dgamma, dbeta = dyt.backward(x, dy, t["alpha"], t["gamma"], dx=dx)
    info_b = dyt.dyt_last_launch_info()
    torch.cuda.synchronize()
    assert (ybuf[:, N:] == 7).all() and (dxbuf[:, N:] == 7).all()  # padding is never written
    out = {"y": H.to_numpy(y.contiguous(), xd), "dx": H.to_numpy(dx.contiguous(), xd),
           "dgamma": H.to_numpy(dgamma, "f32"), "dbeta": H.to_numpy(dbeta, "f32"), "dalpha": float(dalpha.item())}
    H.compare_all(inp, out, M, N, xd, "f32")
    size = 4 if xd == "f32" else 2
    vec = 16 // size
    # whole-vector pitches take the 16-byte kernels (aligned tensors and N a
    # multiple of vec: the plain ones, else the row frame); other pitches run
    # as phases of whole-vector pitch through the same kernels
    pitched = all((p * size) % 16 == 0 for p in (N + pad, N + 2 * pad, N + 3 * pad, N + 4 * pad))
    vectorised = N % vec == 0 and pitched
    k_f = _phases(M, N, (N + pad, N + 3 * pad), size)
    k_b = _phases(M, N, (N + pad, N + 2 * pad, N + 4 * pad), size, backward=True)
    whole_f = all((p * size) % 16 == 0 for p in (N + pad, N + 3 * pad))
    whole_b = all((p * size) % 16 == 0 for p in (N + pad, N + 2 * pad, N + 4 * pad))
    assert info_f["vec"] == (vec if whole_f or k_f > 1 else 1)
    assert info_b["vec"] == (vec if whole_b or k_b > 1 else 1)
    assert info_f["kernels"] == k_f and info_b["kernels"] == k_b + 1
    if pitched:
        assert info_f["shifted"] == info_b["shifted"] == (0 if vectorised else 2)
    assert info_b["pack_rows"] == 1
    if vectorised:  # the same kernels as the contiguous call: the same bits
        ref, _ = H.run_cuda(inp, M, N, xd, "f32")
        for k in ("y", "dx", "dgamma", "dbeta"):
            assert np.array_equal(out[k], ref[k]), k
        assert out["dalpha"] == ref["dalpha"]


def _placed_rows(src, M: int, N: int, off: int, ld: int, fill: float) -> tuple:
    # M rows of N elements, `ld` apart, the first `off` elements past a 16-byte
    # boundary, in a buffer filled with `fill`
    buf = torch.full((M * ld + off + 64,), fill, dtype=src.dtype, device="cuda")
    view = buf[off:off + M * ld].view(M, ld)[:, :N]
    view.copy_(src.reshape(M, N))
    return buf, view


@pytest.mark.parametrize("xd", ["f32", "bf16"])
@pytest.mark.parametrize("N", [1, 3, 17, 100, 255, 520, 4099])
@pytest.mark.parametrize("hx,hd,ho", [(0, 0, 0), (1, 1, 1), (-3, -3, -3), (0, 3, 1), (-1, 0, 2), (2, -1, -1)])
def test_row_frame_rows(xd, N, hx, hd, ho):
    # Strided rows whose pitches are whole 16-byte vectors, with tensors off
    # 16-byte boundaries or a ragged N: each row shifted on its own. NaN
    # between the rows of the inputs (the chunks at a row's ends read some of
    # it; it must reach no result), 7 between the rows of the outputs (never
    # written); elementwise results bit for bit those of the contiguous call,
    # sums within the oracle's bounds.
    import elementwise_reduction_b200 as dyt
    size = 4 if xd == "f32" else 2
    vec = 16 // size
    hx, hd, ho = hx % vec, hd % vec, ho % vec
    if not (hx or hd or ho or N % vec):
        pytest.skip("aligned rows of whole vectors take the plain kernels")
    M = 1201
    base = -(-N // vec) * vec
    inp = make(M, N, xd, "f32")
    t = H.gpu_inputs(inp, xd, "f32")
    _, x = _placed_rows(t["x"], M, N, hx, base + vec, float("nan"))
    _, dy = _placed_rows(t["dy"], M, N, hd, base + 2 * vec, float("nan"))
    zero = torch.zeros(M * N, dtype=t["x"].dtype, device="cuda")
    ybuf, y = _placed_rows(zero, M, N, ho, base + 3 * vec, 7.0)
    dxbuf, dx = _placed_rows(zero, M, N, ho, base, 7.0)
    ymask = torch.ones_like(ybuf, dtype=torch.bool)
    ymask[ho:ho + M * (base + 3 * vec)].view(M, -1)[:, :N] = False
    dxmask = torch.ones_like(dxbuf, dtype=torch.bool)
    dxmask[ho:ho + M * base].view(M, -1)[:, :N] = False
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=y)
    info_f = dyt.dyt_last_launch_info()
    _, dalpha, dgamma, dbeta = dyt.backward(x, dy, t["alpha"], t["gamma"], dx=dx)
    info_b = dyt.dyt_last_launch_info()
    torch.cuda.synchronize()
    assert (ybuf[ymask] == 7).all() and (dxbuf[dxmask] == 7).all()  # nothing outside the rows is written
    # every tensor at the output's offset sh > 0 and N a multiple of vec: the
    # first vector-column also holds each row's last sh elements (3)
    assert info_f["shifted"] == (3 if hx == ho and ho and N % vec == 0 else 2)
    assert info_b["shifted"] == (3 if hx == hd == ho and ho and N % vec == 0 else 2)
    assert info_f["shift"] == info_b["shift"] == ho
    assert info_f["vec"] == info_b["vec"] == vec
    out = {"y": H.to_numpy(y.contiguous(), xd), "dx": H.to_numpy(dx.contiguous(), xd),
           "dgamma": H.to_numpy(dgamma, "f32"), "dbeta": H.to_numpy(dbeta, "f32"), "dalpha": float(dalpha.item())}
    H.compare_all(inp, out, M, N, xd, "f32")
    ref, _ = H.run_cuda(inp, M, N, xd, "f32")
    assert np.array_equal(out["y"], ref["y"]) and np.array_equal(out["dx"], ref["dx"])


@pytest.mark.parametrize("xd,M,N,lds,offs", [
    ("bf16", 8200, 4096, (4100, 4100, 4100), (0, 0, 0)),   # 8200 bytes: 2 phases, forward and backward
    ("bf16", 8200, 4096, (4100, 4100, 4108), (1, 1, 1)),   # 2 phases, every tensor one element off
    ("f32", 4200, 2048, (2050, 2050, 2054), (0, 1, 2)),    # 8200 / 8216 bytes: 2 phases, forward only
    ("bf16", 9000, 2048, (2050, 2054, 2058), (1, 1, 3)),   # 4 phases: the forward's
    ("bf16", 33000, 1024, (1025, 1027, 1029), (0, 5, 2)),  # odd pitches: 8 phases, the forward's
    ("f32", 4001, 17, (17, 21, 19), (3, 0, 1)),            # x adjacent, the others not: too small, one phase
])
def test_phased_rows(xd, M, N, lds, offs):
    # Pitches that are not whole 16-byte vectors: rows j, j + k, ... run as k
    # matrices of whole-vector pitch through the 16-byte kernels. NaN between
    # the inputs' rows, 7 around the outputs (never written); elementwise
    # results bit for bit those of the contiguous call, sums within the
    # oracle's bounds; a workspace too small for the phases runs one phase.
    import elementwise_reduction_b200 as dyt
    size = 4 if xd == "f32" else 2
    vec = 16 // size
    ldx, lddy, ldo = lds
    hx, hd, ho = offs
    inp = make(M, N, xd, "f32")
    t = H.gpu_inputs(inp, xd, "f32")
    _, x = _placed_rows(t["x"], M, N, hx, ldx, float("nan"))
    _, dy = _placed_rows(t["dy"], M, N, hd, lddy, float("nan"))
    zero = torch.zeros(M * N, dtype=t["x"].dtype, device="cuda")
    ybuf, y = _placed_rows(zero, M, N, ho, ldo, 7.0)
    dxbuf, dx = _placed_rows(zero, M, N, ho, ldo, 7.0)
    mask = torch.ones_like(ybuf, dtype=torch.bool)
    mask[ho:ho + M * ldo].view(M, -1)[:, :N] = False
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=y)
    info_f = dyt.dyt_last_launch_info()
    _, dalpha, dgamma, dbeta = dyt.backward(x, dy, t["alpha"], t["gamma"], dx=dx)
    info_b = dyt.dyt_last_launch_info()
    torch.cuda.synchronize()
    assert (ybuf[mask] == 7).all() and (dxbuf[mask] == 7).all()  # nothing outside the rows is written
    k_f, k_b = _phases(M, N, (ldx, ldo), size), _phases(M, N, (ldx, lddy, ldo), size, backward=True)
    assert info_f["kernels"] == k_f and info_b["kernels"] == k_b + 1
    assert info_f["vec"] == (vec if k_f > 1 else 1) and info_b["vec"] == (vec if k_b > 1 else 1)
    out = {"y": H.to_numpy(y.contiguous(), xd), "dx": H.to_numpy(dx.contiguous(), xd),
           "dgamma": H.to_numpy(dgamma, "f32"), "dbeta": H.to_numpy(dbeta, "f32"), "dalpha": float(dalpha.item())}
    H.compare_all(inp, out, M, N, xd, "f32")
    ref, _ = H.run_cuda(inp, M, N, xd, "f32")
    assert np.array_equal(out["y"], ref["y"]) and np.array_equal(out["dx"], ref["dx"])
    # The plain size query covers one phase (the one-element kernels); where
    # that is less than the phases need, the same call runs as one phase.
    small = dyt.workspace(x, t["gamma"])
    fits = small.numel() >= dyt.workspace(x, t["gamma"], dy, dx).numel() or k_b == 1
    dx2 = torch.empty_like(dx)
    _, dalpha2, dgamma2, dbeta2 = dyt.backward(x, dy, t["alpha"], t["gamma"], dx=dx2, ws=small)
    info_1 = dyt.dyt_last_launch_info()
    torch.cuda.synchronize()
    if fits:
        assert info_1["kernels"] == k_b + 1 and info_1["vec"] == (vec if k_b > 1 else 1)
    else:
        assert info_1["kernels"] == 2 and info_1["vec"] == 1
    out2 = {"y": out["y"], "dx": H.to_numpy(dx2.contiguous(), xd), "dgamma": H.to_numpy(dgamma2, "f32"),
            "dbeta": H.to_numpy(dbeta2, "f32"), "dalpha": float(dalpha2.item())}
    H.compare_all(inp, out2, M, N, xd, "f32")


def test_strided_in_place_and_autograd():
    import elementwise_reduction_b200 as dyt
    M, N = 1000, 256
    inp = make(M, N, "bf16", "f32")
    ref, _ = H.run_cuda(inp, M, N, "bf16", "f32")
    t = H.gpu_inputs(inp, "bf16", "f32")
    buf, x = _in_wider_rows(t["x"], M, N, N + 64, 0.0)
    dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=x)  # y over x, same pitch
    assert np.array_equal(H.to_numpy(x.contiguous(), "bf16"), ref["y"])
    # autograd on a strided view: no copy of x, gradients as from the contiguous call
    _, x = _in_wider_rows(t["x"], M, N, N + 64, 0.0)
    x.requires_grad_(True)
    m = dyt.DyT(N, device="cuda")
    with torch.no_grad():
        m.alpha.copy_(t["alpha"]); m.gamma.copy_(t["gamma"]); m.beta.copy_(t["beta"])
    y = m(x)
    y.backward(t["dy"].view(M, N))
    assert np.array_equal(H.to_numpy(y.detach(), "bf16"), ref["y"])
    assert np.array_equal(H.to_numpy(x.grad.contiguous(), "bf16"), ref["dx"])
    assert np.array_equal(H.to_numpy(m.gamma.grad, "f32"), ref["dgamma"])


def test_rows_must_be_evenly_spaced():
    import elementwise_reduction_b200 as dyt
    x = torch.zeros(4, 6, 32, device="cuda")[:, 1:3]  # leading dimensions do not collapse
    one = torch.ones(32, device="cuda")
    with pytest.raises(ValueError):
        dyt.forward(x, one[:1], one, one)
    with pytest.raises(ValueError):
        dyt.forward(torch.zeros(32, 8, device="cuda").t(), one[:1], one, one)


@pytest.mark.parametrize("M,N,xd", [(65537, 32, "bf16"), (3001, 4096, "bf16"), (20000, 255, "f32")])
def test_backward_is_bitwise_deterministic(M, N, xd):
    inp = make(M, N, xd, "f32")
    a, _ = H.run_cuda(inp, M, N, xd, "f32", fwd=False)
    b, _ = H.run_cuda(inp, M, N, xd, "f32", fwd=False)
    for k in ("dx", "dgamma", "dbeta"):
        assert np.array_equal(a[k], b[k])
    assert a["dalpha"] == b["dalpha"] or (np.isnan(a["dalpha"]) and np.isnan(b["dalpha"]))


@pytest.mark.parametrize("M,N,xd", [(65537, 32, "bf16"), (1024, 64, "f32"), (20000, 17, "f32"),
                                    (4096, 4096, "bf16")])
def test_backward_in_cuda_graph_replays_and_with_garbage_workspace(M, N, xd):
    # A fresh workspace holds arbitrary bytes, and a captured graph replays the
    # same launches: both must give the eager bits.
    import elementwise_reduction_b200 as dyt
    inp = make(M, N, xd, "f32")
    t = H.gpu_inputs(inp, xd, "f32")
    x, dy = t["x"].view(M, N), t["dy"].view(M, N)
    ref = [u.clone() for u in dyt.backward(x, dy, t["alpha"], t["gamma"])]
    info = dyt.dyt_last_launch_info()
    ws = dyt.workspace(x, t["gamma"])
    ws.copy_(torch.randint(0, 256, ws.shape, dtype=torch.uint8, device="cuda"))
    outs = [torch.empty_like(u) for u in ref]
    dyt.backward(x, dy, t["alpha"], t["gamma"], dx=outs[0], dalpha=outs[1], dgamma=outs[2], dbeta=outs[3],
                 ws=ws)
    torch.cuda.synchronize()
    for a, b in zip(outs, ref):
        assert torch.equal(a, b)
    stream = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        dyt.backward(x, dy, t["alpha"], t["gamma"], dx=outs[0], dalpha=outs[1], dgamma=outs[2], dbeta=outs[3],
                     ws=ws)  # warm-up on the capture stream
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=stream):
            dyt.backward(x, dy, t["alpha"], t["gamma"], dx=outs[0], dalpha=outs[1], dgamma=outs[2],
                         dbeta=outs[3], ws=ws)
    for _ in range(4):
        for u in outs:
            u.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for a, b in zip(outs, ref):
            assert torch.equal(a, b)
    assert info["kernels"] == 2


@pytest.mark.parametrize("xd", [0, 1, 2])
def test_workspace_bytes_cover_every_vectorised_plan(xd):
    # The size query must cover the plan of every layout a call can have:
    # aligned, shifted (each output offset) and the row frame (wrapped or not).
    from tests.test_abi_cpu import _lib
    lib = _lib()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    vec = 4 if xd == 0 else 8
    for M in (1, 3, 1000, 65537, 100003):
        for N in (1, 3, 8, 17, 32, 100, 255, 256, 513, 4096, 4099, 8192):
            need = lib.dyt_backward_workspace_bytes(M, N, xd, 0)
            assert need > 0
            for layout in (1, 2, 3, 4):
                for shift in (range(vec) if layout >= 2 else [0]):
                    p = lib.dyt_plan_query(M, N, xd, 0, 1, layout, sms, 1, shift=shift)
                    assert p["workspace_bytes"] <= need, (M, N, layout, shift)


def test_workspace_errors():
    import elementwise_reduction_b200 as dyt
    M, N = 100, 64
    x = torch.randn(M, N, device="cuda")
    g = torch.ones(N, device="cuda")
    a = torch.tensor([0.5], device="cuda")
    ws = dyt.workspace(x, g)
    assert ws.numel() >= 16
    with pytest.raises(dyt.DytError) as e:
        dyt.backward(x, x, a, g, ws=ws[:16])
    assert e.value.status == 3
    with pytest.raises(dyt.DytError) as e:
        dyt.backward(x, x, a, g, ws=ws[8:])
    assert e.value.status == 1


@pytest.mark.parametrize("pd", [("bf16", "f32", "f16"), ("f16", "bf16", "f32"), ("f32", "f16", "bf16"),
                                ("bf16", "bf16", "f32")])
@pytest.mark.parametrize("M,N,xd", [(1001, 64, "bf16"), (257, 17, "f32"), (33, 4100, "f16")])
def test_each_parameter_keeps_its_own_dtype(pd, M, N, xd):
    # alpha, gamma and beta in three different dtypes: each gradient comes back
    # in its own parameter's dtype (the page's Summary, "Precision").
    inp = make(M, N, xd, pd)
    out, _ = H.run_cuda(inp, M, N, xd, pd)
    H.compare_all(inp, out, M, N, xd, pd)
    assert out["dgamma"].dtype == oracle.NP_STORAGE[pd[1]] and out["dbeta"].dtype == oracle.NP_STORAGE[pd[2]]


def test_beta_is_not_read_by_the_backward():
    import elementwise_reduction_b200 as dyt
    M, N = 777, 96
    inp = make(M, N, "bf16", "f32")
    t = H.gpu_inputs(inp, "bf16", "f32")
    x, dy = t["x"].view(M, N), t["dy"].view(M, N)
    ref = [u.clone() for u in dyt.backward(x, dy, t["alpha"], t["gamma"])]
    nan_beta = torch.full_like(t["beta"], float("nan"))
    got = dyt.backward(x, dy, t["alpha"], t["gamma"], nan_beta)
    for a, b in zip(got, ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("M,N,alpha", [(200003, 33, 0.9), (100003, 17, 1.3), (65537, 100, float("inf"))])
def test_fp32_sums_meet_the_elementwise_bound(M, N, alpha):
    # Binary32 data of 1e5+ rows: every add of a binary32 running sum would round,
    # enough to break 2e-6 + 1e-5 |o| on columns whose sum is near zero. The
    # kernels' binary64 sums must meet it for dbeta (and for dgamma when t is exact).
    inp = make(M, N, "f32", "f32", alpha=alpha, nonzero=True)
    out, _ = H.run_cuda(inp, M, N, "f32", "f32", fwd=False)
    st = H.compare_all(inp, out, M, N, "f32", "f32")
    assert st["dbeta"]["n_over_strict_elementwise"] == 0
    if np.isinf(alpha):
        assert st["dgamma"]["n_over_strict_elementwise"] == 0


@pytest.mark.parametrize("R,M,N,xd", [(1, 3001, 64, "bf16"), (2, 65537, 32, "bf16"), (3, 10007, 100, "f32"),
                                      (8, 4099, 17, "f32"), (4, 5, 4096, "bf16"), (8, 5, 64, "f16"),
                                      (3, 20000, 255, "f32")])
def test_partials_of_several_ranks_sum_in_one_finalize(R, M, N, xd):
    # R ranks of a row-sharded backward, emulated on one GPU: each rank's stage 1
    # runs on its own rows into its own workspace, then one finalize reads every
    # rank's partials in rank order, as each rank's finalize does through peer
    # pointers. Shards whose rows start off a 16-byte boundary take the
    # one-element kernels; shards with no rows add nothing.
    import elementwise_reduction_b200 as dyt
    from elementwise_reduction_b200.dist import shard_rows
    inp = make(M, N, xd, "f32")
    t = H.gpu_inputs(inp, xd, "f32")
    x, dy = t["x"].view(M, N), t["dy"].view(M, N)
    dx = torch.empty_like(x)
    wss, lays = [], []
    for r in range(R):
        b, e = shard_rows(M, R, r)
        xs, dys, dxs = x[b:e], dy[b:e], dx[b:e]
        ws = dyt.workspace(xs, t["gamma"])
        _, lay = dyt.backward_partials(xs, dys, t["alpha"], t["gamma"], ws, dx=dxs)
        assert lay == dyt.partials_layout(xs, dys, dxs, N)
        wss.append(ws)
        lays.append(lay)
    ptrs = [w.data_ptr() for w in wss]
    da, dg, db = dyt.finalize_partials(ptrs, lays, t["alpha"], t["gamma"], t["beta"])
    torch.cuda.synchronize()
    out = {"dx": H.to_numpy(dx, xd), "dgamma": H.to_numpy(dg, "f32"), "dbeta": H.to_numpy(db, "f32"),
           "dalpha": float(da.item())}
    st = H.compare_all(inp, out, M, N, xd, "f32")
    assert st["dbeta"]["n_over_strict_elementwise"] == 0
    da2, dg2, db2 = dyt.finalize_partials(ptrs, lays, t["alpha"], t["gamma"], t["beta"])  # same bits again
    assert torch.equal(dg, dg2) and torch.equal(db, db2) and torch.equal(da, da2)
    if R == 1:  # one rank: exactly the single-GPU backward
        ref = dyt.backward(x, dy, t["alpha"], t["gamma"], t["beta"])
        for a, b in zip((dx, da, dg, db), ref):
            assert torch.equal(a, b)


def test_finalize_rejects_layouts_outside_their_workspace():
    import elementwise_reduction_b200 as dyt
    M, N = 100, 64
    x = torch.randn(M, N, device="cuda")
    g = torch.ones(N, device="cuda")
    a = torch.tensor([0.5], device="cuda")
    ws = dyt.workspace(x, g)
    _, lay = dyt.backward_partials(x, x, a, g, ws)
    bad = dict(lay, rows=lay["rows"] + 1000)
    with pytest.raises(dyt.DytError) as e:
        dyt.finalize_partials([ws.data_ptr()], [bad], a, g)
    assert e.value.status == 1
    with pytest.raises(dyt.DytError):
        dyt.finalize_partials([ws.data_ptr()] * 9, [lay] * 9, a, g)  # more than 8 ranks


def test_autograd_module_matches_oracle():
    import elementwise_reduction_b200 as dyt
    M, N = 512, 384
    inp = make(M, N, "bf16", "f32", alpha=0.6)
    t = H.gpu_inputs(inp, "bf16", "f32")
    mod = dyt.DyT(N, device="cuda")
    with torch.no_grad():
        mod.alpha.copy_(t["alpha"])
        mod.gamma.copy_(t["gamma"])
        mod.beta.copy_(t["beta"])
    x = t["x"].view(M, N).clone().requires_grad_(True)
    y = mod(x)
    y.backward(t["dy"].view(M, N))
    out = {"y": H.to_numpy(y, "bf16"), "dx": H.to_numpy(x.grad, "bf16"),
           "dgamma": H.to_numpy(mod.gamma.grad, "f32"), "dbeta": H.to_numpy(mod.beta.grad, "f32"),
           "dalpha": float(mod.alpha.grad.item())}
    H.compare_all(inp, out, M, N, "bf16", "f32")


# ---- tanh accuracy over a dense sweep of binary32 inputs -----------------------------------------

def test_tanh_and_sech2_accuracy_sweep():
    import elementwise_reduction_b200 as dyt
    # every 97th positive binary32 pattern from 2^-30 to 64, plus their negatives
    lo, hi = np.float32(2.0 ** -30).view(np.uint32), np.float32(64.0).view(np.uint32)
    bits = np.arange(lo, hi, 97, dtype=np.uint32)
    xs = np.concatenate([bits.view(np.float32), -bits.view(np.float32)])
    n = xs.size
    one = torch.ones(n, device="cuda")
    x = torch.from_numpy(xs).cuda().view(1, n)
    a = torch.tensor([1.0], device="cuda")
    t = dyt.forward(x, a, one, torch.zeros(n, device="cuda")).cpu().numpy().ravel().astype(np.float64)
    dx, _, dg, _ = dyt.backward(x, one.view(1, n), a, one)
    s = dx.cpu().numpy().ravel().astype(np.float64)
    # one row with dy = 1: dgamma[j] is the backward's own t (a binary32 value,
    # exact in its binary64 sum and in the final rounding)
    t_bwd = dg.cpu().numpy().ravel().astype(np.float64)
    X = xs.astype(np.float64)
    rel_t = np.abs(t - np.tanh(X)) / np.abs(np.tanh(X))
    rel_tb = np.abs(t_bwd - np.tanh(X)) / np.abs(np.tanh(X))
    s_ref = 1.0 / np.cosh(X) ** 2
    ok = s_ref > 1e-37  # binary32 normal range
    rel_s = np.abs(s[ok] - s_ref[ok]) / s_ref[ok]
    # The kernel's error model: t within 2^-20.5 relative; 1 - t^2 within 2^-20
    # plus the effect of rounding the exponent argument w = 2|z| log2(e) to
    # binary32, |w| ln2 2^-24 = 2|z| 2^-24.
    print("max rel err t: 2^%.2f" % np.log2(rel_t.max()), " backward t: 2^%.2f" % np.log2(rel_tb.max()),
          " 1-t^2: 2^%.2f" % np.log2(rel_s.max()))
    assert rel_t.max() <= H.T_REL_ERR, rel_t.max()
    # the bound the dgamma tolerance uses: relative, plus an absolute part where
    # |alpha x| < 0.5 (the backward's t takes the exp form for every argument)
    err_tb = np.abs(t_bwd - np.tanh(X))
    assert (err_tb <= H.T_REL_ERR * np.abs(np.tanh(X)) + H.T_ABS_ERR).all(), \
        (err_tb / (H.T_REL_ERR * np.abs(np.tanh(X)) + H.T_ABS_ERR)).max()
    big = np.abs(X) >= 0.5
    assert rel_tb[big].max() <= H.T_REL_ERR, rel_tb[big].max()
    print("backward t: max abs err below 0.5: 2^%.2f" % np.log2(err_tb[~big].max()))
    bound_s = 2.0 ** -20 + 2.0 * np.abs(X[ok]) * 2.0 ** -24
    assert (rel_s <= bound_s).all(), (rel_s / bound_s).max()


# ---- the workloads at full size -----------------------------------------------------------------

@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_workload_full_size(name):
    # Every element of y and dx and every gradient, against the oracle (its
    # elementwise part fanned out over row blocks on the host cores).
    w = workloads.WORKLOADS[name]
    inp = workloads.make_inputs(w)
    out, info = H.run_cuda(inp, w.M, w.N, w.x_dtype, w.p_dtype)
    stats = H.compare_all(inp, out, w.M, w.N, w.x_dtype, w.p_dtype)
    print(name, info, stats)
    assert stats["dbeta"]["n_over_strict_elementwise"] == 0
    if H.t_is_exact(w.alpha) and w.x_dtype == "f32":  # binary64 dgamma terms, each exact
        assert stats["dgamma"]["n_over_strict_elementwise"] == 0
    if w.N <= 256:
        assert info["bwd"]["path"] == 1


@pytest.mark.parametrize("name", list(workloads.VARIANTS))
def test_unaligned_variant_full_size(name):
    # The workload's values with tensors off 16-byte boundaries (the shifted
    # kernels) or rows that are not whole 16-byte vectors (the one-element
    # kernels), checked on every element.
    w = workloads.VARIANTS[name]
    inp = workloads.make_inputs(w)
    out, info = H.run_cuda(inp, w.M, w.N, w.x_dtype, w.p_dtype, offset=w.offset, x_offset=w.x_offset,
                           pitch=w.pitch)
    if w.pitch and (w.pitch * (4 if w.x_dtype == "f32" else 2)) % 16:
        # pitches off whole vectors: phases of whole-vector pitch
        k = _phases(w.M, w.N, (w.pitch,), 4 if w.x_dtype == "f32" else 2)
        k_b = _phases(w.M, w.N, (w.pitch,), 4 if w.x_dtype == "f32" else 2, backward=True)
        assert k > 1 and info["fwd"]["vec"] == (4 if w.x_dtype == "f32" else 8)
        assert info["bwd"]["vec"] == ((4 if w.x_dtype == "f32" else 8) if k_b > 1 else 1)
        assert info["fwd"]["kernels"] == k and info["bwd"]["kernels"] == k_b + 1
    elif w.pitch:  # whole-vector pitches: the row frame (3: with the wrapped first vector-column)
        wrapped = w.offset and w.x_off == w.offset and w.N % (4 if w.x_dtype == "f32" else 8) == 0
        assert info["fwd"]["shifted"] == info["bwd"]["shifted"] == (3 if wrapped else 2)
        assert info["fwd"]["shift"] == info["bwd"]["shift"] == w.offset
    else:
        assert info["fwd"]["shifted"] == 1 and info["bwd"]["shifted"] == 1
        assert info["fwd"]["shift"] == info["bwd"]["shift"] == w.offset
    stats = H.compare_all(inp, out, w.M, w.N, w.x_dtype, w.p_dtype)
    print(name, info, stats)
    assert stats["dbeta"]["n_over_strict_elementwise"] == 0
