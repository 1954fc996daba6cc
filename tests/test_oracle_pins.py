"""Pins of the CPU oracle to things other than itself.

Each check comes from the mathematics of the DyT layer (closed forms, symmetries,
exact rational sums, finite differences), from an independent high-precision
tanh (Python's decimal module), from an independent autodiff (torch, binary64),
or from the facts the Liger-Kernel page states ("fix(dyt): use a 1D grid and
tile small-width rows", Summary). No expected value comes from the CUDA path.
"""
from __future__ import annotations

import decimal
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _inputs(M, N, x_dtype="f32", p_dtype="f32", alpha=0.7, x_std=1.0, seed=11, nonzero=False,
            gamma_std=0.3, beta_std=0.3):
    x = synth.normal(M * N, x_dtype, 0.0, x_std, seed, 1, nonzero=nonzero)
    dy = synth.normal(M * N, x_dtype, 0.0, 1.0, seed, 2, nonzero=nonzero)
    g = synth.normal(N, p_dtype, 1.0, gamma_std, seed, 3)
    b = synth.normal(N, p_dtype, 0.0, beta_std, seed, 4)
    a = np.array([alpha], dtype=oracle.NP_STORAGE[p_dtype])
    return x, dy, a, g, b


def _dec_tanh(v: float) -> decimal.Decimal:
    """tanh at 60 significant digits: odd Taylor series near 0, else exp."""
    with decimal.localcontext() as ctx:
        ctx.prec = 60
        z = decimal.Decimal(v)
        if abs(z) < decimal.Decimal("1e-6"):
            z2 = z * z
            # tanh z = z - z^3/3 + 2 z^5/15 - 17 z^7/315 + O(z^9)
            return z * (1 - z2 / 3 + 2 * z2 * z2 / 15 - 17 * z2 * z2 * z2 / 315)
        if abs(z) > 200:
            return decimal.Decimal(1).copy_sign(z)
        e = (2 * z).exp()
        return (e - 1) / (e + 1)


def test_forward_tanh_matches_decimal():
    xs = [0.0, -0.0, 1e-300, -3e-200, 1e-9, 2.5e-7, 0.001, -0.125, 0.5, 0.54930614433405, 1.0, -2.0,
          3.7, 9.5, -18.0, 19.5, 25.0, 40.0, 700.0, 1e308, -1e308]
    rng = np.random.default_rng(0)
    xs += list(rng.normal(0, 3, 400)) + list(10.0 ** rng.uniform(-12, 2.5, 300))
    x = np.array(xs, dtype=np.float64)
    y = oracle.forward(x, np.array([1.0]), np.ones(x.size), np.full(x.size, -0.0), 1, x.size,
                       "f64", "f64")  # beta = -0 keeps the sign of a zero t
    for xv, yv in zip(x, y):
        want = _dec_tanh(float(xv))
        if want == 0:
            assert yv == 0.0 and math.copysign(1, yv) == math.copysign(1, xv)
            continue
        rel = abs((decimal.Decimal(float(yv)) - want) / want)
        assert rel <= decimal.Decimal(2) ** -51, (xv, yv, want)


def test_alpha_zero_closed_forms():
    M, N = 37, 23
    x, dy, _, g, b = _inputs(M, N)
    a = np.array([0.0], dtype=np.float32)
    y = oracle.forward(x, a, g, b, M, N, "f32", "f32").reshape(M, N)
    assert np.array_equal(y, np.broadcast_to(b.astype(np.float64), (M, N)))
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    assert np.all(r["dx"] == 0.0)
    assert np.all(r["dgamma"] == 0.0)
    X, DY, G = x.astype(np.float64).reshape(M, N), dy.astype(np.float64).reshape(M, N), g.astype(np.float64)
    for j in range(N):
        exact = sum(Fraction(v) for v in DY[:, j])
        assert abs(Fraction(r["dbeta"][j]) - exact) <= Fraction(2.0 ** -50) * r["mag_dbeta"][j]
    # dalpha at alpha = 0 is sum gamma*dy*x, computed here in exact rationals
    exact = sum(Fraction(G[j]) * Fraction(DY[i, j]) * Fraction(X[i, j]) for i in range(M) for j in range(N))
    assert abs(Fraction(r["dalpha"]) - exact) <= Fraction(2.0 ** -48) * Fraction(r["mag_dalpha"])


def test_dbeta_is_exact_column_sum_of_integer_dy():
    M, N = 300, 7
    x, _, a, g, _ = _inputs(M, N)
    dy = np.round(synth.normal(M * N, "f32", 0.0, 40.0, 5, 2)).astype(np.float32)
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    want = dy.astype(np.int64).reshape(M, N).sum(axis=0)
    assert np.array_equal(r["dbeta"], want.astype(np.float64))


def test_alpha_inf_closed_forms_and_page_nan_case():
    M, N = 31, 19
    x, dy, _, g, b = _inputs(M, N, nonzero=True)
    a = np.array([np.inf], dtype=np.float32)
    X, DY = x.astype(np.float64).reshape(M, N), dy.astype(np.float64).reshape(M, N)
    G, B = g.astype(np.float64), b.astype(np.float64)
    y = oracle.forward(x, a, g, b, M, N, "f32", "f32").reshape(M, N)
    want = np.sign(X) * G + B  # tanh(+-inf) = +-1: one binary64 rounding, as in the oracle
    assert np.array_equal(y, want)
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    assert r["dalpha"] == 0.0 and r["mag_dalpha"] == 0.0  # every term carries 1 - t^2 = 0
    assert np.all(np.isnan(r["dx"]))                     # inf * 0 in every element
    for j in range(N):
        exact = sum(Fraction(DY[i, j]) * int(np.sign(X[i, j])) for i in range(M))
        assert abs(Fraction(r["dgamma"][j]) - exact) <= Fraction(2.0 ** -50) * r["mag_dgamma"][j]
    assert np.all(np.isfinite(r["dgamma"])) and np.all(np.isfinite(r["dbeta"]))
    # The page's padding failure: one x = 0 with infinite alpha gives tanh(inf * 0) = NaN,
    # which poisons that column's dgamma and y.
    facts = json.load(open(os.path.join(GOLDEN, "liger_dyt_page_facts.json")))
    assert facts["nan_case"]["expression"] == "tanh(inf * 0)"
    x0 = x.copy()
    x0[5 * N + 3] = 0.0
    y0 = oracle.forward(x0, a, g, b, M, N, "f32", "f32").reshape(M, N)
    assert np.isnan(y0[5, 3]) and np.isfinite(np.delete(y0.ravel(), 5 * N + 3)).all()
    r0 = oracle.backward(x0, dy, a, g, M, N, "f32", "f32")
    assert np.isnan(r0["dgamma"][3]) and np.isfinite(np.delete(r0["dgamma"], 3)).all()


def test_odd_and_even_symmetry_with_zero_beta():
    M, N = 17, 29
    x, dy, a, g, _ = _inputs(M, N, alpha=1.3)
    b = np.zeros(N, dtype=np.float32)
    y = oracle.forward(x, a, g, b, M, N, "f32", "f32")
    yn = oracle.forward(-x, a, g, b, M, N, "f32", "f32")
    assert np.array_equal(yn, -y)
    r, rn = oracle.backward(x, dy, a, g, M, N, "f32", "f32"), oracle.backward(-x, dy, a, g, M, N, "f32", "f32")
    assert np.array_equal(rn["dx"], r["dx"])
    assert np.array_equal(rn["dgamma"], -r["dgamma"])
    assert rn["dalpha"] == -r["dalpha"]
    assert np.array_equal(rn["dbeta"], r["dbeta"])


def test_output_bound_and_linearity_in_dy():
    M, N = 20, 33
    x, dy, _, g, b = _inputs(M, N, x_std=4.0)
    for alpha in (0.01, 1.0, 50.0):
        a = np.array([alpha], dtype=np.float32)
        y = oracle.forward(x, a, g, b, M, N, "f32", "f32").reshape(M, N)
        assert np.all(np.abs(y - b.astype(np.float64)) <= np.abs(g.astype(np.float64)))
    a = np.array([0.9], dtype=np.float32)
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    r2 = oracle.backward(x, (2 * dy).astype(np.float32), a, g, M, N, "f32", "f32")
    for k in ("dx", "dgamma", "dbeta"):
        assert np.array_equal(r2[k], 2 * r[k])
    assert r2["dalpha"] == 2 * r["dalpha"]


def test_row_split_additivity():
    M, N, k = 41, 13, 17
    x, dy, a, g, _ = _inputs(M, N)
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    top = oracle.backward(x[:k * N], dy[:k * N], a, g, k, N, "f32", "f32")
    bot = oracle.backward(x[k * N:], dy[k * N:], a, g, M - k, N, "f32", "f32")
    assert np.array_equal(np.concatenate([top["dx"], bot["dx"]]), r["dx"])
    for key in ("dgamma", "dbeta"):
        assert np.all(np.abs(top[key] + bot[key] - r[key]) <= 1e-14 * r["mag_" + key])
    assert abs(top["dalpha"] + bot["dalpha"] - r["dalpha"]) <= 1e-14 * r["mag_dalpha"]


def _loss(x, dy, a, g, b, M, N):
    """L = sum dy * y in binary64 (the loss whose gradients the backward returns)."""
    return float(np.sum(dy * oracle.forward(x, a, g, b, M, N, "f64", "f64")))


def test_central_finite_differences():
    M, N = 4, 5
    x = synth.normal(M * N, "f64", 0.0, 1.5, 3, 1)
    dy = synth.normal(M * N, "f64", 0.0, 1.0, 3, 2)
    g = synth.normal(N, "f64", 1.0, 0.3, 3, 3)
    b = synth.normal(N, "f64", 0.0, 0.3, 3, 4)
    a = np.array([0.8])
    r = oracle.backward(x, dy, a, g, M, N, "f64", "f64")

    def fd(which, idx):
        base = {"x": x, "g": g, "b": b, "a": a}[which]
        h = 1e-6 * max(1.0, abs(base[idx]))
        vals = []
        for s in (+1, -1):
            p = base.copy()
            p[idx] += s * h
            args = {"x": x, "g": g, "b": b, "a": a}
            args[which] = p
            vals.append(_loss(args["x"], dy, args["a"], args["g"], args["b"], M, N))
        return (vals[0] - vals[1]) / (2 * h)

    for k in range(M * N):
        assert abs(fd("x", k) - r["dx"][k]) <= 1e-7 * (1 + abs(r["dx"][k]))
    for j in range(N):
        assert abs(fd("g", j) - r["dgamma"][j]) <= 1e-7 * (1 + abs(r["dgamma"][j]))
        assert abs(fd("b", j) - r["dbeta"][j]) <= 1e-7 * (1 + abs(r["dbeta"][j]))
    assert abs(fd("a", 0) - r["dalpha"]) <= 1e-7 * (1 + abs(r["dalpha"]))


@pytest.mark.parametrize("M,N,alpha", [(1, 1, 0.3), (1, 3, 2.0), (3, 1, -0.7), (9, 14, 0.45)])
def test_matches_torch_autograd_binary64(M, N, alpha):
    x = synth.normal(M * N, "f64", 0.0, 1.7, 9, 1)
    dy = synth.normal(M * N, "f64", 0.0, 1.0, 9, 2)
    g = synth.normal(N, "f64", 1.0, 0.4, 9, 3)
    b = synth.normal(N, "f64", 0.0, 0.4, 9, 4)
    a = np.array([alpha])
    tx = torch.tensor(x.reshape(M, N), requires_grad=True)
    tg, tb = torch.tensor(g, requires_grad=True), torch.tensor(b, requires_grad=True)
    ta = torch.tensor(alpha, dtype=torch.float64, requires_grad=True)
    ty = tg * torch.tanh(ta * tx) + tb
    (ty * torch.tensor(dy.reshape(M, N))).sum().backward()
    y = oracle.forward(x, a, g, b, M, N, "f64", "f64")
    r = oracle.backward(x, dy, a, g, M, N, "f64", "f64")
    np.testing.assert_allclose(y, ty.detach().numpy().ravel(), rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(r["dx"], tx.grad.numpy().ravel(), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(r["dgamma"], tg.grad.numpy(), rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(r["dbeta"], tb.grad.numpy(), rtol=1e-14, atol=1e-15)
    assert abs(r["dalpha"] - ta.grad.item()) <= 1e-13 * (1 + r["mag_dalpha"])


def test_one_minus_tanh_sq_identity_in_moderate_range():
    # Where 1 - t^2 does not cancel, the oracle's factor equals it (dx = alpha*gamma*dy*(1-t^2)).
    M, N = 1, 200
    x = np.linspace(-6, 6, N)
    dy, g = np.ones(N), np.ones(N)
    r = oracle.backward(x, dy, np.array([1.0]), g, M, N, "f64", "f64")
    t = np.tanh(x)
    np.testing.assert_allclose(r["dx"], 1 - t * t, rtol=1e-9)
    # and it keeps its digits where 1 - t*t has none left
    r = oracle.backward(np.array([30.0]), np.array([1.0]), np.array([1.0]), np.array([1.0]), 1, 1, "f64", "f64")
    assert r["dx"][0] > 0 and abs(r["dx"][0] / (4 * math.exp(-60)) - 1) < 1e-12


def test_empty_shapes():
    e = np.zeros(0, dtype=np.float32)
    a, g = np.array([0.5], dtype=np.float32), np.ones(3, dtype=np.float32)
    assert oracle.forward(e, a, g, g, 0, 3, "f32", "f32").size == 0
    r = oracle.backward(e, e, a, g, 0, 3, "f32", "f32")
    assert np.all(r["dgamma"] == 0) and np.all(r["dbeta"] == 0) and r["dalpha"] == 0.0
    r = oracle.backward(e, e, a, np.zeros(0, np.float32), 5, 0, "f32", "f32")
    assert r["dgamma"].size == 0 and r["dalpha"] == 0.0


# ---- rounding binary64 -> storage dtype --------------------------------------------------


def _grid(dtype):
    """All finite non-negative values of a 16-bit format, ascending, as binary64."""
    bits = np.arange(0, 0x7C00 if dtype == "f16" else 0x7F80, dtype=np.uint16)
    return oracle.decode(bits if dtype == "bf16" else bits.view(np.float16), dtype), bits


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
def test_rounding_is_nearest_ties_to_even_exhaustive(dtype):
    v, bits = _grid(dtype)
    lo, hi = v[:-1], v[1:]
    mid = (lo + hi) / 2  # exact in binary64
    even = np.where(bits[:-1] % 2 == 0, bits[:-1], bits[1:])

    def enc(a):
        r = oracle.round_to(a, dtype)
        return r if dtype == "bf16" else r.view(np.uint16)

    assert np.array_equal(enc(mid), even)
    assert np.array_equal(enc(-mid), even | 0x8000)
    assert np.array_equal(enc(mid - (hi - lo) * 2.0 ** -20), bits[:-1])
    assert np.array_equal(enc(mid + (hi - lo) * 2.0 ** -20), bits[1:])
    assert np.array_equal(enc(v), bits)
    # the largest finite value plus half an ulp overflows (ties to even reaches 2^emax+1)
    top, ulp = v[-1], v[-1] - v[-2]
    assert np.isinf(oracle.round_scalar(top + ulp / 2, dtype))
    assert oracle.round_scalar(top + ulp / 2 * (1 - 2.0 ** -30), dtype) == top
    assert enc(np.array([np.nan]))[0] & 0x7FFF > (0x7F80 if dtype == "bf16" else 0x7C00)
    assert enc(np.array([-np.inf]))[0] == (0xFF80 if dtype == "bf16" else 0xFC00)
    assert enc(np.array([-0.0]))[0] == 0x8000


def test_rounding_matches_library_converters():
    rng = np.random.default_rng(1)
    v = rng.normal(0, 1, 200000) * 10.0 ** rng.uniform(-9, 6, 200000)
    assert np.array_equal(oracle.round_to(v, "f32"), v.astype(np.float32))
    # numpy converts binary64 to binary16 directly with ties to even
    assert np.array_equal(oracle.round_to(v, "f16").view(np.uint16), v.astype(np.float16).view(np.uint16))


def test_decode_matches_library_converters():
    bits = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    d = oracle.decode(bits, "bf16")
    assert np.array_equal(np.isnan(d), np.isnan(t))
    ok = ~np.isnan(t)
    assert np.array_equal(d[ok], t[ok])
    h = bits.view(np.float16)
    d = oracle.decode(h, "f16")
    ok = ~np.isnan(h)
    assert np.array_equal(d[ok], h[ok].astype(np.float64))


# ---- the sum magnitudes that scale the gradient tolerances ---------------------------------------
#
# The oracle also returns S = sum |term| for each gradient sum (dgamma's terms dy t,
# dbeta's dy, dalpha's gamma dy (1 - t^2) x). These set the tolerance of every sum
# comparison, so they are pinned here by an independent computation: numpy's tanh
# and cosh, and math.fsum (a correctly rounded sum), on the same decoded inputs.


def _magnitudes_by_fsum(x, dy, alpha, g, M, N):
    X, DY = x.astype(np.float64).reshape(M, N), dy.astype(np.float64).reshape(M, N)
    G = g.astype(np.float64)
    z = float(alpha) * X
    t = np.tanh(z)
    sech2 = 1.0 / np.cosh(z) ** 2
    mg = np.array([math.fsum(np.abs(DY[:, j] * t[:, j])) for j in range(N)])
    mb = np.array([math.fsum(np.abs(DY[:, j])) for j in range(N)])
    ma = math.fsum(np.abs(G[None, :] * DY * sech2 * X).ravel())
    return mg, mb, ma


@pytest.mark.parametrize("M,N,alpha,seed", [(23, 11, 0.7, 1), (64, 5, 2.5, 2), (7, 40, 0.05, 3)])
def test_sum_magnitudes_match_an_independent_fsum(M, N, alpha, seed):
    x, dy, a, g, _ = _inputs(M, N, alpha=alpha, seed=seed)
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    mg, mb, ma = _magnitudes_by_fsum(x, dy, a[0], g, M, N)
    # index-order binary64 sums of at most 64 * 40 terms: within 1e-12 relative
    np.testing.assert_allclose(r["mag_dgamma"], mg, rtol=1e-12, atol=0)
    np.testing.assert_allclose(r["mag_dbeta"], mb, rtol=1e-12, atol=0)
    assert abs(r["mag_dalpha"] - ma) <= 1e-12 * ma
    # the triangle inequality: a magnitude never falls below its sum's absolute value
    assert np.all(r["mag_dgamma"] >= np.abs(r["dgamma"]))
    assert np.all(r["mag_dbeta"] >= np.abs(r["dbeta"]))
    assert r["mag_dalpha"] >= abs(r["dalpha"])
    # and with terms of both signs it lies strictly above it
    assert np.all(r["mag_dbeta"] > np.abs(r["dbeta"]))


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_sum_magnitudes_equal_the_sums_when_all_terms_share_a_sign(sign):
    # x > 0, dy of one sign, gamma > 0, alpha > 0: every term of each sum has the
    # sign of dy, so sum |term| and |sum term| add the same values in the same order.
    M, N = 50, 9
    x = np.abs(synth.normal(M * N, "f32", 0.0, 1.0, 21, 1, nonzero=True))
    dy = (sign * np.abs(synth.normal(M * N, "f32", 0.0, 1.0, 21, 2, nonzero=True))).astype(np.float32)
    g = np.abs(synth.normal(N, "f32", 1.0, 0.1, 21, 3)).astype(np.float32)
    a = np.array([0.9], dtype=np.float32)
    r = oracle.backward(x, dy, a, g, M, N, "f32", "f32")
    assert np.array_equal(r["mag_dgamma"], np.abs(r["dgamma"]))
    assert np.array_equal(r["mag_dbeta"], np.abs(r["dbeta"]))
    assert r["mag_dalpha"] == abs(r["dalpha"])
    assert np.all(np.sign(r["dbeta"]) == sign)


def test_each_parameter_is_decoded_in_its_own_dtype():
    # alpha in bf16, gamma in fp16, beta in fp32: the oracle must give the same
    # values as with every parameter held exactly in binary64 (decoding is exact).
    M, N = 13, 21
    x, dy, _, _, _ = _inputs(M, N)
    a16 = oracle.round_to(np.array([0.8125]), "bf16")
    g16 = oracle.round_to(synth.normal(N, "f64", 1.0, 0.3, 31, 3), "f16")
    b32 = synth.normal(N, "f32", 0.0, 0.3, 31, 4)
    mixed = ("bf16", "f16", "f32")
    a64, g64, b64 = oracle.decode(a16, "bf16"), oracle.decode(g16, "f16"), b32.astype(np.float64)
    y = oracle.forward(x, a16, g16, b32, M, N, "f32", mixed)
    assert np.array_equal(y, oracle.forward(x, a64, g64, b64, M, N, "f32", "f64"))
    r = oracle.backward(x, dy, a16, g16, M, N, "f32", mixed)
    r64 = oracle.backward(x, dy, a64, g64, M, N, "f32", "f64")
    for k in ("dx", "dgamma", "dbeta", "mag_dgamma", "mag_dbeta"):
        assert np.array_equal(r[k], r64[k]), k
    assert r["dalpha"] == r64["dalpha"] and r["mag_dalpha"] == r64["mag_dalpha"]
