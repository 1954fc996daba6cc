"""Shared test helpers: storage <-> torch, running the CUDA path, comparing with the oracle.

Tolerances (stated once, used by every parity test):
  binary32 y, dx     |g - o| <= 2e-6 + 1e-5 |o|, o the binary64 oracle value.
  16-bit y, dx       at most one unit in the last place from the oracle's value
                     rounded once (ties to even) to the 16-bit format.
  dgamma, dbeta      |g - o| <= 2e-6 + 1e-5 S_j, S_j the magnitude of the column
                     sum (sum of |term|); 16-bit parameters also pass within one
                     unit of the rounded oracle value.
  dalpha             |g - o| <= 1e-5 S, S = sum of |term| (exact when S = 0).
  Everywhere         NaN positions identical; infinities identical with sign.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle

TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}
CODE = {"f32": 0, "bf16": 1, "f16": 2}
ABS_TOL, REL_TOL = 2e-6, 1e-5


# ---- storage conversions ------------------------------------------------------------------

def to_torch(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(a))
    return t.to(device) if device != "cpu" else t


def to_numpy(t: torch.Tensor, dtype: str) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if dtype == "bf16":
        return t.view(torch.int16).numpy().view(np.uint16).ravel()
    return t.numpy().ravel()


def decode(a: np.ndarray, dtype: str) -> np.ndarray:
    return oracle.decode(a, dtype)


# ---- comparisons ---------------------------------------------------------------------------

def ordered16(bits: np.ndarray) -> np.ndarray:
    """16-bit float bit patterns as integers ordered like the values (+0 == -0)."""
    b = bits.astype(np.int64)
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bits16(a: np.ndarray) -> np.ndarray:
    return a.view(np.uint16) if a.dtype != np.uint16 else a


class Mismatch(AssertionError):
    pass


def check_special(g64: np.ndarray, o64: np.ndarray, what: str) -> None:
    gn, on = np.isnan(g64), np.isnan(o64)
    if not np.array_equal(gn, on):
        idx = np.flatnonzero(gn != on)[:5]
        raise Mismatch(f"{what}: NaN positions differ at {idx.tolist()} (gpu {g64[idx]}, oracle {o64[idx]})")
    gi, oi = np.isinf(g64), np.isinf(o64)
    if not (np.array_equal(gi, oi) and np.array_equal(np.sign(g64[gi]), np.sign(o64[oi]))):
        idx = np.flatnonzero(gi != oi)[:5]
        raise Mismatch(f"{what}: infinities differ at {idx.tolist()}")


def check_elementwise(got: np.ndarray, o64: np.ndarray, dtype: str, what: str) -> dict:
    """GPU storage values vs binary64 oracle values, elementwise."""
    g64 = decode(got, dtype)
    check_special(g64, o64, what)
    fin = np.isfinite(o64)
    if dtype == "f32":
        err = np.abs(g64[fin] - o64[fin])
        tol = ABS_TOL + REL_TOL * np.abs(o64[fin])
        bad = err > tol
        if bad.any():
            i = np.flatnonzero(fin)[np.flatnonzero(bad)[:5]]
            raise Mismatch(f"{what}: {bad.sum()} elements out of tolerance, e.g. idx {i.tolist()} gpu "
                           f"{g64[i]} oracle {o64[i]}")
        return {"max_abs_err": float(err.max(initial=0.0)),
                "max_rel_err": float((err / np.maximum(np.abs(o64[fin]), 1e-300)).max(initial=0.0))}
    want = bits16(oracle.round_to(o64, dtype))
    d = np.abs(ordered16(bits16(got))[fin] - ordered16(want)[fin])
    if (d > 1).any():
        i = np.flatnonzero(fin)[np.flatnonzero(d > 1)[:5]]
        raise Mismatch(f"{what}: {(d > 1).sum()} elements more than 1 ulp from the correctly rounded "
                       f"oracle value, e.g. idx {i.tolist()} gpu {g64[i]} oracle {o64[i]}")
    return {"max_ulp": int(d.max(initial=0)), "frac_exact": float((d == 0).mean()) if d.size else 1.0}


def check_sums(got: np.ndarray, o64: np.ndarray, mag: np.ndarray, dtype: str, what: str) -> dict:
    """Reduced outputs (column sums) against the oracle with a sum-magnitude tolerance."""
    g64 = decode(got, dtype)
    check_special(g64, o64, what)
    fin = np.isfinite(o64)
    err = np.abs(g64[fin] - o64[fin])
    ok = err <= ABS_TOL + REL_TOL * mag[fin]
    if dtype != "f32":
        want = bits16(oracle.round_to(o64, dtype))
        ok |= np.abs(ordered16(bits16(got))[fin] - ordered16(want)[fin]) <= 1
    if not ok.all():
        i = np.flatnonzero(fin)[np.flatnonzero(~ok)[:5]]
        raise Mismatch(f"{what}: {(~ok).sum()} sums out of tolerance, e.g. idx {i.tolist()} gpu {g64[i]} "
                       f"oracle {o64[i]} magnitude {mag[i]}")
    strict = err > ABS_TOL + REL_TOL * np.abs(o64[fin])
    return {"max_err_over_mag": float((err / np.maximum(mag[fin], 1e-300)).max(initial=0.0)),
            "n_over_strict_elementwise": int(strict.sum())}


def check_scalar_sum(got: float, o: float, mag: float, what: str, dtype: str = "f32") -> dict:
    if np.isnan(o) or np.isnan(got):
        if not (np.isnan(o) and np.isnan(got)):
            raise Mismatch(f"{what}: gpu {got} oracle {o}")
        return {}
    if np.isinf(o) or np.isinf(got):
        if got != o:
            raise Mismatch(f"{what}: gpu {got} oracle {o}")
        return {}
    err = abs(got - o)
    if dtype != "f32":
        want = bits16(oracle.round_to(np.array([o]), dtype))
        gotb = bits16(oracle.round_to(np.array([got]), dtype))  # got is already on the 16-bit grid
        if abs(int(ordered16(gotb)[0]) - int(ordered16(want)[0])) <= 1:
            return {"err_over_mag": err / mag if mag else 0.0}
    if not err <= REL_TOL * mag:
        raise Mismatch(f"{what}: gpu {got!r} oracle {o!r} |err| {err:.3g} > 1e-5 * magnitude {mag:.6g}")
    return {"err_over_mag": err / mag if mag else 0.0}


# ---- running the CUDA path -------------------------------------------------------------------

def gpu_inputs(inp: dict, x_dtype: str, p_dtype: str) -> dict:
    d = {k: to_torch(inp[k], x_dtype) for k in ("x", "dy")}
    d.update({k: to_torch(inp[k], p_dtype) for k in ("alpha", "gamma", "beta")})
    return d


def run_cuda(inp: dict, M: int, N: int, x_dtype: str, p_dtype: str, fwd: bool = True, bwd: bool = True):
    """Run the C-ABI forward and backward on the device; outputs back as numpy storage."""
    import elementwise_reduction_b200 as dyt

    t = gpu_inputs(inp, x_dtype, p_dtype)
    x = t["x"].view(M, N) if M * N else t["x"]
    out, info = {}, {}
    if fwd:
        y = dyt.forward(x, t["alpha"], t["gamma"], t["beta"])
        info["fwd"] = dyt.dyt_last_launch_info()
        out["y"] = to_numpy(y, x_dtype)
    if bwd:
        dy = t["dy"].view(M, N) if M * N else t["dy"]
        dx, da, dg, db = dyt.backward(x, dy, t["alpha"], t["gamma"])
        info["bwd"] = dyt.dyt_last_launch_info()
        out.update(dx=to_numpy(dx, x_dtype), dgamma=to_numpy(dg, p_dtype), dbeta=to_numpy(db, p_dtype),
                   dalpha=float(decode(to_numpy(da, p_dtype), p_dtype)[0]))
    torch.cuda.synchronize()
    assert dyt.dyt_device_error() == 0, "a pipelined kernel reported a wait that gave up"
    return out, info


def compare_all(inp: dict, out: dict, M: int, N: int, x_dtype: str, p_dtype: str, rows=None) -> dict:
    """Compare every output with the oracle. rows: sampled row indices for y/dx (None = all)."""
    stats = {}
    if rows is None:
        xs, dys, Ms = inp["x"], inp["dy"], M
    else:
        rows = np.asarray(rows)
        xs = inp["x"].reshape(M, N)[rows].ravel()
        dys = inp["dy"].reshape(M, N)[rows].ravel()
        Ms = len(rows)

    def sel(a):
        return a if rows is None else a.reshape(M, N)[rows].ravel()

    if "y" in out:
        y64 = oracle.forward(xs, inp["alpha"], inp["gamma"], inp["beta"], Ms, N, x_dtype, p_dtype)
        stats["y"] = check_elementwise(sel(out["y"]), y64, x_dtype, "y")
    if "dx" in out:
        if rows is None:
            r = oracle.backward(inp["x"], inp["dy"], inp["alpha"], inp["gamma"], M, N, x_dtype, p_dtype)
            dx64 = r["dx"]
        else:
            r = oracle.backward(inp["x"], inp["dy"], inp["alpha"], inp["gamma"], M, N, x_dtype, p_dtype,
                                want_dx=False)
            dx64 = oracle.backward(xs, dys, inp["alpha"], inp["gamma"], Ms, N, x_dtype, p_dtype)["dx"]
        stats["dx"] = check_elementwise(sel(out["dx"]), dx64, x_dtype, "dx")
        stats["dgamma"] = check_sums(out["dgamma"], r["dgamma"], r["mag_dgamma"], p_dtype, "dgamma")
        stats["dbeta"] = check_sums(out["dbeta"], r["dbeta"], r["mag_dbeta"], p_dtype, "dbeta")
        stats["dalpha"] = check_scalar_sum(out["dalpha"], r["dalpha"], r["mag_dalpha"], "dalpha", p_dtype)
    return stats
