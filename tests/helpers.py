"""Shared test helpers: storage <-> torch, running the CUDA path, comparing with the oracle.

Tolerances (stated once, used by every parity test):
  binary32 y, dx     |g - o| <= 2e-6 + 1e-5 |o|, o the binary64 oracle value.
  16-bit y, dx       at most one unit in the last place from the oracle's value
                     rounded once (ties to even) to the 16-bit format.
  dbeta              |g - o| <= 2e-6 + 1e-5 |o| + n 2^-53 S, elementwise (S the sum
                     of |term| of the column, n the number of terms: the binary64
                     summation's own rounding, far below the other terms).
  dgamma             the same, plus eps_t S + abs_t S_beta when t is not exact: the
                     backward's binary32 t is within eps_t |t| + abs_t of tanh
                     (eps_t = 2^-20.5, abs_t = 2^-21; checked by a sweep test), so
                     |sum dy (t_gpu - t)| <= eps_t sum |dy t| + abs_t sum |dy|. With
                     alpha = 0 or +-inf every t is exact (0 or +-1) and the bound
                     is the stated one. Over 16-bit activations the kernels add dgamma in
                     binary32 runs of at most 126 rows (then binary64), which adds
                     126 2^-24 S: in all at most 8.2e-6 S, within the 1e-5 S that
                     the sum-magnitude reading allows.
                     16-bit parameter gradients also pass within one unit of the
                     correctly rounded oracle value.
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


T_REL_ERR = 2.0 ** -20.5  # relative error bound of the kernels' binary32 tanh (checked by a sweep test)
T_ABS_ERR = 2.0 ** -21   # absolute error bound of the backward's t (below |alpha x| = 0.5)
GAMMA_RUN_ERR = 126 * 2.0 ** -24  # binary32 dgamma runs of the 16-bit kernels: at most 126 roundings


def t_is_exact(alpha: float) -> bool:
    """alpha = 0 or +-inf: every t = tanh(alpha x) is exactly 0 or +-1 (or NaN)."""
    return alpha == 0.0 or np.isinf(alpha)


def check_sums(got: np.ndarray, o64: np.ndarray, mag: np.ndarray, dtype: str, what: str, n_terms: int,
               t_err: float = 0.0, extra: np.ndarray | None = None) -> dict:
    """Column sums against the oracle: |g - o| <= 2e-6 + 1e-5 |o| + (n 2^-53 + t_err) S + extra."""
    g64 = decode(got, dtype)
    check_special(g64, o64, what)
    fin = np.isfinite(o64)
    err = np.abs(g64[fin] - o64[fin])
    strict = ABS_TOL + REL_TOL * np.abs(o64[fin])
    ok = err <= strict + (n_terms * 2.0 ** -53 + t_err) * mag[fin] + (0.0 if extra is None else extra[fin])
    if dtype != "f32":
        want = bits16(oracle.round_to(o64, dtype))
        ok |= np.abs(ordered16(bits16(got))[fin] - ordered16(want)[fin]) <= 1
    if not ok.all():
        i = np.flatnonzero(fin)[np.flatnonzero(~ok)[:5]]
        raise Mismatch(f"{what}: {(~ok).sum()} sums out of tolerance, e.g. idx {i.tolist()} gpu {g64[i]} "
                       f"oracle {o64[i]} magnitude {mag[i]}")
    return {"max_err_over_mag": float((err / np.maximum(mag[fin], 1e-300)).max(initial=0.0)),
            "n_over_strict_elementwise": int((err > strict).sum())}


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

def param_dtypes(p_dtype) -> tuple:
    """(alpha, gamma, beta) dtypes from one dtype name or a 3-tuple of them."""
    return (p_dtype,) * 3 if isinstance(p_dtype, str) else tuple(p_dtype)


def gpu_inputs(inp: dict, x_dtype: str, p_dtype) -> dict:
    d = {k: to_torch(inp[k], x_dtype) for k in ("x", "dy")}
    d.update({k: to_torch(inp[k], dt) for k, dt in zip(("alpha", "gamma", "beta"), param_dtypes(p_dtype))})
    return d


def _at_offset(t: torch.Tensor, M: int, N: int, offset: int, pitch: int | None = None) -> torch.Tensor:
    """An M x N copy of t whose first element lies `offset` elements past a 16-byte
    boundary, rows `pitch` elements apart (default N)."""
    ld = pitch or N
    buf = torch.empty(M * ld + offset + 8, dtype=t.dtype, device=t.device)
    m = buf[offset:offset + M * ld].view(M, ld)[:, :N]
    m.copy_(t.reshape(M, N))
    return m


def run_cuda(inp: dict, M: int, N: int, x_dtype: str, p_dtype, fwd: bool = True, bwd: bool = True,
             offset: int = 0, x_offset: int | None = None, pitch: int | None = None):
    """Run the C-ABI forward and backward on the device; outputs back as numpy storage.
    p_dtype: one dtype name for alpha, gamma and beta, or a tuple (alpha, gamma, beta).
    offset: elements by which dy, y and dx (and x, unless x_offset is given) start
    past a 16-byte boundary; pitch: their row pitch in elements (default N)."""
    xo = offset if x_offset is None else x_offset
    placed = bool(offset or xo or pitch) and M * N > 0
    import elementwise_reduction_b200 as dyt

    ad, gd, bd = param_dtypes(p_dtype)
    t = gpu_inputs(inp, x_dtype, p_dtype)
    x = t["x"].view(M, N) if M * N else t["x"]
    if placed:
        x = _at_offset(x, M, N, xo, pitch)
    out, info = {}, {}
    if fwd:
        y = _at_offset(torch.empty((M, N), dtype=x.dtype, device=x.device), M, N, offset, pitch) if placed \
            else None
        y = dyt.forward(x, t["alpha"], t["gamma"], t["beta"], out=y)
        info["fwd"] = dyt.dyt_last_launch_info()
        out["y"] = to_numpy(y, x_dtype)
    if bwd:
        dy = t["dy"].view(M, N) if M * N else t["dy"]
        dxo = None
        if placed:
            dy, dxo = _at_offset(dy, M, N, offset, pitch), _at_offset(torch.empty((M, N), dtype=x.dtype,
                                                                                  device=x.device), M, N, offset,
                                                                      pitch)
        dx, da, dg, db = dyt.backward(x, dy, t["alpha"], t["gamma"], t["beta"], dx=dxo)
        info["bwd"] = dyt.dyt_last_launch_info()
        out.update(dx=to_numpy(dx, x_dtype), dgamma=to_numpy(dg, gd), dbeta=to_numpy(db, bd),
                   dalpha=float(decode(to_numpy(da, ad), ad)[0]))
    torch.cuda.synchronize()
    return out, info


def _alpha_value(inp: dict, p_dtype) -> float:
    return float(decode(np.asarray(inp["alpha"]).ravel()[:1], param_dtypes(p_dtype)[0])[0])


def _row_blocks(M: int, N: int, target: int = 1 << 22):
    rows = max(1, target // max(1, N))
    return [(a, min(M, a + rows)) for a in range(0, M, rows)]


def compare_all(inp: dict, out: dict, M: int, N: int, x_dtype: str, p_dtype, rows=None,
                threads: int | None = None) -> dict:
    """Compare every output with the oracle, y and dx element by element (rows: a
    sample of row indices for y/dx, None = all rows). The elementwise checks run
    over row blocks on `threads` host threads (default: every core this process
    may use); the oracle's gradient sums are one call over the whole matrix in
    index order."""
    import concurrent.futures
    import os

    ad, gd, bd = param_dtypes(p_dtype)
    stats = {}
    X, DY = inp["x"].reshape(M, N) if M * N else inp["x"], inp["dy"].reshape(M, N) if M * N else inp["dy"]
    if rows is not None:
        rows = np.asarray(rows)
        blocks = [(rows, None)]
    else:
        blocks = _row_blocks(M, N) if M * N else []

    def block_check(b):
        sel = b[0] if b[1] is None else slice(b[0], b[1])
        xs, dys = np.ascontiguousarray(X[sel]).ravel(), np.ascontiguousarray(DY[sel]).ravel()
        m = xs.size // N
        res = {}
        if "y" in out:
            y64 = oracle.forward(xs, inp["alpha"], inp["gamma"], inp["beta"], m, N, x_dtype, p_dtype)
            res["y"] = check_elementwise(out["y"].reshape(M, N)[sel].ravel(), y64, x_dtype, "y")
        if "dx" in out:
            dx64 = oracle.backward(xs, dys, inp["alpha"], inp["gamma"], m, N, x_dtype, p_dtype)["dx"]
            res["dx"] = check_elementwise(out["dx"].reshape(M, N)[sel].ravel(), dx64, x_dtype, "dx")
        return res

    if blocks:
        workers = threads or max(1, min(len(blocks), len(os.sched_getaffinity(0))))
        with concurrent.futures.ThreadPoolExecutor(max_workers=workers) as ex:
            parts = list(ex.map(block_check, blocks))
        for k in ("y", "dx"):
            got = [p[k] for p in parts if k in p]
            if got:
                merged = {}
                for st in got:
                    for key, v in st.items():
                        merged[key] = max(merged.get(key, v), v) if key != "frac_exact" else min(merged.get(key, v), v)
                stats[k] = merged
    if "dgamma" in out:
        r = oracle.backward(inp["x"], inp["dy"], inp["alpha"], inp["gamma"], M, N, x_dtype, p_dtype,
                            want_dx=False)
        exact_t = t_is_exact(_alpha_value(inp, p_dtype))
        t_err = (0.0 if exact_t else T_REL_ERR) + (0.0 if x_dtype == "f32" else GAMMA_RUN_ERR)
        t_abs = None if exact_t else T_ABS_ERR * r["mag_dbeta"]
        stats["dgamma"] = check_sums(out["dgamma"], r["dgamma"], r["mag_dgamma"], gd, "dgamma", M, t_err, t_abs)
        stats["dbeta"] = check_sums(out["dbeta"], r["dbeta"], r["mag_dbeta"], bd, "dbeta", M)
        stats["dalpha"] = check_scalar_sum(out["dalpha"], r["dalpha"], r["mag_dalpha"], "dalpha", ad)
    return stats
