"""The DyT workloads: shapes, dtypes and value distributions.

Every tensor is drawn by ``synth.normal`` from seed 0 with its own Philox
stream; N(mu, s) names the mean and the standard deviation. The shapes and
distributions are those of the fused DyT kernel tests described on the
Liger-Kernel page ("fix(dyt): use a 1D grid and tile small-width rows",
Summary and Testing Done): small and ragged widths, 65,537 rows, ragged rows
with infinite alpha, bf16 activations with fp32 parameters; plus two
transformer-sized shapes for bandwidth.
"""
from __future__ import annotations

from dataclasses import dataclass, replace

import numpy as np

from . import STREAM_BETA, STREAM_DY, STREAM_GAMMA, STREAM_X, normal

ITEMSIZE = {"f32": 4, "bf16": 2, "f16": 2, "f64": 8}


@dataclass(frozen=True)
class Workload:
    name: str
    M: int
    N: int
    x_dtype: str          # x, dy, y, dx
    p_dtype: object       # alpha, gamma, beta and their gradients: one dtype name, or a tuple
                          # (alpha, gamma, beta) of names
    alpha: float
    x_std: float = 1.0
    dy_std: float = 1.0
    gamma_mean: float = 1.0
    gamma_std: float = 0.1
    beta_mean: float = 0.0
    beta_std: float = 0.1
    nonzero: bool = False  # redraw x and dy values that are exactly zero
    seed: int = 0
    offset: int = 0        # elements by which dy, y and dx (and x, unless x_offset) start past a
                           # 16-byte boundary
    x_offset: int | None = None  # x's own offset, when it differs
    pitch: int | None = None     # row pitch (elements) of x, dy, y and dx, when not N

    @property
    def x_off(self) -> int:
        return self.offset if self.x_offset is None else self.x_offset

    @property
    def elements(self) -> int:
        return self.M * self.N

    @property
    def param_dtypes(self) -> tuple:
        """(alpha, gamma, beta) dtype names."""
        return (self.p_dtype,) * 3 if isinstance(self.p_dtype, str) else tuple(self.p_dtype)

    def fwd_bytes(self) -> int:
        """Algorithmic bytes of one forward: x in, y out, gamma, beta, alpha in."""
        sa, sg, sb = (ITEMSIZE[d] for d in self.param_dtypes)
        return 2 * self.M * self.N * ITEMSIZE[self.x_dtype] + self.N * (sg + sb) + sa

    def bwd_bytes(self) -> int:
        """Algorithmic bytes of one backward: x, dy in, dx out, gamma, alpha in,
        dgamma, dbeta, dalpha out."""
        sa, sg, sb = (ITEMSIZE[d] for d in self.param_dtypes)
        return 3 * self.M * self.N * ITEMSIZE[self.x_dtype] + self.N * (2 * sg + sb) + 2 * sa

    def with_shape(self, M: int | None = None, N: int | None = None) -> "Workload":
        return replace(self, M=self.M if M is None else M, N=self.N if N is None else N,
                       name=f"{self.name}@{M or self.M}x{N or self.N}")


WORKLOADS = {
    w.name: w
    for w in [
        Workload("c1_f32_1024x64", 1024, 64, "f32", "f32", alpha=0.5),
        Workload("c2_bf16_65537x32", 65537, 32, "bf16", "f32", alpha=0.7),
        Workload("c3_f32_100003x17_inf", 100003, 17, "f32", "f32", alpha=float("inf"), nonzero=True),
        Workload("c3_f32_100003x100_inf", 100003, 100, "f32", "f32", alpha=float("inf"), nonzero=True),
        Workload("c3_f32_100003x255_inf", 100003, 255, "f32", "f32", alpha=float("inf"), nonzero=True),
        Workload("c4_bf16_16384x4096", 16384, 4096, "bf16", "f32", alpha=0.5),
        Workload("c5_bf16_32768x8192", 32768, 8192, "bf16", "f32", alpha=0.3, x_std=2.0, dy_std=2.0,
                 gamma_std=0.2, beta_std=0.2),
    ]
}

# Layout variants of the workloads above: the same values with tensors off
# 16-byte boundaries, which sends them through the shifted 16-byte kernels.
# _off1: every activation tensor one element past a boundary (each input
# vector one aligned chunk); _xoff1: x alone, as a sliced input next to fresh
# outputs (each x vector cut out of two aligned chunks). _pitch4100: rows of
# 4096 elements 4100 apart (8200 bytes, not whole 16-byte vectors), which the
# one-element kernels take. _pitch4104_off1: rows 4104 apart (whole vectors),
# every tensor one element past a boundary; _pitch256: rows of 255 fp32
# elements 256 apart: the row frame, each row shifted on its own.
VARIANTS = {
    w.name: w
    for w in [
        replace(WORKLOADS["c2_bf16_65537x32"], name="c2_bf16_65537x32_off1", offset=1),
        replace(WORKLOADS["c4_bf16_16384x4096"], name="c4_bf16_16384x4096_off1", offset=1),
        replace(WORKLOADS["c4_bf16_16384x4096"], name="c4_bf16_16384x4096_xoff1", x_offset=1),
        replace(WORKLOADS["c4_bf16_16384x4096"], name="c4_bf16_16384x4096_pitch4100", pitch=4100),
        replace(WORKLOADS["c4_bf16_16384x4096"], name="c4_bf16_16384x4096_pitch4104_off1", pitch=4104, offset=1),
        replace(WORKLOADS["c3_f32_100003x255_inf"], name="c3_f32_100003x255_inf_pitch256", pitch=256),
    ]
}

# The configuration whose throughput the benchmark line reports by default: the
# largest one, where the layer moves the most bytes.
DEFAULT_BENCH = "c5_bf16_32768x8192"


def make_params(w: Workload) -> dict:
    p = {
        "alpha": np.array([w.alpha], dtype=np.float64),
        "gamma": normal(w.N, "f64", w.gamma_mean, w.gamma_std, w.seed, STREAM_GAMMA),
        "beta": normal(w.N, "f64", w.beta_mean, w.beta_std, w.seed, STREAM_BETA),
    }
    # Parameters are drawn through binary32 (f64 storage holds the binary32 value) and
    # then encoded in each parameter's dtype.
    return {k: encode(p[k], dt) for k, dt in zip(("alpha", "gamma", "beta"), w.param_dtypes)}


def encode(v64: np.ndarray, dtype: str) -> np.ndarray:
    """Encode float64 values that are already binary32 values into a storage dtype."""
    f32 = np.asarray(v64, dtype=np.float32)
    if dtype == "f32":
        return f32
    if dtype == "f64":
        return f32.astype(np.float64)
    if dtype == "f16":
        return f32.astype(np.float16)
    if dtype == "bf16":
        u = f32.view(np.uint32).astype(np.uint64)
        nan = (u & 0x7FFFFFFF) > 0x7F800000
        r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
        r[nan] = ((u[nan] >> 16) | 0x40).astype(np.uint16)
        return r
    raise ValueError(dtype)


def make_inputs(w: Workload, threads: int | None = None) -> dict:
    """All inputs of one fwd+bwd step of workload ``w`` in storage dtypes."""
    n = w.M * w.N
    d = make_params(w)
    d["x"] = normal(n, w.x_dtype, 0.0, w.x_std, w.seed, STREAM_X, nonzero=w.nonzero, threads=threads)
    d["dy"] = normal(n, w.x_dtype, 0.0, w.dy_std, w.seed, STREAM_DY, nonzero=w.nonzero, threads=threads)
    return d
