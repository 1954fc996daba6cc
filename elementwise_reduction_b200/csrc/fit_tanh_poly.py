"""Fit the small-argument tanh polynomial used by dyt_math.cuh.

tanh(a) = a + a^3 Q(a^2) on [0, T]; Q of degree `deg` is fitted by iteratively
reweighted least squares towards the minimax relative error. Prints the
binary32 coefficients and the error after binary32 evaluation.
"""
import numpy as np

T = 0.5
deg = 3
def tanh_hi(a):  # binary64 is plenty for a fit target at the 1e-10 level
    return np.tanh(a)
u = np.linspace(1e-8, T*T, 20001)
a = np.sqrt(u)
f = (tanh_hi(a) - a) / (a**3)     # Q target (smooth in u)
# series near 0 to avoid cancellation in target
small = a < 1e-2
f[small] = -1/3 + 2/15*u[small] - 17/315*u[small]**2 + 62/2835*u[small]**3
w = np.ones_like(u)
for it in range(30):
    V = np.vander(u, deg+1, increasing=True)
    # relative error of t: a^3 (Q - f) / tanh(a) -> weight a^3/tanh(a) ~ a^2 = u
    W = (a**3 / tanh_hi(a)) * w
    c, *_ = np.linalg.lstsq(V * W[:, None], f * W, rcond=None)
    err = (V @ c - f) * a**3 / tanh_hi(a)
    w *= (1 + 10*np.abs(err)/np.abs(err).max())
print("coeffs", [float(np.float32(x)) for x in c])
print("max rel err (f64 eval)", np.abs(err).max())
# evaluate in float32 arithmetic with fma emulated in f64 then rounded
c32 = [np.float32(x) for x in c]
A = np.float32(np.linspace(0, T, 2000001)).astype(np.float32)
A2 = (A*A).astype(np.float32)
def fma(x,y,z): return np.float32(x.astype(np.float64)*y.astype(np.float64)+z.astype(np.float64))
p = np.full_like(A2, c32[-1])
for k in range(deg-1, -1, -1):
    p = fma(A2, p, np.full_like(A2, c32[k]))
A3 = (A2*A).astype(np.float32)
t = fma(A3, p, A)
ref = np.tanh(A.astype(np.float64))
nz = ref > 0
ulp = np.spacing(ref[nz].astype(np.float32)).astype(np.float64)
print("max err in ulps (fp32 eval):", (np.abs(t[nz]-ref[nz])/ulp).max(), "max rel", (np.abs(t[nz]-ref[nz])/ref[nz]).max())
