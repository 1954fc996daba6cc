/*
 * CPU oracle for the fused Dynamic Tanh (DyT) layer.
 *
 * TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load this library. The product path (the
 * CUDA library and its Python binding) never calls it and shares no code,
 * header, table or constant with it.
 *
 * What it computes (DyT, the layer of the Liger-Kernel page "fix(dyt): use a
 * 1D grid and tile small-width rows", Summary: a scalar alpha, per-column
 * gamma and beta, and the parameter gradients dalpha, dgamma, dbeta). The page
 * names the layer and its gradients but prints no formula; the definitions
 * below are the DyT layer and its exact derivative. For an M x N row-major x:
 *
 *   forward   t[i,j] = tanh(alpha * x[i,j])
 *             y[i,j] = gamma[j] * t[i,j] + beta[j]
 *   backward  (t recomputed from x, as the page's backward kernel does)
 *             dx[i,j]   = alpha * gamma[j] * dy[i,j] * (1 - t[i,j]^2)
 *             dgamma[j] = sum_i dy[i,j] * t[i,j]
 *             dbeta[j]  = sum_i dy[i,j]
 *             dalpha    = sum_{i,j} gamma[j] * dy[i,j] * (1 - t[i,j]^2) * x[i,j]
 *
 * Arithmetic: every input is decoded exactly to binary64 and every step is a
 * binary64 operation; sums run in index order (i outer, j inner), with no
 * blocking or reordering. tanh is the C library's. The factor 1 - t^2 is
 * evaluated as 1 / cosh(z)^2, the same quantity by cosh^2 - sinh^2 = 1: in
 * binary64, 1 - t*t loses all its digits once |z| > 19 while 1/cosh^2 keeps
 * them until it underflows. At z = +-inf both give 0 and at NaN both give NaN.
 * The product for dx is evaluated as ((alpha * gamma) * dy) * (1 - t^2), so
 * an infinite alpha meets the 0 of 1 - t^2 and gives NaN, as the page
 * describes for tanh(inf * 0) in its Summary ("Padding").
 *
 * Results are binary64 arrays; dyt_oracle_round rounds them once, ties to
 * even, to a storage dtype.
 *
 * Built with -ffp-contract=off: no fused multiply-adds are formed.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_F16 = 2, ORACLE_F64 = 3 };

/* ---- storage decoding (exact) ---------------------------------------- */

static double decode_one(const void *p, int64_t i, int dtype) {
  switch (dtype) {
    case ORACLE_F32: return (double)((const float *)p)[i];
    case ORACLE_F64: return ((const double *)p)[i];
    case ORACLE_BF16: {
      /* bf16 is the upper half of a binary32 */
      uint32_t u = (uint32_t)((const uint16_t *)p)[i] << 16;
      float f;
      memcpy(&f, &u, 4);
      return (double)f;
    }
    case ORACLE_F16: {
      _Float16 h;
      memcpy(&h, (const uint16_t *)p + i, 2);
      return (double)h;
    }
  }
  return NAN;
}

static int valid_dtype(int d) { return d >= ORACLE_F32 && d <= ORACLE_F64; }

void dyt_oracle_decode(const void *src, int64_t n, int dtype, double *dst) {
  for (int64_t i = 0; i < n; ++i) dst[i] = decode_one(src, i, dtype);
}

/* ---- 1 - tanh(z)^2 ----------------------------------------------------- */

static double one_minus_tanh_sq(double z) {
  const double c = cosh(z);
  return 1.0 / (c * c);
}

/* ---- forward ----------------------------------------------------------- */

/* y[i*N + j] = gamma[j] * tanh(alpha * x[i*N + j]) + beta[j], binary64.
 * alpha, gamma and beta are stored in a_dtype, g_dtype and b_dtype (each
 * parameter keeps its own dtype, as on the page's Summary, "Precision").
 * Returns 0, or -1 on a bad argument. */
int dyt_oracle_forward(const void *x, int x_dtype, const void *alpha, int a_dtype, const void *gamma,
                       int g_dtype, const void *beta, int b_dtype, int64_t M, int64_t N, double *y) {
  if (M < 0 || N < 0 || !valid_dtype(x_dtype) || !valid_dtype(a_dtype) || !valid_dtype(g_dtype) ||
      !valid_dtype(b_dtype))
    return -1;
  if (M == 0 || N == 0) return 0;
  if (!x || !alpha || !gamma || !beta || !y) return -1;
  double *g = (double *)malloc((size_t)N * sizeof(double));
  double *b = (double *)malloc((size_t)N * sizeof(double));
  if (!g || !b) { free(g); free(b); return -1; }
  dyt_oracle_decode(gamma, N, g_dtype, g);
  dyt_oracle_decode(beta, N, b_dtype, b);
  const double a = decode_one(alpha, 0, a_dtype);
  for (int64_t i = 0; i < M; ++i) {
    for (int64_t j = 0; j < N; ++j) {
      const double xv = decode_one(x, i * N + j, x_dtype);
      const double t = tanh(a * xv);
      y[i * N + j] = g[j] * t + b[j];
    }
  }
  free(g);
  free(b);
  return 0;
}

/* ---- backward ---------------------------------------------------------- */

/*
 * dx (optional, M*N), dgamma[N], dbeta[N], dalpha[1] in binary64.
 * The optional mag_* outputs receive the magnitude of each sum, the sum of the
 * absolute values of its terms: mag_dgamma[j] = sum_i |dy*t|, mag_dbeta[j] =
 * sum_i |dy|, mag_dalpha = sum |gamma*dy*(1-t^2)*x|. They set the error scale
 * of a floating-point sum.
 * alpha and gamma are stored in a_dtype and g_dtype.
 * Returns 0, or -1 on a bad argument.
 */
int dyt_oracle_backward(const void *x, const void *dy, int x_dtype, const void *alpha, int a_dtype,
                        const void *gamma, int g_dtype, int64_t M, int64_t N, double *dx,
                        double *dgamma, double *dbeta, double *dalpha, double *mag_dgamma,
                        double *mag_dbeta, double *mag_dalpha) {
  if (M < 0 || N < 0 || !valid_dtype(x_dtype) || !valid_dtype(a_dtype) || !valid_dtype(g_dtype)) return -1;
  if (!dalpha || (N > 0 && (!dgamma || !dbeta))) return -1;
  for (int64_t j = 0; j < N; ++j) {
    dgamma[j] = 0.0;
    dbeta[j] = 0.0;
    if (mag_dgamma) mag_dgamma[j] = 0.0;
    if (mag_dbeta) mag_dbeta[j] = 0.0;
  }
  *dalpha = 0.0;
  if (mag_dalpha) *mag_dalpha = 0.0;
  if (M == 0 || N == 0) return 0;
  if (!x || !dy || !alpha || !gamma) return -1;
  double *g = (double *)malloc((size_t)N * sizeof(double));
  if (!g) return -1;
  dyt_oracle_decode(gamma, N, g_dtype, g);
  const double a = decode_one(alpha, 0, a_dtype);
  double da = 0.0, da_mag = 0.0;
  for (int64_t i = 0; i < M; ++i) {
    for (int64_t j = 0; j < N; ++j) {
      const int64_t k = i * N + j;
      const double xv = decode_one(x, k, x_dtype);
      const double dyv = decode_one(dy, k, x_dtype);
      const double z = a * xv;
      const double t = tanh(z);
      const double s = one_minus_tanh_sq(z);
      if (dx) dx[k] = ((a * g[j]) * dyv) * s;
      const double dgt = dyv * t;
      dgamma[j] += dgt;
      dbeta[j] += dyv;
      const double term = ((g[j] * dyv) * s) * xv;
      da += term;
      if (mag_dgamma) mag_dgamma[j] += fabs(dgt);
      if (mag_dbeta) mag_dbeta[j] += fabs(dyv);
      da_mag += fabs(term);
    }
  }
  *dalpha = da;
  if (mag_dalpha) *mag_dalpha = da_mag;
  free(g);
  return 0;
}

/* ---- rounding binary64 -> storage dtype, ties to even ------------------ */

/*
 * Round v to the binary format with p significant bits, minimum normal
 * exponent emin and largest finite value maxfinite, ties to even, directly
 * from binary64 (one rounding). Values whose rounded magnitude exceeds
 * maxfinite become infinities; NaN stays NaN.
 */
static double round_to_format(double v, int p, int emin, double maxfinite) {
  if (isnan(v) || isinf(v) || v == 0.0) return v;
  int e;
  (void)frexp(fabs(v), &e); /* |v| = m * 2^e, m in [0.5, 1) */
  int lead = e - 1;          /* exponent of the leading bit */
  if (lead < emin) lead = emin; /* subnormal range: fixed quantum */
  const int q = lead - (p - 1); /* exponent of one unit in the last place */
  const double r = ldexp(nearbyint(ldexp(v, -q)), q);
  if (fabs(r) > maxfinite) return copysign(INFINITY, v);
  return r;
}

double dyt_oracle_round_scalar(double v, int dtype) {
  switch (dtype) {
    case ORACLE_F32: return (double)(float)v;
    case ORACLE_F64: return v;
    case ORACLE_BF16: return round_to_format(v, 8, -126, 0x1.FEp127);
    case ORACLE_F16: return round_to_format(v, 11, -14, 65504.0);
  }
  return NAN;
}

/* out[i] = v[i] rounded once to `dtype` and stored in it (bf16 as raw bits). */
int dyt_oracle_round(const double *v, int64_t n, int dtype, void *out) {
  if (n < 0 || !valid_dtype(dtype)) return -1;
  for (int64_t i = 0; i < n; ++i) {
    const double r = dyt_oracle_round_scalar(v[i], dtype);
    switch (dtype) {
      case ORACLE_F32: ((float *)out)[i] = (float)r; break;
      case ORACLE_F64: ((double *)out)[i] = r; break;
      case ORACLE_BF16: {
        const float f = (float)r; /* exact: r is on the bf16 grid */
        uint32_t u;
        memcpy(&u, &f, 4);
        if (isnan(r)) u = (u & 0x80000000u) | 0x7FC00000u;
        ((uint16_t *)out)[i] = (uint16_t)(u >> 16);
        break;
      }
      case ORACLE_F16: {
        const _Float16 h = (_Float16)r; /* exact: r is on the binary16 grid */
        memcpy((uint16_t *)out + i, &h, 2);
        break;
      }
    }
  }
  return 0;
}
