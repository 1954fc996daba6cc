// Device arithmetic of the fused DyT kernels: tanh and 1 - tanh^2 in binary32,
// the binary64 refinement of a cancelling 16-bit forward output, and storage
// conversions. Written for sm_100a; compiled without fast-math (denormals kept).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <type_traits>

#include "dyt.h"

namespace dyt {

// ---- hardware approximations (special-function unit) ---------------------

// 2^w, flushing results below 2^-126 to 0: used for w >= 0 (results >= 1)
// and for exp(-|z|) whose square gives exp(-2|z|) (see below), where only
// results that square to below the subnormal range are flushed.
__device__ __forceinline__ float ex2_approx(float w) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(w));
  return r;
}


// 1/v for v >= 1 (normal results only).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// ---- tanh(z) and 1 - tanh(z)^2 in binary32 --------------------------------
//
// a = |z|.
//   a <  0.5: tanh z = z + z^3 Q(z^2), Q a degree-3 polynomial fitted to
//             minimise the relative error on [0, 0.5] (fit_tanh_poly.py next to
//             this file; fitted error 1.5e-8, 0.84 ulp after binary32
//             evaluation); odd in z, so the sign needs no handling. 1 - t^2 =
//             fma(-t, t, 1) has no cancellation there (|t| <= 0.47).
//   a >= 0.5, forward (t only): with E = exp(2a) = 2^(2a log2 e) >= e and
//             r = 1 / (1 + E) <= 0.27, tanh a = 1 - 2r (no cancellation).
//   backward t, every a: with e = exp(-2a) (subnormal values kept) and
//             rc = 1 / (1 + e), tanh a = (1 - e) rc: no cancellation for
//             a >= 0.5 (e <= 0.37); below, an absolute error within 2^-21
//             (t only enters the dgamma sum, see dyt_tanh_qsech2).
//   e = exp(-2a) is formed as h^2 with h = 2^(-a log2 e) from the flushing
//             ex2: h is normal for every a < 87.3 (and for larger a, e is
//             below the subnormal range, so 0 is its rounding), and the
//             square, a multiply that keeps subnormals, carries e into the
//             subnormal range without a branch. It costs one multiply; the
//             subnormal-keeping ex2 costs four instructions more per element
//             (15% of the backward's instructions). The relative error is the
//             approximation's doubled plus one rounding.
//   backward 1 - t^2, every a: 1 - tanh^2 a = 4 e rc^2 with e = exp(-2a) in
//             (0, 1] and rc in [1/2, 1]: no cancellation anywhere, accurate to
//             about 2^-21 relative down to the subnormal range, 0 exactly when
//             1 - t^2 rounds to 0, and exactly 1 at z = 0. The kernels carry
//             q = (1 - t^2) / 4 = e rc^2 and multiply it by 4 gamma, which
//             rounds exactly as gamma (1 - t^2) would (scaling by 4 is exact).
//   The sign of z is copied onto t in both forms.
// t(-z) = -t(z) exactly. z = +-inf gives t = +-1, 1 - t^2 = 0; NaN gives NaN.
constexpr float kTanhSplit = 0.5f;
constexpr float k2Log2e = 2.88539008177792681f;  // 2 / ln 2
constexpr float kLog2e = 1.44269504088896341f;   // 1 / ln 2 (exactly half of k2Log2e)
constexpr float kQ0 = -0.333331435918808f;
constexpr float kQ1 = 0.13325883448123932f;
constexpr float kQ2 = -0.053045812994241714f;
constexpr float kQ3 = 0.017242243513464928f;

__device__ __forceinline__ float tanh_small(float z) {
  const float u = z * z;
  float q = fmaf(kQ3, u, kQ2);
  q = fmaf(q, u, kQ1);
  q = fmaf(q, u, kQ0);
  return fmaf(z * u, q, z);
}

__device__ __forceinline__ float dyt_tanh(float z) {
  const float E = ex2_approx(fabsf(z * k2Log2e));
  const float r = rcp_approx(1.0f + E);
  const float t_large = copysignf(fmaf(r, -2.0f, 1.0f), z);
  const float t_small = tanh_small(z);
  return fabsf(z) < kTanhSplit ? t_small : t_large;
}

// exp(-2|z|) as the square of exp(-|z|) (see above).
__device__ __forceinline__ float exp_neg2(float z) {
  const float h = ex2_approx(-fabsf(z * kLog2e));
  return h * h;
}

// The backward's t and q = (1 - tanh(z)^2) / 4 from one evaluation. t only
// enters the dgamma sum, so it takes the exp(-2|z|) form for every z, with no
// polynomial and no select: t = sign(z) (1 - e) / (1 + e). For |z| >= 0.5 this
// is the form above (relative error within 2^-20.5); below, 1 - e loses its
// leading bits and the error is absolute instead, within 2^-21 (e carries the
// exp2 approximation's relative error twice, and 1 - e is exact for e >= 1/2).
// t is exact where it matters for exactness: 0 at z = 0, +-1 at z = +-inf.
__device__ __forceinline__ void dyt_tanh_qsech2(float z, float &t, float &q) {
  const float e = exp_neg2(z);
  const float rc = rcp_approx(1.0f + e);
  t = copysignf(fmaf(e, -1.0f, 1.0f) * rc, z);
  q = (e * rc) * rc;
}

// ---- the same on element pairs (packed f32x2 arithmetic of sm_100) ---------
//
// Identical formulas; the multiplies and adds run as two-lane f32x2
// instructions, halving their issue cost. Every lane is rounded exactly as
// its scalar counterpart (round to nearest even, no fused differences), so a
// pair result equals two scalar results bit for bit.
__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

__device__ __forceinline__ float2 tanh_small2(float2 z) {
  const float2 u = mul2(z, z);
  float2 q = fma2(f2(kQ3), u, f2(kQ2));
  q = fma2(q, u, f2(kQ1));
  q = fma2(q, u, f2(kQ0));
  return fma2(mul2(z, u), q, z);
}

__device__ __forceinline__ float2 dyt_tanh2(float2 z) {
  const float2 w = mul2(z, f2(k2Log2e));
  const float2 ope = add2(make_float2(ex2_approx(fabsf(w.x)), ex2_approx(fabsf(w.y))), f2(1.0f));
  const float2 r = make_float2(rcp_approx(ope.x), rcp_approx(ope.y));
  const float2 tl = fma2(r, f2(-2.0f), f2(1.0f));
  const float2 ts = tanh_small2(z);
  return make_float2(fabsf(z.x) < kTanhSplit ? ts.x : copysignf(tl.x, z.x),
                     fabsf(z.y) < kTanhSplit ? ts.y : copysignf(tl.y, z.y));
}

__device__ __forceinline__ void dyt_tanh_qsech2_2(float2 z, float2 &t, float2 &q) {
  const float2 w = mul2(z, f2(kLog2e));
  const float2 h = make_float2(ex2_approx(-fabsf(w.x)), ex2_approx(-fabsf(w.y)));
  const float2 e = mul2(h, h);  // exp(-2|z|), subnormal values kept
  const float2 ope = add2(e, f2(1.0f));
  const float2 rc = make_float2(rcp_approx(ope.x), rcp_approx(ope.y));
  const float2 tl = mul2(fma2(e, f2(-1.0f), f2(1.0f)), rc);
  q = mul2(mul2(e, rc), rc);
  t = make_float2(copysignf(tl.x, z.x), copysignf(tl.y, z.y));  // see dyt_tanh_qsech2
}

// ---- storage conversions ---------------------------------------------------

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) { return __bfloat162float(v); }
template <>
__device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// One rounding from binary64 (cvt.rn: nearest, ties to even).
template <typename T>
__device__ __forceinline__ T from_f64(double v);
template <>
__device__ __forceinline__ float from_f64<float>(double v) { return (float)v; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_f64<__nv_bfloat16>(double v) {
  unsigned short b;
  asm("cvt.rn.bf16.f64 %0, %1;" : "=h"(b) : "d"(v));
  return __ushort_as_bfloat16(b);
}
template <>
__device__ __forceinline__ __half from_f64<__half>(double v) {
  unsigned short b;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(b) : "d"(v));
  return __ushort_as_half(b);
}

// ---- parameters ----------------------------------------------------------------
//
// alpha, gamma and beta (and their gradients) each carry their own dtype. The
// kernels are instantiated for a parameter type P: float, __nv_bfloat16 or
// __half when all three share it, read through typed read-only pointers; or
// void when they differ, each read by a run-time switch on its dyt_dtype code
// (dt). Parameters are read once per work item, so the switch costs nothing on
// the element path; the typed form, measured, lets the compiler schedule the
// 16-bit forward's row loop better (12% on 16384 x 4096).

template <typename P>
__device__ __forceinline__ float load_param(const P *__restrict__ p, int dt, int64_t i) {
  if constexpr (std::is_void<P>::value) {
    if (dt == DYT_F32) return __ldg(static_cast<const float *>(p) + i);
    const unsigned short u = __ldg(static_cast<const unsigned short *>(p) + i);
    return dt == DYT_BF16 ? __uint_as_float((uint32_t)u << 16) : __half2float(__ushort_as_half(u));
  } else {
    (void)dt;
    return to_f32<P>(__ldg(p + i));
  }
}

// The parameter values at indices col[0..V) as binary32, scaled by `scale`
// (exact: a power of two). With P = void, one dispatch on the dtype for all V
// loads, so the loads are issued back to back and their latencies overlap.
template <int V, typename P>
__device__ __forceinline__ void load_params(const P *__restrict__ p, int dt, const int64_t (&col)[V], float scale,
                                            float (&out)[V]) {
  if constexpr (std::is_void<P>::value) {
    if (dt == DYT_F32) {
      const float *q = static_cast<const float *>(p);
      float v[V];
#pragma unroll
      for (int e = 0; e < V; ++e) v[e] = __ldg(q + col[e]);
#pragma unroll
      for (int e = 0; e < V; ++e) out[e] = scale * v[e];
    } else {
      const unsigned short *q = static_cast<const unsigned short *>(p);
      unsigned short v[V];
#pragma unroll
      for (int e = 0; e < V; ++e) v[e] = __ldg(q + col[e]);
      if (dt == DYT_BF16) {
#pragma unroll
        for (int e = 0; e < V; ++e) out[e] = scale * __uint_as_float((uint32_t)v[e] << 16);
      } else {
#pragma unroll
        for (int e = 0; e < V; ++e) out[e] = scale * __half2float(__ushort_as_half(v[e]));
      }
    }
  } else {
    (void)dt;
    P v[V];
#pragma unroll
    for (int e = 0; e < V; ++e) v[e] = __ldg(p + col[e]);
#pragma unroll
    for (int e = 0; e < V; ++e) out[e] = scale * to_f32<P>(v[e]);
  }
}

// v rounded once (nearest, ties to even) to dtype dt and stored at p[i].
__device__ __forceinline__ void store_param(void *p, int dt, int64_t i, double v) {
  if (dt == DYT_F32) {
    static_cast<float *>(p)[i] = (float)v;
  } else if (dt == DYT_BF16) {
    static_cast<__nv_bfloat16 *>(p)[i] = from_f64<__nv_bfloat16>(v);
  } else {
    static_cast<__half *>(p)[i] = from_f64<__half>(v);
  }
}

// ---- forward output with cancellation refinement ---------------------------
//
// y = gamma * t + beta. The binary32 value carries an error of at most
// eps |gamma t| + 2^-24 |y|, with eps <= 2^-20.5 covering the error of t and of
// z = alpha * x. Since |gamma t| = |y - beta| <= |y| + |beta|, the error is at
// most (eps (1 + 1/tau) + 2^-24) |y| whenever |y| >= tau |beta|. A 16-bit
// output keeps p = 8 (bf16) or 11 (fp16) significant bits, so one unit in its
// last place is at least 2^-p |y|; with tau = 2^-12 (bf16) or 2^-9 (fp16) the
// binary32 value is within that, and the rounded result within one unit of the
// correctly rounded one. Elements with |y| < tau |beta| (cancellation: a few
// in 10^5 for unit-scale data with beta ~ N(0, 0.1), e.g. 87 of the 2.1
// million outputs of a 65537 x 32 bfloat16 forward) are recomputed in binary64
// with the CUDA math library's tanh and rounded once.
template <typename T>
struct CancelGuard;
// kTiny: the type's smallest positive subnormal (the rounding step near 0).
template <>
struct CancelGuard<float> {
  static constexpr bool kOn = false;
  static constexpr float kTau = 0.0f;
  static constexpr float kTiny = 0.0f;
};
template <>
struct CancelGuard<__nv_bfloat16> {
  static constexpr bool kOn = true;
  static constexpr float kTau = 0x1p-12f;
  static constexpr float kTiny = 0x1p-133f;
};
template <>
struct CancelGuard<__half> {
  static constexpr bool kOn = true;
  static constexpr float kTau = 0x1p-9f;
  static constexpr float kTiny = 0x1p-24f;
};

template <typename T>
__device__ __noinline__ T dyt_y_refined(float alpha, float x, float gamma, float beta) {
  const double t = tanh((double)alpha * (double)x);  // the product is exact in binary64
  return from_f64<T>(fma((double)gamma, t, (double)beta));
}

}  // namespace dyt
