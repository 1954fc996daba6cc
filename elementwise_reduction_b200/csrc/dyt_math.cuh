// Device arithmetic of the fused DyT kernels: tanh and 1 - tanh^2 in binary32,
// the binary64 refinement of a cancelling 16-bit forward output, and storage
// conversions. Written for sm_100a; compiled without fast-math (denormals kept).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace dyt {

// ---- hardware approximations (special-function unit) ---------------------

// 2^w. Subnormal results are kept, so exp(-2|z|) decays smoothly to zero.
__device__ __forceinline__ float ex2_approx(float w) {
  float r;
  asm("ex2.approx.f32 %0, %1;" : "=f"(r) : "f"(w));
  return r;
}

// 1/v for v in [1, 2] (the only range it is used on).
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// ---- tanh(z) and 1 - tanh(z)^2 in binary32 --------------------------------
//
// a = |z|.
//   a <  0.5: tanh a = a + a^3 Q(a^2), Q a degree-4 polynomial fitted to
//             minimise the relative error on [0, 0.5] (fit_tanh_poly.py next to
//             this file; fitted error 3.6e-10, 0.67 ulp after binary32
//             evaluation). 1 - t^2 = fma(-t, t, 1) has no cancellation there
//             (t <= 0.47).
//   a >= 0.5: with e = exp(-2a) = 2^(-2a log2 e) in (0, 0.37],
//             tanh a = (1 - e) / (1 + e) and 1 - tanh^2 a = 4e / (1 + e)^2,
//             both free of cancellation; e is one ex2 and 1/(1+e) one rcp.
// tanh is odd: the sign of z is copied onto tanh(a), so t(-z) = -t(z)
// exactly. a = +inf gives t = +-1 and 1 - t^2 = 0; NaN gives NaN in both.
constexpr float kTanhSplit = 0.5f;
constexpr float kMinus2Log2e = -2.88539008177792681f;  // -2 / ln 2
constexpr float kQ0 = -0.333333283662796f;
constexpr float kQ1 = 0.13332964479923248f;
constexpr float kQ2 = -0.053899213671684265f;
constexpr float kQ3 = 0.02129811979830265f;
constexpr float kQ4 = -0.00664772093296051f;

__device__ __forceinline__ float tanh_small(float a) {
  const float u = a * a;
  float q = fmaf(kQ4, u, kQ3);
  q = fmaf(q, u, kQ2);
  q = fmaf(q, u, kQ1);
  q = fmaf(q, u, kQ0);
  return fmaf(a * u, q, a);
}

__device__ __forceinline__ float dyt_tanh(float z) {
  const float a = fabsf(z);
  const float e = ex2_approx(a * kMinus2Log2e);
  const float r = rcp_approx(1.0f + e);
  const float t_large = (1.0f - e) * r;
  const float t_small = tanh_small(a);
  return copysignf(a < kTanhSplit ? t_small : t_large, z);
}

// t = tanh(z) and s = 1 - tanh(z)^2 from one evaluation.
__device__ __forceinline__ void dyt_tanh_sech2(float z, float &t, float &s) {
  const float a = fabsf(z);
  const float e = ex2_approx(a * kMinus2Log2e);
  const float r = rcp_approx(1.0f + e);
  const float t_large = (1.0f - e) * r;
  const float s_large = (4.0f * e) * (r * r);
  const float t_small = tanh_small(a);
  const float s_small = fmaf(-t_small, t_small, 1.0f);
  const bool small = a < kTanhSplit;
  t = copysignf(small ? t_small : t_large, z);
  s = small ? s_small : s_large;
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

// ---- forward output with cancellation refinement ---------------------------
//
// y = gamma * t + beta. The binary32 value carries an error of at most
// eps |gamma t| + 2^-24 |y|, with eps <= 2^-21 covering the error of t and of
// z = alpha * x. A 16-bit output keeps p = 8 (bf16) or 11 (fp16) significant
// bits, so one unit in its last place is at least 2^-p |y|; the binary32 value
// is therefore within one unit whenever |y| >= tau |gamma t| with
// tau = 2^-12 (bf16) or 2^-9 (fp16), with a factor-two margin. Elements below
// that (cancellation, about 1e-3 of unit-scale data) are recomputed in
// binary64 with the CUDA math library's tanh and rounded once, so every
// 16-bit y is within one unit of the correctly rounded value.
template <typename T>
struct CancelGuard;
template <>
struct CancelGuard<float> {
  static constexpr bool kOn = false;
  static constexpr float kTau = 0.0f;
};
template <>
struct CancelGuard<__nv_bfloat16> {
  static constexpr bool kOn = true;
  static constexpr float kTau = 0x1p-12f;
};
template <>
struct CancelGuard<__half> {
  static constexpr bool kOn = true;
  static constexpr float kTau = 0x1p-9f;
};

template <typename T>
__device__ __noinline__ T dyt_y_refined(float alpha, float x, float gamma, float beta) {
  const double t = tanh((double)alpha * (double)x);  // the product is exact in binary64
  return from_f64<T>(fma((double)gamma, t, (double)beta));
}

template <typename T>
__device__ __forceinline__ T dyt_y(float alpha, float x, float gamma, float beta) {
  const float t = dyt_tanh(alpha * x);
  const float y = fmaf(gamma, t, beta);
  if (CancelGuard<T>::kOn && fabsf(y) < fabsf(gamma * t) * CancelGuard<T>::kTau) {
    return dyt_y_refined<T>(alpha, x, gamma, beta);
  }
  return from_f32<T>(y);
}

}  // namespace dyt
