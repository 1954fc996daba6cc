// Definitions of the kernel selectors declared in dyt_select.cuh, and the
// macro that instantiates them (with every kernel they return) for one
// activation dtype.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "dyt_async.cuh"
#include "dyt_select.cuh"

namespace dyt {
namespace launch {

template <typename T, typename P>
FwdKernel<T, P> fwd_kernel_of(bool async, bool packed, int shm) {
  constexpr int V = vec_of<T>(), B = kAsyncBlock, S = kAsyncStagesFwd;
  if (!async) return dyt_fwd_kernel<T, P, kScalarUnrollFwd, kScalarBlock>;
  switch (shm) {
    case 1: return dyt_fwd_async_kernel<T, P, V, B, S, true, 1>;
    case 3: return dyt_fwd_async_kernel<T, P, V, B, S, true, 3>;
    case 9: return dyt_fwd_async_kernel<T, P, V, B, S, false, 9>;
    case 11: return dyt_fwd_async_kernel<T, P, V, B, S, false, 11>;
    case 25: return dyt_fwd_async_kernel<T, P, V, B, S, false, 25>;
  }
  return packed ? dyt_fwd_async_kernel<T, P, V, B, S, true, 0> : dyt_fwd_async_kernel<T, P, V, B, S, false, 0>;
}

template <typename T, typename P, int B, int S>
BwdKernel<T, P> bwd_async_of(bool packed, int shm) {
  constexpr int V = vec_of<T>();
  switch (shm) {
    case 1: return dyt_bwd_async_kernel<T, P, V, B, S, true, 1>;
    case 3: return dyt_bwd_async_kernel<T, P, V, B, S, true, 3>;
    case 7: return dyt_bwd_async_kernel<T, P, V, B, S, true, 7>;
    case 9: return dyt_bwd_async_kernel<T, P, V, B, S, false, 9>;
    case 11: return dyt_bwd_async_kernel<T, P, V, B, S, false, 11>;
    case 15: return dyt_bwd_async_kernel<T, P, V, B, S, false, 15>;
    case 25: return dyt_bwd_async_kernel<T, P, V, B, S, false, 25>;
  }
  return packed ? dyt_bwd_async_kernel<T, P, V, B, S, true, 0> : dyt_bwd_async_kernel<T, P, V, B, S, false, 0>;
}

template <typename T, typename P>
BwdKernel<T, P> bwd_kernel_of(bool async, bool packed, int shm, int block) {
  if (!async) return dyt_bwd_kernel<T, P, kScalarUnrollBwd, kScalarBlock>;
  if (block == kAsyncBlockNarrow) return bwd_async_of<T, P, kAsyncBlockNarrow, kAsyncStagesBwdNarrow>(packed, shm);
  return bwd_async_of<T, P, kAsyncBlock, kAsyncStagesBwd>(packed, shm);
}

}  // namespace launch
}  // namespace dyt

// The selectors for activations of type T and parameters of every type (one
// shared dtype, or void: a run-time dtype per parameter).
#define DYT_INSTANTIATE_SELECTORS_P(T, P)                                                         \
  template dyt::launch::FwdKernel<T, P> dyt::launch::fwd_kernel_of<T, P>(bool, bool, int);       \
  template dyt::launch::BwdKernel<T, P> dyt::launch::bwd_kernel_of<T, P>(bool, bool, int, int);
#define DYT_INSTANTIATE_SELECTORS(T)               \
  DYT_INSTANTIATE_SELECTORS_P(T, float)            \
  DYT_INSTANTIATE_SELECTORS_P(T, __nv_bfloat16)    \
  DYT_INSTANTIATE_SELECTORS_P(T, __half)           \
  DYT_INSTANTIATE_SELECTORS_P(T, void)
