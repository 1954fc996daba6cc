// Per-thread asynchronous-copy DyT kernels for sm_100a (16-byte aligned rows).
//
// Same decomposition, thread mapping, arithmetic and reduction order as the
// register-path kernels in dyt_kernels.cuh. Each thread streams the rows it
// owns (its VEC columns of rows rl, rl + RL, ... of the group) into a private
// ring of S shared-memory slots with 16-byte asynchronous copies
// (cp.async.cg, L2 only), S - 1 rows ahead of the row it computes, and reads
// each slot back after cp.async.wait_group. A thread only ever reads slots it
// filled itself, so no barrier is needed between threads; the data in flight
// (up to (S - 1) x 32 bytes per thread) costs no registers. Each thread visits
// exactly its real rows, so no padded lane is ever computed.
#pragma once

#include <cuda_runtime.h>

#include "dyt_kernels.cuh"

namespace dyt {

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Rows of the current item owned by this thread: first row and count.
__device__ __forceinline__ int64_t thread_rows(int64_t rb, int64_t re, int rl, int RL, int64_t &first) {
  first = rb + rl;
  return first < re ? (re - first + RL - 1) / RL : 0;
}

// ---- forward ------------------------------------------------------------------

template <typename T, typename P, int VEC, int B, int S>
__global__ void __launch_bounds__(B, 1)
    dyt_fwd_async_kernel(const T *__restrict__ x, const P *__restrict__ alpha_p, const P *__restrict__ gamma,
                         const P *__restrict__ beta, T *y, Geom g) {
  using IO = VecIO<T, VEC>;
  static_assert(VEC * sizeof(T) == 16, "16-byte vectors");
  extern __shared__ uint4 ring[];  // [S][B]
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = param(alpha_p, 0);
  uint4 *slot0 = ring + threadIdx.x;
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    int cc, rg;
    item_split(g, item, cc, rg);
    int64_t rb, re;
    group_rows(g, rg, rb, re);
    const int cv = cc * B + ln.cv;
    if (!(ln.live && cv < g.NV)) continue;
    const int64_t c0 = (int64_t)cv * VEC;
    int64_t first;
    const int64_t n = thread_rows(rb, re, ln.rl, g.RL, first);
    const int64_t stride = (int64_t)g.RL * g.N;
    const T *px = x + first * g.N + c0;
    T *py = y + first * g.N + c0;
    // Rows first, parameters second: the parameter loads overlap the copies.
#pragma unroll
    for (int k = 0; k < S - 1; ++k) {
      if (k < n) cp_async16(slot0 + k * B, px + k * stride);
      cp_async_commit();
    }
    float gam[VEC], bet[VEC], bth[VEC];
    fwd_params<T, P, VEC>(gamma, beta, c0, true, gam, bet, bth);
    int s_rd = 0, s_wr = S - 1;
    for (int64_t k = 0; k < n; ++k) {
      if (k + S - 1 < n) cp_async16(slot0 + s_wr * B, px + (k + S - 1) * stride);
      cp_async_commit();
      cp_async_wait<S - 1>();
      const typename IO::Raw rx = *(const typename IO::Raw *)(slot0 + s_rd * B);
      IO::store_raw(py, fwd_vector<T, VEC>(rx, alpha, gam, bet, bth));
      py += stride;
      s_rd = s_rd + 1 == S ? 0 : s_rd + 1;
      s_wr = s_wr + 1 == S ? 0 : s_wr + 1;
    }
    cp_async_wait<0>();
  }
}

// ---- backward, stage 1 ----------------------------------------------------------

template <typename T, typename P, int VEC, int B, int S>
__global__ void __launch_bounds__(B, 1)
    dyt_bwd_async_kernel(const T *__restrict__ x, const T *__restrict__ dy, const P *__restrict__ alpha_p,
                         const P *__restrict__ gamma, T *dx, float *__restrict__ part_dg,
                         float *__restrict__ part_db, double *__restrict__ part_da, Geom g) {
  using IO = VecIO<T, VEC>;
  static_assert(VEC * sizeof(T) == 16, "16-byte vectors");
  // [S][2][B] 16-byte slots; after an item's last row the ring is empty and
  // its first VEC * B floats serve the row-lane reduction.
  extern __shared__ uint4 ring[];
  __shared__ double red_a[B / 32];
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = param(alpha_p, 0);
  float *red = reinterpret_cast<float *>(ring);
  uint4 *slot0 = ring + threadIdx.x;
  double acc_a = 0.0;
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    int cc, rg;
    item_split(g, item, cc, rg);
    int64_t rb, re;
    group_rows(g, rg, rb, re);
    const int cv = cc * B + ln.cv;
    const bool col_ok = ln.live && cv < g.NV;
    const int64_t c0 = (int64_t)cv * VEC;
    float gam[VEC];
    BwdAcc<VEC> acc;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      acc.g[e] = 0.0f;
      acc.b[e] = 0.0f;
    }
    if (col_ok) {
      int64_t first;
      const int64_t n = thread_rows(rb, re, ln.rl, g.RL, first);
      const int64_t stride = (int64_t)g.RL * g.N;
      const T *px = x + first * g.N + c0;
      const T *pd = dy + first * g.N + c0;
      T *pdx = dx + first * g.N + c0;
      // Rows first, parameters second: the gamma loads overlap the copies.
#pragma unroll
      for (int k = 0; k < S - 1; ++k) {
        if (k < n) {
          cp_async16(slot0 + (2 * k) * B, px + k * stride);
          cp_async16(slot0 + (2 * k + 1) * B, pd + k * stride);
        }
        cp_async_commit();
      }
#pragma unroll
      for (int e = 0; e < VEC; ++e) gam[e] = 4.0f * param(gamma, c0 + e);  // 4 gamma (see bwd_vector)
      int s_rd = 0, s_wr = S - 1;
      for (int64_t k = 0; k < n; ++k) {
        if (k + S - 1 < n) {
          cp_async16(slot0 + (2 * s_wr) * B, px + (k + S - 1) * stride);
          cp_async16(slot0 + (2 * s_wr + 1) * B, pd + (k + S - 1) * stride);
        }
        cp_async_commit();
        cp_async_wait<S - 1>();
        const typename IO::Raw rx = *(const typename IO::Raw *)(slot0 + (2 * s_rd) * B);
        const typename IO::Raw rd = *(const typename IO::Raw *)(slot0 + (2 * s_rd + 1) * B);
        float2 ca = make_float2(0.0f, 0.0f);
        IO::store_raw(pdx, bwd_vector<T, VEC, false>(rx, rd, alpha, gam, acc, ca, true));
        acc_a += (double)ca.x;
        acc_a += (double)ca.y;
        pdx += stride;
        s_rd = s_rd + 1 == S ? 0 : s_rd + 1;
        s_wr = s_wr + 1 == S ? 0 : s_wr + 1;
      }
      cp_async_wait<0>();
    }
    // ---- item done: per-(group, column) partials ----
    float *pg = part_dg + (int64_t)rg * g.N;
    float *pb = part_db + (int64_t)rg * g.N;
    if (g.RL == 1) {
      if (col_ok) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          pg[c0 + e] = acc.g[e];
          pb[c0 + e] = acc.b[e];
        }
      }
    } else {
      __syncthreads();  // every thread's ring is drained: reuse it for the reduction
      if ((32 % g.NV) == 0) {
        // the chunk's columns start at 0 on the row-tiled path (one chunk)
        lane_reduce_warps<VEC, B>(acc.g, acc.b, red, g, ln, 0, pg, pb);
      } else {
#pragma unroll
        for (int e = 0; e < VEC; ++e) red[e * B + threadIdx.x] = acc.g[e];
        __syncthreads();
        lane_tree<VEC, B>(red, g, ln);
        if (col_ok && ln.rl == 0) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) pg[c0 + e] = red[e * B + threadIdx.x];
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < VEC; ++e) red[e * B + threadIdx.x] = acc.b[e];
        __syncthreads();
        lane_tree<VEC, B>(red, g, ln);
        if (col_ok && ln.rl == 0) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) pb[c0 + e] = red[e * B + threadIdx.x];
        }
        __syncthreads();
      }
    }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) acc_a += __shfl_down_sync(0xFFFFFFFFu, acc_a, off);
  if ((threadIdx.x & 31) == 0) red_a[threadIdx.x >> 5] = acc_a;
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int w = 0; w < B / 32; ++w) s += red_a[w];
    part_da[blockIdx.x] = s;
  }
}

}  // namespace dyt
