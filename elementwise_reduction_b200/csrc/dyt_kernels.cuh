// Fused DyT forward / backward kernels for sm_100a.
//
// Work decomposition (one 1D persistent grid, the page's Summary "Launch
// limit": rows never sit on grid dimension 1, so M is unbounded):
//   - a thread owns one vector-column cv (VEC consecutive columns; VEC = 16
//     bytes / element size, or 1 for unaligned or ragged rows) and keeps its
//     gamma/beta in registers;
//   - row-tiled path (NV = N / VEC <= B / 2, the page's narrow rows): RL =
//     B / NV row lanes share a CTA step, so one step covers RL * U whole rows
//     (the page's Summary "Small widths": several rows per tile);
//   - row-per-CTA path (wider rows): RL = 1, every thread works on every row
//     of the CTA, columns spread across threads; rows wider than B * VEC are
//     split into column chunks;
//   - rows are cut into nrg balanced contiguous groups; a work item is
//     (column chunk, row group) and CTA b takes items b, b + grid, ... (a
//     static schedule: the same inputs always give the same bits).
// Backward sums: each thread accumulates its columns in binary32 over at most
// 96 rows per group (the host sizes the groups so), the
// row lanes of a CTA are added by a fixed-order tree in shared memory, and
// each (group, column) partial goes to the workspace; dalpha is carried in
// binary64 per thread, reduced per CTA in a fixed order. The finalize kernel
// adds the partials in binary64 in a fixed order.
// Lanes outside [0,M) x [0,N) never enter a sum: their contribution is
// dropped by a select after the arithmetic (the page's Summary, "Padding").
#pragma once

#include <cuda_runtime.h>

#include "dyt_math.cuh"

namespace dyt {

struct Geom {
  int64_t M;   // rows
  int64_t N;   // columns
  int NV;      // vector-columns per row (N / VEC)
  int RL;      // row lanes per CTA step (1 on the row-per-CTA path)
  int ncc;     // column chunks (of B vector-columns)
  int nrg;     // row groups
  int nitems;  // ncc * nrg
};

// Rows [begin, end) of group rg when [0, M) is cut into nrg balanced groups.
__device__ __forceinline__ void group_rows(int64_t M, int nrg, int rg, int64_t &begin, int64_t &end) {
  const int64_t q = M / nrg, rem = M % nrg;
  begin = (int64_t)rg * q + (rg < rem ? rg : rem);
  end = begin + q + (rg < rem ? 1 : 0);
}

// ---- global memory access --------------------------------------------------

// Streaming 16-byte load through the non-coherent path, not kept in L1.
__device__ __forceinline__ uint4 ld_stream16(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st16(void *p, const uint4 &v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

template <typename T>
__device__ __forceinline__ T ld_scalar(const T *p) {
  return __ldg(p);
}

// VEC elements of T as raw storage, with float conversion.
template <typename T, int VEC>
struct VecIO;

template <typename T>
struct VecIO<T, 1> {
  using Raw = T;
  static __device__ __forceinline__ Raw load(const T *p) { return ld_scalar(p); }
  static __device__ __forceinline__ Raw zero() { return from_f32<T>(0.0f); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[1]) { f[0] = to_f32<T>(r); }
  static __device__ __forceinline__ void store(T *p, const float (&f)[1]) { *p = from_f32<T>(f[0]); }
  static __device__ __forceinline__ void set(Raw &r, int, T v) { r = v; }
  static __device__ __forceinline__ Raw pack(const float (&f)[1]) { return from_f32<T>(f[0]); }
  static __device__ __forceinline__ void store_raw(T *p, const Raw &r) { *p = r; }
};

template <>
struct VecIO<float, 4> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const float *p) { return ld_stream16(p); }
  static __device__ __forceinline__ Raw zero() { return make_uint4(0, 0, 0, 0); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[4]) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
  }
  static __device__ __forceinline__ Raw pack(const float (&f)[4]) {
    return make_uint4(__float_as_uint(f[0]), __float_as_uint(f[1]), __float_as_uint(f[2]),
                      __float_as_uint(f[3]));
  }
  static __device__ __forceinline__ void set(Raw &r, int e, float v) {
    const uint32_t u = __float_as_uint(v);
    if (e == 0) r.x = u;
    else if (e == 1) r.y = u;
    else if (e == 2) r.z = u;
    else r.w = u;
  }
  static __device__ __forceinline__ void store_raw(float *p, const Raw &r) { st16(p, r); }
};

// Two 16-bit values per 32-bit word, element 2i in the low half.
__device__ __forceinline__ uint32_t word_of(const uint4 &r, int w) {
  return w == 0 ? r.x : w == 1 ? r.y : w == 2 ? r.z : r.w;
}
__device__ __forceinline__ void set_word(uint4 &r, int w, uint32_t v) {
  if (w == 0) r.x = v;
  else if (w == 1) r.y = v;
  else if (w == 2) r.z = v;
  else r.w = v;
}

template <>
struct VecIO<__nv_bfloat16, 8> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const __nv_bfloat16 *p) { return ld_stream16(p); }
  static __device__ __forceinline__ Raw zero() { return make_uint4(0, 0, 0, 0); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[8]) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t u = word_of(r, w);
      f[2 * w] = __uint_as_float(u << 16);
      f[2 * w + 1] = __uint_as_float(u & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ Raw pack(const float (&f)[8]) {
    Raw r;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t u;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(f[2 * w + 1]), "f"(f[2 * w]));
      set_word(r, w, u);
    }
    return r;
  }
  static __device__ __forceinline__ void set(Raw &r, int e, __nv_bfloat16 v) {
    const uint32_t b = __bfloat16_as_ushort(v);
    const uint32_t u = word_of(r, e >> 1);
    set_word(r, e >> 1, (e & 1) ? ((u & 0x0000FFFFu) | (b << 16)) : ((u & 0xFFFF0000u) | b));
  }
  static __device__ __forceinline__ void store_raw(__nv_bfloat16 *p, const Raw &r) { st16(p, r); }
};

template <>
struct VecIO<__half, 8> {
  using Raw = uint4;
  static __device__ __forceinline__ Raw load(const __half *p) { return ld_stream16(p); }
  static __device__ __forceinline__ Raw zero() { return make_uint4(0, 0, 0, 0); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[8]) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t u = word_of(r, w);
      f[2 * w] = __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu)));
      f[2 * w + 1] = __half2float(__ushort_as_half((unsigned short)(u >> 16)));
    }
  }
  static __device__ __forceinline__ Raw pack(const float (&f)[8]) {
    Raw r;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t u;
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(f[2 * w + 1]), "f"(f[2 * w]));
      set_word(r, w, u);
    }
    return r;
  }
  static __device__ __forceinline__ void set(Raw &r, int e, __half v) {
    const uint32_t b = __half_as_ushort(v);
    const uint32_t u = word_of(r, e >> 1);
    set_word(r, e >> 1, (e & 1) ? ((u & 0x0000FFFFu) | (b << 16)) : ((u & 0xFFFF0000u) | b));
  }
  static __device__ __forceinline__ void store_raw(__half *p, const Raw &r) { st16(p, r); }
};

template <typename P>
__device__ __forceinline__ float param(const P *p, int64_t i) {
  return to_f32<P>(ld_scalar(p + i));
}

// Thread -> (row lane, vector-column) of the CTA.
struct Lane {
  int rl;     // row lane
  int cv;     // vector-column within the chunk
  bool live;  // false for threads past RL * NV on the row-tiled path
};

__device__ __forceinline__ Lane lane_of(const Geom &g, int tid) {
  Lane l;
  if (g.RL > 1) {
    l.rl = tid / g.NV;
    l.cv = tid - l.rl * g.NV;
    l.live = l.rl < g.RL;
  } else {
    l.rl = 0;
    l.cv = tid;
    l.live = true;
  }
  return l;
}

// ---- forward -----------------------------------------------------------------

template <typename T, typename P, int VEC, int U, int B>
__global__ void __launch_bounds__(B, 1)
    dyt_fwd_kernel(const T *__restrict__ x, const P *__restrict__ alpha_p, const P *__restrict__ gamma,
                   const P *__restrict__ beta, T *y, Geom g) {
  using IO = VecIO<T, VEC>;
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = param(alpha_p, 0);
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    const int cc = item % g.ncc, rg = item / g.ncc;
    int64_t rb, re;
    group_rows(g.M, g.nrg, rg, rb, re);
    const int cv = cc * B + ln.cv;
    const bool col_ok = ln.live && cv < g.NV;
    if (!col_ok) continue;
    const int64_t c0 = (int64_t)cv * VEC;
    float gam[VEC], bet[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      gam[e] = param(gamma, c0 + e);
      bet[e] = param(beta, c0 + e);
    }
    const int64_t step = (int64_t)g.RL * U;
    for (int64_t r0 = rb + ln.rl; r0 < re; r0 += step) {
      typename IO::Raw raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = r0 + (int64_t)u * g.RL;
        raw[u] = row < re ? IO::load(x + row * g.N + c0) : IO::zero();
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = r0 + (int64_t)u * g.RL;
        if (row >= re) continue;
        float xf[VEC], yf[VEC];
        IO::unpack(raw[u], xf);
        bool cancel_any = false;
        bool cancel[VEC];
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const float t = dyt_tanh(alpha * xf[e]);
          yf[e] = fmaf(gam[e], t, bet[e]);
          cancel[e] = CancelGuard<T>::kOn && fabsf(yf[e]) < fabsf(gam[e] * t) * CancelGuard<T>::kTau;
          cancel_any |= cancel[e];
        }
        typename IO::Raw out = IO::pack(yf);
        if (CancelGuard<T>::kOn && cancel_any) {
#pragma unroll
          for (int e = 0; e < VEC; ++e)
            if (cancel[e]) IO::set(out, e, dyt_y_refined<T>(alpha, xf[e], gam[e], bet[e]));
        }
        IO::store_raw(y + row * g.N + c0, out);
      }
    }
  }
}

// ---- backward, stage 1 ---------------------------------------------------------

// Fixed-order tree over the RL row lanes of a CTA: lane rl absorbs lane rl + h,
// h = ceil(n / 2), until one lane is left. red[] holds B * VEC floats laid out
// by thread; afterwards lane 0's entries hold the CTA sums.
template <int VEC, int B>
__device__ __forceinline__ void lane_tree(float *red, const Geom &g, const Lane &ln) {
  for (int n = g.RL; n > 1;) {
    const int h = (n + 1) >> 1;
    if (ln.live && ln.rl < n - h) {
      const int src = (threadIdx.x + h * g.NV) * VEC;
#pragma unroll
      for (int e = 0; e < VEC; ++e) red[threadIdx.x * VEC + e] += red[src + e];
    }
    __syncthreads();
    n = h;
  }
}

template <typename T, typename P, int VEC, int U, int B>
__global__ void __launch_bounds__(B, 1)
    dyt_bwd_kernel(const T *__restrict__ x, const T *__restrict__ dy, const P *__restrict__ alpha_p,
                   const P *__restrict__ gamma, T *dx, float *__restrict__ part_dg,
                   float *__restrict__ part_db, double *__restrict__ part_da, Geom g) {
  using IO = VecIO<T, VEC>;
  __shared__ float red[B * VEC];
  __shared__ double red_a[B / 32];
  // Let the finalize kernel, launched as a programmatic dependent, get
  // scheduled early; it still waits for this grid to finish before reading.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = param(alpha_p, 0);
  double acc_a = 0.0;
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    const int cc = item % g.ncc, rg = item / g.ncc;
    int64_t rb, re;
    group_rows(g.M, g.nrg, rg, rb, re);
    const int cv = cc * B + ln.cv;
    const bool col_ok = ln.live && cv < g.NV;
    const int64_t c0 = (int64_t)cv * VEC;
    float gam[VEC], acc_g[VEC], acc_b[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      gam[e] = col_ok ? param(gamma, c0 + e) : 0.0f;
      acc_g[e] = 0.0f;
      acc_b[e] = 0.0f;
    }
    if (col_ok) {
      const int64_t step = (int64_t)g.RL * U;
      for (int64_t r0 = rb + ln.rl; r0 < re; r0 += step) {
        typename IO::Raw rx[U], rdy[U];
        bool rok[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t row = r0 + (int64_t)u * g.RL;
          rok[u] = row < re;
          rx[u] = rok[u] ? IO::load(x + row * g.N + c0) : IO::zero();
          rdy[u] = rok[u] ? IO::load(dy + row * g.N + c0) : IO::zero();
        }
        float ca = 0.0f;
#pragma unroll
        for (int u = 0; u < U; ++u) {
          float xf[VEC], dyf[VEC], dxf[VEC];
          IO::unpack(rx[u], xf);
          IO::unpack(rdy[u], dyf);
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            float t, s;
            dyt_tanh_sech2(alpha * xf[e], t, s);
            const float gdys = (gam[e] * dyf[e]) * s;  // gamma * dy * (1 - t^2)
            dxf[e] = alpha * gdys;
            // Padded rows were loaded as zeros and went through the arithmetic
            // above; their results are dropped here, after it.
            acc_g[e] = rok[u] ? fmaf(dyf[e], t, acc_g[e]) : acc_g[e];
            acc_b[e] = rok[u] ? acc_b[e] + dyf[e] : acc_b[e];
            ca = rok[u] ? fmaf(gdys, xf[e], ca) : ca;
          }
          if (rok[u]) IO::store_raw(dx + (r0 + (int64_t)u * g.RL) * g.N + c0, IO::pack(dxf));
        }
        acc_a += (double)ca;
      }
    }
    // Per-(group, column) partials.
    float *pg = part_dg + (int64_t)rg * g.N;
    float *pb = part_db + (int64_t)rg * g.N;
    if (g.RL == 1) {
      if (col_ok) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          pg[c0 + e] = acc_g[e];
          pb[c0 + e] = acc_b[e];
        }
      }
    } else {
#pragma unroll
      for (int e = 0; e < VEC; ++e) red[threadIdx.x * VEC + e] = acc_g[e];
      __syncthreads();
      lane_tree<VEC, B>(red, g, ln);
      if (col_ok && ln.rl == 0) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) pg[c0 + e] = red[threadIdx.x * VEC + e];
      }
      __syncthreads();
#pragma unroll
      for (int e = 0; e < VEC; ++e) red[threadIdx.x * VEC + e] = acc_b[e];
      __syncthreads();
      lane_tree<VEC, B>(red, g, ln);
      if (col_ok && ln.rl == 0) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) pb[c0 + e] = red[threadIdx.x * VEC + e];
      }
      __syncthreads();
    }
  }
  // dalpha partial of this CTA: warp shuffle, then warps in order.
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

// ---- backward, stage 2 -------------------------------------------------------

// Block of 256 threads = CT columns x (256 / CT) lanes. Lane l adds partials
// l, l + L, ... of its column in binary64, then a fixed-order tree adds the
// lanes; the sum is rounded once to P. Block 0 also reduces dalpha.
constexpr int kFinThreads = 256;

template <typename P>
__global__ void __launch_bounds__(kFinThreads)
    dyt_finalize_kernel(const float *__restrict__ part_dg, const float *__restrict__ part_db,
                        const double *__restrict__ part_da, P *dgamma, P *dbeta, P *dalpha,
                        int64_t N, int nrg, int nda, int CT) {
  __shared__ double sg[kFinThreads], sb[kFinThreads];
  // Wait until the stage-1 grid has finished and its writes are visible.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int tid = threadIdx.x;
  const int L = kFinThreads / CT;
  const int lane = tid / CT, c = tid - lane * CT;
  const int64_t col = (int64_t)blockIdx.x * CT + c;
  double a = 0.0, b = 0.0;
  if (col < N) {
    for (int r = lane; r < nrg; r += L) {
      a += (double)part_dg[(int64_t)r * N + col];
      b += (double)part_db[(int64_t)r * N + col];
    }
  }
  sg[tid] = a;
  sb[tid] = b;
  __syncthreads();
  for (int n = L; n > 1;) {
    const int h = (n + 1) >> 1;
    if (lane < n - h) {
      sg[tid] += sg[tid + h * CT];
      sb[tid] += sb[tid + h * CT];
    }
    __syncthreads();
    n = h;
  }
  if (lane == 0 && col < N) {
    dgamma[col] = from_f64<P>(sg[tid]);
    dbeta[col] = from_f64<P>(sb[tid]);
  }
  if (blockIdx.x == 0) {
    __syncthreads();
    double s = 0.0;
    for (int i = tid; i < nda; i += kFinThreads) s += part_da[i];
    sg[tid] = s;
    __syncthreads();
    for (int n = kFinThreads; n > 1; n >>= 1) {
      if (tid < n / 2) sg[tid] += sg[tid + n / 2];
      __syncthreads();
    }
    if (tid == 0) dalpha[0] = from_f64<P>(sg[0]);
  }
}

}  // namespace dyt
