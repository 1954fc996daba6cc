// TMA-pipelined DyT kernels for sm_100a (16-byte aligned rows).
//
// Same work decomposition, thread mapping, arithmetic and reduction order as
// the register-path kernels in dyt_kernels.cuh; only the way x (and dy) reach
// the threads differs. One thread per CTA streams tiles of whole rows into a
// ring of S shared-memory stages with 1D bulk copies (cp.async.bulk, the TMA
// engine; no multicast), each stage guarded by two mbarriers:
//   full[s]  completes when the stage's bytes have landed (expect_tx),
//   empty[s] completes when every warp has finished reading the stage.
// The data in flight lives in shared memory, not in registers, so a CTA keeps
// S tiles (up to ~190 KB) of loads outstanding while it computes.
//
// Every wait is bounded. A wait that runs out sets the CTA's abort flag and
// the library's device error word (read by dyt_device_error); from then on no
// copy is issued, no wait blocks, and before returning thread 0 waits (again
// bounded) for the copies it already issued.
#pragma once

#include <cuda_runtime.h>

#include "dyt_kernels.cuh"

namespace dyt {

// Device-wide sticky error word: bit 0 = a pipeline wait ran out.
__device__ unsigned int g_dyt_device_error = 0u;
constexpr unsigned int kErrWaitTimeout = 1u;

// ---- mbarrier and bulk-copy primitives --------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// Global -> shared bulk copy of `bytes` (multiple of 16, both addresses 16-byte
// aligned), completing on mbarrier `bar`.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(bar)
               : "memory");
}

// Bounded wait on an mbarrier phase. Returns false when it gave up (or the
// CTA had already aborted); the first give-up raises the abort flag.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t spin_limit) {
  for (uint32_t i = 0; i < spin_limit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  *abort_flag = 1;
  atomicOr(&g_dyt_device_error, kErrWaitTimeout);
  return false;
}

// ---- the tile sequence of a CTA ---------------------------------------------------

// Tiles are SR consecutive rows of one work item (column chunk x row group),
// walked item by item; producer and consumers step through the same sequence.
struct TileCursor {
  int64_t r;   // first row of the current tile
  int64_t re;  // end of the item's rows
  int item;    // current item index (blockIdx.x + k * gridDim.x)
};

__device__ __forceinline__ int item_cc(const Geom &g, int item) { return item % g.ncc; }
__device__ __forceinline__ int item_rg(const Geom &g, int item) { return item / g.ncc; }

__device__ __forceinline__ bool cursor_begin(TileCursor &c, const Geom &g, int item) {
  for (; item < g.nitems; item += gridDim.x) {
    int64_t rb, re;
    group_rows(g, item_rg(g, item), rb, re);
    c.item = item;
    c.r = rb;
    c.re = re;
    if (rb < re) return true;
  }
  c.item = g.nitems;
  return false;
}

// Advance by one tile of SR rows; returns false past the CTA's last tile.
__device__ __forceinline__ bool cursor_next(TileCursor &c, const Geom &g, int SR) {
  c.r += SR;
  if (c.r < c.re) return true;
  return cursor_begin(c, g, c.item + gridDim.x);
}

struct TmaGeom {
  int SR;          // rows per tile (= RL * U)
  int U;           // rows per row lane per tile
  int pitch;       // bytes per tile row in shared memory (one column chunk)
  int stages;      // S
  uint32_t spin;   // bounded-wait iteration limit
};

// Issue the copies of one tile (x, and dy when D is not null) into stage s.
template <typename T>
__device__ __forceinline__ void issue_tile(const TileCursor &c, const Geom &g, const TmaGeom &tg, int B,
                                           int VEC, const T *x, const T *d, char *stage, uint32_t bar) {
  const int64_t rows = (c.re - c.r) < tg.SR ? (c.re - c.r) : tg.SR;
  const int64_t col0 = (int64_t)item_cc(g, c.item) * B * VEC;
  const int64_t cols = (g.N - col0) < (int64_t)B * VEC ? (g.N - col0) : (int64_t)B * VEC;
  const uint32_t row_bytes = (uint32_t)(cols * sizeof(T));
  const uint32_t tensor_bytes = (uint32_t)rows * row_bytes;
  const uint32_t half = (uint32_t)tg.SR * (uint32_t)tg.pitch;  // dy follows x in the stage
  mbar_arrive_expect_tx(bar, d ? 2 * tensor_bytes : tensor_bytes);
  const uint32_t dst = smem_u32(stage);
  if (g.ncc == 1) {  // whole rows: one contiguous copy per tensor
    bulk_g2s(dst, x + c.r * g.N, tensor_bytes, bar);
    if (d) bulk_g2s(dst + half, d + c.r * g.N, tensor_bytes, bar);
  } else {  // one row segment per copy
    for (int64_t i = 0; i < rows; ++i) {
      bulk_g2s(dst + (uint32_t)i * tg.pitch, x + (c.r + i) * g.N + col0, row_bytes, bar);
      if (d) bulk_g2s(dst + half + (uint32_t)i * tg.pitch, d + (c.r + i) * g.N + col0, row_bytes, bar);
    }
  }
}

// Shared-memory layout of the pipelined kernels (dynamic):
//   [S stages of stage_bytes][full[S]][empty[S]][abort flag]
__device__ __forceinline__ uint32_t bar_full(char *base, const TmaGeom &tg, int stage_bytes, int s) {
  return smem_u32(base + (size_t)tg.stages * stage_bytes + 8 * s);
}
__device__ __forceinline__ uint32_t bar_empty(char *base, const TmaGeom &tg, int stage_bytes, int s) {
  return smem_u32(base + (size_t)tg.stages * stage_bytes + 8 * (tg.stages + s));
}

template <int B>
__device__ __forceinline__ volatile int *pipeline_setup(char *base, const TmaGeom &tg, int stage_bytes) {
  volatile int *abort_flag = (volatile int *)(base + (size_t)tg.stages * stage_bytes + 16 * tg.stages);
  if (threadIdx.x == 0) {
    for (int s = 0; s < tg.stages; ++s) {
      mbar_init(bar_full(base, tg, stage_bytes, s), 1);
      mbar_init(bar_empty(base, tg, stage_bytes, s), B / 32);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  return abort_flag;
}

// Thread 0, before the CTA exits: wait (bounded) until every copy it issued has
// landed, so no copy can still target this CTA's shared memory afterwards.
__device__ __forceinline__ void pipeline_drain(char *base, const TmaGeom &tg, int stage_bytes, int64_t issued,
                                               int64_t consumed, volatile int *abort_flag) {
  for (int64_t k = consumed; k < issued; ++k) {
    const int s = (int)(k % tg.stages);
    const uint32_t parity = (uint32_t)((k / tg.stages) & 1);
    const uint32_t bar = bar_full(base, tg, stage_bytes, s);
    for (uint32_t i = 0; i < tg.spin; ++i)
      if (mbar_try_wait(bar, parity)) break;
  }
  (void)abort_flag;
}

// Stage index and phase parity of the k-th tile, carried incrementally.
struct Ring {
  int s = 0;
  uint32_t parity = 0;
  __device__ __forceinline__ void next(int stages) {
    if (++s == stages) {
      s = 0;
      parity ^= 1u;
    }
  }
};

// Producer state, touched by thread 0 only (kept in shared memory so that it
// costs the other threads no registers).
struct Producer {
  TileCursor cur;
  int64_t issued, consumed;
  int more;
};

// ---- forward ----------------------------------------------------------------------

template <typename T, typename P, int VEC, int B>
__global__ void __launch_bounds__(B, 1)
    dyt_fwd_tma_kernel(const T *__restrict__ x, const P *__restrict__ alpha_p, const P *__restrict__ gamma,
                       const P *__restrict__ beta, T *y, Geom g, TmaGeom tg) {
  using IO = VecIO<T, VEC>;
  extern __shared__ __align__(128) char smem[];
  __shared__ Producer prod;
  pdl_prologue();
  const int stage_bytes = tg.SR * tg.pitch;
  volatile int *abort_flag = pipeline_setup<B>(smem, tg, stage_bytes);
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = param(alpha_p, 0);
  if (threadIdx.x == 0) {  // fill the ring
    prod.issued = prod.consumed = 0;
    prod.more = cursor_begin(prod.cur, g, blockIdx.x);
    for (int s = 0; s < tg.stages && prod.more; ++s) {
      issue_tile<T>(prod.cur, g, tg, B, VEC, x, (const T *)nullptr,
                    smem + (size_t)s * stage_bytes, bar_full(smem, tg, stage_bytes, s));
      ++prod.issued;
      prod.more = cursor_next(prod.cur, g, tg.SR);
    }
  }
  TileCursor cons;
  Ring ring;
  bool more = cursor_begin(cons, g, blockIdx.x);
  int cur_item = -1;
  float gam[VEC], bet[VEC], bth[VEC];
  int64_t c0 = 0;
  bool col_ok = false;
  while (more) {
    if (cons.item != cur_item) {  // new item: this thread's columns and parameters
      cur_item = cons.item;
      const int cv = item_cc(g, cur_item) * B + ln.cv;
      col_ok = ln.live && cv < g.NV;
      c0 = (int64_t)cv * VEC;
      fwd_params<T, P, VEC>(gamma, beta, c0, col_ok, gam, bet, bth);
    }
    const bool have = mbar_wait(bar_full(smem, tg, stage_bytes, ring.s), ring.parity, abort_flag, tg.spin);
    if (have && col_ok) {
      const char *st = smem + (size_t)ring.s * stage_bytes + (size_t)ln.cv * (VEC * sizeof(T));
      for (int u = 0; u < tg.U; ++u) {
        const int ri = ln.rl + u * g.RL;
        const int64_t row = cons.r + ri;
        if (row < cons.re) {
          const typename IO::Raw rx = *(const typename IO::Raw *)(st + (size_t)ri * tg.pitch);
          IO::store_raw(y + row * g.N + c0, fwd_vector<T, VEC>(rx, alpha, gam, bet, bth));
        }
      }
    }
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar_empty(smem, tg, stage_bytes, ring.s));
    if (threadIdx.x == 0) {
      ++prod.consumed;
      if (prod.more && !*abort_flag &&
          mbar_wait(bar_empty(smem, tg, stage_bytes, ring.s), ring.parity, abort_flag, tg.spin)) {
        // every warp has released this stage: refill it
        issue_tile<T>(prod.cur, g, tg, B, VEC, x, (const T *)nullptr, smem + (size_t)ring.s * stage_bytes,
                      bar_full(smem, tg, stage_bytes, ring.s));
        ++prod.issued;
        prod.more = cursor_next(prod.cur, g, tg.SR);
      }
    }
    ring.next(tg.stages);
    more = cursor_next(cons, g, tg.SR);
  }
  if (threadIdx.x == 0) pipeline_drain(smem, tg, stage_bytes, prod.issued, prod.consumed, abort_flag);
}

// ---- backward, stage 1 ---------------------------------------------------------

template <typename T, typename P, int VEC, int B>
__global__ void __launch_bounds__(B, 1)
    dyt_bwd_tma_kernel(const T *__restrict__ x, const T *__restrict__ dy, const P *__restrict__ alpha_p,
                       const P *__restrict__ gamma, T *dx, float *__restrict__ part_dg,
                       float *__restrict__ part_db, double *__restrict__ part_da, Geom g, TmaGeom tg) {
  using IO = VecIO<T, VEC>;
  extern __shared__ __align__(128) char smem[];
  __shared__ float red[VEC * B];
  __shared__ double red_a[B / 32];
  __shared__ Producer prod;
  pdl_prologue();
  const int stage_bytes = 2 * tg.SR * tg.pitch;
  volatile int *abort_flag = pipeline_setup<B>(smem, tg, stage_bytes);
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = param(alpha_p, 0);
  if (threadIdx.x == 0) {  // fill the ring
    prod.issued = prod.consumed = 0;
    prod.more = cursor_begin(prod.cur, g, blockIdx.x);
    for (int s = 0; s < tg.stages && prod.more; ++s) {
      issue_tile<T>(prod.cur, g, tg, B, VEC, x, dy, smem + (size_t)s * stage_bytes,
                    bar_full(smem, tg, stage_bytes, s));
      ++prod.issued;
      prod.more = cursor_next(prod.cur, g, tg.SR);
    }
  }
  double acc_a = 0.0;
  TileCursor cons;
  Ring ring;
  bool more = cursor_begin(cons, g, blockIdx.x);
  while (more) {
    // ---- one work item: this thread's columns, fresh sums ----
    const int item = cons.item;
    const int cv = item_cc(g, item) * B + ln.cv;
    const bool col_ok = ln.live && cv < g.NV;
    const int64_t c0 = (int64_t)cv * VEC;
    float gam[VEC];
    BwdAcc<VEC> acc;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      gam[e] = col_ok ? 4.0f * param(gamma, c0 + e) : 0.0f;  // 4 gamma (see bwd_vector)
      acc.g[e] = 0.0f;
      acc.b[e] = 0.0f;
    }
    while (more && cons.item == item) {
      const bool have = mbar_wait(bar_full(smem, tg, stage_bytes, ring.s), ring.parity, abort_flag, tg.spin);
      if (have && col_ok) {
        const char *st = smem + (size_t)ring.s * stage_bytes + (size_t)ln.cv * (VEC * sizeof(T));
        const char *sd = st + (size_t)tg.SR * tg.pitch;
        const bool full_tile = cons.r + (int64_t)(tg.SR - 1) < cons.re;
        float2 ca = make_float2(0.0f, 0.0f);
        for (int u = 0; u < tg.U; ++u) {
          const int ri = ln.rl + u * g.RL;
          const int64_t row = cons.r + ri;
          const typename IO::Raw rx = *(const typename IO::Raw *)(st + (size_t)ri * tg.pitch);
          const typename IO::Raw rd = *(const typename IO::Raw *)(sd + (size_t)ri * tg.pitch);
          if (full_tile) {
            IO::store_raw(dx + row * g.N + c0, bwd_vector<T, VEC, false>(rx, rd, alpha, gam, acc, ca, VEC));
          } else {  // the item's last, ragged tile: padded rows are dropped after the arithmetic
            const bool ok = row < cons.re;
            const typename IO::Raw o = bwd_vector<T, VEC, true>(rx, rd, alpha, gam, acc, ca, ok ? VEC : 0);
            if (ok) IO::store_raw(dx + row * g.N + c0, o);
          }
        }
        acc_a += (double)ca.x;
        acc_a += (double)ca.y;
      }
      __syncwarp();
      if ((threadIdx.x & 31) == 0) mbar_arrive(bar_empty(smem, tg, stage_bytes, ring.s));
      if (threadIdx.x == 0) {
        ++prod.consumed;
        if (prod.more && !*abort_flag &&
            mbar_wait(bar_empty(smem, tg, stage_bytes, ring.s), ring.parity, abort_flag, tg.spin)) {
          issue_tile<T>(prod.cur, g, tg, B, VEC, x, dy, smem + (size_t)ring.s * stage_bytes,
                        bar_full(smem, tg, stage_bytes, ring.s));
          ++prod.issued;
          prod.more = cursor_next(prod.cur, g, tg.SR);
        }
      }
      ring.next(tg.stages);
      more = cursor_next(cons, g, tg.SR);
    }
    // ---- item done: per-(group, column) partials ----
    const int rg = item_rg(g, item);
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
  if (threadIdx.x == 0) pipeline_drain(smem, tg, stage_bytes, prod.issued, prod.consumed, abort_flag);
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

// ---- self-test of the bounded wait -----------------------------------------------

// Waits on an mbarrier phase that nothing completes, with the given limit; the
// wait must give up, raise the device error word and return.
__global__ void dyt_wait_timeout_selftest_kernel(uint32_t spin_limit, int *gave_up) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  const bool ok = mbar_wait(smem_u32(&bar), 0, (volatile int *)&abort_flag, spin_limit);
  if (threadIdx.x == 0) *gave_up = ok ? 0 : 1;
}

}  // namespace dyt
