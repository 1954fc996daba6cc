// Per-thread asynchronous-copy DyT kernels for sm_100a (16-byte vectors): the
// kernels every 16-byte aligned matrix takes.
//
// Same decomposition, thread mapping and arithmetic as the one-element
// kernels in dyt_kernels.cuh; the row lanes of a CTA are added by a register
// reduce-scatter when NV divides 32, otherwise by the same fixed-order tree.
// Each thread streams the rows it owns
// (its VEC columns of rows rl, rl + RL, ... of the group) into a private ring
// of S shared-memory slots with 16-byte asynchronous copies (cp.async.cg, L2
// only), S - 1 rows ahead of the row it computes, and reads each slot back
// after cp.async.wait_group. A thread only ever reads slots it filled itself,
// so no barrier is needed between threads; the data in flight (up to
// (S - 1) x 32 bytes per thread) costs no registers. Each thread visits
// exactly its real rows; only the one vector that straddles the end of a
// packed matrix holds padding, which is masked after the arithmetic.
#pragma once

#include <cuda_runtime.h>

#include "dyt_kernels.cuh"

namespace dyt {

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
// The same copy reading only the first src_bytes (0..16) of the source and
// zero-filling the rest of the slot: nothing past src + src_bytes is read.
__device__ __forceinline__ void cp_async16_zfill(void *smem_dst, const void *gmem_src, uint32_t src_bytes) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gmem_src), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Matrix columns of the VEC elements of the vector at offset c0 of a row:
// c0 + e, or on the packed path (c0 + e) mod Nc, where c0 < VEC * Nc.
template <int VEC, bool PK>
__device__ __forceinline__ void vector_columns(int64_t c0, int64_t Nc, int64_t (&col)[VEC]) {
  if constexpr (PK) {
    int64_t c = c0;
    while (c >= Nc) c -= Nc;  // at most VEC - 1 times
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      col[e] = c;
      c = c + 1 == Nc ? 0 : c + 1;
    }
  } else {
#pragma unroll
    for (int e = 0; e < VEC; ++e) col[e] = c0 + e;
  }
}

// The first n (< VEC) elements of a 16-byte vector, one by one: the vector
// that straddles the end of a packed matrix.
template <typename T, int VEC>
__device__ __forceinline__ void store_first(T *p, const uint4 &r, int n) {
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    if (e < n) {
      if constexpr (sizeof(T) == 4) {
        *reinterpret_cast<uint32_t *>(p + e) = word_of(r, e);
      } else {
        const uint32_t u = word_of(r, e >> 1);
        *reinterpret_cast<unsigned short *>(p + e) = (unsigned short)((e & 1) ? (u >> 16) : (u & 0xFFFFu));
      }
    }
  }
}

// Start pulling into L2 the rows this CTA copies first: those of its first
// work item, at most as many as the rings hold (S - 1 steps). This runs before
// griddepcontrol.wait, while the preceding grid may still be writing. That is
// safe: a prefetch changes no memory state, and the ring copies after the wait
// read L2 (cp.async.cg), so a line written later is read in its final state.
// Rows are 16-byte aligned on this path, so every range below is too. ld: the
// tensor's row pitch in elements.
template <typename T, int VEC, int B, int S, bool PK>
__device__ __forceinline__ void prefetch_first_rows_l2(const T *p, int64_t ld, const Geom &g) {
  if (!g.l2_prefetch || threadIdx.x >= 32 || (int)blockIdx.x >= g.nitems) return;  // warp 0 issues them
  int cc, rg;
  item_split(g, blockIdx.x, cc, rg);
  int64_t rb, re;
  group_rows(g, rg, rb, re);
  const int64_t rows = min(re - rb, (int64_t)(S - 1) * g.RL);
  if (rows <= 0) return;
  constexpr uint32_t kPiece = 16384;
  // Ranges end at the matrix's last element (a packed matrix's last row may
  // be short) and are rounded down to whole 16-byte units.
  if (g.ncc == 1 && ld == g.N) {  // whole, adjacent rows: one range, cut into pieces
    const int64_t bytes = (min(rows * g.N, g.total - rb * g.N) * (int64_t)sizeof(T)) & ~(int64_t)15;
    const int64_t k = threadIdx.x;
    if (k * kPiece < bytes) {
      const uint32_t n = (uint32_t)min((int64_t)kPiece, bytes - k * kPiece);
      const char *a = reinterpret_cast<const char *>(p + rb * g.N) + k * kPiece;
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
    }
  } else if (threadIdx.x < rows) {  // one column chunk of each row
    const int64_t c0 = (int64_t)cc * B * VEC;
    const int64_t at = (rb + threadIdx.x) * ld + c0;
    int64_t n = min((int64_t)B * VEC, g.N - c0);
    if (PK) n = min(n, g.total - at);  // packed rows are adjacent (ld = N)
    n = (n * (int64_t)sizeof(T)) & ~(int64_t)15;
    if (n > 0)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p + at), "r"((uint32_t)n) : "memory");
  }
}

// Rows of the current item owned by this thread: first row and count. A group
// has at most kMaxRowsPerLane * RL rows (the host caps it), so the quotient is
// formed with the host's multiply-high constant, exactly, instead of a 64-bit
// division.
__device__ __forceinline__ int64_t thread_rows(const Geom &g, int64_t rb, int64_t re, int rl, int64_t &first) {
  first = rb + rl;
  if (first >= re) return 0;
  const uint32_t n = (uint32_t)(re - first) + (uint32_t)(g.RL - 1);
  return g.RL == 1 ? (int64_t)n : (int64_t)__umulhi(n, g.rl_magic);
}

// ---- forward ------------------------------------------------------------------

// Real elements of the vector at offset c0 of (packed) row `row`: VEC, except
// in the vector that straddles the end of a packed matrix; 0 past it.
__device__ __forceinline__ int64_t vector_real(const Geom &g, int64_t row, int64_t c0) {
  return g.total - (row * g.N + c0);
}

// Trims a thread's row count on the packed path: drops a last vector that
// lies wholly past the matrix and returns the real elements of the last one
// (VEC when it is whole).
template <int VEC, bool PK>
__device__ __forceinline__ int last_vector_real(const Geom &g, int64_t first, int64_t c0, int64_t &n) {
  if (!PK || n <= 0) return VEC;
  const int64_t r = vector_real(g, first + (n - 1) * g.RL, c0);
  if (r <= 0) {
    --n;  // only the matrix's last pack is short, so the one before is whole
    return VEC;
  }
  return r < VEC ? (int)r : VEC;
}

template <typename T, typename P, int VEC, int B, int S, bool PK>
__global__ void __launch_bounds__(B, 1)
    dyt_fwd_async_kernel(const T *__restrict__ x, const P *__restrict__ alpha_p, const P *__restrict__ gamma_p,
                         const P *__restrict__ beta_p, ParamTypes pt, T *y, Geom g) {
  using IO = VecIO<T, VEC>;
  static_assert(VEC * sizeof(T) == 16, "16-byte vectors");
  extern __shared__ uint4 ring[];  // [S][B]
  prefetch_first_rows_l2<T, VEC, B, S, PK>(x, g.ldx, g);
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = load_param<P>(alpha_p, pt.alpha, 0);
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
    int64_t n = thread_rows(g, rb, re, ln.rl, first);
    const int nl = last_vector_real<VEC, PK>(g, first, c0, n);
    const uint32_t last_bytes = (uint32_t)(nl * (int)sizeof(T));
    const int64_t sx = (int64_t)g.RL * g.ldx, sy = (int64_t)g.RL * g.ldo;
    const T *px = x + first * g.ldx + c0;
    T *py = y + first * g.ldo + c0;
    // Rows first, parameters second: the parameter loads overlap the copies.
#pragma unroll
    for (int k = 0; k < S - 1; ++k) {
      if (k < n) {
        if (PK) cp_async16_zfill(slot0 + k * B, px + k * sx, k == n - 1 ? last_bytes : 16u);
        else cp_async16(slot0 + k * B, px + k * sx);
      }
      cp_async_commit();
    }
    int64_t col[VEC];
    vector_columns<VEC, PK>(c0, g.Nc, col);
    float gam[VEC], bet[VEC], bth[VEC];
    fwd_params_at<T, VEC, P>(gamma_p, beta_p, pt, col, gam, bet, bth);
    int s_rd = 0, s_wr = S - 1;
    for (int64_t k = 0; k < n; ++k) {
      const int64_t kn = k + S - 1;
      if (kn < n) {
        if (PK) cp_async16_zfill(slot0 + s_wr * B, px + kn * sx, kn == n - 1 ? last_bytes : 16u);
        else cp_async16(slot0 + s_wr * B, px + kn * sx);
      }
      cp_async_commit();
      cp_async_wait<S - 1>();
      const typename IO::Raw rx = *(const typename IO::Raw *)(slot0 + s_rd * B);
      const typename IO::Raw ry = fwd_vector<T, VEC>(rx, alpha, gam, bet, bth);
      if (PK && k == n - 1 && nl < VEC) store_first<T, VEC>(py, ry, nl);  // zero-filled tail: not stored
      else IO::store_raw(py, ry);
      py += sy;
      s_rd = s_rd + 1 == S ? 0 : s_rd + 1;
      s_wr = s_wr + 1 == S ? 0 : s_wr + 1;
    }
    cp_async_wait<0>();
  }
}

// ---- backward, stage 1 ----------------------------------------------------------

template <typename T, typename P, int VEC, int B, int S, bool PK>
__global__ void __launch_bounds__(B, 1)
    dyt_bwd_async_kernel(const T *__restrict__ x, const T *__restrict__ dy, const P *__restrict__ alpha_p,
                         const P *__restrict__ gamma_p, ParamTypes pt, T *dx, double *__restrict__ part_dg,
                         double *__restrict__ part_db, double *__restrict__ part_da, Geom g) {
  using IO = VecIO<T, VEC>;
  constexpr bool EXACT_G = ExactGamma<T>::value;
  constexpr int kRunBlocks = kGammaRunRows / S;  // unrolled blocks of S rows per binary32 dgamma run
  static_assert(VEC * sizeof(T) == 16, "16-byte vectors");
  static_assert(2 * VEC * sizeof(double) <= 2 * S * 16, "the reduction fits in the drained ring");
  static_assert(kRunBlocks >= 1, "a dgamma run holds at least one block");
  // [S][2][B] 16-byte slots; after an item's last row the ring is empty and
  // its first 2 VEC * B binary64 values (at most 64 KB) serve the row-lane
  // reduction. Without EXACT_G, [VEC][B] binary64 dgamma totals follow the
  // ring (each thread's own, flushed from its binary32 runs).
  extern __shared__ uint4 ring[];
  __shared__ double red_a[B / 32];
  prefetch_first_rows_l2<T, VEC, B, S, PK>(x, g.ldx, g);
  prefetch_first_rows_l2<T, VEC, B, S, PK>(dy, g.ldd, g);
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = load_param<P>(alpha_p, pt.alpha, 0);
  double *red = reinterpret_cast<double *>(ring);
  double *gtot = reinterpret_cast<double *>(ring + 2 * S * B) + threadIdx.x;  // [e * B]
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
    BwdAcc<VEC, EXACT_G> acc;
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      acc.g[e] = 0;
      acc.b[e] = 0.0;
      if (!EXACT_G) gtot[e * B] = 0.0;
    }
    if (col_ok) {
      int64_t first;
      int64_t n = thread_rows(g, rb, re, ln.rl, first);
      const int nl = last_vector_real<VEC, PK>(g, first, c0, n);
      const uint32_t last_bytes = (uint32_t)(nl * (int)sizeof(T));
      const int nn = (int)n;  // at most kMaxRowsPerLane: the host caps a group's rows per lane
      const int64_t sx = (int64_t)g.RL * g.ldx, sd = (int64_t)g.RL * g.ldd, so = (int64_t)g.RL * g.ldo;
      const T *px = x + first * g.ldx + c0;  // the next rows to copy (advanced, not re-derived)
      const T *pd = dy + first * g.ldd + c0;
      T *pdx = dx + first * g.ldo + c0;
      // Rows first, parameters second: the gamma loads overlap the copies.
      // Row r lives in slot r mod S; the loop below is unrolled by S so that
      // every slot index is a constant.
#pragma unroll
      for (int k = 0; k < S - 1; ++k) {
        if (k < nn) {
          if (PK) {
            const uint32_t b = k == nn - 1 ? last_bytes : 16u;
            cp_async16_zfill(slot0 + (2 * k) * B, px, b);
            cp_async16_zfill(slot0 + (2 * k + 1) * B, pd, b);
          } else {
            cp_async16(slot0 + (2 * k) * B, px);
            cp_async16(slot0 + (2 * k + 1) * B, pd);
          }
        }
        px += sx;
        pd += sd;
        cp_async_commit();
      }
      int64_t col[VEC];
      vector_columns<VEC, PK>(c0, g.Nc, col);
      load_params<VEC, P>(gamma_p, pt.gamma, col, 4.0f, gam);  // 4 gamma (see bwd_vector)
      int run = 0;  // blocks in the current binary32 dgamma run
      for (int k0 = 0; k0 < nn; k0 += S) {
        float2 ca = make_float2(0.0f, 0.0f);  // this block's dalpha terms (at most S VEC / 2 per lane)
#pragma unroll
        for (int j = 0; j < S; ++j) {
          const int k = k0 + j;
          if (k >= nn) break;
          if (k + S - 1 < nn) {  // rows k + S - 1 into slot (j + S - 1) mod S
            const int sw = (j + S - 1) % S;
            if (PK) {
              const uint32_t b = k + S - 1 == nn - 1 ? last_bytes : 16u;
              cp_async16_zfill(slot0 + (2 * sw) * B, px, b);
              cp_async16_zfill(slot0 + (2 * sw + 1) * B, pd, b);
            } else {
              cp_async16(slot0 + (2 * sw) * B, px);
              cp_async16(slot0 + (2 * sw + 1) * B, pd);
            }
          }
          px += sx;
          pd += sd;
          cp_async_commit();
          cp_async_wait<S - 1>();
          const typename IO::Raw rx = *(const typename IO::Raw *)(slot0 + (2 * j) * B);
          const typename IO::Raw rd = *(const typename IO::Raw *)(slot0 + (2 * j + 1) * B);
          if (PK && k == nn - 1 && nl < VEC) {  // the straddling vector: its zero-filled tail is dropped
            store_first<T, VEC>(pdx, bwd_vector<T, VEC, true, EXACT_G>(rx, rd, alpha, gam, acc, ca, nl), nl);
          } else {
            IO::store_raw(pdx, bwd_vector<T, VEC, false, EXACT_G>(rx, rd, alpha, gam, acc, ca, VEC));
          }
          pdx += so;
        }
        acc_a += (double)ca.x;
        acc_a += (double)ca.y;
        if (!EXACT_G && ++run == kRunBlocks) {  // end of a binary32 dgamma run
          run = 0;
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            gtot[e * B] += (double)acc.g[e];
            acc.g[e] = 0;
          }
        }
      }
      cp_async_wait<0>();
    }
    // ---- item done: per-(group, column) partials ----
    double ag[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) ag[e] = EXACT_G ? (double)acc.g[e] : gtot[e * B] + (double)acc.g[e];
    double *pg = part_dg + (int64_t)rg * g.N;
    double *pb = part_db + (int64_t)rg * g.N;
    if (g.RL == 1) {
      if (col_ok) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          pg[c0 + e] = ag[e];
          pb[c0 + e] = acc.b[e];
        }
      }
    } else {
      __syncthreads();  // every thread's ring is drained: reuse it for the reduction
      if ((32 % g.NV) == 0) {
        // the chunk's columns start at 0 on the row-tiled path (one chunk)
        lane_reduce_warps<VEC, B>(ag, acc.b, red, g, ln, 0, pg, pb);
      } else {  // dgamma and dbeta sums in one tree: 2 VEC values per thread
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          red[e * B + threadIdx.x] = ag[e];
          red[(VEC + e) * B + threadIdx.x] = acc.b[e];
        }
        __syncthreads();
        lane_tree<2 * VEC, B>(red, g, ln);
        if (col_ok && ln.rl == 0) {
#pragma unroll
          for (int e = 0; e < VEC; ++e) {
            pg[c0 + e] = red[e * B + threadIdx.x];
            pb[c0 + e] = red[(VEC + e) * B + threadIdx.x];
          }
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
