// The DyT backward's finalize kernel (stage 2): the binary64 partial sums of
// one or several stage-1 launches (ranks) added in a fixed order and rounded
// once per gradient. Kept apart from the stage-1 kernels so that only the
// translation unit that launches it defines it.
#pragma once

#include "dyt_kernels.cuh"

namespace dyt {

// ---- backward, stage 2 -------------------------------------------------------

// The binary64 partial sums that one stage-1 launch left, possibly in another
// GPU's memory (a peer mapping): rows x N dgamma and dbeta partials, nda dalpha
// partials.
constexpr int kMaxRanks = 8;
struct RankParts {
  const double *dg;
  const double *db;
  const double *da;
  int rows;
  int nda;
};
struct PartsSet {
  RankParts r[kMaxRanks];
  int nranks;
};

// Block of 256 threads = CT columns x L lanes (L = 256 / CT, chosen on the host
// so that a lane reads at most a few partials of a rank), thread = lane * CT +
// column. For each rank in order, lane l adds that rank's partials l, l + L,
// ... of its column in binary64, in that order; each batch of four is loaded
// before any is added, so a lane waits for one round trip per batch. The lanes
// of a column are then added by a fixed-order warp butterfly (lanes CT apart
// share a warp when CT < 32) and the warps' results by one thread per column,
// in warp order: the rank's column total. The ranks' totals are added in rank
// order (the first one starts the sum), and the result is rounded once to the
// gradient's dtype. The last block also reduces dalpha the same way. With one
// rank this is the single-GPU finalize; with several it is the cross-GPU sum of
// a row-sharded backward, each rank's partials read through peer loads.
constexpr int kFinThreads = 256;

__device__ __forceinline__ double fin_rank_column(const RankParts &rp, int64_t N, int64_t col, int lane, int L,
                                                  bool ok, double &b_out) {
  double a = 0.0, b = 0.0;
  if (ok) {
    for (int r = lane; r < rp.rows; r += 4 * L) {
      double va[4], vb[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int rk = r + k * L;
        va[k] = rk < rp.rows ? rp.dg[(int64_t)rk * N + col] : 0.0;  // + 0 leaves a sum unchanged
        vb[k] = rk < rp.rows ? rp.db[(int64_t)rk * N + col] : 0.0;
      }
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        a += va[k];
        b += vb[k];
      }
    }
  }
  b_out = b;
  return a;
}

__global__ void __launch_bounds__(kFinThreads)
    dyt_finalize_kernel(PartsSet ps, GradOut out, int64_t N, int CT) {
  __shared__ double sg[kFinThreads], sb[kFinThreads], sa[kFinThreads / 32];
  // Wait until the stage-1 grid has finished and its writes are visible, then
  // let the next grid in the stream get scheduled (it waits for this one to
  // finish before touching memory).
  pdl_prologue();
  const int tid = threadIdx.x;
  const int L = kFinThreads / CT;
  const int lane = tid / CT, c = tid - lane * CT;
  const int64_t col = (int64_t)blockIdx.x * CT + c;
  const bool da_block = blockIdx.x == gridDim.x - 1;
  const int stride = CT < 32 ? 32 : CT;  // one value per warp and column (CT < 32), else one per lane
  double tg = 0.0, tb = 0.0, ta = 0.0;   // the ranks' totals so far (threads tid < CT, and 0 for dalpha)
  for (int r = 0; r < ps.nranks; ++r) {
    const RankParts &rp = ps.r[r];
    // dalpha partials: thread i adds i, i + 256, ...; the first is loaded here
    // and added only after the column loads below are under way.
    const double da0 = da_block && tid < rp.nda ? rp.da[tid] : 0.0;
    double b;
    double a = fin_rank_column(rp, N, col, lane, L, col < N, b);
    // Lanes of a column within a warp: a butterfly (both partners of an
    // exchange form the same sum, so every lane ends with identical bits).
    for (int off = CT; off < 32; off <<= 1) {
      a += __shfl_xor_sync(0xFFFFFFFFu, a, off);
      b += __shfl_xor_sync(0xFFFFFFFFu, b, off);
    }
    if (r > 0) __syncthreads();  // the previous rank's totals have been read
    sg[tid] = a;
    sb[tid] = b;
    if (da_block) {
      double da = 0.0 + da0;
      for (int i = tid + kFinThreads; i < rp.nda; i += kFinThreads) da += rp.da[i];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) da += __shfl_xor_sync(0xFFFFFFFFu, da, off);
      if ((tid & 31) == 0) sa[tid >> 5] = da;
    }
    __syncthreads();
    if (tid < CT && col < N) {
      double sgc = 0.0, sbc = 0.0;
      for (int k = 0; k < kFinThreads / stride; ++k) {
        sgc += sg[k * stride + tid];
        sbc += sb[k * stride + tid];
      }
      tg = r == 0 ? sgc : tg + sgc;
      tb = r == 0 ? sbc : tb + sbc;
    }
    if (da_block && tid == 0) {
      double s = 0.0;
      for (int w = 0; w < kFinThreads / 32; ++w) s += sa[w];
      ta = r == 0 ? s : ta + s;
    }
  }
  if (tid < CT && col < N) {
    store_param(out.dgamma, out.gamma_dt, col, tg);
    store_param(out.dbeta, out.beta_dt, col, tb);
  }
  if (da_block && tid == 0) store_param(out.dalpha, out.alpha_dt, 0, ta);
}

}  // namespace dyt
