// C ABI of the fused DyT layer (declared in include/dyt.h): argument checks,
// launch planning and kernel dispatch. All device work is in the kernels of
// dyt_kernels.cuh, dyt_async.cuh and dyt_tma.cuh.
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "dyt.h"
#include "dyt_kernels.cuh"
#include "dyt_tma.cuh"
#include "dyt_async.cuh"

namespace {

using dyt::Geom;

thread_local dyt_launch_info t_info = {};
thread_local int t_cuda_err = 0;

// Tuning constants (compile-time; -D overrides them for sweeps).
#ifndef DYT_FWD_UNROLL_VEC
#define DYT_FWD_UNROLL_VEC 2
#endif
#ifndef DYT_BWD_UNROLL_VEC
#define DYT_BWD_UNROLL_VEC 2
#endif
#ifndef DYT_FWD_UNROLL_SCALAR
#define DYT_FWD_UNROLL_SCALAR 8
#endif
#ifndef DYT_BWD_UNROLL_SCALAR
#define DYT_BWD_UNROLL_SCALAR 8
#endif
// Pipeline of the 16-byte aligned path: 0 = loads into registers, 1 = CTA-wide
// bulk-copy (TMA) ring, 2 = per-thread asynchronous-copy ring.
#ifndef DYT_PIPE
#define DYT_PIPE 2
#endif
#define DYT_USE_TMA (DYT_PIPE == 1)
#ifndef DYT_ASYNC_STAGES_FWD
#define DYT_ASYNC_STAGES_FWD 8
#endif
#ifndef DYT_ASYNC_STAGES_BWD
#define DYT_ASYNC_STAGES_BWD 6
#endif
#ifndef DYT_TILE_BYTES
#define DYT_TILE_BYTES 32768
#endif
#ifndef DYT_MAX_STAGES
#define DYT_MAX_STAGES 8
#endif
// Inputs read by one launch below which the L2 prefetch of the first rows is
// skipped (bytes).
#ifndef DYT_PREFETCH_MIN_BYTES
#define DYT_PREFETCH_MIN_BYTES (1 << 20)
#endif
constexpr int kBlock = 1024;          // threads per CTA of the main kernels
constexpr uint32_t kSpinLimit = 1u << 22;  // bounded mbarrier waits (iterations)
constexpr int kMaxDynSmem = 227 * 1024;
#ifndef DYT_ASYNC_BLOCK
#define DYT_ASYNC_BLOCK 512
#endif
constexpr int kAsyncBlock = DYT_ASYNC_BLOCK;  // one CTA per SM: up to 128 registers a thread
constexpr int kAsyncStagesFwd = DYT_ASYNC_STAGES_FWD;
constexpr int kAsyncStagesBwd = DYT_ASYNC_STAGES_BWD;
constexpr int kMaxRowsPerLane = 128;  // sequential binary32 adds per thread per group
constexpr int64_t kPrefetchMinBytes = DYT_PREFETCH_MIN_BYTES;

constexpr int kFwdUnrollVec = DYT_FWD_UNROLL_VEC;        // rows in flight per thread, 16-byte access
constexpr int kBwdUnrollVec = DYT_BWD_UNROLL_VEC;
constexpr int kFwdUnrollScalar = DYT_FWD_UNROLL_SCALAR;  // rows in flight per thread, scalar access
constexpr int kBwdUnrollScalar = DYT_BWD_UNROLL_SCALAR;

dyt_status cuda_fail(cudaError_t e) {
  t_cuda_err = (int)e;
  return DYT_ERR_CUDA;
}

size_t dsize(dyt_dtype d) { return d == DYT_F32 ? 4 : 2; }
bool valid_dtype(int d) { return d == DYT_F32 || d == DYT_BF16 || d == DYT_F16; }
bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- per-device facts and per-kernel occupancy (cached, thread-safe) -------

std::mutex g_mu;
std::unordered_map<int, int> g_sms;                   // device -> SM count
std::unordered_map<uint64_t, int> g_occ;              // (device, kernel) -> CTAs per SM

dyt_status current_sms(int *dev_out, int *sms_out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_sms.find(dev);
    if (it != g_sms.end()) {
      *dev_out = dev;
      *sms_out = it->second;
      return DYT_OK;
    }
  }
  int sms = 0;
  e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(g_mu);
  g_sms[dev] = sms;
  *dev_out = dev;
  *sms_out = sms;
  return DYT_OK;
}

dyt_status occupancy(int dev, const void *kernel, int block, int *ctas) {
  const uint64_t key = ((uint64_t)(uint32_t)dev << 48) ^ (uint64_t)(uintptr_t)kernel;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_occ.find(key);
    if (it != g_occ.end()) {
      *ctas = it->second;
      return DYT_OK;
    }
  }
  int n = 0;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, block, 0);
  if (e != cudaSuccess) return cuda_fail(e);
  if (n < 1) n = 1;
  std::lock_guard<std::mutex> lk(g_mu);
  g_occ[key] = n;
  *ctas = n;
  return DYT_OK;
}

// ---- launch plan ---------------------------------------------------------------

struct Plan {
  Geom g;
  int block;  // threads per CTA of the main kernel
  int vec;
  int unroll;
  int grid;
  int path;
  bool tma;
  bool async;
  bool packed;  // ragged N on 16-byte aligned rows: packs of vec rows (see dyt_kernels.cuh)
  bool too_big; // the group or item count would not fit the kernels' int indices
  dyt::TmaGeom tg;
  size_t smem;  // dynamic shared memory of the pipelined kernel
  size_t ws_dg, ws_db, ws_da, ws_total;  // workspace byte offsets / sizes
};

size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

// vec: elements per access (1 or 16 / element size). ctas_per_sm from the
// kernel's occupancy. packed: N is not a multiple of vec, and the matrix is
// laid out as ceil(M / vec) packs of vec rows, each of pitch vec * N. The
// plan depends only on (M, N, vec, packed, SM count, occupancy).
Plan make_plan(int64_t M_rows, int64_t N_cols, int vec, bool backward, int sms, int ctas_per_sm,
               int block = kBlock, bool packed = false, int64_t elem_bytes = 4) {
  Plan p = {};
  p.block = block;
  p.vec = vec;
  p.packed = packed;
  const int64_t M = packed ? ceil_div(M_rows, (int64_t)vec) : M_rows;
  const int64_t N = packed ? (int64_t)vec * N_cols : N_cols;
  p.unroll = backward ? (vec > 1 ? kBwdUnrollVec : kBwdUnrollScalar)
                      : (vec > 1 ? kFwdUnrollVec : kFwdUnrollScalar);
  const int64_t NV = N / vec;
  Geom &g = p.g;
  g.M = M;
  g.N = N;
  g.Nc = N_cols;
  g.total = M_rows * N_cols;
  g.ldx = g.ldd = g.ldo = N;  // adjacent rows; the strided entry points override this
  g.NV = (int)NV;
  if (NV <= block / 2) {
    g.RL = block / (int)NV;
    g.ncc = 1;
    p.path = 1;
  } else {
    g.RL = 1;
    g.ncc = (int)ceil_div(NV, block);
    p.path = 2;
  }
  const int64_t target = (int64_t)sms * ctas_per_sm;
  // One wave of items: `fill` row groups per column chunk, fill * ncc <= target
  // (at least one group), but no group thinner than one row per lane.
  int64_t fill = target / g.ncc;
  if (fill < 1) fill = 1;
  const int64_t rows_per_lane_min = ceil_div(M, (int64_t)g.RL);
  if (fill > rows_per_lane_min) fill = rows_per_lane_min;
  int64_t nrg = fill;
  // Cap the rows a lane adds in one group; keep the group count a multiple of
  // the fill so every CTA gets the same number of items.
  const int64_t max_rows = (int64_t)g.RL * kMaxRowsPerLane;
  if (ceil_div(M, nrg) > max_rows) nrg = ceil_div(ceil_div(M, max_rows), fill) * fill;
  // Shapes this large cannot be allocated on any device, but the plan must not
  // wrap around for them either.
  p.too_big = nrg * g.ncc > (int64_t)INT32_MAX;
  if (p.too_big) nrg = 1;
  g.nrg = (int)nrg;
  g.nitems = (int)(nrg * g.ncc);
  g.gq = M / nrg;
  g.grem = M % nrg;
  g.nv_magic = NV >= 2 ? (uint32_t)((((uint64_t)1 << 32) + (uint64_t)NV - 1) / (uint64_t)NV) : 0u;
  g.rl_magic = g.RL >= 2 ? (uint32_t)((((uint64_t)1 << 32) + (uint64_t)g.RL - 1) / (uint64_t)g.RL) : 0u;
  // L2 prefetch of the first rows (pipelined kernels): worth its issue cost
  // only when the launch reads enough that its inputs are unlikely to be
  // resident in L2 already and each CTA's first rows take a DRAM round trip
  // or more; below kPrefetchMinBytes it is skipped.
  g.l2_prefetch = (int64_t)(backward ? 2 : 1) * M_rows * N_cols * elem_bytes >= kPrefetchMinBytes;
  int64_t grid = fill * g.ncc;
  if (grid > target) grid = target;
  if (grid > g.nitems) grid = g.nitems;
  p.grid = (int)grid;
  p.ws_dg = 0;
  p.ws_db = align16((size_t)nrg * (size_t)N * sizeof(float));
  p.ws_da = p.ws_db + align16((size_t)nrg * (size_t)N * sizeof(float));
  p.ws_total = p.ws_da + align16((size_t)p.grid * sizeof(double));
  return p;
}

// Tiles of the pipelined kernels: about DYT_TILE_BYTES per stage, as many
// stages as fit next to the kernel's static shared memory.
void plan_tma(Plan &p, size_t elem, bool backward, int static_smem) {
  const dyt::Geom &g = p.g;
  const int64_t chunk_cols = g.ncc == 1 ? g.N : (int64_t)kBlock * p.vec;
  dyt::TmaGeom &tg = p.tg;
  tg.pitch = (int)(chunk_cols * (int64_t)elem);
  const int ntensors = backward ? 2 : 1;
  const int64_t per_u = (int64_t)g.RL * tg.pitch * ntensors;  // bytes per row per lane
  int64_t U = DYT_TILE_BYTES / per_u;
  if (U < 1) U = 1;
  const int64_t rows_per_group = ceil_div(g.M, g.nrg);
  const int64_t u_cap = ceil_div(rows_per_group, g.RL);
  if (U > u_cap) U = u_cap;
  if (U > kMaxRowsPerLane) U = kMaxRowsPerLane;
  tg.U = (int)U;
  tg.SR = g.RL * tg.U;
  const int64_t stage = (int64_t)tg.SR * tg.pitch * ntensors;
  int64_t S = (kMaxDynSmem - static_smem - 16 * DYT_MAX_STAGES - 64) / stage;
  if (S > DYT_MAX_STAGES) S = DYT_MAX_STAGES;
  tg.stages = (int)S;
  tg.spin = kSpinLimit;
  p.smem = (size_t)S * stage + 16 * S + 16;
  p.tma = S >= 2;
  p.unroll = tg.U;
}

// ---- kernel tables ---------------------------------------------------------------

template <typename T>
constexpr int vec_of() {
  return 16 / (int)sizeof(T);
}

template <typename T, typename P>
const void *fwd_kernel(int vec) {
  if (vec > 1) return (const void *)dyt::dyt_fwd_kernel<T, P, vec_of<T>(), kFwdUnrollVec, kBlock>;
  return (const void *)dyt::dyt_fwd_kernel<T, P, 1, kFwdUnrollScalar, kBlock>;
}

template <typename T, typename P>
const void *bwd_kernel(int vec) {
  if (vec > 1) return (const void *)dyt::dyt_bwd_kernel<T, P, vec_of<T>(), kBwdUnrollVec, kBlock>;
  return (const void *)dyt::dyt_bwd_kernel<T, P, 1, kBwdUnrollScalar, kBlock>;
}

template <typename F>
dyt_status with_types(dyt_dtype xd, dyt_dtype pd, F &&f) {
  auto with_p = [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    switch (pd) {
      case DYT_F32: return f(T{}, float{});
      case DYT_BF16: return f(T{}, __nv_bfloat16{});
      case DYT_F16: return f(T{}, __half{});
    }
    return DYT_ERR_UNSUPPORTED_DTYPE;
  };
  switch (xd) {
    case DYT_F32: return with_p(float{});
    case DYT_BF16: return with_p(__nv_bfloat16{});
    case DYT_F16: return with_p(__half{});
  }
  return DYT_ERR_UNSUPPORTED_DTYPE;
}

dyt_status check_shape(int64_t M, int64_t N, dyt_dtype xd, dyt_dtype pd) {
  if (!valid_dtype(xd) || !valid_dtype(pd)) return DYT_ERR_UNSUPPORTED_DTYPE;
  if (M < 0 || N < 0 || N > INT32_MAX) return DYT_ERR_INVALID_VALUE;
  if (N > 0 && M > INT64_MAX / N / 8) return DYT_ERR_INVALID_VALUE;
  // group and item counts are ints
  if (M > ((int64_t)1 << 40)) return DYT_ERR_INVALID_VALUE;
  return DYT_OK;
}

// Row pitches: at least N, and the last element of every tensor addressable.
dyt_status check_pitch(int64_t M, int64_t N, int64_t ld) {
  if (ld < N) return DYT_ERR_INVALID_VALUE;
  if (M > 1 && ld > 0 && (M - 1) > (INT64_MAX / 8 - N) / ld) return DYT_ERR_INVALID_VALUE;
  return DYT_OK;
}

// A row pitch of whole 16-byte vectors.
bool vec_pitch(int64_t ld, size_t elem) { return ((uint64_t)ld * elem) % 16 == 0; }

dyt_launch_info describe(int op, const Plan *p, int kernels, size_t ws) {
  dyt_launch_info i = {};
  i.op = op;
  i.kernels = kernels;
  i.workspace_bytes = (int64_t)ws;
  if (p) {
    i.path = p->path;
    i.vec = p->vec;
    i.block = p->block;
    i.grid = p->grid;
    i.row_lanes = p->g.RL;
    i.pack_rows = p->packed ? p->vec : 1;
    i.rows_per_step = p->g.RL * p->unroll * i.pack_rows;
    i.col_chunks = p->g.ncc;
    i.row_groups = p->g.nrg;
    i.tma_stages = p->tma ? p->tg.stages : 0;
    i.async_stages = p->async ? (op == 2 ? kAsyncStagesBwd : kAsyncStagesFwd) : 0;
  }
  return i;
}

void record(int op, const Plan *p, int kernels, size_t ws) { t_info = describe(op, p, kernels, ws); }

// Columns per thread in the pipelined kernels (their shared-memory reads are
// 4 elements wide; the bulk copies move whole rows regardless).
constexpr int kTmaVec = 4;

template <typename T, typename P>
const void *tma_kernel(bool backward) {
  return backward ? (const void *)dyt::dyt_bwd_tma_kernel<T, P, kTmaVec, kBlock>
                  : (const void *)dyt::dyt_fwd_tma_kernel<T, P, kTmaVec, kBlock>;
}

template <typename T, typename P, bool PK>
const void *async_kernel(bool backward) {
  return backward ? (const void *)dyt::dyt_bwd_async_kernel<T, P, vec_of<T>(), kAsyncBlock, kAsyncStagesBwd, PK>
                  : (const void *)dyt::dyt_fwd_async_kernel<T, P, vec_of<T>(), kAsyncBlock, kAsyncStagesFwd, PK>;
}

// Static shared memory of a kernel and, once, the opt-in to the largest
// dynamic shared memory (cached per device and kernel).
std::unordered_map<uint64_t, int> g_static_smem;

dyt_status prepare_tma_kernel(int dev, const void *kernel, int *static_smem) {
  const uint64_t key = ((uint64_t)(uint32_t)dev << 48) ^ (uint64_t)(uintptr_t)kernel;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_static_smem.find(key);
    if (it != g_static_smem.end()) {
      *static_smem = it->second;
      return DYT_OK;
    }
  }
  cudaFuncAttributes a;
  cudaError_t e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return cuda_fail(e);
  const int dyn = kMaxDynSmem - (int)a.sharedSizeBytes;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(g_mu);
  g_static_smem[key] = (int)a.sharedSizeBytes;
  *static_smem = (int)a.sharedSizeBytes;
  return DYT_OK;
}

// Plan for given pointers' alignment on the current device.
// Which kernels a call takes. aligned: every tensor starts on a 16-byte
// boundary; pitched: every row pitch is a whole number of 16-byte vectors;
// adjacent: every pitch is N. v: elements per 16-byte vector.
struct PathChoice {
  bool packed;  // ragged N on adjacent rows: packs of v rows through the 16-byte kernels
  int vec;      // elements per access: v, or 1 for the scalar kernels
  bool tma;     // the CTA-wide bulk-copy pipeline (compile-time option)
  bool async;   // the per-thread asynchronous-copy rings
};

PathChoice choose_path(int64_t N, int v, bool aligned, bool pitched, bool adjacent) {
  PathChoice c;
  // A pack of v adjacent rows is a whole number of vectors whatever N is.
  c.packed = DYT_PIPE == 2 && aligned && adjacent && N % v != 0;
  const bool vec_ok = aligned && (c.packed || (pitched && N % v == 0));
  c.tma = DYT_USE_TMA && vec_ok && adjacent;
  c.vec = vec_ok && (!DYT_USE_TMA || c.tma) ? v : 1;
  c.async = DYT_PIPE == 2 && c.vec > 1;
  return c;
}

// aligned, pitched, adjacent: as for choose_path.
template <typename T, typename P>
dyt_status plan_for(int64_t M, int64_t N, bool aligned, bool pitched, bool adjacent, bool backward, Plan *out) {
  int dev = 0, sms = 0;
  dyt_status st = current_sms(&dev, &sms);
  if (st != DYT_OK) return st;
  // Ragged rows of an aligned matrix go through the asynchronous-copy
  // kernels as packs; unaligned matrices take the scalar kernels.
  const PathChoice pc = choose_path(N, vec_of<T>(), aligned, pitched, adjacent);
  const bool packed = pc.packed, use_tma = pc.tma, use_async = pc.async;
  const int vec = pc.vec;
  const void *k = use_tma     ? tma_kernel<T, P>(backward)
                  : use_async ? (packed ? async_kernel<T, P, true>(backward) : async_kernel<T, P, false>(backward))
                  : backward  ? bwd_kernel<T, P>(vec)
                              : fwd_kernel<T, P>(vec);
  int occ = 1;
  int static_smem = 0;
  if (use_tma || use_async) {
    st = prepare_tma_kernel(dev, k, &static_smem);
    if (st != DYT_OK) return st;
  } else {
    st = occupancy(dev, k, kBlock, &occ);
    if (st != DYT_OK) return st;
  }
  *out = make_plan(M, N, use_tma ? kTmaVec : vec, backward, sms, occ, use_async ? kAsyncBlock : kBlock, packed,
                   (int64_t)sizeof(T));
  if (out->too_big) return DYT_ERR_INVALID_VALUE;
  out->tma = false;
  out->async = use_async;
  if (use_tma) plan_tma(*out, sizeof(T), backward, static_smem);
  if (use_async) {
    out->smem = backward ? (size_t)kAsyncStagesBwd * 2 * kAsyncBlock * 16 : (size_t)kAsyncStagesFwd * kAsyncBlock * 16;
    out->unroll = 1;
  }
  return DYT_OK;
}

}  // namespace

extern "C" {

dyt_status dyt_forward(const void *x, const void *alpha, const void *gamma, const void *beta, void *y,
                       int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                       dyt_stream_t stream) {
  return dyt_forward_strided(x, N, alpha, gamma, beta, y, N, M, N, x_dtype, param_dtype, stream);
}

dyt_status dyt_forward_strided(const void *x, int64_t ldx, const void *alpha, const void *gamma,
                               const void *beta, void *y, int64_t ldy, int64_t M, int64_t N,
                               dyt_dtype x_dtype, dyt_dtype param_dtype, dyt_stream_t stream) {
  dyt_status st = check_shape(M, N, x_dtype, param_dtype);
  if (st != DYT_OK) return st;
  if (check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, ldy) != DYT_OK) return DYT_ERR_INVALID_VALUE;
  if (M == 0 || N == 0) {
    record(1, nullptr, 0, 0);
    return DYT_OK;
  }
  if (!x || !alpha || !gamma || !beta || !y) return DYT_ERR_INVALID_VALUE;
  return with_types(x_dtype, param_dtype, [&](auto tx, auto tp) -> dyt_status {
    using T = decltype(tx);
    using P = decltype(tp);
    constexpr int V = vec_of<T>();
    Plan p;
    dyt_status s = plan_for<T, P>(M, N, aligned16(x) && aligned16(y),
                                  vec_pitch(ldx, sizeof(T)) && vec_pitch(ldy, sizeof(T)), ldx == N && ldy == N,
                                  false, &p);
    if (s != DYT_OK) return s;
    if (!p.packed) {
      p.g.ldx = ldx;
      p.g.ldo = ldy;
    }
    // Programmatic dependent launch: the kernel may be scheduled while its
    // predecessor in the stream drains; its first instruction waits
    // (griddepcontrol.wait) for that predecessor, so stream order holds.
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(p.block);
    cfg.stream = (cudaStream_t)stream;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (p.tma) {
      cfg.dynamicSmemBytes = p.smem;
      e = cudaLaunchKernelEx(&cfg, dyt::dyt_fwd_tma_kernel<T, P, kTmaVec, kBlock>, (const T *)x, (const P *)alpha,
                             (const P *)gamma, (const P *)beta, (T *)y, p.g, p.tg);
    } else if (p.async) {
      cfg.dynamicSmemBytes = p.smem;
      if (p.packed)
        e = cudaLaunchKernelEx(&cfg, dyt::dyt_fwd_async_kernel<T, P, V, kAsyncBlock, kAsyncStagesFwd, true>,
                               (const T *)x, (const P *)alpha, (const P *)gamma, (const P *)beta, (T *)y, p.g);
      else
        e = cudaLaunchKernelEx(&cfg, dyt::dyt_fwd_async_kernel<T, P, V, kAsyncBlock, kAsyncStagesFwd, false>,
                               (const T *)x, (const P *)alpha, (const P *)gamma, (const P *)beta, (T *)y, p.g);
    } else if (p.vec > 1)
      e = cudaLaunchKernelEx(&cfg, dyt::dyt_fwd_kernel<T, P, V, kFwdUnrollVec, kBlock>,
                             (const T *)x, (const P *)alpha, (const P *)gamma, (const P *)beta, (T *)y,
                             p.g);
    else
      e = cudaLaunchKernelEx(&cfg, dyt::dyt_fwd_kernel<T, P, 1, kFwdUnrollScalar, kBlock>, (const T *)x,
                             (const P *)alpha, (const P *)gamma, (const P *)beta, (T *)y, p.g);
    if (e != cudaSuccess) return cuda_fail(e);
    record(1, &p, 1, 0);
    return DYT_OK;
  });
}

size_t dyt_backward_workspace_bytes(int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype) {
  if (check_shape(M, N, x_dtype, param_dtype) != DYT_OK) return 0;
  if (M == 0 || N == 0) return 0;
  size_t need = 0;
  dyt_status st = with_types(x_dtype, param_dtype, [&](auto tx, auto tp) -> dyt_status {
    using T = decltype(tx);
    using P = decltype(tp);
    // The vectorised and the scalar plan may differ; cover both.
    for (int v = 0; v < 2; ++v) {
      Plan p;
      dyt_status s = plan_for<T, P>(M, N, v == 1, v == 1, true, true, &p);
      if (s != DYT_OK) return s;
      if (p.ws_total > need) need = p.ws_total;
    }
    return DYT_OK;
  });
  return st == DYT_OK ? need : 0;
}

dyt_status dyt_backward(const void *x, const void *dy, const void *alpha, const void *gamma, void *dx,
                        void *dgamma, void *dbeta, void *dalpha, int64_t M, int64_t N,
                        dyt_dtype x_dtype, dyt_dtype param_dtype, void *workspace,
                        size_t workspace_bytes, dyt_stream_t stream) {
  return dyt_backward_strided(x, N, dy, N, alpha, gamma, dx, N, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype,
                              workspace, workspace_bytes, stream);
}

dyt_status dyt_backward_strided(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                                const void *gamma, void *dx, int64_t lddx, void *dgamma, void *dbeta,
                                void *dalpha, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                                void *workspace, size_t workspace_bytes, dyt_stream_t stream) {
  dyt_status st = check_shape(M, N, x_dtype, param_dtype);
  if (st != DYT_OK) return st;
  if (check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, lddy) != DYT_OK || check_pitch(M, N, lddx) != DYT_OK)
    return DYT_ERR_INVALID_VALUE;
  if (!dalpha || (N > 0 && (!dgamma || !dbeta))) return DYT_ERR_INVALID_VALUE;
  cudaStream_t s = (cudaStream_t)stream;
  const size_t ps = dsize(param_dtype);
  if (M == 0 || N == 0) {
    // Empty sums: every gradient is +0 (all-zero bits in each dtype).
    cudaError_t e = cudaSuccess;
    if (N > 0) {
      e = cudaMemsetAsync(dgamma, 0, (size_t)N * ps, s);
      if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, (size_t)N * ps, s);
    }
    if (e == cudaSuccess) e = cudaMemsetAsync(dalpha, 0, ps, s);
    if (e != cudaSuccess) return cuda_fail(e);
    record(2, nullptr, 0, 0);
    return DYT_OK;
  }
  if (!x || !dy || !alpha || !gamma || !dx || !workspace) return DYT_ERR_INVALID_VALUE;
  if (!aligned16(workspace)) return DYT_ERR_INVALID_VALUE;
  return with_types(x_dtype, param_dtype, [&](auto tx, auto tp) -> dyt_status {
    using T = decltype(tx);
    using P = decltype(tp);
    constexpr int V = vec_of<T>();
    Plan p;
    const size_t es = sizeof(T);
    dyt_status r = plan_for<T, P>(M, N, aligned16(x) && aligned16(dy) && aligned16(dx),
                                  vec_pitch(ldx, es) && vec_pitch(lddy, es) && vec_pitch(lddx, es),
                                  ldx == N && lddy == N && lddx == N, true, &p);
    if (r != DYT_OK) return r;
    if (!p.packed) {
      p.g.ldx = ldx;
      p.g.ldd = lddy;
      p.g.ldo = lddx;
    }
    if (workspace_bytes < p.ws_total) return DYT_ERR_WORKSPACE_TOO_SMALL;
    char *ws = (char *)workspace;
    float *pdg = (float *)(ws + p.ws_dg);
    float *pdb = (float *)(ws + p.ws_db);
    double *pda = (double *)(ws + p.ws_da);

    cudaLaunchAttribute pdl[1];  // see dyt_forward
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(p.block);
    cfg.stream = s;
    cfg.attrs = pdl;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (p.tma) {
      cfg.dynamicSmemBytes = p.smem;
      e = cudaLaunchKernelEx(&cfg, dyt::dyt_bwd_tma_kernel<T, P, kTmaVec, kBlock>, (const T *)x, (const T *)dy,
                             (const P *)alpha, (const P *)gamma, (T *)dx, pdg, pdb, pda, p.g, p.tg);
    } else if (p.async) {
      cfg.dynamicSmemBytes = p.smem;
      if (p.packed)
        e = cudaLaunchKernelEx(&cfg, dyt::dyt_bwd_async_kernel<T, P, V, kAsyncBlock, kAsyncStagesBwd, true>,
                               (const T *)x, (const T *)dy, (const P *)alpha, (const P *)gamma, (T *)dx, pdg, pdb,
                               pda, p.g);
      else
        e = cudaLaunchKernelEx(&cfg, dyt::dyt_bwd_async_kernel<T, P, V, kAsyncBlock, kAsyncStagesBwd, false>,
                               (const T *)x, (const T *)dy, (const P *)alpha, (const P *)gamma, (T *)dx, pdg, pdb,
                               pda, p.g);
    } else if (p.vec > 1)
      e = cudaLaunchKernelEx(&cfg, dyt::dyt_bwd_kernel<T, P, V, kBwdUnrollVec, kBlock>,
                             (const T *)x, (const T *)dy, (const P *)alpha, (const P *)gamma, (T *)dx,
                             pdg, pdb, pda, p.g);
    else
      e = cudaLaunchKernelEx(&cfg, dyt::dyt_bwd_kernel<T, P, 1, kBwdUnrollScalar, kBlock>, (const T *)x,
                             (const T *)dy, (const P *)alpha, (const P *)gamma, (T *)dx, pdg, pdb, pda,
                             p.g);
    if (e != cudaSuccess) return cuda_fail(e);

    // Stage 2, as a programmatic dependent launch: it may start while stage 1
    // drains and waits (griddepcontrol.wait) for stage 1's results.
    // The partials form (nrg x pack rows) rows of N columns: a packed row group
    // holds vec partial rows, one per row of the pack, in pack order.
    const int nparts = p.g.nrg * (p.packed ? p.vec : 1);
    // Lanes per column: enough that each lane reads at most four partials.
    int L = 1;
    while (L < dyt::kFinThreads && (int64_t)L * 4 < nparts) L <<= 1;
    const int CT = dyt::kFinThreads / L;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t fcfg = {};
    fcfg.gridDim = dim3((unsigned)ceil_div(N, CT));
    fcfg.blockDim = dim3(dyt::kFinThreads);
    fcfg.stream = s;
    fcfg.attrs = attr;
    fcfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&fcfg, dyt::dyt_finalize_kernel<P>, (const float *)pdg, (const float *)pdb,
                           (const double *)pda, (P *)dgamma, (P *)dbeta, (P *)dalpha, (int64_t)N,
                           nparts, p.grid, CT);
    if (e != cudaSuccess) return cuda_fail(e);
    record(2, &p, 2, p.ws_total);
    return DYT_OK;
  });
}

const char *dyt_status_string(dyt_status status) {
  switch (status) {
    case DYT_OK: return "DYT_OK";
    case DYT_ERR_INVALID_VALUE: return "DYT_ERR_INVALID_VALUE: bad pointer, size or alignment";
    case DYT_ERR_UNSUPPORTED_DTYPE: return "DYT_ERR_UNSUPPORTED_DTYPE";
    case DYT_ERR_WORKSPACE_TOO_SMALL: return "DYT_ERR_WORKSPACE_TOO_SMALL";
    case DYT_ERR_CUDA: return "DYT_ERR_CUDA: the CUDA runtime refused a query or a launch";
  }
  return "DYT_ERR_UNKNOWN";
}

int dyt_last_cuda_error(void) { return t_cuda_err; }

dyt_status dyt_device_error(unsigned int *word, int clear) {
  if (!word) return DYT_ERR_INVALID_VALUE;
  cudaError_t e = cudaMemcpyFromSymbol(word, dyt::g_dyt_device_error, sizeof(unsigned int));
  if (e != cudaSuccess) return cuda_fail(e);
  if (clear) {
    const unsigned int zero = 0;
    e = cudaMemcpyToSymbol(dyt::g_dyt_device_error, &zero, sizeof(unsigned int));
    if (e != cudaSuccess) return cuda_fail(e);
  }
  return DYT_OK;
}

dyt_status dyt_selftest_wait_timeout(unsigned int spin_limit, int *gave_up, dyt_stream_t stream) {
  if (!gave_up || spin_limit == 0) return DYT_ERR_INVALID_VALUE;
  dyt::dyt_wait_timeout_selftest_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(spin_limit, gave_up);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e);
  return DYT_OK;
}

dyt_status dyt_plan_query(int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype, int backward,
                          int vectorized, int sm_count, int ctas_per_sm, dyt_launch_info *out) {
  if (!out || sm_count < 1 || ctas_per_sm < 1) return DYT_ERR_INVALID_VALUE;
  dyt_status st = check_shape(M, N, x_dtype, param_dtype);
  if (st != DYT_OK) return st;
  const int op = backward ? 2 : 1;
  if (M == 0 || N == 0) {
    *out = describe(op, nullptr, 0, 0);
    return DYT_OK;
  }
  const int v = 16 / (int)dsize(x_dtype);
  const PathChoice pc = choose_path(N, v, vectorized != 0, vectorized != 0, true);  // adjacent rows
  const bool packed = pc.packed, use_tma = pc.tma, use_async = pc.async;
  const int vec = pc.vec;
  Plan p = make_plan(M, N, use_tma ? kTmaVec : vec, backward != 0, sm_count, ctas_per_sm,
                     use_async ? kAsyncBlock : kBlock, packed, (int64_t)dsize(x_dtype));
  if (p.too_big) return DYT_ERR_INVALID_VALUE;
  p.tma = false;
  p.async = use_async;
  if (p.async) p.unroll = 1;
  if (use_tma) plan_tma(p, dsize(x_dtype), backward != 0, backward ? 17 * 1024 : 256);
  *out = describe(op, &p, backward ? 2 : 1, backward ? p.ws_total : 0);
  return DYT_OK;
}

dyt_status dyt_last_launch_info(dyt_launch_info *out) {
  if (!out) return DYT_ERR_INVALID_VALUE;
  *out = t_info;
  return DYT_OK;
}

}  // extern "C"

// ---- backward without a caller-provided workspace ---------------------------------
//
// For callers that cannot allocate device memory themselves (an embedding
// application owning all device memory, or loops that cannot afford
// cudaMalloc's implicit synchronisation): the scratch is a fixed file-scope
// device array. Host code only ever sees a stand-in for its name, so the
// device address is looked up with cudaGetSymbolAddress, once per device,
// with that device current, and handed to the kernels.

namespace {

static __device__ __align__(256) unsigned char g_dyt_noalloc_scratch[DYT_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
std::unordered_map<int, void *> g_noalloc_ptr;  // device -> address of the array

dyt_status noalloc_scratch(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  auto it = g_noalloc_ptr.find(dev);
  if (it != g_noalloc_ptr.end()) {
    *out = it->second;
    return DYT_OK;
  }
  void *p = nullptr;
  e = cudaGetSymbolAddress(&p, g_dyt_noalloc_scratch);
  if (e != cudaSuccess) return cuda_fail(e);
  g_noalloc_ptr[dev] = p;
  *out = p;
  return DYT_OK;
}

}  // namespace

extern "C" dyt_status dyt_backward_noalloc(const void *x, const void *dy, const void *alpha, const void *gamma,
                                           void *dx, void *dgamma, void *dbeta, void *dalpha, int64_t M,
                                           int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                                           dyt_stream_t stream) {
  void *scratch = nullptr;
  const dyt_status st = noalloc_scratch(&scratch);
  if (st != DYT_OK) return st;
  // dyt_backward checks the arguments and rejects, before launching, a shape
  // whose scratch need exceeds the array (DYT_ERR_WORKSPACE_TOO_SMALL).
  return dyt_backward(x, dy, alpha, gamma, dx, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype, scratch,
                      DYT_NOALLOC_SCRATCH_BYTES, stream);
}
