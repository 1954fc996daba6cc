// C ABI of the fused DyT layer (declared in include/dyt.h): argument checks,
// launch planning and kernel dispatch. All device work is in the kernels of
// dyt_async.cuh and dyt_kernels.cuh (stage 1 and the forward, selected through
// dyt_select.cuh and compiled per activation dtype in dyt_inst_*.cu) and
// dyt_finalize.cuh (the finalize, compiled here).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <algorithm>
#include <cstring>
#include <mutex>
#include <unordered_map>

#include "dyt.h"
#include "dyt_finalize.cuh"
#include "dyt_select.cuh"

namespace {

using dyt::Geom;
using namespace dyt::launch;

thread_local dyt_launch_info t_info = {};
thread_local int t_cuda_err = 0;


// A CUDA runtime call failed: keep its code for dyt_last_cuda_error and clear
// the runtime's last-error state, so that the failure, reported by our status,
// does not surface again in the caller's next CUDA call.
dyt_status cuda_fail(cudaError_t e) {
  t_cuda_err = (int)e;
  (void)cudaGetLastError();
  return DYT_ERR_CUDA;
}

size_t dsize(int d) { return d == DYT_F32 ? 4 : 2; }
bool valid_dtype(int d) { return d == DYT_F32 || d == DYT_BF16 || d == DYT_F16; }
bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
// A pointer to whole elements of `bytes` bytes (the kernels' loads need it).
bool elem_aligned(const void *p, size_t bytes) { return ((uintptr_t)p & (bytes - 1)) == 0; }
// Elements between the 16-byte boundary below p and p.
int shift_of(const void *p, size_t elem) { return (int)(((uintptr_t)p & 15u) / elem); }
// Two pointers at the same offset past a 16-byte boundary.
bool same_offset(const void *a, const void *b) { return (((uintptr_t)a ^ (uintptr_t)b) & 15u) == 0; }
int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// ---- per-device facts and per-kernel occupancy (cached, thread-safe) -------

std::mutex g_mu;
std::unordered_map<int, int> g_sms;                   // device -> SM count
std::unordered_map<uint64_t, int> g_occ;              // (device, kernel) -> CTAs per SM
std::unordered_map<uint64_t, int> g_smem_ready;       // (device, kernel) -> dynamic shared memory opted in

uint64_t kernel_key(int dev, const void *kernel) {
  return ((uint64_t)(uint32_t)dev << 48) ^ (uint64_t)(uintptr_t)kernel;
}

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
  const uint64_t key = kernel_key(dev, kernel);
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

// Opt a kernel in to `bytes` of dynamic shared memory, once per device.
dyt_status prepare_smem(int dev, const void *kernel, int bytes) {
  const uint64_t key = kernel_key(dev, kernel);
  {
    std::lock_guard<std::mutex> lk(g_mu);
    auto it = g_smem_ready.find(key);
    if (it != g_smem_ready.end() && it->second >= bytes) return DYT_OK;
  }
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return cuda_fail(e);
  std::lock_guard<std::mutex> lk(g_mu);
  g_smem_ready[key] = bytes;
  return DYT_OK;
}

// ---- launch plan ---------------------------------------------------------------

struct Plan {
  Geom g;
  int block;    // threads per CTA of the main kernel
  int vec;      // elements per access: 16 / element size, or 1 for the one-element kernels
  int unroll;   // rows in flight per thread on the one-element kernels (1 on the 16-byte path)
  int grid;
  int path;     // 1 = row-tiled, 2 = row-per-CTA
  bool async;   // the 16-byte per-thread copy rings
  bool packed;  // the packed-layout kernels: a ragged N (packs of vec rows) or the flat shifted kernels
  bool shifted; // the shifted kernels: tensors not all 16-byte aligned, or strided rows of a ragged N
                // (see dyt_async.cuh)
  bool rowframe;  // of those, the row frame: strided rows, each shifted on its own
  bool wrap;      // the row frame with a wrapped vector-column (see make_plan)
  int shm;      // their mode: 0 = not shifted, else 1 | 2 (x's vectors cut out of two chunks) | 4 (dy's)
                // | 8 (the row frame)
  int pack_rows;  // matrix rows per row of the packed layout: vec for a ragged N, else 1
  bool too_big; // the group or item count would not fit the kernels' int indices
  size_t smem;  // dynamic shared memory of the 16-byte kernel
  size_t ws_dg, ws_db, ws_da, ws_total;  // workspace byte offsets / sizes
};

size_t align16(size_t v) { return (v + 15) & ~(size_t)15; }

// Dynamic shared memory of a 16-byte kernel: its per-thread ring of 16-byte
// slots (the backward holds x and dy in each slot pair) and, in a backward
// over 16-bit activations, each thread's binary64 dgamma totals (16-byte
// vectors of elem_bytes-byte elements).
size_t async_stages(bool backward, int block) {
  return !backward ? kAsyncStagesFwd : block == kAsyncBlockNarrow ? kAsyncStagesBwdNarrow : kAsyncStagesBwd;
}
// The shifted kernels hold two 16-byte chunks per slot and tensor.
size_t async_smem(bool backward, int block, size_t elem_bytes, bool shifted) {
  const size_t ch = shifted ? 2 : 1;
  if (!backward) return (size_t)kAsyncStagesFwd * ch * block * 16;
  const size_t totals = elem_bytes == 4 ? 0 : (16 / elem_bytes) * (size_t)block * sizeof(double);
  return async_stages(true, block) * 2 * ch * block * 16 + totals;
}

// vec: elements per access (1 or 16 / element size). ctas_per_sm from the
// kernel's occupancy. ragged: N is not a multiple of vec, and the matrix is
// laid out as packs of vec rows, each of pitch vec * N. shifted: the flat
// shifted kernels, whose packed layout (packs of vec rows for a ragged N, else
// of one row) starts the matrix at position sh, the output's offset past a
// 16-byte boundary in elements. rowframe: the row frame, each matrix row laid
// out on its own from position sh of a row of ceil((N + sh) / vec) vectors;
// wrap (N a multiple of vec, sh > 0, every input at the output's offset): of
// N / vec vectors instead, the first holding the row's last sh elements too.
// The plan depends only on these arguments.
Plan make_plan(int64_t M_rows, int64_t N_cols, int vec, bool backward, bool async, int sms, int ctas_per_sm,
               bool ragged, bool shifted, bool rowframe, bool wrap, int sh, int64_t elem_bytes) {
  Plan p = {};
  p.vec = vec;
  p.async = async;
  p.packed = ragged || shifted;
  p.shifted = shifted || rowframe;
  p.rowframe = rowframe;
  p.wrap = rowframe && wrap;
  p.pack_rows = ragged ? vec : 1;
  // the matrix's end in the (packed) layout; the row frame: a row's end in its frame
  const int64_t end = rowframe ? N_cols + sh : M_rows * N_cols + (shifted ? sh : 0);
  const int64_t N = p.wrap ? N_cols : rowframe ? ceil_div(end, (int64_t)vec) * vec : (int64_t)p.pack_rows * N_cols;
  const int64_t M = p.packed ? ceil_div(end, N) : M_rows;
  const int64_t NV = N / vec;
  p.block = !async ? kScalarBlock : backward && NV <= kNarrowMaxNV ? kAsyncBlockNarrow : kAsyncBlock;
  const int block = p.block;
  p.unroll = async ? 1 : (backward ? kScalarUnrollBwd : kScalarUnrollFwd);
  p.smem = async ? async_smem(backward, block, (size_t)elem_bytes, p.shifted) : 0;
  Geom &g = p.g;
  g.M = M;
  g.N = N;
  g.Nc = N_cols;
  g.total = end;
  g.sh = p.shifted ? sh : 0;
  g.ldx = g.ldd = g.ldo = N;  // adjacent rows; the strided calls override this
  g.NV = (int)NV;
  if (NV <= block / 2) {
    g.RL = block / (int)NV;
    g.ncc = 1;
    g.cw = block;
    p.path = 1;
  } else {
    g.RL = 1;
    g.ncc = (int)ceil_div(NV, block);
    // Chunks of equal width in whole warps: 513 vectors as 288 + 225, not as
    // 512 + 1, which would leave the CTAs of every second item nearly idle.
    g.cw = async ? (int)std::min<int64_t>(block, ceil_div(ceil_div(NV, (int64_t)g.ncc), 32) * 32) : block;
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
  // Cap the rows a lane visits in one group; keep the group count a multiple
  // of the fill so every CTA gets the same number of items.
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
  // (the row frame's rows are strided: no prefetch)
  g.l2_prefetch = !rowframe && (int64_t)(backward ? 2 : 1) * M_rows * N_cols * elem_bytes >= kPrefetchMinBytes;
  int64_t grid = fill * g.ncc;
  if (grid > target) grid = target;
  if (grid > g.nitems) grid = g.nitems;
  p.grid = (int)grid;
  // Workspace: binary64 partial sums of dgamma and dbeta per (group, row of a
  // pack, column), and of dalpha per CTA.
  const size_t width = (size_t)p.pack_rows * (size_t)N_cols;  // partials per group
  p.ws_dg = 0;
  p.ws_db = align16((size_t)nrg * width * sizeof(double));
  p.ws_da = p.ws_db + align16((size_t)nrg * width * sizeof(double));
  p.ws_total = p.ws_da + align16((size_t)p.grid * sizeof(double));
  return p;
}

// ---- kernel tables ---------------------------------------------------------------

template <typename T, typename P>
const void *main_kernel(bool backward, bool async, bool packed, int shm, int block) {
  return backward ? (const void *)bwd_kernel_of<T, P>(async, packed, shm, block)
                  : (const void *)fwd_kernel_of<T, P>(async, packed, shm);
}

// The parameter type of the kernels for these parameter dtypes: the shared
// dtype when all are equal (typed, read-only loads), else void (a run-time
// switch per parameter). f receives a Tag<P>.
template <typename P>
struct Tag {
  using type = P;
};
template <typename F>
dyt_status with_ptype(int ad, int gd, int bd, F &&f) {
  if (ad == gd && gd == bd) {
    switch (ad) {
      case DYT_F32: return f(Tag<float>{});
      case DYT_BF16: return f(Tag<__nv_bfloat16>{});
      case DYT_F16: return f(Tag<__half>{});
    }
    return DYT_ERR_UNSUPPORTED_DTYPE;
  }
  return f(Tag<void>{});
}

template <typename F>
dyt_status with_xtype(int xd, F &&f) {
  switch (xd) {
    case DYT_F32: return f(float{});
    case DYT_BF16: return f(__nv_bfloat16{});
    case DYT_F16: return f(__half{});
  }
  return DYT_ERR_UNSUPPORTED_DTYPE;
}

dyt_status check_shape(int64_t M, int64_t N, int xd) {
  if (!valid_dtype(xd)) return DYT_ERR_UNSUPPORTED_DTYPE;
  if (M < 0 || N < 0 || N > INT32_MAX) return DYT_ERR_INVALID_VALUE;
  if (N > 0 && M > INT64_MAX / N / 8) return DYT_ERR_INVALID_VALUE;
  // group and item counts are ints
  if (M > ((int64_t)1 << 40)) return DYT_ERR_INVALID_VALUE;
  return DYT_OK;
}

dyt_status check_param_dtypes(int ad, int gd, int bd) {
  return valid_dtype(ad) && valid_dtype(gd) && valid_dtype(bd) ? DYT_OK : DYT_ERR_UNSUPPORTED_DTYPE;
}

// Row pitches: at least N, and the last element of every tensor addressable.
dyt_status check_pitch(int64_t M, int64_t N, int64_t ld) {
  if (ld < N) return DYT_ERR_INVALID_VALUE;
  if (M > 1 && ld > 0 && (M - 1) > (INT64_MAX / 8 - N) / ld) return DYT_ERR_INVALID_VALUE;
  return DYT_OK;
}

// A row pitch of whole 16-byte vectors.
bool vec_pitch(int64_t ld, size_t elem) { return ((uint64_t)ld * elem) % 16 == 0; }

// Rows ld elements apart: a row's offset past a 16-byte boundary repeats
// every 16 / (lowest set bit of ld * elem mod 16) rows (1, 2, 4 or 8).
int pitch_period(int64_t ld, size_t elem) {
  const uint64_t r = ((uint64_t)ld * elem) & 15u;
  return r == 0 ? 1 : (int)(16u / (unsigned)(r & (~r + 1u)));
}

// Rows of phase j of k: j, j + k, ... below M.
int64_t phase_rows(int64_t M, int k, int j) { return (M - j + k - 1) / k; }

// Phases of a strided call (not every pitch N) whose pitches are not all whole
// 16-byte vectors: k = the longest period of its tensors' pitches. Rows j,
// j + k, j + 2k, ... then form a matrix of pitch k * ld (whole vectors) for
// every tensor, which the 16-byte kernels take (aligned, or the row frame);
// the call runs its k phases one after another. 1: no phases (the pitches are
// whole vectors, the rows are adjacent, or a phase would move fewer than
// min_bytes per tensor, which the one-element kernels take in one launch).
int phases_of(int64_t M, int64_t N, const int64_t *lds, int n, size_t elem, int64_t min_bytes) {
  int k = 1;
  bool adjacent = true;
  for (int i = 0; i < n; ++i) {
    k = std::max(k, pitch_period(lds[i], elem));
    adjacent = adjacent && lds[i] == N;
  }
  if (adjacent || k == 1 || M < k) return 1;
  if (phase_rows(M, k, k - 1) * N * (int64_t)elem < min_bytes) return 1;  // the smallest phase
  return k;
}

// The backward runs phases only for k = 2: every phase leaves a full set of
// binary64 partials (k times the finalize's reads) after a launch of its own.
// Measured against the one-element kernels (us): 16384 x 4096 bf16, pitch
// 4100 (2 phases) 154.6 -> 117.7; 100003 x 255 fp32, pitch 257 (4 phases)
// 75.0 -> 87.6; 16384 x 4096 bf16, pitch 4097 (8 phases) 153.8 -> 231.9. The
// forward gains at every k: 130.0 -> 61.0, 54.0 -> 50.5, 128.8 -> 96.5.
int bwd_phases(int k) { return k == 2 ? 2 : 1; }

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
    i.pack_rows = p->pack_rows;
    i.shifted = p->wrap ? 3 : p->rowframe ? 2 : p->shifted ? 1 : 0;
    i.shift = p->g.sh;
    i.rows_per_step = p->g.RL * p->unroll * i.pack_rows;
    i.col_chunks = p->g.ncc;
    i.row_groups = p->g.nrg;
    i.async_stages = p->async ? (int)async_stages(op != 1, p->block) : 0;
  }
  return i;
}

void record(int op, const Plan *p, int kernels, size_t ws) { t_info = describe(op, p, kernels, ws); }

// Which kernels a call takes. aligned: every tensor starts on a 16-byte
// boundary; pitched: every row pitch is a whole number of 16-byte vectors;
// adjacent: every pitch is N. v: elements per 16-byte vector. Every pointer
// is a whole number of elements (checked before).
struct PathChoice {
  bool ragged;    // ragged N on adjacent rows: packs of v rows through the 16-byte kernels
  bool shifted;   // adjacent rows not all 16-byte aligned: the flat shifted 16-byte kernels
  bool rowframe;  // strided rows of whole-vector pitches, not all aligned or of a ragged N: the row frame
  bool async;     // the 16-byte kernels (per-thread copy rings)
  int vec;        // elements per access: v, or 1 for the one-element kernels
};

PathChoice choose_path(int64_t N, int v, bool aligned, bool pitched, bool adjacent) {
  PathChoice c;
  c.shifted = !aligned && adjacent;
  // A pack of v adjacent rows is a whole number of vectors whatever N is.
  c.ragged = adjacent && N % v != 0;
  // Whole-vector pitches keep every row's offset past a boundary the same.
  c.rowframe = !adjacent && pitched && (!aligned || N % v != 0);
  c.async = c.shifted || c.rowframe || (aligned && (c.ragged || (pitched && N % v == 0)));
  if (!c.async) c.ragged = false;
  c.vec = c.async ? v : 1;
  return c;
}

// The plan for tensors of type T with the given layout on the current device;
// sh: the output's offset past a 16-byte boundary, in elements; win: for the
// shifted kernels, 2 if x's offset differs from the output's, | 4 if dy's does.
template <typename T, typename P>
dyt_status plan_for(int64_t M, int64_t N, bool aligned, bool pitched, bool adjacent, int sh, int win,
                    bool backward, Plan *out) {
  int dev = 0, sms = 0;
  dyt_status st = current_sms(&dev, &sms);
  if (st != DYT_OK) return st;
  const PathChoice pc = choose_path(N, vec_of<T>(), aligned, pitched, adjacent);
  if (pc.async) {
    // One CTA per SM by construction (__launch_bounds__(B, 1), ring sized for it).
    const bool wrap = pc.rowframe && sh > 0 && N % pc.vec == 0 && win == 0;
    *out = make_plan(M, N, pc.vec, backward, true, sms, 1, pc.ragged, pc.shifted, pc.rowframe, wrap, sh,
                     (int64_t)sizeof(T));
    if (out->too_big) return DYT_ERR_INVALID_VALUE;
    // dy alone off the output's offset runs the kernel that cuts both inputs
    out->shm = !out->shifted ? 0
                             : (out->rowframe ? 8 : 0) | (out->wrap ? 16 : 0) | ((win & 4) ? 7 : 1 | (win & 2));
    return prepare_smem(dev, main_kernel<T, P>(backward, true, out->packed, out->shm, out->block),
                        (int)out->smem);
  }
  int occ = 1;
  st = occupancy(dev, main_kernel<T, P>(backward, false, false, 0, kScalarBlock), kScalarBlock, &occ);
  if (st != DYT_OK) return st;
  *out = make_plan(M, N, pc.vec, backward, false, sms, occ, false, false, false, false, 0, (int64_t)sizeof(T));
  if (out->too_big) return DYT_ERR_INVALID_VALUE;
  return DYT_OK;
}

// Programmatic dependent launch: the kernel may be scheduled while its
// predecessor in the stream drains; its first instruction waits
// (griddepcontrol.wait) for that predecessor, so stream order holds.
struct PdlConfig {
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg;
  PdlConfig(unsigned grid, unsigned block, size_t smem, cudaStream_t s) {
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
  }
};

using MemGetAddressRangeFn = CUresult (*)(CUdeviceptr *, size_t *, CUdeviceptr);

// The partials' layout in the workspace of a backward plan.
dyt_partials_layout layout_of(const Plan &p) {
  dyt_partials_layout l = {};
  l.bytes = (int64_t)p.ws_total;
  l.off_dgamma = (int64_t)p.ws_dg;
  l.off_dbeta = (int64_t)p.ws_db;
  l.off_dalpha = (int64_t)p.ws_da;
  // (nrg x pack rows) rows of N: a packed row group holds pack_rows partial
  // rows, one per row of the pack, in pack order.
  l.rows = p.g.nrg * p.pack_rows;
  l.dalpha_parts = p.grid;
  return l;
}

// The layout facts of a backward call's tensors: aligned, pitched, adjacent
// (see choose_path), the output's offset past a 16-byte boundary and which
// inputs' offsets differ from it (see plan_for).
struct LayoutArgs {
  bool aligned, pitched, adjacent;
  int sh, win;
};
template <typename T>
LayoutArgs stage1_layout_args(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *dx,
                              int64_t lddx, int64_t N) {
  const size_t es = sizeof(T);
  return {aligned16(x) && aligned16(dy) && aligned16(dx),
          vec_pitch(ldx, es) && vec_pitch(lddy, es) && vec_pitch(lddx, es), ldx == N && lddy == N && lddx == N,
          shift_of(dx, es), (same_offset(x, dx) ? 0 : 2) | (same_offset(dy, dx) ? 0 : 4)};
}
template <typename T, typename P>
dyt_status plan_for(int64_t M, int64_t N, LayoutArgs a, bool backward, Plan *out) {
  return plan_for<T, P>(M, N, a.aligned, a.pitched, a.adjacent, a.sh, a.win, backward, out);
}

// The gradient pointers hold whole elements of their dtypes.
bool grads_aligned(const void *dgamma, const void *dbeta, const void *dalpha, int ad, int gd, int bd) {
  return elem_aligned(dgamma, dsize(gd)) && elem_aligned(dbeta, dsize(bd)) && elem_aligned(dalpha, dsize(ad));
}

// Every gradient +0 (all-zero bits in each dtype): the empty sums.
dyt_status zero_gradients(int64_t N, void *dgamma, void *dbeta, void *dalpha, dyt_dtype ad, dyt_dtype gd,
                          dyt_dtype bd, cudaStream_t s) {
  cudaError_t e = cudaSuccess;
  if (N > 0) {
    e = cudaMemsetAsync(dgamma, 0, (size_t)N * dsize(gd), s);
    if (e == cudaSuccess) e = cudaMemsetAsync(dbeta, 0, (size_t)N * dsize(bd), s);
  }
  if (e == cudaSuccess) e = cudaMemsetAsync(dalpha, 0, dsize(ad), s);
  return e == cudaSuccess ? DYT_OK : cuda_fail(e);
}

// Stage 1 of the backward (M, N > 0, arguments checked): dx and the binary64
// partial sums in the workspace, laid out as *lay describes.
dyt_status bwd_stage1(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha, const void *gamma,
                      void *dx, int64_t lddx, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype alpha_dtype,
                      dyt_dtype gamma_dtype, void *workspace, size_t workspace_bytes, cudaStream_t s, Plan *plan,
                      dyt_partials_layout *lay) {
  if (!x || !dy || !alpha || !gamma || !dx || !workspace) return DYT_ERR_INVALID_VALUE;
  if (!aligned16(workspace)) return DYT_ERR_INVALID_VALUE;
  const size_t es = dsize(x_dtype);
  if (!elem_aligned(x, es) || !elem_aligned(dy, es) || !elem_aligned(dx, es) ||
      !elem_aligned(alpha, dsize(alpha_dtype)) || !elem_aligned(gamma, dsize(gamma_dtype)))
    return DYT_ERR_INVALID_VALUE;
  const dyt::ParamTypes pt = {(int)alpha_dtype, (int)gamma_dtype, (int)gamma_dtype};
  // beta is not read: the kernels' parameter type follows alpha and gamma.
  return with_xtype(x_dtype, [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    return with_ptype(alpha_dtype, gamma_dtype, gamma_dtype, [&](auto tp) -> dyt_status {
    using P = typename decltype(tp)::type;
    Plan &p = *plan;
    dyt_status r = plan_for<T, P>(M, N, stage1_layout_args<T>(x, ldx, dy, lddy, dx, lddx, N), true, &p);
    if (r != DYT_OK) return r;
    if (!p.packed) {
      p.g.ldx = ldx;
      p.g.ldd = lddy;
      p.g.ldo = lddx;
    }
    if (workspace_bytes < p.ws_total) return DYT_ERR_WORKSPACE_TOO_SMALL;
    char *ws = (char *)workspace;
    double *pdg = (double *)(ws + p.ws_dg);
    double *pdb = (double *)(ws + p.ws_db);
    double *pda = (double *)(ws + p.ws_da);
    const P *pa = (const P *)alpha, *pg = (const P *)gamma;
    PdlConfig lc(p.grid, p.block, p.smem, s);
    const cudaError_t e = cudaLaunchKernelEx(&lc.cfg, bwd_kernel_of<T, P>(p.async, p.packed, p.shm, p.block),
                                             (const T *)x, (const T *)dy, pa, pg, pt, (T *)dx, pdg, pdb, pda, p.g);
    if (e != cudaSuccess) return cuda_fail(e);
    *lay = layout_of(p);
    return DYT_OK;
    });
  });
}

// Stage 2 (N > 0, dtypes checked): the partials of `nranks` workspaces summed
// in binary64 in a fixed order (rank by rank), each gradient rounded once.
// Launched as a programmatic dependent: it may start while its predecessor in
// the stream drains and waits (griddepcontrol.wait) for its results.
// The workspace bytes stage 1 needs for these tensors (the plan only;
// nothing is launched). The plans do not depend on the parameter type.
dyt_status stage1_bytes(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *dx, int64_t lddx,
                        int64_t M, int64_t N, dyt_dtype x_dtype, size_t *out) {
  return with_xtype(x_dtype, [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    Plan p;
    const dyt_status r = plan_for<T, float>(M, N, stage1_layout_args<T>(x, ldx, dy, lddy, dx, lddx, N), true, &p);
    if (r == DYT_OK) *out = p.ws_total;
    return r;
  });
}

dyt_status bwd_finalize(const void *const *wss, const dyt_partials_layout *lay, int nranks, int64_t N, void *dgamma,
                        void *dbeta, void *dalpha, dyt_dtype ad, dyt_dtype gd, dyt_dtype bd, cudaStream_t s) {
  dyt::PartsSet ps = {};
  ps.nranks = nranks;
  int64_t rows_max = 0;
  for (int r = 0; r < nranks; ++r) {
    const dyt_partials_layout &l = lay[r];
    if (l.rows < 0 || l.dalpha_parts < 0) return DYT_ERR_INVALID_VALUE;
    if (l.rows > 0 || l.dalpha_parts > 0) {
      const char *w = (const char *)wss[r];
      if (!w || !aligned16(w)) return DYT_ERR_INVALID_VALUE;
      const int64_t part_bytes = (int64_t)l.rows * N * (int64_t)sizeof(double);
      if (l.off_dgamma < 0 || l.off_dbeta < 0 || l.off_dalpha < 0 || l.off_dgamma + part_bytes > l.bytes ||
          l.off_dbeta + part_bytes > l.bytes || l.off_dalpha + (int64_t)l.dalpha_parts * 8 > l.bytes)
        return DYT_ERR_INVALID_VALUE;
      ps.r[r].dg = (const double *)(w + l.off_dgamma);
      ps.r[r].db = (const double *)(w + l.off_dbeta);
      ps.r[r].da = (const double *)(w + l.off_dalpha);
    }
    ps.r[r].rows = l.rows;
    ps.r[r].nda = l.dalpha_parts;
    if (l.rows > rows_max) rows_max = l.rows;
  }
  // Lanes per column: enough that each lane reads at most four partials of a
  // rank. Every rank that finalizes the same layouts picks the same L, so all
  // get the same bits.
  int L = 1;
  while (L < dyt::kFinThreads && (int64_t)L * 4 < rows_max) L <<= 1;
  const int CT = dyt::kFinThreads / L;
  const dyt::GradOut go = {dgamma, dbeta, dalpha, (int)gd, (int)bd, (int)ad};
  PdlConfig fc((unsigned)ceil_div(N, CT), dyt::kFinThreads, 0, s);
  const cudaError_t e = cudaLaunchKernelEx(&fc.cfg, dyt::dyt_finalize_kernel, ps, go, (int64_t)N, CT);
  return e == cudaSuccess ? DYT_OK : cuda_fail(e);
}

}  // namespace

extern "C" {

dyt_status dyt_forward(const void *x, const void *alpha, const void *gamma, const void *beta, void *y,
                       int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                       dyt_stream_t stream) {
  return dyt_forward_ex(x, N, alpha, gamma, beta, y, N, M, N, x_dtype, param_dtype, param_dtype, param_dtype,
                        stream);
}

dyt_status dyt_forward_strided(const void *x, int64_t ldx, const void *alpha, const void *gamma,
                               const void *beta, void *y, int64_t ldy, int64_t M, int64_t N,
                               dyt_dtype x_dtype, dyt_dtype param_dtype, dyt_stream_t stream) {
  return dyt_forward_ex(x, ldx, alpha, gamma, beta, y, ldy, M, N, x_dtype, param_dtype, param_dtype, param_dtype,
                        stream);
}

dyt_status dyt_forward_ex(const void *x, int64_t ldx, const void *alpha, const void *gamma, const void *beta,
                          void *y, int64_t ldy, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype alpha_dtype,
                          dyt_dtype gamma_dtype, dyt_dtype beta_dtype, dyt_stream_t stream) {
  dyt_status st = check_shape(M, N, x_dtype);
  if (st == DYT_OK) st = check_param_dtypes(alpha_dtype, gamma_dtype, beta_dtype);
  if (st != DYT_OK) return st;
  if (check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, ldy) != DYT_OK) return DYT_ERR_INVALID_VALUE;
  if (M == 0 || N == 0) {
    record(1, nullptr, 0, 0);
    return DYT_OK;
  }
  if (!x || !alpha || !gamma || !beta || !y) return DYT_ERR_INVALID_VALUE;
  const size_t es = dsize(x_dtype);
  if (!elem_aligned(x, es) || !elem_aligned(y, es) || !elem_aligned(alpha, dsize(alpha_dtype)) ||
      !elem_aligned(gamma, dsize(gamma_dtype)) || !elem_aligned(beta, dsize(beta_dtype)))
    return DYT_ERR_INVALID_VALUE;
  const dyt::ParamTypes pt = {(int)alpha_dtype, (int)gamma_dtype, (int)beta_dtype};
  const int64_t lds[2] = {ldx, ldy};
  const int k = phases_of(M, N, lds, 2, es, kPhaseMinBytesFwd);  // 1 unless the pitches call for phases
  return with_xtype(x_dtype, [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    return with_ptype(alpha_dtype, gamma_dtype, beta_dtype, [&](auto tp) -> dyt_status {
    using P = typename decltype(tp)::type;
    Plan p;
    for (int j = 0; j < k; ++j) {  // phase j: rows j, j + k, ...
      const T *xj = (const T *)x + j * ldx;
      T *yj = (T *)y + j * ldy;
      const int64_t lx = k * ldx, ly = k * ldy, Mj = phase_rows(M, k, j);
      dyt_status s = plan_for<T, P>(Mj, N, aligned16(xj) && aligned16(yj),
                                    vec_pitch(lx, sizeof(T)) && vec_pitch(ly, sizeof(T)), lx == N && ly == N,
                                    shift_of(yj, sizeof(T)), same_offset(xj, yj) ? 0 : 2, false, &p);
      if (s != DYT_OK) return s;
      if (!p.packed) {
        p.g.ldx = lx;
        p.g.ldo = ly;
      }
      const P *pa = (const P *)alpha, *pg = (const P *)gamma, *pb = (const P *)beta;
      PdlConfig lc(p.grid, p.block, p.smem, (cudaStream_t)stream);
      const cudaError_t e = cudaLaunchKernelEx(&lc.cfg, fwd_kernel_of<T, P>(p.async, p.packed, p.shm), xj, pa, pg,
                                               pb, pt, yj, p.g);
      if (e != cudaSuccess) return cuda_fail(e);
    }
    record(1, &p, k, 0);
    return DYT_OK;
    });
  });
}

size_t dyt_backward_workspace_bytes(int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype) {
  if (check_shape(M, N, x_dtype) != DYT_OK || !valid_dtype(param_dtype)) return 0;
  if (M == 0 || N == 0) return 0;
  size_t need = 0;
  dyt_status st = with_xtype(x_dtype, [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    // The aligned (adjacent or strided), the shifted and the row-frame (one
    // per output offset) and the one-element plans may differ; cover them
    // all. The plans do not depend on P.
    constexpr int V = vec_of<T>();
    for (int v = -3; v < 3 * V; ++v) {
      Plan p;
      const dyt_status s = v == -3    ? plan_for<T, float>(M, N, true, true, true, 0, 0, true, &p)
                           : v == -2  ? plan_for<T, float>(M, N, true, true, false, 0, 0, true, &p)
                           : v == -1  ? plan_for<T, float>(M, N, false, false, false, 0, 0, true, &p)
                           : v < V    ? plan_for<T, float>(M, N, false, false, true, v, 0, true, &p)
                           : v < 2 * V ? plan_for<T, float>(M, N, false, true, false, v - V, 0, true, &p)
                                       : plan_for<T, float>(M, N, false, true, false, v - 2 * V, 2, true, &p);
      if (s != DYT_OK) return s;
      if (p.ws_total > need) need = p.ws_total;
    }
    return DYT_OK;
  });
  return st == DYT_OK ? need : 0;
}

size_t dyt_backward_workspace_bytes_strided(int64_t M, int64_t N, int64_t ldx, int64_t lddy, int64_t lddx,
                                            dyt_dtype x_dtype, dyt_dtype param_dtype) {
  const size_t plain = dyt_backward_workspace_bytes(M, N, x_dtype, param_dtype);
  if (plain == 0 || check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, lddy) != DYT_OK ||
      check_pitch(M, N, lddx) != DYT_OK)
    return plain;
  const int64_t lds[3] = {ldx, lddy, lddx};
  const int k = bwd_phases(phases_of(M, N, lds, 3, dsize(x_dtype), kPhaseMinBytesBwd));
  if (k == 1) return plain;
  // Each phase's region: the largest plan its rows can take, whatever the
  // tensors' offsets (aligned, or the row frame at any output offset, its
  // inputs at that offset or not).
  size_t need = 0;
  const dyt_status st = with_xtype(x_dtype, [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    constexpr int V = vec_of<T>();
    for (int j = 0; j < k; ++j) {
      const int64_t Mj = phase_rows(M, k, j);
      size_t region = 0;
      for (int v = -1; v < 2 * V; ++v) {
        Plan p;
        const dyt_status s = v < 0   ? plan_for<T, float>(Mj, N, true, true, false, 0, 0, true, &p)
                             : v < V ? plan_for<T, float>(Mj, N, false, true, false, v, 0, true, &p)
                                     : plan_for<T, float>(Mj, N, false, true, false, v - V, 2, true, &p);
        if (s != DYT_OK) return s;
        region = std::max(region, p.ws_total);
      }
      need += align16(region);
    }
    return DYT_OK;
  });
  return st == DYT_OK ? std::max(plain, need) : 0;
}

dyt_status dyt_backward(const void *x, const void *dy, const void *alpha, const void *gamma, const void *beta,
                        void *dx, void *dgamma, void *dbeta, void *dalpha, int64_t M, int64_t N,
                        dyt_dtype x_dtype, dyt_dtype param_dtype, void *workspace, size_t workspace_bytes,
                        dyt_stream_t stream) {
  return dyt_backward_ex(x, N, dy, N, alpha, gamma, beta, dx, N, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype,
                         param_dtype, param_dtype, workspace, workspace_bytes, stream);
}

dyt_status dyt_backward_strided(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                                const void *gamma, const void *beta, void *dx, int64_t lddx, void *dgamma,
                                void *dbeta, void *dalpha, int64_t M, int64_t N, dyt_dtype x_dtype,
                                dyt_dtype param_dtype, void *workspace, size_t workspace_bytes,
                                dyt_stream_t stream) {
  return dyt_backward_ex(x, ldx, dy, lddy, alpha, gamma, beta, dx, lddx, dgamma, dbeta, dalpha, M, N, x_dtype,
                         param_dtype, param_dtype, param_dtype, workspace, workspace_bytes, stream);
}

dyt_status dyt_backward_ex(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                           const void *gamma, const void *beta, void *dx, int64_t lddx, void *dgamma, void *dbeta,
                           void *dalpha, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype alpha_dtype,
                           dyt_dtype gamma_dtype, dyt_dtype beta_dtype, void *workspace, size_t workspace_bytes,
                           dyt_stream_t stream) {
  (void)beta;  // the gradients do not depend on beta; only its dtype (beta_dtype) is used
  dyt_status st = check_shape(M, N, x_dtype);
  if (st == DYT_OK) st = check_param_dtypes(alpha_dtype, gamma_dtype, beta_dtype);
  if (st != DYT_OK) return st;
  if (check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, lddy) != DYT_OK || check_pitch(M, N, lddx) != DYT_OK)
    return DYT_ERR_INVALID_VALUE;
  if (!dalpha || (N > 0 && (!dgamma || !dbeta))) return DYT_ERR_INVALID_VALUE;
  if (!grads_aligned(dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype)) return DYT_ERR_INVALID_VALUE;
  if (M == 0 || N == 0) {
    st = zero_gradients(N, dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype, (cudaStream_t)stream);
    if (st == DYT_OK) record(2, nullptr, 0, 0);
    return st;
  }
  // Pitches that call for phases (see phases_of): one stage 1 per phase, each
  // in its own workspace region, and one finalize over the phases' partials
  // in phase order. When the regions do not fit in the workspace given, the
  // call runs as one phase (the one-element kernels).
  const size_t es = dsize(x_dtype);
  const int64_t lds[3] = {ldx, lddy, lddx};
  int k = bwd_phases(phases_of(M, N, lds, 3, es, kPhaseMinBytesBwd));
  size_t off[dyt::kMaxRanks + 1] = {0};
  static_assert(dyt::kMaxRanks >= 8, "the finalize takes up to 8 partial sets");
  if (k > 1) {
    if (!x || !dy || !dx || !elem_aligned(x, es) || !elem_aligned(dy, es) || !elem_aligned(dx, es))
      return DYT_ERR_INVALID_VALUE;
    for (int j = 0; j < k; ++j) {
      size_t b = 0;
      st = stage1_bytes((const char *)x + j * ldx * es, k * ldx, (const char *)dy + j * lddy * es, k * lddy,
                        (const char *)dx + j * lddx * es, k * lddx, phase_rows(M, k, j), N, x_dtype, &b);
      if (st != DYT_OK) return st;
      off[j + 1] = off[j] + align16(b);
    }
    if (off[k] > workspace_bytes) k = 1;
  }
  Plan p;
  dyt_partials_layout lay[dyt::kMaxRanks];
  const void *wss[dyt::kMaxRanks];
  for (int j = 0; j < k; ++j) {
    char *ws = (char *)workspace + off[j];
    st = bwd_stage1((const char *)x + j * ldx * es, k * ldx, (const char *)dy + j * lddy * es, k * lddy, alpha,
                    gamma, (char *)dx + j * lddx * es, k * lddx, phase_rows(M, k, j), N, x_dtype, alpha_dtype,
                    gamma_dtype, ws, k == 1 ? workspace_bytes : off[j + 1] - off[j], (cudaStream_t)stream, &p,
                    &lay[j]);
    if (st != DYT_OK) return st;
    wss[j] = ws;
  }
  st = bwd_finalize(wss, lay, k, N, dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype,
                    (cudaStream_t)stream);
  if (st != DYT_OK) return st;
  record(2, &p, k + 1, k == 1 ? p.ws_total : off[k]);
  return DYT_OK;
}

dyt_status dyt_backward_partials(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                                 const void *gamma, void *dx, int64_t lddx, int64_t M, int64_t N, dyt_dtype x_dtype,
                                 dyt_dtype alpha_dtype, dyt_dtype gamma_dtype, void *workspace,
                                 size_t workspace_bytes, dyt_partials_layout *layout, dyt_stream_t stream) {
  if (!layout) return DYT_ERR_INVALID_VALUE;
  dyt_status st = check_shape(M, N, x_dtype);
  if (st == DYT_OK) st = check_param_dtypes(alpha_dtype, gamma_dtype, DYT_F32);
  if (st != DYT_OK) return st;
  if (check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, lddy) != DYT_OK || check_pitch(M, N, lddx) != DYT_OK)
    return DYT_ERR_INVALID_VALUE;
  if (M == 0 || N == 0) {  // no rows: no partials (a rank with an empty shard adds nothing)
    *layout = dyt_partials_layout{};
    record(3, nullptr, 0, 0);
    return DYT_OK;
  }
  Plan p;
  st = bwd_stage1(x, ldx, dy, lddy, alpha, gamma, dx, lddx, M, N, x_dtype, alpha_dtype, gamma_dtype, workspace,
                  workspace_bytes, (cudaStream_t)stream, &p, layout);
  if (st == DYT_OK) record(3, &p, 1, p.ws_total);
  return st;
}

dyt_status dyt_partials_layout_query(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *dx,
                                     int64_t lddx, int64_t M, int64_t N, dyt_dtype x_dtype,
                                     dyt_partials_layout *layout) {
  if (!layout) return DYT_ERR_INVALID_VALUE;
  dyt_status st = check_shape(M, N, x_dtype);
  if (st != DYT_OK) return st;
  if (check_pitch(M, N, ldx) != DYT_OK || check_pitch(M, N, lddy) != DYT_OK || check_pitch(M, N, lddx) != DYT_OK)
    return DYT_ERR_INVALID_VALUE;
  if (M == 0 || N == 0) {
    *layout = dyt_partials_layout{};
    return DYT_OK;
  }
  return with_xtype(x_dtype, [&](auto tx) -> dyt_status {
    using T = decltype(tx);
    Plan p;
    const dyt_status r = plan_for<T, float>(M, N, stage1_layout_args<T>(x, ldx, dy, lddy, dx, lddx, N), true, &p);
    if (r == DYT_OK) *layout = layout_of(p);
    return r;
  });
}

dyt_status dyt_finalize_partials(const void *const *workspaces, const dyt_partials_layout *layouts, int nranks,
                                 int64_t N, void *dgamma, void *dbeta, void *dalpha, dyt_dtype alpha_dtype,
                                 dyt_dtype gamma_dtype, dyt_dtype beta_dtype, dyt_stream_t stream) {
  if (!workspaces || !layouts || nranks < 1 || nranks > DYT_MAX_RANKS) return DYT_ERR_INVALID_VALUE;
  dyt_status st = check_param_dtypes(alpha_dtype, gamma_dtype, beta_dtype);
  if (st != DYT_OK) return st;
  if (N < 0 || N > INT32_MAX) return DYT_ERR_INVALID_VALUE;
  if (!dalpha || (N > 0 && (!dgamma || !dbeta))) return DYT_ERR_INVALID_VALUE;
  if (!grads_aligned(dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype)) return DYT_ERR_INVALID_VALUE;
  if (N == 0)
    return zero_gradients(N, dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype, (cudaStream_t)stream);
  st = bwd_finalize(workspaces, layouts, nranks, N, dgamma, dbeta, dalpha, alpha_dtype, gamma_dtype, beta_dtype,
                    (cudaStream_t)stream);
  if (st == DYT_OK) record(4, nullptr, 1, 0);
  return st;
}

dyt_status dyt_ipc_export(const void *ptr, dyt_ipc_handle *out) {
  if (!ptr || !out) return DYT_ERR_INVALID_VALUE;
  static MemGetAddressRangeFn get_range = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuMemGetAddressRange", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_range = (MemGetAddressRangeFn)f;
  });
  if (!get_range) return cuda_fail(cudaErrorNotSupported);
  CUdeviceptr base = 0;
  size_t size = 0;
  if (get_range(&base, &size, (CUdeviceptr)(uintptr_t)ptr) != CUDA_SUCCESS) return cuda_fail(cudaErrorInvalidValue);
  cudaIpcMemHandle_t h;
  const cudaError_t e = cudaIpcGetMemHandle(&h, (void *)(uintptr_t)base);
  if (e != cudaSuccess) return cuda_fail(e);
  static_assert(sizeof(h) == sizeof(out->bytes), "CUDA IPC handles are 64 bytes");
  memcpy(out->bytes, &h, sizeof(h));
  out->offset = (int64_t)((uintptr_t)ptr - (uintptr_t)base);
  return DYT_OK;
}

dyt_status dyt_ipc_import(const dyt_ipc_handle *handle, void **ptr) {
  if (!handle || !ptr || handle->offset < 0) return DYT_ERR_INVALID_VALUE;
  cudaIpcMemHandle_t h;
  memcpy(&h, handle->bytes, sizeof(h));
  void *base = nullptr;
  const cudaError_t e = cudaIpcOpenMemHandle(&base, h, cudaIpcMemLazyEnablePeerAccess);
  if (e != cudaSuccess) return cuda_fail(e);
  *ptr = (char *)base + handle->offset;
  return DYT_OK;
}

dyt_status dyt_ipc_close(void *ptr, const dyt_ipc_handle *handle) {
  if (!ptr || !handle || handle->offset < 0) return DYT_ERR_INVALID_VALUE;
  const cudaError_t e = cudaIpcCloseMemHandle((char *)ptr - handle->offset);
  if (e != cudaSuccess) return cuda_fail(e);
  return DYT_OK;
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

dyt_status dyt_plan_query(int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype, int backward, int layout,
                          int shift, int sm_count, int ctas_per_sm, dyt_launch_info *out) {
  if (!out || sm_count < 1 || ctas_per_sm < 1) return DYT_ERR_INVALID_VALUE;
  dyt_status st = check_shape(M, N, x_dtype);
  if (st == DYT_OK && !valid_dtype(param_dtype)) st = DYT_ERR_UNSUPPORTED_DTYPE;
  if (st != DYT_OK) return st;
  const int v = 16 / (int)dsize(x_dtype);
  if (layout < 0 || layout > 4 || (layout >= 2 && (shift < 0 || shift >= v))) return DYT_ERR_INVALID_VALUE;
  const int op = backward ? 2 : 1;
  if (M == 0 || N == 0) {
    *out = describe(op, nullptr, 0, 0);
    return DYT_OK;
  }
  // layout 0: rows that are not whole 16-byte vectors; 1: contiguous and
  // 16-byte aligned; 2: contiguous, the output `shift` elements past a
  // boundary; 3 / 4: strided rows of whole-vector pitches, the output `shift`
  // elements past a boundary, every input at its offset (3) or not (4).
  const bool strided = layout == 3 || layout == 4;
  const PathChoice pc = choose_path(N, v, layout == 1 || (layout == 3 && shift == 0), layout == 1 || strided,
                                    layout == 1 || layout == 2);
  const bool wrap = pc.rowframe && layout == 3 && shift > 0 && N % v == 0;
  // The 16-byte kernels always run one CTA per SM.
  Plan p = make_plan(M, N, pc.vec, backward != 0, pc.async, sm_count, pc.async ? 1 : ctas_per_sm, pc.ragged,
                     pc.shifted, pc.rowframe, wrap, layout >= 2 ? shift : 0, (int64_t)dsize(x_dtype));
  if (p.too_big) return DYT_ERR_INVALID_VALUE;
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
// device address is looked up with cudaGetSymbolAddress, with the device
// current, and handed to the kernels. The lookup runs once per device context
// and is cached under the driver's unique context id, so a context that
// cudaDeviceReset ended, and the fresh one that replaces it, never share an
// address.

namespace {

static __device__ __align__(256) unsigned char g_dyt_noalloc_scratch[DYT_NOALLOC_SCRATCH_BYTES];

std::mutex g_noalloc_mu;
std::unordered_map<uint64_t, void *> g_noalloc_ptr;  // context id -> address of the array

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// The driver's unique id of the current context, in *id; false when no
// context is current yet or the driver cannot say.
bool context_id(uint64_t *id) {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = (CtxGetCurrentFn)f;
    f = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &f, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = (CtxGetIdFn)f;
  });
  CUcontext ctx = nullptr;
  unsigned long long v = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx || get_id(ctx, &v) != CUDA_SUCCESS)
    return false;
  *id = (uint64_t)v;
  return true;
}

// The array's device address in the current context. Looked up once per
// context; without a context id (no context current yet, or a driver that
// cannot name it) the lookup runs and is cached only once the id is known.
dyt_status noalloc_scratch(void **out) {
  uint64_t id = 0;
  bool known = context_id(&id);
  if (known) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    auto it = g_noalloc_ptr.find(id);
    if (it != g_noalloc_ptr.end()) {
      *out = it->second;
      return DYT_OK;
    }
  }
  void *p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_dyt_noalloc_scratch);  // also creates the context if needed
  if (e != cudaSuccess) return cuda_fail(e);
  if (!known) known = context_id(&id);
  if (known) {
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    g_noalloc_ptr[id] = p;
  }
  *out = p;
  return DYT_OK;
}

}  // namespace

extern "C" dyt_status dyt_backward_noalloc(const void *x, const void *dy, const void *alpha, const void *gamma,
                                           const void *beta, void *dx, void *dgamma, void *dbeta, void *dalpha,
                                           int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                                           dyt_stream_t stream) {
  // Shape and dtype errors, and empty shapes (which need no scratch), are
  // settled before the scratch is looked up.
  dyt_status st = check_shape(M, N, x_dtype);
  if (st == DYT_OK && !valid_dtype(param_dtype)) st = DYT_ERR_UNSUPPORTED_DTYPE;
  if (st != DYT_OK) return st;
  if (M == 0 || N == 0)
    return dyt_backward(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype, nullptr,
                        0, stream);
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != DYT_OK) return st;
  // dyt_backward checks the arguments and rejects, before launching, a shape
  // whose scratch need exceeds the array (DYT_ERR_WORKSPACE_TOO_SMALL).
  return dyt_backward(x, dy, alpha, gamma, beta, dx, dgamma, dbeta, dalpha, M, N, x_dtype, param_dtype, scratch,
                      DYT_NOALLOC_SCRATCH_BYTES, stream);
}
