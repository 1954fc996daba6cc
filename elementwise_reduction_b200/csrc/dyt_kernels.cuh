// Fused DyT forward / backward for sm_100a: the pieces every kernel shares,
// the kernels for matrices that are not 16-byte aligned (one element per
// access), and the finalize of the backward.
//
// Work decomposition (one 1D persistent grid, the page's Summary "Launch
// limit": rows never sit on grid dimension 1, so M is unbounded):
//   - a thread owns one vector-column cv (VEC consecutive columns; VEC = 16
//     bytes / element size on the 16-byte path, 1 here) and keeps its gamma
//     and beta in registers;
//   - packed rows (16-byte aligned matrix, N not a multiple of VEC): VEC
//     consecutive rows always span exactly N 16-byte vectors, so such a pack
//     is treated as one row of pitch VEC * N with NV = N vector-columns; the
//     element e of vector-column cv then lies in matrix column
//     (cv * VEC + e) mod N, fixed for the thread. The last pack may hold
//     fewer than VEC rows: its vectors past the matrix are not read, and the
//     one vector that straddles the end is zero-filled and masked;
//   - row-tiled path (NV = N / VEC <= B / 2, the page's narrow rows): RL =
//     B / NV row lanes share a CTA step, so one step covers RL whole rows
//     (the page's Summary "Small widths": several rows per tile);
//   - row-per-CTA path (wider rows): RL = 1, every thread works on every row
//     of the CTA's group, columns spread across threads; rows wider than
//     B * VEC are split into column chunks;
//   - rows are cut into nrg balanced contiguous groups; a work item is
//     (column chunk, row group) and CTA b takes items b, b + grid, ... (a
//     static schedule: the same inputs always give the same bits).
// Backward sums: each thread accumulates dbeta of its columns in binary64, and
// dgamma in binary64 (binary32 activations) or in binary32 runs of at most
// kGammaRunRows rows flushed into binary64 (16-bit activations); the row
// lanes of a CTA are added in binary64 in a fixed order, and each (group,
// column) partial goes to the workspace in binary64; dalpha is carried in
// binary64 per thread (binary32 within a few rows) and reduced per CTA in a
// fixed order. The finalize adds the partials in binary64 in a fixed order and
// rounds each gradient once.
// Lanes outside [0,M) x [0,N) never enter a sum: their contribution is
// dropped by a select after the arithmetic (the page's Summary, "Padding").
#pragma once

#include <cuda_runtime.h>

#include <type_traits>

#include "dyt_math.cuh"

namespace dyt {

struct Geom {
  int64_t M;      // rows (packs of VEC rows on the packed path)
  int64_t N;      // elements of a row (VEC x Nc on the packed path): the partials' pitch
  int64_t Nc;     // columns of the matrix (= N unless packed)
  int64_t total;  // elements of the matrix (its rows x Nc): later ones are padding (packed path)
  int64_t ldx;    // row pitches in elements (= N when packed): x,
  int64_t ldd;    //   dy,
  int64_t ldo;    //   and the output (y or dx)
  int NV;         // vector-columns per row (N / VEC)
  int RL;         // row lanes per CTA step (1 on the row-per-CTA path)
  int ncc;        // column chunks
  int cw;         // vector-columns per column chunk (at most B; the 16-byte kernels read it)
  int nrg;        // row groups
  int nitems;     // ncc * nrg
  int64_t gq;     // M / nrg     (computed on the host: the kernels divide nothing)
  int64_t grem;   // M % nrg
  uint32_t nv_magic;  // ceil(2^32 / NV) for NV >= 2: tid / NV = umulhi(tid, nv_magic), tid < 1024
  uint32_t rl_magic;  // ceil(2^32 / RL) for RL >= 2: n / RL = umulhi(n, rl_magic) for n < 2^32 / RL
  int l2_prefetch;    // the 16-byte kernels prefetch their first rows into L2 (large inputs only)
  int sh;             // shifted kernels: the output's offset past a 16-byte boundary, in elements
                      // (0 .. VEC - 1); its matrix starts at position sh of the packed layout
};

// The parameters' dtypes (dyt_dtype codes), read by the kernels instantiated
// with P = void (parameters of different dtypes); beta is read by the forward
// only.
struct ParamTypes {
  int alpha;
  int gamma;
  int beta;
};

// Where the finalize writes the parameter gradients, each in its parameter's dtype.
struct GradOut {
  void *dgamma;
  void *dbeta;
  void *dalpha;
  int gamma_dt;
  int beta_dt;
  int alpha_dt;
};

// Where the shifted kernels keep the partial sums of position q of a packed
// row. The matrix starts at position sh there, so position q holds column
// (q - sh) mod Nc; slot q - sh (mod N) holds the same column modulo Nc, which
// is all the finalize reads (it adds slot j into column j mod Nc).
__device__ __forceinline__ int64_t shifted_slot(const Geom &g, int64_t q) {
  const int64_t r = q - g.sh;
  return r < 0 ? r + g.N : r;
}

// Rows [begin, end) of group rg when [0, M) is cut into nrg balanced groups.
__device__ __forceinline__ void group_rows(const Geom &g, int rg, int64_t &begin, int64_t &end) {
  begin = (int64_t)rg * g.gq + (rg < g.grem ? rg : g.grem);
  end = begin + g.gq + (rg < g.grem ? 1 : 0);
}

// Work item -> (column chunk, row group); a single chunk needs no division.
__device__ __forceinline__ void item_split(const Geom &g, int item, int &cc, int &rg) {
  if (g.ncc == 1) {
    cc = 0;
    rg = item;
  } else {
    cc = item % g.ncc;
    rg = item / g.ncc;
  }
}

// ---- global memory access --------------------------------------------------

__device__ __forceinline__ void st16(void *p, const uint4 &v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// VEC elements of T as raw storage, with float conversion.
template <typename T, int VEC>
struct VecIO;

template <typename T>
struct VecIO<T, 1> {
  using Raw = T;
  static constexpr int kPairs = 0;
  static __device__ __forceinline__ Raw load(const T *p) { return __ldg(p); }
  static __device__ __forceinline__ Raw zero() { return from_f32<T>(0.0f); }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[1]) { f[0] = to_f32<T>(r); }
  static __device__ __forceinline__ void set(Raw &r, int, T v) { r = v; }
  static __device__ __forceinline__ Raw pack(const float (&f)[1]) { return from_f32<T>(f[0]); }
  static __device__ __forceinline__ void store_raw(T *p, const Raw &r) { *p = r; }
};

template <>
struct VecIO<float, 4> {
  using Raw = uint4;
  static constexpr int kPairs = 2;
  static __device__ __forceinline__ void unpack2(const Raw &r, float2 (&f)[2]) {
    f[0] = make_float2(__uint_as_float(r.x), __uint_as_float(r.y));
    f[1] = make_float2(__uint_as_float(r.z), __uint_as_float(r.w));
  }
  static __device__ __forceinline__ Raw pack2(const float2 (&f)[2]) {
    return make_uint4(__float_as_uint(f[0].x), __float_as_uint(f[0].y), __float_as_uint(f[1].x),
                      __float_as_uint(f[1].y));
  }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[4]) {
    f[0] = __uint_as_float(r.x);
    f[1] = __uint_as_float(r.y);
    f[2] = __uint_as_float(r.z);
    f[3] = __uint_as_float(r.w);
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
  static constexpr int kPairs = 4;
  static __device__ __forceinline__ void unpack2(const Raw &r, float2 (&f)[4]) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t u = word_of(r, w);
      f[w] = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    }
  }
  static __device__ __forceinline__ Raw pack2(const float2 (&f)[4]) {
    Raw r;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t u;
      asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(f[w].y), "f"(f[w].x));
      set_word(r, w, u);
    }
    return r;
  }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[8]) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t u = word_of(r, w);
      f[2 * w] = __uint_as_float(u << 16);
      f[2 * w + 1] = __uint_as_float(u & 0xFFFF0000u);
    }
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
  static constexpr int kPairs = 4;
  static __device__ __forceinline__ void unpack2(const Raw &r, float2 (&f)[4]) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t u = word_of(r, w);
      f[w] = __half22float2(*reinterpret_cast<const __half2 *>(&u));
    }
  }
  static __device__ __forceinline__ Raw pack2(const float2 (&f)[4]) {
    Raw r;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      uint32_t u;
      asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(u) : "f"(f[w].y), "f"(f[w].x));
      set_word(r, w, u);
    }
    return r;
  }
  static __device__ __forceinline__ void unpack(const Raw &r, float (&f)[8]) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t u = word_of(r, w);
      f[2 * w] = __half2float(__ushort_as_half((unsigned short)(u & 0xFFFFu)));
      f[2 * w + 1] = __half2float(__ushort_as_half((unsigned short)(u >> 16)));
    }
  }
  static __device__ __forceinline__ void set(Raw &r, int e, __half v) {
    const uint32_t b = __half_as_ushort(v);
    const uint32_t u = word_of(r, e >> 1);
    set_word(r, e >> 1, (e & 1) ? ((u & 0x0000FFFFu) | (b << 16)) : ((u & 0xFFFF0000u) | b));
  }
  static __device__ __forceinline__ void store_raw(__half *p, const Raw &r) { st16(p, r); }
};

// Bytes of dynamic shared memory this launch was given.
__device__ __forceinline__ uint32_t dynamic_smem_bytes() {
  uint32_t r;
  asm("mov.u32 %0, %%dynamic_smem_size;" : "=r"(r));
  return r;
}

// Start of every main kernel: wait until the preceding grid in the stream has
// completed and its memory is visible (a no-op without a programmatic
// predecessor), then let the next grid get scheduled. The kernels read and
// write no global memory before this (the 16-byte kernels only issue L2
// prefetch hints, which change no memory state), so programmatic launch keeps
// stream order.
__device__ __forceinline__ void pdl_prologue() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Thread -> (row lane, vector-column) of the CTA.
struct Lane {
  int rl;     // row lane
  int cv;     // vector-column within the chunk
  bool live;  // false for threads past RL * NV on the row-tiled path, past cw on the other
};

__device__ __forceinline__ Lane lane_of(const Geom &g, int tid) {
  Lane l;
  if (g.RL > 1) {
    l.rl = g.NV == 1 ? tid : (int)__umulhi((unsigned)tid, g.nv_magic);
    l.cv = tid - l.rl * g.NV;
    l.live = l.rl < g.RL;
  } else {
    l.rl = 0;
    l.cv = tid;
    l.live = tid < g.cw;
  }
  return l;
}

// ---- forward -----------------------------------------------------------------

// y for one vector of VEC elements (one row, VEC columns).
// bth[e] = tau |beta[e]|: below it the binary32 value may have cancelled.
template <typename T, int VEC>
__device__ __forceinline__ typename VecIO<T, VEC>::Raw fwd_vector(const typename VecIO<T, VEC>::Raw &rx,
                                                                 float alpha, const float (&gam)[VEC],
                                                                 const float (&bet)[VEC],
                                                                 const float (&bth)[VEC]) {
  using IO = VecIO<T, VEC>;
  typename IO::Raw out;
  bool cancel_any = false;
  if constexpr (IO::kPairs > 0) {
    constexpr int H = IO::kPairs;
    float2 x2[H], y2[H];
    IO::unpack2(rx, x2);
#pragma unroll
    for (int h = 0; h < H; ++h) {
      const float2 t = dyt_tanh2(mul2(f2(alpha), x2[h]));
      y2[h] = fma2(make_float2(gam[2 * h], gam[2 * h + 1]), t, make_float2(bet[2 * h], bet[2 * h + 1]));
      if (CancelGuard<T>::kOn)
        cancel_any |= (fabsf(y2[h].x) < bth[2 * h]) | (fabsf(y2[h].y) < bth[2 * h + 1]);
    }
    out = IO::pack2(y2);
    if (CancelGuard<T>::kOn && cancel_any) {
      // Rare: find the cancelling elements again from the rounded outputs.
      // Rounding moves |y| by at most max(2^-8 |y|, kTiny / 2) (relative
      // above the subnormal range, half a subnormal step within it), so
      // |y| < bth implies |round(y)| < bth (1 + 2^-7) + kTiny: the test below
      // flags every element the binary32 test flagged (and at most a few
      // more, whose binary64 value is as good). Those get the binary64 value.
      float yr[VEC], xf[VEC];
      IO::unpack(out, yr);
      IO::unpack(rx, xf);
#pragma unroll
      for (int e = 0; e < VEC; ++e)
        if (fabsf(yr[e]) < fmaf(bth[e], 1.0f + 0x1p-7f, CancelGuard<T>::kTiny))
          IO::set(out, e, dyt_y_refined<T>(alpha, xf[e], gam[e], bet[e]));
    }
  } else {
    float xf[VEC], yf[VEC];
    IO::unpack(rx, xf);
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      yf[e] = fmaf(gam[e], dyt_tanh(alpha * xf[e]), bet[e]);
      if (CancelGuard<T>::kOn) cancel_any |= fabsf(yf[e]) < bth[e];
    }
    out = IO::pack(yf);
    if (CancelGuard<T>::kOn && cancel_any) {
#pragma unroll
      for (int e = 0; e < VEC; ++e)
        if (fabsf(yf[e]) < bth[e]) IO::set(out, e, dyt_y_refined<T>(alpha, xf[e], gam[e], bet[e]));
    }
  }
  return out;
}

// gamma, beta and the cancellation thresholds of the VEC columns col[e] (not
// necessarily consecutive).
template <typename T, int VEC, typename P>
__device__ __forceinline__ void fwd_params_at(const P *__restrict__ gamma, const P *__restrict__ beta,
                                              const ParamTypes &pt, const int64_t (&col)[VEC], float (&gam)[VEC],
                                              float (&bet)[VEC], float (&bth)[VEC]) {
  load_params<VEC, P>(gamma, pt.gamma, col, 1.0f, gam);
  load_params<VEC, P>(beta, pt.beta, col, 1.0f, bet);
#pragma unroll
  for (int e = 0; e < VEC; ++e) bth[e] = fabsf(bet[e]) * CancelGuard<T>::kTau;
}

// Forward for matrices that are not 16-byte aligned: one element per access,
// U rows in flight per thread.
template <typename T, typename P, int U, int B>
__global__ void __launch_bounds__(B, 1)
    dyt_fwd_kernel(const T *__restrict__ x, const P *__restrict__ alpha_p, const P *__restrict__ gamma_p,
                   const P *__restrict__ beta_p, ParamTypes pt, T *y, Geom g) {
  using IO = VecIO<T, 1>;
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = load_param<P>(alpha_p, pt.alpha, 0);
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    int cc, rg;
    item_split(g, item, cc, rg);
    int64_t rb, re;
    group_rows(g, rg, rb, re);
    const int cv = cc * B + ln.cv;
    if (!(ln.live && cv < g.NV)) continue;
    const int64_t col[1] = {cv};
    float gam[1], bet[1], bth[1];
    fwd_params_at<T, 1, P>(gamma_p, beta_p, pt, col, gam, bet, bth);
    const int64_t step = (int64_t)g.RL * U;
    for (int64_t r0 = rb + ln.rl; r0 < re; r0 += step) {
      T raw[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = r0 + (int64_t)u * g.RL;
        raw[u] = row < re ? IO::load(x + row * g.ldx + cv) : IO::zero();
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t row = r0 + (int64_t)u * g.RL;
        if (row < re) IO::store_raw(y + row * g.ldo + cv, fwd_vector<T, 1>(raw[u], alpha, gam, bet, bth));
      }
    }
  }
}

// ---- backward, stage 1 ---------------------------------------------------------

// Fixed-order tree over the RL row lanes of a CTA: lane rl absorbs lane rl + h,
// h = ceil(n / 2), until one lane is left. red[] holds V * B binary64 values,
// element-major (red[e * B + thread]); afterwards lane 0's entries hold the CTA
// sums.
template <int V, int B>
__device__ __forceinline__ void lane_tree(double *red, const Geom &g, const Lane &ln) {
  for (int n = g.RL; n > 1;) {
    const int h = (n + 1) >> 1;
    if (ln.live && ln.rl < n - h) {
      const int src = threadIdx.x + h * g.NV;
#pragma unroll
      for (int e = 0; e < V; ++e) red[e * B + threadIdx.x] += red[e * B + src];
    }
    __syncthreads();
    n = h;
  }
}

// CTA sums of the row lanes when NV divides 32: every warp then holds 32 / NV
// whole row lanes of the same NV vector-columns, so their sums are formed in
// registers by a reduce-scatter over lane offsets NV, 2 NV, ... 16. The 2 VEC
// values of a thread (VEC dgamma sums, then VEC dbeta sums) are halved at each
// level: the partner with the offset bit clear keeps the lower half, the
// other the upper half, and each adds the half the partner sent, so one
// exchange moves half of what a full butterfly would. When one value is left
// before the offsets run out, the remaining levels are a butterfly (both
// partners form the same sum). The order of every sum is fixed. Each warp
// then holds each of its 2 NV VEC sums once; one pass over the warps in order
// adds them. red[] holds (B / 32) x 2 NV VEC binary64 values. Results go to
// out_g / out_b (row of the group's partials) at the thread's positions; MAP
// 1: at their shifted_slot (flat shifted layout); MAP 2: at position - sh,
// padding positions skipped (row frame).
template <int VEC, int B, int MAP>
__device__ __forceinline__ void lane_reduce_warps(const double (&vg)[VEC], const double (&vb)[VEC], double *red,
                                                  const Geom &g, const Lane &ln, int64_t c0_chunk,
                                                  double *out_g, double *out_b) {
  constexpr int V2 = 2 * VEC;
  double v[V2];
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    v[e] = vg[e];
    v[VEC + e] = vb[e];
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int start = 0;     // index (in 0 .. 2 VEC - 1) of this thread's first kept value
  int m = V2;        // values kept
  bool dup = false;  // a butterfly level ran: lanes with its bit set hold copies
  int off = g.NV;
#pragma unroll
  for (int i = 0; i < 5; ++i) {
    const int h = V2 >> (i + 1);  // a constant once unrolled
    if (off < 32) {
      const bool up = (lane & off) != 0;
      if (h >= 1) {
#pragma unroll
        for (int j = 0; j < h; ++j) {
          const double send = up ? v[j] : v[j + h];
          const double recv = __shfl_xor_sync(0xFFFFFFFFu, send, off);
          v[j] = (up ? v[j + h] : v[j]) + recv;
        }
        start += up ? h : 0;
        m = h;
      } else {
        v[0] += __shfl_xor_sync(0xFFFFFFFFu, v[0], off);
        dup = dup || up;
      }
      off <<= 1;
    }
  }
  const int width = g.NV * VEC;  // values per warp and sum
  if (!dup) {
#pragma unroll
    for (int j = 0; j < V2; ++j) {
      if (j < m) {
        const int idx = start + j, which = idx >= VEC, e = idx - which * VEC;
        red[(2 * warp + which) * width + ln.cv * VEC + e] = v[j];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 2 * width; i += B) {  // 2 width can exceed B (NV = 32 with B = 256)
    const int which = i / width, k = i - which * width;
    double sum = 0.0;
    for (int w = 0; w < B / 32; ++w) sum += red[(2 * w + which) * width + k];
    const int64_t q = c0_chunk + k;
    if constexpr (MAP == 2) {
      if (q >= g.sh && q - g.sh < g.Nc) (which ? out_b : out_g)[q - g.sh] = sum;
    } else {
      (which ? out_b : out_g)[MAP == 1 ? shifted_slot(g, q) : q] = sum;
    }
  }
  __syncthreads();
}

// Whether a kernel over activations of type T adds the dgamma terms in
// binary64 (exact products dy * t, no rounding of the running sum). The
// 16-bit kernels carry twice the elements per byte, and a binary32 -> binary64
// conversion per term would take the special-function pipe (shared with the
// exp2 and reciprocal of tanh) past its rate: they add dgamma in binary32
// runs of at most kGammaRunRows rows, each flushed into a binary64 total.
template <typename T>
struct ExactGamma {
  static constexpr bool value = sizeof(T) == 4;
};
constexpr int kGammaRunRows = 126;

// Per-thread backward state for VEC columns. dbeta is always a binary64 sum:
// its terms dy are exact there, so the sum carries no rounding error until the
// final one. dgamma is binary64 (EXACT_G) or the current binary32 run.
template <int VEC, bool EXACT_G>
struct BwdAcc {
  using GT = typename std::conditional<EXACT_G, double, float>::type;
  GT g[VEC];      // sum of dy * t over this group's rows (or the current run)
  double b[VEC];  // sum of dy
};

// One vector (one row, VEC columns): dx out, sums in. g4[e] = 4 gamma[e]
// (with q = (1 - t^2) / 4, g4 * dy * q rounds exactly as gamma * dy * (1 - t^2)).
// dbeta's terms dy, and with EXACT_G dgamma's terms dy * t (a product of two
// binary32 values), are exact in binary64; ca collects the dalpha terms of the
// row in binary32 (the caller moves it into binary64 every few rows).
// MASKED: only the elements whose bit is set in vmask are real (none for a
// padded row; the vectors that straddle the start or the end of a packed
// matrix hold some); the others are computed like any other and their
// results dropped afterwards.
template <typename T, int VEC, bool MASKED, bool EXACT_G>
__device__ __forceinline__ typename VecIO<T, VEC>::Raw bwd_vector(const typename VecIO<T, VEC>::Raw &rx,
                                                                 const typename VecIO<T, VEC>::Raw &rdy,
                                                                 float alpha, const float (&g4)[VEC],
                                                                 BwdAcc<VEC, EXACT_G> &acc, float2 &ca,
                                                                 uint32_t vmask) {
  using IO = VecIO<T, VEC>;
  if constexpr (IO::kPairs > 0) {
    constexpr int H = IO::kPairs;
    float2 x2[H], dy2[H], dx2[H];
    IO::unpack2(rx, x2);
    IO::unpack2(rdy, dy2);
#pragma unroll
    for (int h = 0; h < H; ++h) {
      float2 t, q;
      dyt_tanh_qsech2_2(mul2(f2(alpha), x2[h]), t, q);
      const float2 gdys = mul2(mul2(make_float2(g4[2 * h], g4[2 * h + 1]), dy2[h]), q);  // gamma dy (1-t^2)
      dx2[h] = mul2(f2(alpha), gdys);
      const double d0 = (double)dy2[h].x, d1 = (double)dy2[h].y;
      using GT = typename BwdAcc<VEC, EXACT_G>::GT;
      GT ng0, ng1;
      if constexpr (EXACT_G) {
        ng0 = fma(d0, (double)t.x, acc.g[2 * h]);
        ng1 = fma(d1, (double)t.y, acc.g[2 * h + 1]);
      } else {
        const float2 ng = fma2(dy2[h], t, make_float2(acc.g[2 * h], acc.g[2 * h + 1]));
        ng0 = ng.x;
        ng1 = ng.y;
      }
      double nb0 = acc.b[2 * h] + d0, nb1 = acc.b[2 * h + 1] + d1;
      float2 nca = fma2(gdys, x2[h], ca);
      if (MASKED) {  // drop padded elements' results, after the arithmetic
        const bool okx = (vmask >> (2 * h)) & 1u, oky = (vmask >> (2 * h + 1)) & 1u;
        ng0 = okx ? ng0 : acc.g[2 * h];
        nb0 = okx ? nb0 : acc.b[2 * h];
        ng1 = oky ? ng1 : acc.g[2 * h + 1];
        nb1 = oky ? nb1 : acc.b[2 * h + 1];
        nca = make_float2(okx ? nca.x : ca.x, oky ? nca.y : ca.y);
      }
      acc.g[2 * h] = ng0;
      acc.g[2 * h + 1] = ng1;
      acc.b[2 * h] = nb0;
      acc.b[2 * h + 1] = nb1;
      ca = nca;
    }
    return IO::pack2(dx2);
  } else {
    float xf[VEC], dyf[VEC], dxf[VEC];
    IO::unpack(rx, xf);
    IO::unpack(rdy, dyf);
#pragma unroll
    for (int e = 0; e < VEC; ++e) {
      float t, q;
      dyt_tanh_qsech2(alpha * xf[e], t, q);
      const float gdys = (g4[e] * dyf[e]) * q;
      dxf[e] = alpha * gdys;
      static_assert(EXACT_G, "the one-element kernels add dgamma in binary64");
      const double d = (double)dyf[e];
      const double ng = fma(d, (double)t, acc.g[e]), nb = acc.b[e] + d;
      const float nca = fmaf(gdys, xf[e], ca.x);
      const bool ok = (vmask >> e) & 1u;
      acc.g[e] = (MASKED && !ok) ? acc.g[e] : ng;
      acc.b[e] = (MASKED && !ok) ? acc.b[e] : nb;
      ca.x = (MASKED && !ok) ? ca.x : nca;
    }
    return IO::pack(dxf);
  }
}

// Backward stage 1 for matrices that are not 16-byte aligned: one element
// per access, U rows in flight per thread.
template <typename T, typename P, int U, int B>
__global__ void __launch_bounds__(B, 1)
    dyt_bwd_kernel(const T *__restrict__ x, const T *__restrict__ dy, const P *__restrict__ alpha_p,
                   const P *__restrict__ gamma_p, ParamTypes pt, T *dx, double *__restrict__ part_dg,
                   double *__restrict__ part_db, double *__restrict__ part_da, Geom g) {
  using IO = VecIO<T, 1>;
  __shared__ double red[2 * B];
  __shared__ double red_a[B / 32];
  // Let the finalize kernel, launched as a programmatic dependent, get
  // scheduled early; it still waits for this grid to finish before reading.
  pdl_prologue();

  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = load_param<P>(alpha_p, pt.alpha, 0);
  double acc_a = 0.0;
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    int cc, rg;
    item_split(g, item, cc, rg);
    int64_t rb, re;
    group_rows(g, rg, rb, re);
    const int cv = cc * B + ln.cv;
    const bool col_ok = ln.live && cv < g.NV;
    float gam[1] = {col_ok ? 4.0f * load_param<P>(gamma_p, pt.gamma, cv) : 0.0f};  // 4 gamma (see bwd_vector)
    BwdAcc<1, true> acc;
    acc.g[0] = 0.0;
    acc.b[0] = 0.0;
    if (col_ok) {
      const int64_t step = (int64_t)g.RL * U;
      for (int64_t r0 = rb + ln.rl; r0 < re; r0 += step) {
        T rx[U], rdy[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int64_t row = r0 + (int64_t)u * g.RL;
          const bool ok = row < re;
          rx[u] = ok ? IO::load(x + row * g.ldx + cv) : IO::zero();
          rdy[u] = ok ? IO::load(dy + row * g.ldd + cv) : IO::zero();
        }
        float2 ca = make_float2(0.0f, 0.0f);
        if (r0 + (int64_t)(U - 1) * g.RL < re) {  // every row of the step is real
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int64_t row = r0 + (int64_t)u * g.RL;
            IO::store_raw(dx + row * g.ldo + cv, bwd_vector<T, 1, false, true>(rx[u], rdy[u], alpha, gam, acc, ca, 1));
          }
        } else {  // ragged last step of the group
#pragma unroll
          for (int u = 0; u < U; ++u) {
            const int64_t row = r0 + (int64_t)u * g.RL;
            const bool ok = row < re;
            const T d = bwd_vector<T, 1, true, true>(rx[u], rdy[u], alpha, gam, acc, ca, ok ? 1 : 0);
            if (ok) IO::store_raw(dx + row * g.ldo + cv, d);
          }
        }
        acc_a += (double)ca.x;
      }
    }
    // Per-(group, column) partials.
    double *pg = part_dg + (int64_t)rg * g.N;
    double *pb = part_db + (int64_t)rg * g.N;
    if (g.RL == 1) {
      if (col_ok) {
        pg[cv] = acc.g[0];
        pb[cv] = acc.b[0];
      }
    } else {
      red[threadIdx.x] = acc.g[0];
      red[B + threadIdx.x] = acc.b[0];
      __syncthreads();
      lane_tree<2, B>(red, g, ln);
      if (col_ok && ln.rl == 0) {
        pg[cv] = red[threadIdx.x];
        pb[cv] = red[B + threadIdx.x];
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

}  // namespace dyt
