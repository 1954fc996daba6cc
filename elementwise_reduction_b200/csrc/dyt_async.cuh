// Per-thread asynchronous-copy DyT kernels for sm_100a (16-byte vectors): the
// kernels every 16-byte aligned matrix takes, and (shifted kernels, below)
// every contiguous matrix off 16-byte boundaries.
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
// (S - 1) x 32 bytes per thread, twice that in the shifted kernels) costs no
// registers. Each thread visits exactly its real rows; only the vectors that
// straddle the start or the end of a packed matrix hold padding, which is
// masked after the arithmetic.
#pragma once

#include <cuda_runtime.h>

#include <type_traits>

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
// c0 + e, or on the packed path (c0 + e) mod Nc, where -VEC < c0 < VEC * Nc
// (the shifted kernels pass the vector's offset minus sh).
template <int VEC, bool PK>
__device__ __forceinline__ void vector_columns(int64_t c0, int64_t Nc, int64_t (&col)[VEC]) {
  if constexpr (PK) {
    int64_t c = c0;
    while (c < 0) c += Nc;    // the shifted layout: c0 - sh, sh < VEC
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

// Row frame: matrix columns c + e of the VEC elements of a vector starting
// at column c (c + e may fall in the row's padding, below 0 or at N and
// beyond: those elements are masked, and get column 0 or N - 1 so that every
// parameter load stays inside the parameter vectors).
template <int VEC>
__device__ __forceinline__ void row_frame_columns(int64_t c, int64_t Nc, int64_t (&col)[VEC]) {
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    const int64_t v = c + e;
    col[e] = v < 0 ? 0 : v >= Nc ? Nc - 1 : v;
  }
}

// The elements of a 16-byte vector whose bit is set in m, one by one: the
// vectors that hold padding (a packed matrix's straddling vector, the shifted
// layouts' partial vectors). Its masks are runs of set bits; storing a run as
// aligned 8-, 4- and 2-byte pieces (a loop, or straight-line code) made the
// kernels slower: the flat shifted backward on 16384 x 4096 bf16 one element
// off 76.6 -> 85.0 us, the row frame's forward 63.8 -> 83.1 us.
template <typename T, int VEC>
__device__ __forceinline__ void store_mask(T *p, const uint4 &r, uint32_t m) {
#pragma unroll
  for (int e = 0; e < VEC; ++e) {
    if ((m >> e) & 1u) {
      if constexpr (sizeof(T) == 4) {
        *reinterpret_cast<uint32_t *>(p + e) = word_of(r, e);
      } else {
        const uint32_t u = word_of(r, e >> 1);
        *reinterpret_cast<unsigned short *>(p + e) = (unsigned short)((e & 1) ? (u >> 16) : (u & 0xFFFFu));
      }
    }
  }
}

// ---- shifted kernels: contiguous tensors off 16-byte boundaries ----------------
//
// The packed layout is laid over the output with its matrix starting at
// position sh (the output's offset past a 16-byte boundary, in elements), so
// every output vector is a whole, aligned 16-byte vector. An input whose
// offset differs from the output's by d bytes (mod 16) holds the elements of
// output vector k in bytes [d, d + 16) of its two aligned chunks k and k + 1:
// both are copied into the thread's slot and the vector is cut out of them.

// What the shifted kernels need of one input tensor.
struct ShIn {
  const char *a;     // 16-byte aligned: its first chunk under position 0 of the layout
  int d;             // byte offset of a vector in its two chunks (0: the vector is one chunk)
  uintptr_t lo, hi;  // the tensor's bytes [lo, hi)
};

// rf: the row frame (rows ld elements apart, position 0 of row 0's frame
// sh elements before p); [lo, hi) is then the tensor's span, from its first
// element to its last: the bytes between its rows (the chunks at a row's two
// ends reach into them) lie inside it.
template <typename T>
__device__ __forceinline__ ShIn shifted_input(const T *p, const Geom &g, int64_t ld, bool rf) {
  ShIn s;
  const uintptr_t f = (uintptr_t)p - (uintptr_t)g.sh * sizeof(T);  // where position 0 falls in this tensor
  s.d = (int)(f & 15u);
  s.a = reinterpret_cast<const char *>(f - (uintptr_t)s.d);
  s.lo = (uintptr_t)p;
  s.hi = s.lo + (uintptr_t)(rf ? (g.M - 1) * ld + g.Nc : g.total - g.sh) * sizeof(T);
  return s;
}

// A 16-byte chunk (at a, 16-byte aligned) of a tensor whose bytes are
// [lo, hi), elements of ES bytes: copied whole when it lies inside; only its
// first hi - a bytes (the rest of the slot zero-filled) when the tensor ends in
// it; element by element from lo when the tensor starts in it; not at all when
// it holds none of the tensor. Nothing outside [lo, hi) is read. The slot bytes
// not written hold stale values, which only padded elements take.
template <int ES>
__device__ __forceinline__ void copy_chunk_checked(uint4 *slot, const char *a, uintptr_t lo, uintptr_t hi) {
  const uintptr_t ua = (uintptr_t)a;
  if (ua >= hi || ua + 16u <= lo) return;
  if (ua >= lo) {
    const uintptr_t n = hi - ua;
    cp_async16_zfill(slot, a, n < 16u ? (uint32_t)n : 16u);
    return;
  }
  const int b1 = hi - ua < 16u ? (int)(hi - ua) : 16;
  char *dst = reinterpret_cast<char *>(slot);
  for (int b = (int)(lo - ua); b < b1; b += ES) {
    if constexpr (ES == 4) *reinterpret_cast<uint32_t *>(dst + b) = *reinterpret_cast<const uint32_t *>(a + b);
    else *reinterpret_cast<unsigned short *>(dst + b) = *reinterpret_cast<const unsigned short *>(a + b);
  }
}

// One input's chunks of a row into its slot (chunk 0 at slot, chunk 1 at
// slot + B): plain copies on the rows where every copy lies inside the tensor
// (fast), checked ones elsewhere.
// W: the kernel cuts windows out of this input (its offset may differ from
// the output's); without W its vectors are single chunks (d = 0).
// wb (row frame, wrapped vector-column only; W is then false): the second
// chunk lies wb bytes after the first (the row's last elements).
template <typename T, int B, bool W>
__device__ __forceinline__ void copy_shifted(uint4 *slot, const T *src, const ShIn &s, bool fast,
                                             uintptr_t wb = 0) {
  const char *a = reinterpret_cast<const char *>(src);
  if (fast) {
    cp_async16(slot, a);
    if (W && s.d) cp_async16(slot + B, a + 16);
    if (!W && wb) cp_async16(slot + B, a + wb);
  } else {
    copy_chunk_checked<(int)sizeof(T)>(slot, a, s.lo, s.hi);
    if (W && s.d) copy_chunk_checked<(int)sizeof(T)>(slot + B, a + 16, s.lo, s.hi);
    if (!W && wb) copy_chunk_checked<(int)sizeof(T)>(slot + B, a + wb, s.lo, s.hi);
  }
}

// The row frame's wrapped vector-column (SHM bit 4: N a multiple of VEC, every
// tensor at the output's offset sh > 0): vector-column 0 of a row holds the
// row's last sh elements at positions 0 .. sh - 1 (from the chunk N elements
// on, the slot's second half) and its first VEC - sh at positions sh .. VEC - 1
// (the first half), so a row spans N / VEC vectors as if it were aligned.
// m: the bytes of positions 0 .. sh - 1.
__device__ __forceinline__ uint4 wrap_bytes_mask(int sh, int es) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int nb = sh * es - 4 * i;  // bytes of this word below the cut
    w[i] = nb >= 4 ? 0xFFFFFFFFu : nb <= 0 ? 0u : (1u << (8 * nb)) - 1u;
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 read_wrapped(const uint4 *slot, int B, const uint4 &m) {
  const uint4 a = slot[0], b = slot[B];
  return make_uint4((a.x & ~m.x) | (b.x & m.x), (a.y & ~m.y) | (b.y & m.y), (a.z & ~m.z) | (b.z & m.z),
                    (a.w & ~m.w) | (b.w & m.w));
}

// The input vector of a row from its slot: with W, bytes [d, d + 16) of its
// two chunks (chunk 0 at slot, chunk 1 at slot + B), read as 32-bit words
// d / 4 .. d / 4 + 3 (+ one more, and 16-bit funnel shifts, when d is not a
// multiple of 4: 16-bit elements at an odd offset). Measured against two
// 16-byte loads with the window picked by selects and funnel shifts, on 16384
// x 4096 bf16 with x one element off: backward 97.3 -> 93.4 us, forward 64.4
// -> 63.9 us.
template <int B, bool W>
__device__ __forceinline__ uint4 read_shifted(const uint4 *slot, const ShIn &s) {
  if constexpr (W) {
    const char *base = reinterpret_cast<const char *>(slot);
    const int q = s.d >> 2;
    uint32_t v[5];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int p = q + i;  // word p of the two chunks
      v[i] = *reinterpret_cast<const uint32_t *>(base + (p < 4 ? 4 * p : 16 * B + 4 * (p - 4)));
    }
    if (s.d & 3) {
      v[4] = *reinterpret_cast<const uint32_t *>(base + 16 * B + 4 * q);  // word q + 4, in chunk 1
      return make_uint4(__byte_perm(v[0], v[1], 0x5432), __byte_perm(v[1], v[2], 0x5432),
                        __byte_perm(v[2], v[3], 0x5432), __byte_perm(v[3], v[4], 0x5432));
    }
    return make_uint4(v[0], v[1], v[2], v[3]);
  } else {
    return *slot;
  }
}

// Whether row k of a thread is one of its whole-vector rows [k_lo, k_hi).
__device__ __forceinline__ bool fast_row(int k, int k_lo, int k_hi) {
  return (unsigned)(k - k_lo) < (unsigned)(k_hi - k_lo);
}

// Real elements (bits) of the output vector at position pos of the layout:
// those in [sh, total).
template <int VEC>
__device__ __forceinline__ uint32_t shifted_mask(const Geom &g, int64_t pos) {
  const int lo = pos < g.sh ? (int)(g.sh - pos) : 0;
  const int64_t rem = g.total - pos;
  const int hi = rem <= 0 ? 0 : rem < VEC ? (int)rem : VEC;
  return ((1u << hi) - 1u) & ~((1u << lo) - 1u);
}

// The L2 prefetch of prefetch_first_rows_l2 for the shifted kernels: the same
// rows of the layout, clipped to the 16-byte units that lie wholly inside the
// tensor, so nothing outside it is touched.
template <typename T, int VEC, int B, int S>
__device__ __forceinline__ void prefetch_shifted_rows_l2(const ShIn &s, const Geom &g) {
  if (!g.l2_prefetch || threadIdx.x >= 32 || (int)blockIdx.x >= g.nitems) return;  // warp 0 issues them
  int cc, rg;
  item_split(g, blockIdx.x, cc, rg);
  int64_t rb, re;
  group_rows(g, rg, rb, re);
  const int64_t rows = min(re - rb, (int64_t)(S - 1) * g.RL);
  if (rows <= 0) return;
  const uintptr_t lo = (s.lo + 15u) & ~(uintptr_t)15, hi = s.hi & ~(uintptr_t)15;
  constexpr uintptr_t kPiece = 16384;
  uintptr_t a, e;
  if (g.ncc == 1) {  // whole rows: one range, cut into pieces
    a = (uintptr_t)s.a + (uintptr_t)(rb * g.N) * sizeof(T) + threadIdx.x * kPiece;
    e = (uintptr_t)s.a + (uintptr_t)((rb + rows) * g.N) * sizeof(T);
    if (e > a + kPiece) e = a + kPiece;
  } else {  // one column chunk of each row
    if (threadIdx.x >= rows) return;
    const int64_t c0 = (int64_t)cc * g.cw * VEC;
    a = (uintptr_t)s.a + (uintptr_t)((rb + threadIdx.x) * g.N + c0) * sizeof(T);
    e = a + (uintptr_t)min((int64_t)g.cw * VEC, g.N - c0) * sizeof(T);
  }
  if (a < lo) a = lo;
  if (e > hi) e = hi;
  if (a < e)
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"((uint32_t)(e - a)) : "memory");
}

// Whether input chunk(s) at a lie inside the tensor from below / from above.
__device__ __forceinline__ bool shifted_lo_ok(const ShIn &s, const void *a) { return (uintptr_t)a >= s.lo; }
__device__ __forceinline__ bool shifted_hi_ok(const ShIn &s, const void *a) {
  return (uintptr_t)a + (s.d ? 32u : 16u) <= s.hi;
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
    const int64_t c0 = (int64_t)cc * g.cw * VEC;
    const int64_t at = (rb + threadIdx.x) * ld + c0;
    int64_t n = min((int64_t)g.cw * VEC, g.N - c0);
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

// SHM != 0: the shifted kernels (contiguous tensors not all 16-byte aligned;
// PK holds): ring slots of two chunks, the packed layout laid over the output
// with its matrix from position g.sh, rows whose copies or output vector reach
// past a tensor's ends handled one by one (checked copies, masked stores).
// SHM bit 1: x's offset differs from y's, so its vectors are cut out of two
// chunks. SHM bit 3: the row frame (RF) instead of the flat packed layout:
// strided rows, each laid out on its own from position sh (see row_frame_*);
// bit 4 (WR): with its wrapped vector-column (see read_wrapped).
template <typename T, typename P, int VEC, int B, int S, bool PK, int SHM>
__global__ void __launch_bounds__(B, 1)
    dyt_fwd_async_kernel(const T *__restrict__ x, const P *__restrict__ alpha_p, const P *__restrict__ gamma_p,
                         const P *__restrict__ beta_p, ParamTypes pt, T *y, Geom g) {
  using IO = VecIO<T, VEC>;
  constexpr bool SH = SHM != 0, WX = (SHM & 2) != 0, RF = (SHM & 8) != 0, WR = (SHM & 16) != 0;
  constexpr bool FL = SH && !RF;  // the flat shifted layout
  static_assert(!WR || (RF && !WX), "the wrapped column: row frame, inputs at the output's offset");
  static_assert(VEC * sizeof(T) == 16, "16-byte vectors");
  static_assert(PK == FL || (PK && !SH), "the flat shifted kernels use the packed layout, the row frame does not");
  constexpr int CH = SH ? 2 : 1;  // 16-byte chunks per slot
  extern __shared__ uint4 ring[];  // [S][CH][B]
  // A launch whose shared memory cannot hold the ring writes nothing (the
  // host sizes it from the same constants; this only keeps a mismatch from
  // reaching past the allocation).
  if (dynamic_smem_bytes() < (uint32_t)(S * CH * B * 16)) return;
  ShIn ix = {};
  if constexpr (SH) ix = shifted_input(x, g, g.ldx, RF);
  if constexpr (FL) {
    prefetch_shifted_rows_l2<T, VEC, B, S>(ix, g);
  } else if constexpr (!RF) {
    prefetch_first_rows_l2<T, VEC, B, S, PK>(x, g.ldx, g);
  }
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = load_param<P>(alpha_p, pt.alpha, 0);
  uint4 *slot0 = ring + threadIdx.x;
  const T *xb = SH ? reinterpret_cast<const T *>(ix.a) : x;  // position 0 of the layout
  T *yb = SH ? y - g.sh : y;
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    int cc, rg;
    item_split(g, item, cc, rg);
    int64_t rb, re;
    group_rows(g, rg, rb, re);
    const int cv = cc * g.cw + ln.cv;
    if (!(ln.live && cv < g.NV)) continue;
    const int64_t c0 = (int64_t)cv * VEC;
    int64_t first;
    int64_t n = thread_rows(g, rb, re, ln.rl, first);
    const int nl = last_vector_real<VEC, PK>(g, first, c0, n);
    const uint32_t last_bytes = (uint32_t)(nl * (int)sizeof(T));
    const int64_t sx = (int64_t)g.RL * g.ldx, sy = (int64_t)g.RL * g.ldo;
    const T *px = xb + first * g.ldx + c0;
    T *py = yb + first * g.ldo + c0;
    // SH: rows [k_lo, k_hi) copy whole chunks (and FL: store whole vectors);
    // the others (at most a few at each end of the matrix; RF: the tensor's
    // first and last rows) copy element by element.
    const int64_t pos0 = first * g.N + c0, dpos = (int64_t)g.RL * g.N;  // layout positions
    int k_lo = 0, k_hi = (int)n;  // n is at most kMaxRowsPerLane
    // RF: the real elements of the thread's vectors are the same in every row
    const uint32_t rmask = RF ? shifted_mask<VEC>(g, c0) : 0xFFu;
    const bool rstore = !RF || rmask == (1u << VEC) - 1u;
    // WR: vector-column 0 is the wrapped one; its second chunk lies N on
    const bool wrap = WR && cv == 0;
    const int64_t wn = wrap ? g.Nc : 0;
    const uint4 wm = wrap_bytes_mask(WR ? g.sh : 0, (int)sizeof(T));
    const uint32_t wlo = ~((1u << g.sh) - 1u) & ((1u << VEC) - 1u), whi = (1u << g.sh) - 1u;
    if constexpr (SH) {
      while (k_lo < n && !((RF || pos0 + k_lo * dpos >= g.sh) && shifted_lo_ok(ix, px + k_lo * sx))) ++k_lo;
      while (k_hi > k_lo &&
             !((RF || pos0 + (k_hi - 1) * dpos + VEC <= g.total) && shifted_hi_ok(ix, px + (k_hi - 1) * sx + wn)))
        --k_hi;
    }
    // Rows first, parameters second: the parameter loads overlap the copies.
#pragma unroll
    for (int k = 0; k < S - 1; ++k) {
      if (k < n) {
        if constexpr (SH)
          copy_shifted<T, B, WX>(slot0 + k * CH * B, px + k * sx, ix, fast_row(k, k_lo, k_hi), wn * sizeof(T));
        else if (PK) cp_async16_zfill(slot0 + k * B, px + k * sx, k == n - 1 ? last_bytes : 16u);
        else cp_async16(slot0 + k * B, px + k * sx);
      }
      cp_async_commit();
    }
    int64_t col[VEC];
    if constexpr (WR) vector_columns<VEC, true>(c0 - g.sh, g.Nc, col);  // (c0 + e - sh) mod N
    else if constexpr (RF) row_frame_columns<VEC>(c0 - g.sh, g.Nc, col);
    else vector_columns<VEC, PK>(SH ? c0 - g.sh : c0, g.Nc, col);
    float gam[VEC], bet[VEC], bth[VEC];
    fwd_params_at<T, VEC, P>(gamma_p, beta_p, pt, col, gam, bet, bth);
    int s_rd = 0, s_wr = S - 1;
    if constexpr (SH) {
      // One ring step: copy row k + S - 1, then compute and store row k. CHK:
      // the step tests whether its rows are whole-vector rows; iterations
      // [k_lo, k_hi - S + 1) need no test (both rows lie in [k_lo, k_hi)).
      int64_t k = 0;
      auto step = [&](auto chk) {
        constexpr bool CHK = decltype(chk)::value;
        const int64_t kn = k + S - 1;
        if (!CHK || kn < n)
          copy_shifted<T, B, WX>(slot0 + s_wr * CH * B, px + kn * sx, ix, !CHK || fast_row((int)kn, k_lo, k_hi),
                                 wn * sizeof(T));
        cp_async_commit();
        cp_async_wait<S - 1>();
        const uint4 v = WR && wrap ? read_wrapped(slot0 + s_rd * CH * B, B, wm)
                                   : read_shifted<B, WX>(slot0 + s_rd * CH * B, ix);
        const typename IO::Raw ry = fwd_vector<T, VEC>(v, alpha, gam, bet, bth);
        if (WR && wrap) {  // the row's first VEC - sh elements, then its last sh
          store_mask<T, VEC>(py, ry, wlo);
          store_mask<T, VEC>(py + g.Nc, ry, whi);
        } else if (!rstore) store_mask<T, VEC>(py, ry, rmask);  // RF: the row's padding is not stored
        else if (RF || !CHK || fast_row((int)k, k_lo, k_hi)) IO::store_raw(py, ry);
        else store_mask<T, VEC>(py, ry, shifted_mask<VEC>(g, pos0 + k * dpos));  // padding: not stored
        py += sy;
        s_rd = s_rd + 1 == S ? 0 : s_rd + 1;
        s_wr = s_wr + 1 == S ? 0 : s_wr + 1;
        ++k;
      };
      const int64_t f1 = max((int64_t)k_lo, (int64_t)k_hi - (S - 1));
      if (f1 - k_lo >= 2 * S) {  // enough unchecked steps to pay for the phases
        while (k < k_lo) step(std::true_type{});
        while (k < f1) step(std::false_type{});
      }
      while (k < n) step(std::true_type{});
    } else {
      int64_t k = 0;
      // fp32 rows two at a time while both are whole, for threads with at least
      // 2 S rows (as the backward's pairs; here only the 4-element vectors
      // gain: 100003 x 100 fp32 16.35 -> 14.33 us, 100003 x 255 38.25 ->
      // 37.25 us, while the 16-bit forward lost 2% and threads with a few rows
      // lose a little). Same bits as the one-row loop.
      if constexpr (sizeof(T) == 4) {
        const int64_t np = PK && nl < VEC ? n - 1 : n;  // the masked last vector stays below
        for (; n >= 2 * S && k + 1 < np; k += 2) {
          cp_async_wait<S - 3>();  // rows k and k + 1 have landed
          const int s_rd1 = s_rd + 1 == S ? 0 : s_rd + 1;
          const typename IO::Raw rx0 = *(const typename IO::Raw *)(slot0 + s_rd * B);
          const typename IO::Raw rx1 = *(const typename IO::Raw *)(slot0 + s_rd1 * B);
          const int s_wr1 = s_wr + 1 == S ? 0 : s_wr + 1;
          const int64_t k1 = k + S - 1, k2 = k + S;
          if (k1 < n) {
            if (PK) cp_async16_zfill(slot0 + s_wr * B, px + k1 * sx, k1 == n - 1 ? last_bytes : 16u);
            else cp_async16(slot0 + s_wr * B, px + k1 * sx);
          }
          cp_async_commit();
          if (k2 < n) {
            if (PK) cp_async16_zfill(slot0 + s_wr1 * B, px + k2 * sx, k2 == n - 1 ? last_bytes : 16u);
            else cp_async16(slot0 + s_wr1 * B, px + k2 * sx);
          }
          cp_async_commit();
          const typename IO::Raw ry0 = fwd_vector<T, VEC>(rx0, alpha, gam, bet, bth);
          const typename IO::Raw ry1 = fwd_vector<T, VEC>(rx1, alpha, gam, bet, bth);
          IO::store_raw(py, ry0);
          IO::store_raw(py + sy, ry1);
          py += 2 * sy;
          s_rd = s_rd1 + 1 == S ? 0 : s_rd1 + 1;
          s_wr = s_wr1 + 1 == S ? 0 : s_wr1 + 1;
        }
      }
      for (; k < n; ++k) {
        const int64_t kn = k + S - 1;
        if (kn < n) {
          if (PK) cp_async16_zfill(slot0 + s_wr * B, px + kn * sx, kn == n - 1 ? last_bytes : 16u);
          else cp_async16(slot0 + s_wr * B, px + kn * sx);
        }
        cp_async_commit();
        cp_async_wait<S - 1>();
        const typename IO::Raw rx = *(const typename IO::Raw *)(slot0 + s_rd * B);
        const typename IO::Raw ry = fwd_vector<T, VEC>(rx, alpha, gam, bet, bth);
        if (PK && k == n - 1 && nl < VEC) store_mask<T, VEC>(py, ry, (1u << nl) - 1u);  // zero-filled tail: not stored
        else IO::store_raw(py, ry);
        py += sy;
        s_rd = s_rd + 1 == S ? 0 : s_rd + 1;
        s_wr = s_wr + 1 == S ? 0 : s_wr + 1;
      }
    }
    cp_async_wait<0>();
  }
}

// ---- backward, stage 1 ----------------------------------------------------------

// SHM != 0: as the forward's shifted kernels, x and dy each with their own
// offset: bit 1 cuts x's vectors out of two chunks, bit 2 dy's; bit 3 the row
// frame, bit 4 its wrapped vector-column.
template <typename T, typename P, int VEC, int B, int S, bool PK, int SHM>
__global__ void __launch_bounds__(B, 1)
    dyt_bwd_async_kernel(const T *__restrict__ x, const T *__restrict__ dy, const P *__restrict__ alpha_p,
                         const P *__restrict__ gamma_p, ParamTypes pt, T *dx, double *__restrict__ part_dg,
                         double *__restrict__ part_db, double *__restrict__ part_da, Geom g) {
  using IO = VecIO<T, VEC>;
  constexpr bool SH = SHM != 0, WX = (SHM & 2) != 0, WD = (SHM & 4) != 0, RF = (SHM & 8) != 0;
  constexpr bool WR = (SHM & 16) != 0;
  constexpr bool FL = SH && !RF;  // the flat shifted layout
  static_assert(!WR || (RF && !WX && !WD), "the wrapped column: row frame, inputs at the output's offset");
  constexpr bool EXACT_G = ExactGamma<T>::value;
  constexpr int kRunBlocks = kGammaRunRows / S;  // unrolled blocks of S rows per binary32 dgamma run
  constexpr int CH = SH ? 2 : 1;                 // 16-byte chunks per slot
  static_assert(VEC * sizeof(T) == 16, "16-byte vectors");
  static_assert(PK == FL || (PK && !SH), "the flat shifted kernels use the packed layout, the row frame does not");
  static_assert(2 * VEC * sizeof(double) <= 2 * S * 16, "the reduction fits in the drained ring");
  static_assert(kRunBlocks >= 1, "a dgamma run holds at least one block");
  // [S][2][CH][B] 16-byte slots (x, then dy); after an item's last row the
  // ring is empty and its first 2 VEC * B binary64 values (at most 64 KB) serve
  // the row-lane reduction. Without EXACT_G, [VEC][B] binary64 dgamma totals
  // follow the ring (each thread's own, flushed from its binary32 runs).
  extern __shared__ uint4 ring[];
  __shared__ double red_a[B / 32];
  // A launch whose shared memory cannot hold the ring and the dgamma totals
  // writes nothing (see the forward).
  if (dynamic_smem_bytes() < (uint32_t)(2 * S * CH * B * 16 + (EXACT_G ? 0 : VEC * B * 8))) return;
  ShIn ix = {}, id = {};
  if constexpr (SH) {
    ix = shifted_input(x, g, g.ldx, RF);
    id = shifted_input(dy, g, g.ldd, RF);
  }
  if constexpr (FL) {
    prefetch_shifted_rows_l2<T, VEC, B, S>(ix, g);
    prefetch_shifted_rows_l2<T, VEC, B, S>(id, g);
  } else if constexpr (!RF) {
    prefetch_first_rows_l2<T, VEC, B, S, PK>(x, g.ldx, g);
    prefetch_first_rows_l2<T, VEC, B, S, PK>(dy, g.ldd, g);
  }
  pdl_prologue();
  const Lane ln = lane_of(g, threadIdx.x);
  const float alpha = load_param<P>(alpha_p, pt.alpha, 0);
  double *red = reinterpret_cast<double *>(ring);
  double *gtot = reinterpret_cast<double *>(ring + 2 * S * CH * B) + threadIdx.x;  // [e * B]
  uint4 *slot0 = ring + threadIdx.x;
  const T *xb = SH ? reinterpret_cast<const T *>(ix.a) : x;  // position 0 of the layout
  const T *db = SH ? reinterpret_cast<const T *>(id.a) : dy;
  T *dxb = SH ? dx - g.sh : dx;
  double acc_a = 0.0;
  for (int item = blockIdx.x; item < g.nitems; item += gridDim.x) {
    int cc, rg;
    item_split(g, item, cc, rg);
    int64_t rb, re;
    group_rows(g, rg, rb, re);
    const int cv = cc * g.cw + ln.cv;
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
      const T *px = xb + first * g.ldx + c0;  // the next rows to copy (advanced, not re-derived)
      const T *pd = db + first * g.ldd + c0;
      T *pdx = dxb + first * g.ldo + c0;
      // SH: rows [k_lo, k_hi) copy whole chunks (and FL: store whole
      // vectors); the others (at most a few at each end of the matrix; RF:
      // the tensors' first and last rows) copy element by element.
      const int64_t pos0 = first * g.N + c0, dpos = (int64_t)g.RL * g.N;  // layout positions
      int k_lo = 0, k_hi = nn;
      // RF: the real elements of the thread's vectors are the same in every row
      const uint32_t rmask = RF ? shifted_mask<VEC>(g, c0) : 0xFFu;
      const bool rstore = !RF || rmask == (1u << VEC) - 1u;
      // WR: vector-column 0 is the wrapped one; its second chunk lies N on
      const bool wrap = WR && cv == 0;
      const int64_t wn = wrap ? g.Nc : 0;
      const uintptr_t wb = (uintptr_t)wn * sizeof(T);
      const uint4 wm = wrap_bytes_mask(WR ? g.sh : 0, (int)sizeof(T));
      const uint32_t wlo = ~((1u << g.sh) - 1u) & ((1u << VEC) - 1u), whi = (1u << g.sh) - 1u;
      if constexpr (SH) {
        while (k_lo < nn && !((RF || pos0 + k_lo * dpos >= g.sh) && shifted_lo_ok(ix, px + k_lo * sx) &&
                              shifted_lo_ok(id, pd + k_lo * sd)))
          ++k_lo;
        while (k_hi > k_lo &&
               !((RF || pos0 + (k_hi - 1) * dpos + VEC <= g.total) && shifted_hi_ok(ix, px + (k_hi - 1) * sx + wn) &&
                 shifted_hi_ok(id, pd + (k_hi - 1) * sd + wn)))
          --k_hi;
      }
      // Rows first, parameters second: the gamma loads overlap the copies.
      // Row r lives in slot r mod S; the loop below is unrolled by S so that
      // every slot index is a constant.
#pragma unroll
      for (int k = 0; k < S - 1; ++k) {
        if (k < nn) {
          if constexpr (SH) {
            const bool fast = fast_row(k, k_lo, k_hi);
            copy_shifted<T, B, WX>(slot0 + (2 * k) * CH * B, px, ix, fast, wb);
            copy_shifted<T, B, WD>(slot0 + (2 * k + 1) * CH * B, pd, id, fast, wb);
          } else if (PK) {
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
      if constexpr (WR) vector_columns<VEC, true>(c0 - g.sh, g.Nc, col);  // (c0 + e - sh) mod N
      else if constexpr (RF) row_frame_columns<VEC>(c0 - g.sh, g.Nc, col);
      else vector_columns<VEC, PK>(SH ? c0 - g.sh : c0, g.Nc, col);
      load_params<VEC, P>(gamma_p, pt.gamma, col, 4.0f, gam);  // 4 gamma (see bwd_vector)
      int run = 0;  // blocks in the current binary32 dgamma run
      for (int k0 = 0; k0 < nn; k0 += S) {
        float2 ca = make_float2(0.0f, 0.0f);  // this block's dalpha terms (at most S VEC / 2 per lane)
        // Rows k0 .. k0 + S - 1. CHK: the rows and their copies are tested
        // (ends of the matrix, the shifted kernels' partial vectors); the
        // shifted kernels skip the tests on blocks whose rows and copies all
        // lie in [k_lo, k_hi).
        auto block = [&](auto chk) {
          constexpr bool CHK = decltype(chk)::value;
          // 512-thread CTAs, whole blocks (aligned or packed rows; the packed
          // matrix's last, partial vector stays on the one-row loop): rows two
          // at a time.
          // One wait covers rows k and k + 1; both are read, the next two
          // copies are issued (the prefetch distance stays S - 1 rows), and
          // the two rows are computed together: twice the independent work
          // between stalls for the CTA's 16 warps. The sums take the rows in
          // the same order, so the bits are those of the one-row loop.
          // Measured (B200, interleaved CUDA graphs): 32768 x 8192 bf16
          // 278.4 -> 263.2 us, 16384 x 4096 bf16 74.8 -> 72.7 us, 100003 x 255
          // fp32 (packed) 61.7 -> 59.6 us; the narrow 256-thread CTAs gained
          // nothing and keep the one-row loop. (The forward, tried the same
          // way, lost 2% on the bf16 shapes.)
          if constexpr (!SH && S % 2 == 0 && B >= 512) {
            if (k0 + S < nn || (k0 + S == nn && (!PK || nl == VEC))) {
#pragma unroll
              for (int j = 0; j < S; j += 2) {
                const int k = k0 + j;
                cp_async_wait<S - 3>();  // rows k and k + 1 have landed
                const typename IO::Raw rx0 = *(const typename IO::Raw *)(slot0 + (2 * j) * B);
                const typename IO::Raw rd0 = *(const typename IO::Raw *)(slot0 + (2 * j + 1) * B);
                const typename IO::Raw rx1 = *(const typename IO::Raw *)(slot0 + (2 * j + 2) * B);
                const typename IO::Raw rd1 = *(const typename IO::Raw *)(slot0 + (2 * j + 3) * B);
                if (k + S - 1 < nn) {  // row k + S - 1 into slot (j + S - 1) mod S
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
                if (k + S < nn) {  // row k + S into slot j (read above)
                  if (PK) {
                    const uint32_t b = k + S == nn - 1 ? last_bytes : 16u;
                    cp_async16_zfill(slot0 + (2 * j) * B, px, b);
                    cp_async16_zfill(slot0 + (2 * j + 1) * B, pd, b);
                  } else {
                    cp_async16(slot0 + (2 * j) * B, px);
                    cp_async16(slot0 + (2 * j + 1) * B, pd);
                  }
                }
                px += sx;
                pd += sd;
                cp_async_commit();
                const typename IO::Raw o0 = bwd_vector<T, VEC, false, EXACT_G>(rx0, rd0, alpha, gam, acc, ca, 0xFFu);
                const typename IO::Raw o1 = bwd_vector<T, VEC, false, EXACT_G>(rx1, rd1, alpha, gam, acc, ca, 0xFFu);
                IO::store_raw(pdx, o0);
                IO::store_raw(pdx + so, o1);
                pdx += 2 * so;
              }
              return;
            }
          }
#pragma unroll
          for (int j = 0; j < S; ++j) {
            const int k = k0 + j;
            if (CHK && k >= nn) break;
            if (!CHK || k + S - 1 < nn) {  // rows k + S - 1 into slot (j + S - 1) mod S
              const int sw = (j + S - 1) % S;
              if constexpr (SH) {
                const bool fast = !CHK || fast_row(k + S - 1, k_lo, k_hi);
                copy_shifted<T, B, WX>(slot0 + (2 * sw) * CH * B, px, ix, fast, wb);
                copy_shifted<T, B, WD>(slot0 + (2 * sw + 1) * CH * B, pd, id, fast, wb);
              } else if (PK) {
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
            typename IO::Raw rx, rd;
            if constexpr (WR) {
              if (wrap) {
                rx = read_wrapped(slot0 + (2 * j) * CH * B, B, wm);
                rd = read_wrapped(slot0 + (2 * j + 1) * CH * B, B, wm);
              } else {
                rx = *(slot0 + (2 * j) * CH * B);
                rd = *(slot0 + (2 * j + 1) * CH * B);
              }
            } else if constexpr (SH) {
              rx = read_shifted<B, WX>(slot0 + (2 * j) * CH * B, ix);
              rd = read_shifted<B, WD>(slot0 + (2 * j + 1) * CH * B, id);
            } else {
              rx = *(const typename IO::Raw *)(slot0 + (2 * j) * B);
              rd = *(const typename IO::Raw *)(slot0 + (2 * j + 1) * B);
            }
            if constexpr (RF) {
              // One computation for every thread, masked by the thread's own
              // mask (the wrapped vector-column holds no padding), so that no
              // warp runs it twice for its partial vectors: on 16384 x 4096
              // bf16, pitch 4104, every tensor one element off, warp 0
              // computing twice held the other warps at the item's barrier
              // (ncu: barrier stalls 2.58 per issue against 0.07; 127 -> 98 us
              // with one computation). Only the stores differ.
              const typename IO::Raw o = bwd_vector<T, VEC, !WR, EXACT_G>(rx, rd, alpha, gam, acc, ca, rmask);
              if (WR && wrap) {  // the row's first VEC - sh elements, then its last sh
                store_mask<T, VEC>(pdx, o, wlo);
                store_mask<T, VEC>(pdx + g.Nc, o, whi);
              } else if (!rstore) {
                store_mask<T, VEC>(pdx, o, rmask);  // the row's padding is dropped
              } else {
                IO::store_raw(pdx, o);
              }
            } else if (FL && CHK && !fast_row(k, k_lo, k_hi)) {  // padding of the shifted layout: dropped
              const uint32_t m = shifted_mask<VEC>(g, pos0 + k * dpos);
              store_mask<T, VEC>(pdx, bwd_vector<T, VEC, true, EXACT_G>(rx, rd, alpha, gam, acc, ca, m), m);
            } else if (!SH && PK && k == nn - 1 && nl < VEC) {  // the straddling vector: its zero-filled tail is dropped
              const uint32_t m = (1u << nl) - 1u;
              store_mask<T, VEC>(pdx, bwd_vector<T, VEC, true, EXACT_G>(rx, rd, alpha, gam, acc, ca, m), m);
            } else {
              IO::store_raw(pdx, bwd_vector<T, VEC, false, EXACT_G>(rx, rd, alpha, gam, acc, ca, 0xFFu));
            }
            pdx += so;
          }
        };
        if constexpr (SH && B >= 512) {  // narrow rows (256-thread CTAs) give each thread few rows
          if (k0 >= k_lo && k0 + 2 * S - 2 < k_hi) block(std::false_type{});
          else block(std::true_type{});
        } else {
          block(std::true_type{});
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
    // a row of partials holds N (RF: Nc, the columns) values
    double *pg = part_dg + (int64_t)rg * (RF ? g.Nc : g.N);
    double *pb = part_db + (int64_t)rg * (RF ? g.Nc : g.N);
    if (g.RL == 1) {
      if (col_ok) {
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          const int64_t q = c0 + e;
          if constexpr (RF && !WR) {
            if (q >= g.sh && q - g.sh < g.Nc) {
              pg[q - g.sh] = ag[e];
              pb[q - g.sh] = acc.b[e];
            }
          } else {
            const int64_t at = SH ? shifted_slot(g, q) : q;
            pg[at] = ag[e];
            pb[at] = acc.b[e];
          }
        }
      }
    } else {
      __syncthreads();  // every thread's ring is drained: reuse it for the reduction
      if ((32 % g.NV) == 0) {
        // the chunk's columns start at 0 on the row-tiled path (one chunk)
        lane_reduce_warps<VEC, B, RF && !WR ? 2 : SH ? 1 : 0>(ag, acc.b, red, g, ln, 0, pg, pb);
      } else {  // dgamma and dbeta sums: 2 VEC values per thread, added over the row lanes in order
#pragma unroll
        for (int e = 0; e < VEC; ++e) {
          red[e * B + threadIdx.x] = ag[e];
          red[(VEC + e) * B + threadIdx.x] = acc.b[e];
        }
        __syncthreads();
        // Thread t = i NV + v forms value i (dgamma e = i, then dbeta e = i - VEC)
        // of vector-column v: lane 0 + lane 1 + ... (thread rl NV + v holds lane
        // rl). One barrier instead of a fixed-order tree of ceil(log2 RL)
        // barrier-separated levels: 100003 x 17 fp32 backward 10.0 -> 9.7 us,
        // 65537 x 24 bf16 10.4 -> 9.1 us, 100003 x 100 fp32 25.4 -> 24.9 us.
        for (int t = threadIdx.x; t < 2 * VEC * g.NV; t += B) {
          const int i = t / g.NV, v = t - i * g.NV;
          const double *src = red + i * B + v;
          double sum = 0.0;
          for (int r = 0; r < g.RL; ++r) sum += src[r * g.NV];
          const int e = i < VEC ? i : i - VEC;
          double *out = i < VEC ? pg : pb;
          const int64_t q = (int64_t)v * VEC + e;
          if constexpr (RF && !WR) {
            if (q >= g.sh && q - g.sh < g.Nc) out[q - g.sh] = sum;
          } else {
            out[SH ? shifted_slot(g, q) : q] = sum;
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
