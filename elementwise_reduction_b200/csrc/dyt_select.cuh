// Which kernel a launch plan runs: the launch constants the host planning and
// the kernel instantiations share, and the selectors that return a kernel
// pointer. The selectors are defined in dyt_select_impl.cuh and instantiated
// once per activation dtype (dyt_inst_f32.cu, dyt_inst_bf16.cu,
// dyt_inst_f16.cu), so that the kernels compile in parallel.
#pragma once

#include <cstdint>

#include "dyt_kernels.cuh"

namespace dyt {
namespace launch {

constexpr int kScalarBlock = 1024;      // threads per CTA of the one-element kernels
constexpr int kScalarUnrollFwd = 8;     // rows in flight per thread there
constexpr int kScalarUnrollBwd = 8;
constexpr int kAsyncBlock = 512;        // 16-byte kernels: one CTA per SM, up to 128 registers a thread
constexpr int kAsyncStagesFwd = 8;      // ring slots per thread (forward: x)
constexpr int kAsyncStagesBwd = 6;      // ring slots per thread (backward: x and dy)
// The backward over narrow rows (at most kNarrowMaxNV 16-byte vectors per row)
// runs 256-thread CTAs with deeper rings: each thread then visits twice the
// rows, and the per-thread fixed work (group bounds, ring prologue, parameter
// loads, the row-lane reduction) is spread over twice the elements. Measured
// on B200: 65537 x 32 bf16 9.2 -> 8.2 us, 100003 x 17 fp32 11.3 -> 10.0 us,
// 100003 x 100 fp32 26.9 -> 25.0 us; 128 threads and 12 slots were slower.
constexpr int kAsyncBlockNarrow = 256;
constexpr int kAsyncStagesBwdNarrow = 8;
constexpr int kNarrowMaxNV = 32;
// Rows one lane adds per group, at most. The kernels count a thread's rows with
// a multiply-high by ceil(2^32 / RL), exact for counts below 2^32 / RL; a
// count stays below 2049 RL, and 2049 RL^2 < 2^32 for every RL <= 1024.
constexpr int kMaxRowsPerLane = 2048;
// Strided rows whose pitches are not whole 16-byte vectors run as k phases
// (rows j, j + k, ...) of whole-vector pitch only when each phase moves at
// least this many bytes per tensor (forward / backward); smaller calls take
// the one-element kernels in one launch. Each phase is a launch of its own,
// with its fixed costs, and the backward's phases each leave a full partial
// set. Measured (bf16, 4096 columns, pitch 4100, two phases): 600 rows
// forward 8.8 -> 9.0 us, 2000 rows forward 20.0 -> 15.0 but backward 28.1 ->
// 41.9, 16384 rows backward 154.6 -> 117.7; eight phases of 375 rows x 255
// columns forward 4.0 -> 30.5 us.
constexpr int64_t kPhaseMinBytesFwd = (int64_t)8 << 20;
constexpr int64_t kPhaseMinBytesBwd = (int64_t)32 << 20;
// Inputs read by one launch below which the L2 prefetch of the first rows is
// skipped (bytes): smaller inputs are likely resident in L2 already.
constexpr int64_t kPrefetchMinBytes = 1 << 20;

template <typename T>
constexpr int vec_of() {
  return 16 / (int)sizeof(T);
}

template <typename T, typename P>
using FwdKernel = void (*)(const T *, const P *, const P *, const P *, ParamTypes, T *, Geom);
template <typename T, typename P>
using BwdKernel = void (*)(const T *, const T *, const P *, const P *, ParamTypes, T *, double *, double *,
                           double *, Geom);

// The forward kernel of a plan: the 16-byte kernels (aligned, packed or
// shifted) or the one-element kernel. shm: the shifted kernels' mode (0 = not
// shifted; else 1, | 2 when x's vectors are cut out of two chunks, | 8 for the
// row frame, | 16 for its wrapped vector-column).
template <typename T, typename P>
FwdKernel<T, P> fwd_kernel_of(bool async, bool packed, int shm);

// Stage 1 of the backward of a plan; narrow rows run on 256-thread CTAs. shm:
// as for the forward, | 4 for dy (a mode with bit 2 alone runs as 7).
template <typename T, typename P>
BwdKernel<T, P> bwd_kernel_of(bool async, bool packed, int shm, int block);

}  // namespace launch
}  // namespace dyt
