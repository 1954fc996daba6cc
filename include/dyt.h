/*
 * dyt.h -- C ABI of the fused Dynamic Tanh (DyT) layer for NVIDIA B200 (sm_100a).
 *
 * The layer is the one of the Liger-Kernel pull request "fix(dyt): use a 1D
 * grid and tile small-width rows" (Summary): a scalar alpha, per-column gamma
 * and beta, a fused forward kernel and a fused backward kernel that returns
 * dx and the parameter gradients dalpha, dgamma and dbeta. For an M x N
 * row-major activation x:
 *
 *   forward   y[i,j]    = gamma[j] * tanh(alpha * x[i,j]) + beta[j]
 *   backward  t[i,j]    = tanh(alpha * x[i,j])            (recomputed, not saved)
 *             dx[i,j]   = alpha * gamma[j] * dy[i,j] * (1 - t[i,j]^2)
 *             dgamma[j] = sum_i dy[i,j] * t[i,j]
 *             dbeta[j]  = sum_i dy[i,j]
 *             dalpha    = sum_{i,j} gamma[j] * dy[i,j] * (1 - t[i,j]^2) * x[i,j]
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Pointers: every tensor pointer is a DEVICE pointer (or memory the device
 *   can address, such as managed memory), alpha included, so no call reads
 *   device memory on the host or synchronises. The caller owns every buffer,
 *   the workspace included; the library allocates nothing and keeps no state
 *   other than the calling thread's last-launch record.
 * - Layout: x, dy, y and dx are row-major M x N arrays, contiguous (row
 *   stride N elements) for dyt_forward / dyt_backward and with a row pitch
 *   per tensor for the *_strided entry points. gamma, beta, dgamma and dbeta
 *   hold N elements; alpha and
 *   dalpha hold one. Every pointer must hold whole elements of its dtype
 *   (2- or 4-byte aligned; others give DYT_ERR_INVALID_VALUE); beyond that
 *   any alignment is accepted. 16-byte aligned tensors take the vectorised
 *   path, for any N (a ragged N is streamed in packs of 16 / element-size
 *   rows, which always span whole 16-byte vectors). Contiguous tensors that
 *   are not all 16-byte aligned take the shifted vectorised kernels: whole
 *   16-byte vectors of the output, each input vector cut out of two aligned
 *   16-byte chunks; no byte outside a tensor is read or written.
 * - Dtypes (the page's Summary, "Precision"): x, dy, y and dx share x_dtype,
 *   so y and dx come back in x's dtype. Each parameter gradient comes back in
 *   its parameter's dtype: dalpha in alpha's, dgamma in gamma's, dbeta in
 *   beta's. The *_ex entry points take the three parameter dtypes one by one;
 *   the others take one param_dtype for all three. Element arithmetic is
 *   binary32; the parameter-gradient sums are binary64 throughout, rounded
 *   once to the gradient's dtype.
 * - Outputs are overwritten, never accumulated into.
 * - Aliasing: y may alias x, and dx may alias x or dy (each element is read
 *   before the same thread writes it). Any other overlap is undefined.
 * - Sizes: M, N >= 0 and M * N * element size must fit in int64. M is not
 *   limited by the CUDA grid (the page's Summary, "Launch limit": more than
 *   65,535 rows must launch): the grid is one-dimensional and persistent.
 * - Asynchrony: calls only enqueue work on `stream` (0 = legacy default
 *   stream) and return. DYT_ERR_CUDA reports a launch error; a fault in a
 *   kernel surfaces at the caller's next synchronisation. No call aborts, and
 *   no failure is reported as DYT_OK.
 * - Results are deterministic: the same inputs on the same device give the
 *   same bits (static schedule, fixed reduction order, no atomics in sums).
 * - Every argument error is reported by a status code before anything is
 *   launched. No kernel waits on another CTA, grid or device; the only waits
 *   are hardware completion waits (a thread's own asynchronous copies, the
 *   preceding grid in the stream).
 */
#ifndef DYT_H_
#define DYT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as the CUDA runtime's cudaStream_t. */
typedef struct CUstream_st *dyt_stream_t;

typedef enum dyt_dtype {
  DYT_F32 = 0,  /* IEEE binary32 */
  DYT_BF16 = 1, /* bfloat16 */
  DYT_F16 = 2   /* IEEE binary16 */
} dyt_dtype;

typedef enum dyt_status {
  DYT_OK = 0,
  DYT_ERR_INVALID_VALUE = 1,       /* null pointer, negative size, size overflow, bad enum */
  DYT_ERR_UNSUPPORTED_DTYPE = 2,   /* dtype enum outside dyt_dtype */
  DYT_ERR_WORKSPACE_TOO_SMALL = 3, /* workspace_bytes < dyt_backward_workspace_bytes(...) */
  DYT_ERR_CUDA = 4                 /* the CUDA runtime refused a query or a launch */
} dyt_status;

/*
 * Forward: y = gamma * tanh(alpha * x) + beta, one kernel launch.
 *   x      [M*N] x_dtype, read
 *   alpha  [1]   param_dtype, read on the device
 *   gamma  [N]   param_dtype, read
 *   beta   [N]   param_dtype, read
 *   y      [M*N] x_dtype, written (may alias x)
 * Each y element is rounded once to x_dtype. For 16-bit x_dtype an element
 * whose binary32 value of gamma*t + beta may have cancelled (|y| < tau |beta|,
 * tau = 2^-12 for bf16 and 2^-9 for fp16) is recomputed in binary64, so every y is
 * within one unit in the last place of the correctly rounded value.
 * M * N == 0 launches nothing. Null pointers with M * N > 0 give
 * DYT_ERR_INVALID_VALUE.
 */
dyt_status dyt_forward(const void *x, const void *alpha, const void *gamma, const void *beta,
                       void *y, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                       dyt_stream_t stream);

/*
 * Bytes of device workspace dyt_backward needs for this shape on the CURRENT
 * device (the grid, and with it the number of partial sums, depends on the
 * device's SM count). Returns 0 for invalid arguments or when no workspace is
 * needed (M * N == 0).
 */
size_t dyt_backward_workspace_bytes(int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype);

/*
 * Backward: recomputes t = tanh(alpha * x) and writes dx, dgamma, dbeta and
 * dalpha. Two kernel launches on `stream`: the fused elementwise pass, which
 * also writes binary64 partial sums to the workspace (per row group and column
 * for dgamma and dbeta, per CTA for dalpha), and a finalize pass that adds the
 * partials in binary64 in a fixed order and rounds each gradient once.
 *   x, dy     [M*N] x_dtype, read
 *   alpha     [1]   param_dtype, read on the device
 *   gamma     [N]   param_dtype, read
 *   beta      [N]   param_dtype, not read: the gradients do not depend on beta.
 *                   May be NULL. (It is part of the call so that the layer's
 *                   parameters travel together; dbeta takes beta's dtype.)
 *   dx        [M*N] x_dtype, written (may alias x or dy)
 *   dgamma    [N]   param_dtype, written
 *   dbeta     [N]   param_dtype, written
 *   dalpha    [1]   param_dtype, written
 *   workspace device scratch of at least dyt_backward_workspace_bytes(M, N,
 *             x_dtype, param_dtype) bytes, 16-byte aligned, owned by the
 *             caller; its contents on entry do not matter and on exit are
 *             unspecified. Two calls in flight at once need two workspaces.
 * Contributions of lanes outside [0,M) x [0,N) are removed by a select after
 * the arithmetic, never by multiplying with a mask (the page's Summary,
 * "Padding"), so alpha = +inf cannot put NaN into the sums through them.
 * With M * N == 0: dgamma and dbeta (when N > 0) and dalpha are set to zero,
 * and no workspace is used.
 */
dyt_status dyt_backward(const void *x, const void *dy, const void *alpha, const void *gamma, const void *beta,
                        void *dx, void *dgamma, void *dbeta, void *dalpha, int64_t M, int64_t N,
                        dyt_dtype x_dtype, dyt_dtype param_dtype, void *workspace, size_t workspace_bytes,
                        dyt_stream_t stream);

/*
 * dyt_forward and dyt_backward over row-strided matrices: row i of a tensor
 * starts ld elements after row i - 1 (ld >= N), each with its own pitch
 * (ldx, ldy; ldx, lddy, lddx). The page's kernels take contiguous rows; this
 * leading-dimension form has no counterpart there. With the same kernels
 * (see below) it gives the same bits as the contiguous call on the same rows.
 * dyt_forward / dyt_backward are these with every pitch = N.
 * Padding between rows is never written. When every pitch times the
 * element size is a multiple of 16 bytes, the vectorised kernels run: the
 * aligned ones for 16-byte aligned tensors and N a multiple of 16 / element
 * size, else the row frame (each row laid out on its own as the shifted
 * kernels lay out a contiguous matrix: whole 16-byte vectors of the output,
 * masked at the row's two ends). The row frame copies the inputs in aligned
 * 16-byte chunks, so it reads the padding bytes that share a chunk with a
 * row's first or last elements (always between the tensor's first and last
 * elements); their values reach no result. The other kernels read no
 * padding. Pitches that are not whole 16-byte vectors (pitch times element
 * size a multiple of 8, 4 or 2 bytes: a row's offset past a boundary then
 * repeats every k = 2, 4 or 8 rows) run as k phases, rows j, j + k, ... of
 * pitch k * ld each through the kernels above, when every phase moves at
 * least 8 MiB per tensor (forward, any k) or 32 MiB per tensor (backward,
 * k = 2, and the workspace holds both phases' partials:
 * dyt_backward_workspace_bytes_strided; the finalize then adds the phases'
 * partials in phase order). Otherwise they take the one-element kernels.
 * y may alias x (dx may alias x or
 * dy) only with equal pitches. A pitch below N, or (M - 1) * ld + N beyond
 * the int64 limit of byte offsets, gives DYT_ERR_INVALID_VALUE.
 * dyt_backward_workspace_bytes covers every strided call (one phase);
 * dyt_backward_workspace_bytes_strided also covers the phases its pitches
 * call for (and is at least dyt_backward_workspace_bytes). Both return 0 for
 * invalid arguments or when no workspace is needed.
 */
size_t dyt_backward_workspace_bytes_strided(int64_t M, int64_t N, int64_t ldx, int64_t lddy, int64_t lddx,
                                            dyt_dtype x_dtype, dyt_dtype param_dtype);
dyt_status dyt_forward_strided(const void *x, int64_t ldx, const void *alpha, const void *gamma,
                               const void *beta, void *y, int64_t ldy, int64_t M, int64_t N,
                               dyt_dtype x_dtype, dyt_dtype param_dtype, dyt_stream_t stream);
dyt_status dyt_backward_strided(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                                const void *gamma, const void *beta, void *dx, int64_t lddx, void *dgamma,
                                void *dbeta, void *dalpha, int64_t M, int64_t N, dyt_dtype x_dtype,
                                dyt_dtype param_dtype, void *workspace, size_t workspace_bytes,
                                dyt_stream_t stream);

/*
 * The general forms: row pitches as in the *_strided calls, and one dtype per
 * parameter (the page's Summary, "Precision": each parameter gradient takes
 * its own parameter's dtype). alpha is read as alpha_dtype, gamma as
 * gamma_dtype, beta as beta_dtype; the backward writes dalpha in alpha_dtype,
 * dgamma in gamma_dtype and dbeta in beta_dtype (beta itself is not read and
 * may be NULL). Every other entry point above is one of these with all
 * pitches N and/or all three parameter dtypes equal, and gives the same bits
 * as this call with those arguments. An invalid dtype code gives
 * DYT_ERR_UNSUPPORTED_DTYPE; the workspace size does not depend on the
 * parameter dtypes.
 */
dyt_status dyt_forward_ex(const void *x, int64_t ldx, const void *alpha, const void *gamma, const void *beta,
                          void *y, int64_t ldy, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype alpha_dtype,
                          dyt_dtype gamma_dtype, dyt_dtype beta_dtype, dyt_stream_t stream);
dyt_status dyt_backward_ex(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                           const void *gamma, const void *beta, void *dx, int64_t lddx, void *dgamma, void *dbeta,
                           void *dalpha, int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype alpha_dtype,
                           dyt_dtype gamma_dtype, dyt_dtype beta_dtype, void *workspace, size_t workspace_bytes,
                           dyt_stream_t stream);

/*
 * The backward in two halves, for a row-sharded backward over several GPUs.
 * The page's gradients are sums over ALL rows (Summary, "Padding" and
 * "Precision"), so ranks that each hold some rows of x and dy must add their
 * partial sums once; here that addition is the finalize itself, reading every
 * rank's binary64 partials through peer pointers, in rank order, rounding once.
 * dyt_backward is dyt_backward_partials followed by dyt_finalize_partials over
 * its one workspace, and gives the same bits.
 *
 * dyt_backward_partials: stage 1 only. Writes dx and leaves binary64 partial
 * sums in the workspace (at least dyt_backward_workspace_bytes bytes); *layout
 * receives where they are. Arguments as for dyt_backward_ex (no beta). M * N ==
 * 0 launches nothing and gives an empty layout (rows = dalpha_parts = 0).
 *
 * dyt_partials_layout_query: the layout dyt_backward_partials would report for
 * these tensors on the current device, without launching or reading anything
 * (the pointers are looked at for their alignment only). Ranks exchange these
 * once, so that every rank finalizes with the same layouts.
 *
 * dyt_finalize_partials: dgamma, dbeta (when N > 0) and dalpha from the
 * partials of nranks (1 <= nranks <= DYT_MAX_RANKS) workspaces. workspaces is a
 * HOST array of pointers the current device can read (its own workspace, or
 * another GPU's through dyt_ipc_import); layouts the matching host array.
 * Every column is summed per rank in a fixed order, the ranks' totals are
 * added in rank order, and each gradient is rounded once to its dtype. Ranks
 * that pass the same workspaces and layouts in the same order get the same
 * bits. One kernel launch; the caller orders it after every rank's
 * dyt_backward_partials (on other GPUs: a barrier such as a one-element NCCL
 * all-reduce on the stream) and keeps the workspaces untouched until every
 * rank's finalize has run. Layouts that point outside their own `bytes` give
 * DYT_ERR_INVALID_VALUE.
 */
#define DYT_MAX_RANKS 8

typedef struct dyt_partials_layout {
  int64_t bytes;        /* workspace bytes the partials occupy */
  int64_t off_dgamma;   /* byte offsets, in the workspace, of the dgamma partials, */
  int64_t off_dbeta;    /*   the dbeta partials */
  int64_t off_dalpha;   /*   and the dalpha partials */
  int32_t rows;         /* partial rows: N binary64 values each, for dgamma and for dbeta */
  int32_t dalpha_parts; /* binary64 dalpha partials */
} dyt_partials_layout;

dyt_status dyt_backward_partials(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *alpha,
                                 const void *gamma, void *dx, int64_t lddx, int64_t M, int64_t N, dyt_dtype x_dtype,
                                 dyt_dtype alpha_dtype, dyt_dtype gamma_dtype, void *workspace,
                                 size_t workspace_bytes, dyt_partials_layout *layout, dyt_stream_t stream);
dyt_status dyt_partials_layout_query(const void *x, int64_t ldx, const void *dy, int64_t lddy, const void *dx,
                                     int64_t lddx, int64_t M, int64_t N, dyt_dtype x_dtype,
                                     dyt_partials_layout *layout);
dyt_status dyt_finalize_partials(const void *const *workspaces, const dyt_partials_layout *layouts, int nranks,
                                 int64_t N, void *dgamma, void *dbeta, void *dalpha, dyt_dtype alpha_dtype,
                                 dyt_dtype gamma_dtype, dyt_dtype beta_dtype, dyt_stream_t stream);

/*
 * Sharing a workspace with the other processes of a node (CUDA IPC), so that
 * their finalize can read its partials over NVLink with plain loads.
 * dyt_ipc_export: a handle for the device allocation holding ptr, and ptr's
 * byte offset in it (the memory must come from cudaMalloc, directly or through
 * a caching allocator that uses it). dyt_ipc_import: in another process, a
 * pointer to the same bytes, readable from the current device (peer access is
 * enabled on first use). dyt_ipc_close: releases an imported pointer.
 * Failures report DYT_ERR_CUDA (dyt_last_cuda_error gives the reason).
 */
typedef struct dyt_ipc_handle {
  unsigned char bytes[64]; /* the CUDA IPC memory handle of the allocation */
  int64_t offset;          /* the pointer's byte offset in that allocation */
} dyt_ipc_handle;

dyt_status dyt_ipc_export(const void *ptr, dyt_ipc_handle *out);
dyt_status dyt_ipc_import(const dyt_ipc_handle *handle, void **ptr);
dyt_status dyt_ipc_close(void *ptr, const dyt_ipc_handle *handle);

/* Static, human-readable name of a status. Never NULL. */
const char *dyt_status_string(dyt_status status);

/* The cudaError_t value behind the calling thread's last DYT_ERR_CUDA (0 if
 * none). When a call returns DYT_ERR_CUDA it has also cleared the CUDA
 * runtime's last-error state (cudaGetLastError), so the failure is reported
 * once, by the status; a sticky error (a fault in an earlier kernel) stays. */
int dyt_last_cuda_error(void);

/*
 * Launch geometry of the calling thread's last successful dyt_forward or
 * dyt_backward call, so tests can check which path ran.
 */
typedef struct dyt_launch_info {
  int op;            /* 1 = forward, 2 = backward, 3 = backward stage 1 (dyt_backward_partials),
                        4 = finalize (dyt_finalize_partials), 0 = none yet */
  int path;          /* 0 = nothing launched, 1 = row-tiled (several rows per CTA step),
                        2 = row-per-CTA (one row per CTA step, columns across threads) */
  int vec;           /* elements per vector access (1 = the one-element kernels) */
  int block;         /* threads per CTA */
  int grid;          /* CTAs of the main kernel (1D) */
  int row_lanes;     /* rows (packs of pack_rows rows) one CTA step covers side by side */
  int rows_per_step; /* matrix rows one CTA step covers in total */
  int col_chunks;    /* column chunks the grid is split into */
  int row_groups;    /* row groups (= partial sums per column) */
  int kernels;       /* kernels this call launched */
  int async_stages;  /* per-thread asynchronous-copy ring slots (0 = the one-element kernels) */
  int pack_rows;     /* 1, or vec on the packed path: a matrix of adjacent rows whose N is not a
                        multiple of vec is streamed as packs of vec rows (vec x N elements,
                        exactly N 16-byte vectors) */
  int shifted;       /* 1 = the flat shifted 16-byte kernels (adjacent rows, tensors not all
                        16-byte aligned); 2 = the row frame (strided rows whose pitches are
                        whole 16-byte vectors, tensors not all 16-byte aligned or N not a
                        multiple of vec: each row shifted on its own); 3 = the row frame
                        with a wrapped first vector-column (N a multiple of vec, every
                        tensor shift elements off: the first vector of a row also holds
                        its last shift elements, so a row spans N / vec vectors); 0
                        otherwise */
  int shift;         /* shifted kernels: the output's offset past a 16-byte boundary, in
                        elements (0 .. vec - 1); 0 otherwise */
  int64_t workspace_bytes;
} dyt_launch_info;

dyt_status dyt_last_launch_info(dyt_launch_info *out);

/*
 * The launch plan dyt_forward (backward = 0) or dyt_backward (backward != 0)
 * would use for this shape on a device with `sm_count` SMs running
 * `ctas_per_sm` CTAs of the kernel each, for tensors laid out as `layout`
 * says: 0 = rows that are not whole 16-byte vectors (the one-element kernels),
 * 1 = contiguous and 16-byte aligned (a ragged N gets the packed form,
 * out->pack_rows > 1), 2 = contiguous with the output `shift` elements past a
 * 16-byte boundary (the shifted kernels), 3 = strided rows (pitches not N)
 * whose pitches are whole 16-byte vectors, every tensor `shift` elements past
 * a 16-byte boundary (the row frame unless shift is 0 and N a multiple of
 * vec), 4 = as 3 with the inputs at other offsets than the output (`shift`
 * is read for layouts 2 to 4 only).
 * Host arithmetic only: touches no device, so the planning is testable
 * without a GPU. out->kernels is the number of kernels the call would launch
 * and out->workspace_bytes the workspace it needs.
 * Errors: as the shape checks of dyt_forward, or DYT_ERR_INVALID_VALUE for
 * out == NULL, sm_count / ctas_per_sm < 1, a layout outside 0..4 or a shift
 * outside 0 .. 16 / element size - 1.
 */
dyt_status dyt_plan_query(int64_t M, int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype,
                          int backward, int layout, int shift, int sm_count, int ctas_per_sm,
                          dyt_launch_info *out);

/*
 * Backward without a caller-provided workspace (no counterpart in the paper:
 * it exists for callers that cannot allocate device memory themselves, such as
 * code embedded in a host application that owns all device memory through its
 * own pool, or latency-critical loops where cudaMalloc's implicit device
 * synchronisation is not acceptable).
 *
 * Same arguments, results and errors as dyt_backward, minus the workspace: the
 * scratch comes from a fixed array of DYT_NOALLOC_SCRATCH_BYTES bytes that the
 * library keeps in device memory (every device that loads the library holds it
 * until the process exits). The call allocates nothing.
 * - The first call on each device looks the array's device address up
 *   (cudaGetSymbolAddress) with that device current, and keeps it for that
 *   device's context; make that first call before any stream capture. After a
 *   cudaDeviceReset, the next call on the device is such a first call again:
 *   the address is cached under the driver's context id, never reused across
 *   contexts.
 * - Shapes whose scratch need (dyt_backward_workspace_bytes) exceeds
 *   DYT_NOALLOC_SCRATCH_BYTES are rejected with DYT_ERR_WORKSPACE_TOO_SMALL
 *   before anything is launched.
 * - Every call on a device shares the one array, which keeps the last call's
 *   contents; nothing in it has to start at zero (each call rewrites every
 *   partial sum before reading it). Calls that overlap on the GPU (on
 *   different streams, or from different host threads without ordering) race
 *   on the array and give undefined results: order them on one stream.
 */
#define DYT_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)

dyt_status dyt_backward_noalloc(const void *x, const void *dy, const void *alpha, const void *gamma,
                                const void *beta, void *dx, void *dgamma, void *dbeta, void *dalpha, int64_t M,
                                int64_t N, dyt_dtype x_dtype, dyt_dtype param_dtype, dyt_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DYT_H_ */
