/*
 * fp8ds.h -- C ABI of libfp8ds.so, the FP8 delayed-scaling linear hot path
 * for NVIDIA B200 (sm_100a).
 *
 * Sources of the method (web pages; cited by title and section):
 *   [TE820]  "[PyTorch] Refactor FP8 workspaces in linear modules"
 *            (TransformerEngine PR #820): one cached FP8 weight workspace per
 *            linear; a Float8Tensor keeps a private scale-inverse that scale
 *            updates do not touch until its data is rewritten; lazy transpose
 *            cache; is_first_microbatch.
 *   [TE761]  "CPU Overhead of te.Linear FP8 Layers" (TransformerEngine issue
 *            #761): the DelayedScaling recipe (HYBRID format, amax history
 *            length 16, amax_compute_algo "max"), the TEBlock workload, and
 *            the per-linear launch overhead that motivates few launches.
 *   [F8E312] "support delayed scaling of weight in float8 all-gather"
 *            (float8_experimental PR #312): amax buffers of all linears
 *            gathered into one tensor and synced once per step.
 *   [PTFP8]  "Accelerating PyTorch Training Workloads with FP8 -- Part 2"
 *            (PyTorch-native FP8 data types): float8_e4m3fn / float8_e5m2
 *            finfo table, the worked cast example, torch._scaled_mm.
 *
 * Conventions for every call:
 *   - Pointers are DEVICE pointers unless stated otherwise; the caller owns all
 *     memory (tensors, weight cache, meta arrays).  The library allocates
 *     nothing, keeps no device state between calls (except the error word read
 *     by fp8ds_device_status) and never synchronises: every call only enqueues
 *     work on `stream` (NULL = the legacy default stream).
 *   - Scalars that the method updates on the device (scale, amax, scale_inv)
 *     are passed as device pointers, so a sequence of calls can be captured
 *     in a CUDA graph.
 *   - Tensors are dense row-major.  FP8 data are raw bytes (uint8).
 *   - Return value: FP8DS_OK, or an error detected on the host before any
 *     launch (nothing is enqueued then), or FP8DS_ERR_CUDA if a launch failed.
 *     fp8ds_last_error() gives a message for the calling thread.
 */
#ifndef FP8DS_H
#define FP8DS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FP8DS_OK = 0,
    FP8DS_ERR_INVALID_ARG = 1,   /* null pointer, bad size, misalignment */
    FP8DS_ERR_UNSUPPORTED = 2,   /* valid but not implemented combination */
    FP8DS_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed */
    FP8DS_ERR_TIMEOUT = 4        /* a bounded device wait gave up (device word) */
} fp8ds_status;

/* FP8 formats [PTFP8 finfo table]: E4M3FN (max 448, no inf) and E5M2 (max 57344). */
typedef enum { FP8DS_E4M3 = 0, FP8DS_E5M2 = 1 } fp8ds_format;

/* High-precision element types. */
typedef enum { FP8DS_F32 = 0, FP8DS_BF16 = 1 } fp8ds_dtype;

/*
 * Storage order of a GEMM operand.  K_MAJOR: a [m, k] / b [n, k] row-major
 * (k contiguous, the "TN" layout of torch._scaled_mm(a, b.t())).  MN_MAJOR:
 * a [k, m] / b [k, n] row-major -- the tensor as its producer wrote it,
 * read transposed by the tensor core (sm_100's tcgen05 reads 8-bit operands
 * in either order, so no FP8 transpose has to be materialised).
 */
typedef enum { FP8DS_K_MAJOR = 0, FP8DS_MN_MAJOR = 1 } fp8ds_major;

/*
 * Amax used by the update [TE761 recipe: amax_compute_algo, "max" in the
 * repro]: MAX = the max over the history window; MOST_RECENT = the amax
 * recorded in the current step alone (the recipe parameter's other choice).
 */
typedef enum { FP8DS_AMAX_MAX = 0, FP8DS_AMAX_MOST_RECENT = 1 } fp8ds_amax_algo;

/* A cudaStream_t. */
typedef struct CUstream_st *fp8ds_stream;

/*
 * fp8_quantize -- per-tensor cast of a flat tensor [PTFP8 worked cast example;
 * TE820 Float8Tensor scale-inverse].
 *
 *   y[i]       = sat_rne_fp8(fl32(x[i] * *scale))   for i < n
 *   *amax      = max(*amax, max_i |x[i]|)           (unscaled input, NaN ignored)
 *   *scale_inv = fl32(1 / *scale)                   (the tensor's private copy)
 *
 * sat_rne_fp8 rounds to nearest, ties to even, saturates to +-max (also +-inf),
 * keeps the sign of zero and maps NaN to 0x7F.
 *   x        [n] fp32 or bf16 (x_dtype).
 *   scale    [1] fp32, read on the device.
 *   y        [n] uint8 FP8 codes of format `fmt`.
 *   amax     [1] fp32 or NULL.  Atomically max-ed into, so it must hold a
 *            non-negative value (normally slot 0 of the tensor's amax history).
 *   scale_inv[1] fp32 or NULL.
 * Errors: FP8DS_ERR_INVALID_ARG if n < 0 or a required pointer is NULL.
 * n == 0 enqueues only the scale_inv write.
 */
fp8ds_status fp8_quantize(const void *x, fp8ds_dtype x_dtype, int64_t n, fp8ds_format fmt,
                          const float *scale, uint8_t *y, float *amax, float *scale_inv,
                          fp8ds_stream stream);

/*
 * fp8_cast_transpose_amax -- fp8_quantize of a 2-D tensor that also writes the
 * FP8 transpose [TE820: FP8 weight workspace and its transpose cache; the
 * transposes feed the backward GEMMs].
 *
 *   y[r,c]  = sat_rne_fp8(fl32(x[r,c] * *scale))     y  [rows, cols]
 *   yt[c,r] = y[r,c]                                  yt [cols, rows] (NULL: skipped)
 *   amax, scale_inv as in fp8_quantize.
 * Errors: FP8DS_ERR_INVALID_ARG for negative sizes or NULL x / scale / y.
 * Any sizes are accepted; 16-byte aligned pointers with cols % 8 == 0 and
 * rows % 16 == 0 take the vectorised path.
 */
fp8ds_status fp8_cast_transpose_amax(const void *x, fp8ds_dtype x_dtype, int64_t rows,
                                     int64_t cols, fp8ds_format fmt, const float *scale,
                                     uint8_t *y, uint8_t *yt, float *amax, float *scale_inv,
                                     fp8ds_stream stream);

/*
 * fp8_cast_transpose_amax_noop -- fp8_cast_transpose_amax with a device-side
 * skip flag (TE's noop flag) [TE820: with CUDA graphs the choice of casting or
 * reusing the cached weight must be made on the GPU at replay time].
 *   noop_flag  device int32, read by the kernel when it runs: non-zero ->
 *              nothing is written (y, yt, amax, scale_inv keep their values);
 *              zero -> exactly fp8_cast_transpose_amax.
 * Errors: as fp8_cast_transpose_amax; FP8DS_ERR_INVALID_ARG for a NULL flag.
 */
fp8ds_status fp8_cast_transpose_amax_noop(const void *x, fp8ds_dtype x_dtype, int64_t rows,
                                          int64_t cols, fp8ds_format fmt, const float *scale,
                                          uint8_t *y, uint8_t *yt, float *amax, float *scale_inv,
                                          const int32_t *noop_flag, fp8ds_stream stream);

/*
 * fp8_cast_transpose_amax_pair -- two independent fp8_cast_transpose_amax
 * calls of one input dtype and one FP8 format, issued as one kernel launch
 * where possible [TE820 and TE761: per-call launches of small kernels are the
 * CPU and launch overhead the pages set out to remove; a linear's forward
 * casts its input and its weight back to back].  Tensor a is cast exactly as
 * fp8_cast_transpose_amax(x_a, ..., scale_a, y_a, yt_a, amax_a, scale_inv_a),
 * tensor b exactly as fp8_cast_transpose_amax_noop(x_b, ..., noop_b) (or the
 * plain call when noop_b is NULL).  One launch when both tensors suit the TMA
 * path (x and y 16-byte aligned, cols % 8 == 0, rows % 16 == 0) and both or
 * neither have a transpose output; otherwise two launches, one per tensor.
 * The results are the same bytes either way (amax is a max, so its order
 * does not matter).  Tensors a and b must not overlap in memory, except that
 * they may share scale, amax or scale_inv only if the caller wants their
 * combined effect (amax is atomically maxed).
 * Errors: as fp8_cast_transpose_amax, for either tensor.
 */
fp8ds_status fp8_cast_transpose_amax_pair(const void *x_a, int64_t rows_a, int64_t cols_a,
                                          const float *scale_a, uint8_t *y_a, uint8_t *yt_a,
                                          float *amax_a, float *scale_inv_a, const void *x_b,
                                          int64_t rows_b, int64_t cols_b, const float *scale_b,
                                          uint8_t *y_b, uint8_t *yt_b, float *amax_b,
                                          float *scale_inv_b, const int32_t *noop_b,
                                          fp8ds_dtype x_dtype, fp8ds_format fmt, fp8ds_stream stream);

/*
 * One tensor of fp8_cast_transpose_amax_multi: the arguments of
 * fp8_cast_transpose_amax_noop gathered in a struct (host memory; the
 * pointers inside are device pointers).
 */
typedef struct {
    const void *x;             /* [rows, cols] row-major input (x_dtype) */
    fp8ds_dtype x_dtype;
    int64_t rows;
    int64_t cols;
    fp8ds_format fmt;
    const float *scale;        /* [1] fp32, read on the device */
    uint8_t *y;                /* [rows, cols] FP8 codes */
    uint8_t *yt;               /* [cols, rows] FP8 transpose, or NULL */
    float *amax;               /* [1] atomic-max target, or NULL */
    float *scale_inv;          /* [1] private scale_inv, or NULL */
    const int32_t *noop_flag;  /* device int32 or NULL: non-zero at run time skips this tensor */
} fp8ds_cast_job;

/*
 * fp8_cast_transpose_amax_multi -- many independent casts in one kernel
 * launch [TE820: the FP8 weight workspaces of all linears refreshed together
 * ("fewer kernel launches"); TE761: the CPU time of launching per-tensor
 * kernels is the overhead to remove].  Job i gives exactly the bytes of
 * fp8_cast_transpose_amax_noop(jobs[i].x, ..., jobs[i].noop_flag) (the plain
 * call when noop_flag is NULL): y, yt, the amax max-ed into *amax and
 * *scale_inv.  Jobs may mix input dtypes, formats, shapes and transpose or
 * none; a job with no elements only writes its scale_inv.
 *   jobs      host array of num_jobs job records (read during the call only;
 *             the job list is copied into the launch, so a captured CUDA graph
 *             replays it).
 * Up to 256 jobs go into one launch; a longer list is split into consecutive
 * launches of up to 256.  Outputs of different jobs must not overlap (amax /
 * scale_inv targets may be shared only if their combined effect is wanted).
 * Errors: FP8DS_ERR_INVALID_ARG for num_jobs < 0, a NULL jobs array, any job
 * that fp8_cast_transpose_amax would reject, or a job with a transpose whose
 * rows or cols reach 2^31; nothing is enqueued then.
 */
fp8ds_status fp8_cast_transpose_amax_multi(const fp8ds_cast_job *jobs, int32_t num_jobs,
                                           fp8ds_stream stream);

/*
 * fp8_cast_transpose_amax_dynamic -- dynamic scaling, for comparison with the
 * delayed recipe [F8E312: delayed vs dynamic scaling; "delayed scaling is
 * theoretically faster than dynamic scaling (less memory reads)" is the
 * page's claim this measures].  The scale comes from the tensor itself, so
 * the input is read twice:
 *   *amax      = max |x|                         (overwritten; NaN ignored)
 *   *scale     = fl32(fp8_max / *amax) if that amax is > 0 and finite and the
 *                quotient finite; otherwise the value passed in is kept
 *   *scale_inv = fl32(1 / *scale)                (if not NULL)
 *   y, yt      = fp8_cast_transpose_amax(x, fmt, scale) (no amax accumulation)
 * Arguments and layouts as fp8_cast_transpose_amax; scale is in/out, amax
 * required.  Enqueues a 4-byte memset and three kernels on `stream`.
 * Errors: as fp8_cast_transpose_amax; FP8DS_ERR_INVALID_ARG for NULL amax.
 */
fp8ds_status fp8_cast_transpose_amax_dynamic(const void *x, fp8ds_dtype x_dtype, int64_t rows,
                                             int64_t cols, fp8ds_format fmt, float *scale,
                                             uint8_t *y, uint8_t *yt, float *amax,
                                             float *scale_inv, fp8ds_stream stream);

/*
 * fp8_transpose -- the FP8 transpose cache of a tensor that arrived already
 * cast [TE820: transpose_2d(cache=True) fills a Float8Tensor's transpose;
 * F8E312: a weight all-gathered in FP8 still needs its transpose for the
 * backward]:  yt[c, r] = y[r, c], bytes copied unchanged.
 *   y [rows, cols] uint8, yt [cols, rows] uint8 (must not overlap y).
 * 16-byte aligned pointers with rows and cols multiples of 16 take the
 * vectorised path; other shapes are still transposed exactly.
 * Errors: FP8DS_ERR_INVALID_ARG for negative sizes, NULL or aliasing pointers.
 */
fp8ds_status fp8_transpose(const uint8_t *y, int64_t rows, int64_t cols, uint8_t *yt,
                           fp8ds_stream stream);

/*
 * fp8_update_scales -- the delayed-scaling recipe update of T FP8 meta tensors
 * in ONE launch [TE820 "FP8 scale update kernel"; TE761 DelayedScaling(
 * amax_history_len=16, amax_compute_algo="max"); F8E312 amax buffers of all
 * linears handled together].  For every t < num_tensors:
 *
 *   a          = max_h amax_history[h, t]   (algo MAX: window of hist_len steps)
 *                amax_history[0, t]          (algo MOST_RECENT: this step's amax)
 *   scale[t]   = fl32(fp8_max(formats[t]) / a)  if a > 0, a finite and the
 *                quotient finite; otherwise scale[t] is kept
 *   scale_inv[t] = fl32(1 / scale[t])                   (the meta's copy; FP8
 *                tensors keep the private copy written by their cast)
 *   amax_history[:, t] rolled by one: h <- h+1 (slot hist_len-1 receives the
 *                current amax of slot 0), then slot 0 = 0 for the next step.
 *
 *   amax_history [hist_len, num_tensors] fp32, slot-major (row 0 = the amaxes
 *                recorded in the current step; contiguous, so a cross-rank
 *                max-reduction of row 0 is one contiguous buffer).
 *   scale, scale_inv [num_tensors] fp32;  formats [num_tensors] uint8 (fp8ds_format).
 * Errors: FP8DS_ERR_INVALID_ARG for num_tensors < 0, hist_len < 1 or NULL
 * pointers; FP8DS_ERR_UNSUPPORTED for an unknown algo.
 */
fp8ds_status fp8_update_scales(int64_t num_tensors, int32_t hist_len, float *amax_history,
                               float *scale, float *scale_inv, const uint8_t *formats,
                               fp8ds_amax_algo algo, fp8ds_stream stream);

/*
 * fp8_gemm -- scaled FP8 GEMM with a dequantising epilogue [PTFP8
 * torch._scaled_mm: two FP8 operands, their scale factors, optional bias,
 * chosen output dtype; TE761 HYBRID: e4m3 x e4m3 forward, e5m2 x e4m3 for
 * gradients].
 *
 *   d[m,n] = (sum_k dec(a[m,k]) * dec(b[n,k])) * *a_scale_inv * *b_scale_inv
 *            (+ bias[n])                       accumulated in fp32
 *
 *   a [m, k] uint8 FP8 (a_fmt), row-major (k contiguous)
 *   b [n, k] uint8 FP8 (b_fmt), row-major (k contiguous): the "TN" layout of
 *     torch._scaled_mm(a, b.t())
 *   a_scale_inv, b_scale_inv [1] fp32 (normally the operands' private copies)
 *   bias [n] (bias_dtype) or NULL
 *   d [m, n] fp32 or bf16 (d_dtype)
 * Requirements (TMA): k % 16 == 0, a/b/d 16-byte aligned, n % 8 == 0 for bf16
 * and n % 4 == 0 for fp32 output.  m, n, k > 0.
 * Errors: FP8DS_ERR_INVALID_ARG when a requirement fails; FP8DS_ERR_CUDA if
 * the tensor maps cannot be encoded or the launch fails.  A device-side wait
 * that exceeds its time limit aborts the kernel and sets the error word read
 * by fp8ds_device_status (the output is then undefined).
 */
fp8ds_status fp8_gemm(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv,
                      const uint8_t *b, fp8ds_format b_fmt, const float *b_scale_inv,
                      const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype,
                      int64_t m, int64_t n, int64_t k, fp8ds_stream stream);

/*
 * fp8_gemm_workspace_size -- bytes of workspace that let fp8_gemm_ex use the
 * stream-K schedule on the current device (a few tens of MB on B200).  Host
 * only; no device work.
 */
fp8ds_status fp8_gemm_workspace_size(size_t *bytes);

/*
 * fp8_gemm_plan -- the tile schedule that fp8_gemm, fp8_gemm_ex,
 * fp8_gemm_cast and the linear calls take for an m x n x k product on the
 * current device; it has no counterpart on the pages (it tells a caller
 * whether a workspace would change anything).  Host only; no device work.
 *   info [5] int64, written:
 *     info[0]  1: CTA-pair tiles (m > 128); 0: one-CTA tiles of 128 x 256
 *     info[1]  pair tiles of 256 (1) or 512 (2) rows x 256 columns; 0 for
 *              one-CTA tiles
 *     info[2]  number of tiles
 *     info[3]  1 if a workspace (fp8_gemm_ex, fp8_gemm_noalloc) turns the
 *              launch into the stream-K schedule, else 0
 *     info[4]  CTA pairs (one-CTA tiles: CTAs) resident at once
 * Errors: FP8DS_ERR_INVALID_ARG for a NULL info or m, n, k not positive.
 */
fp8ds_status fp8_gemm_plan(int64_t m, int64_t n, int64_t k, int64_t *info);

/*
 * fp8_gemm_ex -- fp8_gemm with a caller-owned device workspace.  When the
 * tiles would leave a ragged last wave of CTA pairs (fp8_gemm_plan, info[3]),
 * the whole waves still run as whole tiles and the k-blocks of the remaining
 * tiles are shared out equally among all pairs ("stream-K"); a tile split
 * between consecutive pairs is combined through the workspace in a fixed
 * order: each pair that holds a later part stores its fp32 partial
 * accumulator there (after adding the part after it, if any) and publishes
 * it, and the pair that holds the tile's first k-blocks adds it and writes D.
 * The result satisfies the same bounds as fp8_gemm (the partials are added
 * in fp32) and is the same bits on every run.  On B200 the whole-tile
 * schedule of fp8_gemm still measured faster on the MLP shapes (8192 x 2048
 * x 8192: 99-100 us against 91-93 us): the schedule alone would save about
 * 3 us, and storing and reloading the partials costs about 9.  The stream-K
 * schedule is for cases where a profile shows the ragged last wave
 * dominating.
 *   workspace  16-byte aligned device memory of at least
 *              fp8_gemm_workspace_size() bytes, ZERO-FILLED before its first
 *              use; the library leaves its publication words at zero after
 *              every completed call.  NULL (or fewer bytes) means fp8_gemm.
 *              Calls that may run concurrently must not share a workspace.
 * Errors: as fp8_gemm; FP8DS_ERR_INVALID_ARG for an unaligned workspace.
 */
fp8ds_status fp8_gemm_ex(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv,
                         const uint8_t *b, fp8ds_format b_fmt, const float *b_scale_inv,
                         const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype,
                         int64_t m, int64_t n, int64_t k, void *workspace, size_t workspace_bytes,
                         fp8ds_stream stream);

/*
 * fp8_gemm_noalloc -- fp8_gemm_ex for callers that cannot allocate device
 * memory: the stream-K scratch is an 80 MiB array inside the library (held by
 * every device that loads it until the process exits) instead of a workspace
 * argument.  The pages have no counterpart; it exists because some callers
 * must not call cudaMalloc -- for example a program whose device memory is
 * all handed to a framework's caching allocator or reserved by a serving
 * engine at start-up, or C code that only receives tensor pointers and owns
 * no allocator -- yet want the same GEMM.
 *   Arguments, layouts and results as fp8_gemm.  Calls no allocator (no
 *   cudaMalloc/cudaFree, no library routine that allocates).  When the
 *   shape's tiles leave a ragged last wave of CTA pairs (the stream-K case)
 *   it enqueues a 4 KiB memset of the scratch's publication words and the
 *   GEMM on `stream`; otherwise only the GEMM, exactly as fp8_gemm.
 *   The first call on a device looks up the scratch's device address (a
 *   runtime query, done once per device with that device current); make that
 *   first call before any stream capture on the device.  The address, like
 *   the library's other per-device settings (kernel attributes, occupancy
 *   figures), is kept for the life of the process: after cudaDeviceReset on
 *   a device, do not call the library on that device again.
 *   All calls share the one scratch: calls that may overlap on the GPU (other
 *   streams, other threads) race and must be ordered by the caller.
 * Errors: as fp8_gemm; FP8DS_ERR_INVALID_ARG if the device needs more
 * stream-K scratch than the 80 MiB array holds (more than 79 CTA pairs).
 */
fp8ds_status fp8_gemm_noalloc(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv,
                              const uint8_t *b, fp8ds_format b_fmt, const float *b_scale_inv,
                              const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype,
                              int64_t m, int64_t n, int64_t k, fp8ds_stream stream);

/*
 * fp8_gemm_major -- fp8_gemm with either storage order per operand
 * (fp8ds_major).  Same result as fp8_gemm on the transposed operands:
 *   d[m,n] = (sum_k A(m,k) B(n,k)) * *a_scale_inv * *b_scale_inv (+ bias[n])
 *   A(m,k) = a[m*k + k'] (K_MAJOR) or a[k*m + m'] (MN_MAJOR), likewise B.
 * The backward of a linear needs no transposed copies with it: the wgrad
 * dW = dY^T X reads dY8 [tokens, out] and X8 [tokens, in] MN-major, the
 * dgrad dX = dY W reads W8 [out, in] MN-major (the pages' TE and
 * float8_experimental designs cast transposes because Hopper's FP8 tensor
 * cores read only K-major operands).
 * Requirements: as fp8_gemm, except that k % 16 == 0 is needed only with a
 * K-major operand; m % 16 == 0 for an MN-major a, n % 16 == 0 for an
 * MN-major b.  Errors: as fp8_gemm; FP8DS_ERR_INVALID_ARG for an unknown
 * layout.
 */
fp8ds_status fp8_gemm_major(const uint8_t *a, fp8ds_format a_fmt, fp8ds_major a_major,
                            const float *a_scale_inv, const uint8_t *b, fp8ds_format b_fmt,
                            fp8ds_major b_major, const float *b_scale_inv, const void *bias,
                            fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype, int64_t m,
                            int64_t n, int64_t k, fp8ds_stream stream);

/*
 * fp8_gemm_cast -- the GEMM with an FP8 output for the next layer [PTFP8
 * torch._scaled_mm with out_dtype=float8_e4m3fn, returning the output and its
 * amax].  Reading used here: the FP8 output is the cast that the next layer
 * would apply to this GEMM's bf16 output, done inside the epilogue, so fusing
 * changes no result:
 *   h[m,n]   = bf16_rne((sum_k dec(a[m,k]) dec(b[n,k])) * *a_scale_inv
 *              * *b_scale_inv (+ bias[n]))      exactly fp8_gemm's bf16 output
 *   d8[m,n]  = sat_rne_fp8(fl32(h[m,n] * *out_scale))  (out_fmt)
 *   d8t[n,m] = d8[m,n]                              (if d8t is not NULL)
 *   *out_amax = max(*out_amax, max |h|)             (if not NULL; NaN ignored)
 *   *out_scale_inv = fl32(1 / *out_scale)           (if not NULL)
 * i.e. fp8_cast_transpose_amax(h, out_fmt, out_scale, d8, d8t, out_amax,
 * out_scale_inv) without h ever reaching memory.  out_scale is normally the
 * next layer's delayed scale (meta.scale[t]) and out_amax its history slot 0
 * (amax_history[0, t]).
 *   a, b, bias, m, n, k, formats: as fp8_gemm; a_major / b_major as
 *   fp8_gemm_major (the fused dgrad of a linear without a weight transpose
 *   reads w8 MN-major).
 *   d8 [m, n] uint8, d8t [n, m] uint8 or NULL; out_scale [1] fp32.
 * Requirements: as fp8_gemm, plus n % 16 == 0, m % 16 == 0 when d8t is not
 * NULL, d8 / d8t 16-byte aligned.  Errors: as fp8_gemm.
 */
fp8ds_status fp8_gemm_cast(const uint8_t *a, fp8ds_format a_fmt, fp8ds_major a_major,
                           const float *a_scale_inv, const uint8_t *b, fp8ds_format b_fmt,
                           fp8ds_major b_major, const float *b_scale_inv, const void *bias,
                           fp8ds_dtype bias_dtype, int64_t m, int64_t n, int64_t k,
                           fp8ds_format out_fmt, const float *out_scale, uint8_t *d8, uint8_t *d8t,
                           float *out_amax, float *out_scale_inv, fp8ds_stream stream);

/*
 * Packed FP8 meta of T tensors (the DelayedScaling state [TE761; F8E312
 * _amax_history_buffer / _scale_buffer]).  All arrays are caller-owned device
 * memory; amax_history is [hist_len, num_tensors] slot-major, zero-filled and
 * scale = 1 at initialisation (no amax-init pass).
 */
typedef struct {
    float *amax_history;
    float *scale;
    float *scale_inv;
    const uint8_t *formats;
    int64_t num_tensors;
    int32_t hist_len;
} fp8ds_meta;

/*
 * One linear layer y = x . w^T + bias with its FP8 weight cache [TE820]:
 * w8 / w8t hold the e4m3 weight and its transpose, w_scale_inv the private
 * scale-inverse they were cast with.  meta_in / meta_w / meta_grad index the
 * packed meta (input, weight, output-gradient tensors).  cache_valid is a host
 * flag that fp8_linear_fwd sets once the cache holds a cast weight; set it to
 * 0 to force the next forward to refresh the cache.
 */
typedef struct {
    const float *w;            /* [out_features, in_features] fp32 master weight */
    const void *bias;          /* [out_features] or NULL */
    fp8ds_dtype bias_dtype;
    int64_t in_features;
    int64_t out_features;
    uint8_t *w8;               /* [out_features, in_features] cached FP8 weight */
    uint8_t *w8t;              /* [in_features, out_features] cached FP8 transpose, or NULL
                                  (then the backward reads w8 MN-major) */
    float *w_scale_inv;        /* [1] private scale_inv of the cached weight */
    int32_t meta_in, meta_w, meta_grad;
    int32_t cache_valid;
    void *workspace;           /* NULL or the GEMM workspace of fp8_gemm_ex */
    size_t workspace_bytes;
    const int32_t *w_noop_flag; /* NULL or a device int32: see fp8_linear_fwd */
} fp8ds_linear;

/*
 * fp8_linear_fwd -- FP8 forward of one linear [TE820; TE761 HYBRID: e4m3]:
 *   1. cast x -> x8 (and x8t if not NULL) with meta.scale[meta_in], amax into
 *      amax_history[0, meta_in], private scale_inv into *x_scale_inv;
 *   2. if is_first_microbatch is -1 (None: always), 1 (True: refresh and keep),
 *      or 0 (False) with no valid cache: cast w -> w8 and w8t (if not NULL) with
 *      meta.scale[meta_w], amax into amax_history[0, meta_w], private
 *      scale_inv into *w_scale_inv; sets cache_valid.  With 0 and a valid
 *      cache the cached weight and its frozen scale_inv are reused;
 *   3. y = fp8_gemm(x8, w8, *x_scale_inv, *w_scale_inv, bias).
 * When x is fp32 and the weight is recast, steps 1 and 2 are one launch
 * (fp8_cast_transpose_amax_pair) where the shapes allow; the bytes are the
 * same as with two.
 * With lin->w_noop_flag set, step 2 is decided on the device instead [TE820:
 * a CUDA graph captured around the forward must not bake in the weight-cache
 * decision]: the weight cast is always enqueued and skips itself while
 * *w_noop_flag != 0 at run time (the cache and its frozen scale_inv stay);
 * is_first_microbatch is then ignored for the weight.  Write 0 to the flag
 * for a microbatch that must refresh the cache, 1 for the others.
 *   x [m, in_features] (x_dtype); y [m, out_features] (y_dtype);
 *   x8 [m, in_features], x8t [in_features, m] or NULL (fp8_linear_bwd reads
 *   x8t; fp8_linear_bwd_ex reads x8 MN-major when x8t is NULL).
 * The delayed-scaling update is not part of the forward: call
 * fp8_update_scales once per step over the whole meta.
 * Errors: as the calls it makes; nothing is enqueued if the arguments fail.
 */
fp8ds_status fp8_linear_fwd(fp8ds_linear *lin, const fp8ds_meta *meta, const void *x,
                            fp8ds_dtype x_dtype, int64_t m, void *y, fp8ds_dtype y_dtype,
                            int32_t is_first_microbatch, uint8_t *x8, uint8_t *x8t,
                            float *x_scale_inv, fp8ds_stream stream);

/*
 * fp8_linear_refresh_weights -- refresh the FP8 weight caches of many linears
 * in one launch [TE820: one weight workspace per linear, refreshed when
 * is_first_microbatch is True or None; TE761: per-linear launch overhead].
 * For every lins[i]: cast w -> w8 (and w8t if not NULL) in e4m3 with
 * meta.scale[meta_w], amax into amax_history[0, meta_w], private scale_inv
 * into *w_scale_inv (honouring w_noop_flag), exactly as fp8_linear_fwd's
 * weight cast, then set cache_valid = 1.  The forwards that follow pass
 * is_first_microbatch = 0 to use the refreshed caches.  `extra` (may be NULL
 * with num_extra = 0) lists further casts of the same launch, e.g. a layer's
 * input (then forwarded with fp8ds_fp8_io.in_cast).  All casts go through
 * fp8_cast_transpose_amax_multi (one launch for up to 256 casts).
 *   lins      host array of num_lins handle pointers.
 * Errors: FP8DS_ERR_INVALID_ARG for an incomplete handle, a meta index out of
 * range, or an invalid extra job; nothing is enqueued then and no cache_valid
 * flag changes.
 */
fp8ds_status fp8_linear_refresh_weights(fp8ds_linear *const *lins, int32_t num_lins,
                                        const fp8ds_meta *meta, const fp8ds_cast_job *extra,
                                        int32_t num_extra, fp8ds_stream stream);

/*
 * fp8_linear_bwd -- FP8 backward of one linear [TE761 HYBRID: e5m2 gradients]:
 *   1. cast dy -> e5m2 dy8 and dy8t with meta.scale[meta_grad], amax into
 *      amax_history[0, meta_grad], private scale_inv into *dy_scale_inv;
 *   2. dgrad (if dx != NULL): dx[m, in] = dy8 . (w8t)^T with
 *      *dy_scale_inv * *w_scale_inv (the cached weight's private copy);
 *   3. wgrad: dw[out, in] (fp32) = dy8t . (x8t)^T with *dy_scale_inv * *x_scale_inv.
 *   dy [m, out_features] (dy_dtype); x8t [in_features, m] and x_scale_inv from
 *   the forward; dy8 [m, out_features], dy8t [out_features, m] workspaces.
 *   dy8t may be NULL (no gradient transpose is written; the wgrad reads dy8
 *   MN-major), and a linear without w8t has its dgrad read w8 MN-major (see
 *   fp8_gemm_major; out_features % 16 == 0 / in_features % 16 == 0 then).
 * Requires lin->cache_valid.  Errors: as the calls it makes.
 */
fp8ds_status fp8_linear_bwd(const fp8ds_linear *lin, const fp8ds_meta *meta, const void *dy,
                            fp8ds_dtype dy_dtype, int64_t m, const uint8_t *x8t,
                            const float *x_scale_inv, void *dx, fp8ds_dtype dx_dtype,
                            float *dw, uint8_t *dy8, uint8_t *dy8t, float *dy_scale_inv,
                            fp8ds_stream stream);

/*
 * Options of fp8_linear_fwd_ex / fp8_linear_bwd_ex: how the FP8 tensors pass
 * between consecutive linears without a separate cast (zero-initialise, set
 * out_meta = -1 for "no FP8 output").
 *   in_cast   non-zero: the input (forward) or output gradient (backward) is
 *             already cast -- x8 / x8t / x_scale_inv (dy8 / dy8t /
 *             dy_scale_inv) hold it, written by the neighbouring layer's
 *             fused epilogue, which also recorded its amax -- so x (dy) may be
 *             NULL and no cast is enqueued.
 *   out_meta  >= 0: the forward output (backward dgrad) is cast in the GEMM
 *             epilogue as fp8_gemm_cast does, with meta.scale[out_meta]
 *             (format e4m3 forward, e5m2 backward: HYBRID), its amax recorded
 *             in amax_history[0, out_meta]; y (dx) is not written.  -1: none.
 *   out8      [m, out_features] forward / [m, in_features] backward codes.
 *   out8t     their transpose, or NULL.
 *   out_scale_inv  [1] private scale_inv of out8 (fl32(1 / scale)).
 * With both, an MLP hands H and dH from GEMM to GEMM in FP8: fc1's forward
 * writes fc2's x8 / x8t (out_meta = fc2's meta_in) and fc2's backward writes
 * fc1's dy8 / dy8t (out_meta = fc1's meta_grad).  The results are those of
 * the unfused calls: the same bytes, amaxes and scales.
 */
typedef struct {
    int32_t in_cast;
    int32_t out_meta;
    uint8_t *out8;
    uint8_t *out8t;
    float *out_scale_inv;
} fp8ds_fp8_io;

/* fp8_linear_fwd with the options above (io may be NULL: same as fp8_linear_fwd). */
fp8ds_status fp8_linear_fwd_ex(fp8ds_linear *lin, const fp8ds_meta *meta, const void *x,
                               fp8ds_dtype x_dtype, int64_t m, void *y, fp8ds_dtype y_dtype,
                               int32_t is_first_microbatch, uint8_t *x8, uint8_t *x8t,
                               float *x_scale_inv, const fp8ds_fp8_io *io, fp8ds_stream stream);

/*
 * fp8_linear_bwd with the options above (io may be NULL), and with every
 * transposed copy optional (fp8_gemm_major reads the untransposed tensors):
 *   x8t NULL  -> the wgrad reads x8 [m, in_features] (required then);
 *   dy8t NULL -> the gradient cast writes no transpose and the wgrad reads
 *                dy8 [m, out_features];
 *   lin->w8t NULL (also accepted by the forward, which then writes no weight
 *                transpose) -> the dgrad reads w8 [out_features, in_features].
 * MN-major reads need in_features % 16 == 0 and out_features % 16 == 0.
 */
fp8ds_status fp8_linear_bwd_ex(const fp8ds_linear *lin, const fp8ds_meta *meta, const void *dy,
                               fp8ds_dtype dy_dtype, int64_t m, const uint8_t *x8, const uint8_t *x8t,
                               const float *x_scale_inv, void *dx, fp8ds_dtype dx_dtype,
                               float *dw, uint8_t *dy8, uint8_t *dy8t, float *dy_scale_inv,
                               const fp8ds_fp8_io *io, fp8ds_stream stream);

/* Message describing the last error returned on the calling thread ("" if none). */
const char *fp8ds_last_error(void);

/*
 * fp8ds_device_status -- reads the device error word that kernels set when a
 * bounded wait gives up (0 = none, otherwise FP8DS_ERR_TIMEOUT in the low byte
 * and the site in the upper bytes).  Synchronises the current device.  If
 * `clear` is non-zero the word is reset to 0.  Returns FP8DS_ERR_CUDA if the
 * read fails.
 */
fp8ds_status fp8ds_device_status(int32_t *code_out, int32_t clear);

/*
 * fp8ds_test_stream_k_withhold -- test setting for the error path of the
 * stream-K GEMM; it has no counterpart on the pages and changes nothing the
 * method computes.  With withhold != 0, every stream-K launch issued after
 * the call (fp8_gemm_ex, fp8_gemm_noalloc and the linear calls with a
 * workspace) runs with the CTA pairs that compute the later k-blocks of a
 * split tile NOT publishing their partial sums: the pairs that own those
 * tiles wait for a publication that never comes, give up after wait_ns
 * nanoseconds (0: the default limit of 2 s), record FP8DS_ERR_TIMEOUT with
 * site code 5 (the partial-sum wait) in the device error word
 * (fp8ds_device_status: (5 << 8) | FP8DS_ERR_TIMEOUT), leave their split
 * tiles unwritten and exit; the launch ends and the context stays usable.
 * withhold = 0 (and wait_ns = 0) restores normal operation.  A process-wide
 * host setting read when a GEMM is enqueued; a graph captured meanwhile
 * keeps it.  Always returns FP8DS_OK.
 */
fp8ds_status fp8ds_test_stream_k_withhold(int32_t withhold, uint64_t wait_ns);

/* Library version string. */
const char *fp8ds_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8DS_H */
