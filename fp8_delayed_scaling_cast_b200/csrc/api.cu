// C ABI of libfp8ds.so: argument checks, error reporting and the FP8 linear
// forward/backward glue.  Every numeric step runs in the kernels of cast.cu,
// update.cu and gemm_sm100.cu; this file only validates and enqueues.
#include <stdarg.h>
#include <stdio.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "fp8ds_internal.h"

namespace fp8ds {

namespace {
thread_local char g_msg[512] = "";

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool valid_fmt(int f) { return f == FP8DS_E4M3 || f == FP8DS_E5M2; }
bool valid_dtype(int d) { return d == FP8DS_F32 || d == FP8DS_BF16; }
}  // namespace

void set_error(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
}

void clear_error() { g_msg[0] = '\0'; }

int num_sms() {
    // per device; concurrent first calls may both query and store the same value
    static std::atomic<int> cached[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}
}  // namespace

bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t read_device_error(int32_t *out, bool clear) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    int32_t g = 0, c = 0;
    if ((e = read_gemm_error(&g, clear)) != cudaSuccess) return e;
    if ((e = read_cast_error(&c, clear)) != cudaSuccess) return e;
    *out = g != 0 ? g : c;
    return cudaSuccess;
}

static fp8ds_status cuda_status(cudaError_t e, const char *what) {
    if (e == cudaSuccess) return FP8DS_OK;
    set_error("%s: %s", what, cudaGetErrorString(e));
    return FP8DS_ERR_CUDA;
}

static fp8ds_status invalid(const char *fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_msg, sizeof g_msg, fmt, ap);
    va_end(ap);
    return FP8DS_ERR_INVALID_ARG;
}

// ------------------------------------------------------------------ checks --

static fp8ds_status check_cast(const char *fn, const void *x, int x_dtype, int64_t a, int64_t b, int fmt,
                               const float *scale, const uint8_t *y) {
    if (a < 0 || b < 0) return invalid("%s: negative size", fn);
    if (scale == nullptr) return invalid("%s: scale must not be NULL", fn);
    if ((x == nullptr || y == nullptr) && a != 0 && b != 0)
        return invalid("%s: x and y must not be NULL for a non-empty tensor", fn);
    if (!valid_dtype(x_dtype)) return invalid("%s: unknown input dtype %d", fn, x_dtype);
    if (!valid_fmt(fmt)) return invalid("%s: unknown FP8 format %d", fn, fmt);
    return FP8DS_OK;
}

// a_mn / b_mn: the operand is stored MN-major ([k, m] / [k, n] row-major);
// its row pitch is then m (n) bytes instead of k, which the tensor map needs
// to be a multiple of 16.
static fp8ds_status check_gemm_layout(const uint8_t *a, int fa, const float *sa, bool a_mn, const uint8_t *b, int fb,
                                      const float *sb, bool b_mn, const void *bias, int bias_dtype, const void *d,
                                      int d_dtype, int64_t m, int64_t n, int64_t k) {
    if (a == nullptr || b == nullptr || d == nullptr || sa == nullptr || sb == nullptr)
        return invalid("fp8_gemm: a, b, d and the scale_inv pointers must not be NULL");
    if (!valid_fmt(fa) || !valid_fmt(fb)) return invalid("fp8_gemm: unknown FP8 format");
    if (!valid_dtype(d_dtype) || (bias != nullptr && !valid_dtype(bias_dtype)))
        return invalid("fp8_gemm: unknown output or bias dtype");
    if (m <= 0 || n <= 0 || k <= 0) return invalid("fp8_gemm: m, n, k must be positive");
    if (m > 0x7FFFFFFF || n > 0x7FFFFFFF || k > 0x7FFFFFFF) return invalid("fp8_gemm: size exceeds 2^31-1");
    if ((!a_mn || !b_mn) && k % 16 != 0)
        return invalid("fp8_gemm: k (%lld) must be a multiple of 16 for a K-major operand", (long long)k);
    if (a_mn && m % 16 != 0) return invalid("fp8_gemm: m (%lld) must be a multiple of 16 for an MN-major a", (long long)m);
    if (b_mn && n % 16 != 0) return invalid("fp8_gemm: n (%lld) must be a multiple of 16 for an MN-major b", (long long)n);
    if (d_dtype == FP8DS_BF16 && n % 8 != 0) return invalid("fp8_gemm: n must be a multiple of 8 for bf16 output");
    if (d_dtype == FP8DS_F32 && n % 4 != 0) return invalid("fp8_gemm: n must be a multiple of 4 for fp32 output");
    if (!aligned16(a) || !aligned16(b) || !aligned16(d))
        return invalid("fp8_gemm: a, b and d must be 16-byte aligned");
    return FP8DS_OK;
}

// Extra conditions of a GEMM whose output is FP8 codes (row pitch n bytes,
// transposed pitch m bytes: both multiples of 16 for the tensor maps).
static fp8ds_status check_cast_out(const char *fn, const uint8_t *d8, const uint8_t *d8t, const float *scale,
                                   int64_t m, int64_t n) {
    if (d8 == nullptr || scale == nullptr) return invalid("%s: the FP8 output and its scale must not be NULL", fn);
    if (n % 16 != 0) return invalid("%s: n (%lld) must be a multiple of 16 for FP8 output", fn, (long long)n);
    if (d8t != nullptr && m % 16 != 0)
        return invalid("%s: m (%lld) must be a multiple of 16 for the transposed FP8 output", fn, (long long)m);
    if (!aligned16(d8) || (d8t != nullptr && !aligned16(d8t)))
        return invalid("%s: the FP8 outputs must be 16-byte aligned", fn);
    return FP8DS_OK;
}

static fp8ds_status check_gemm(const uint8_t *a, int fa, const float *sa, const uint8_t *b, int fb,
                               const float *sb, const void *bias, int bias_dtype, const void *d, int d_dtype,
                               int64_t m, int64_t n, int64_t k) {
    return check_gemm_layout(a, fa, sa, false, b, fb, sb, false, bias, bias_dtype, d, d_dtype, m, n, k);
}

static fp8ds_status check_meta(const char *fn, const fp8ds_meta *meta, int32_t idx) {
    if (meta == nullptr || meta->amax_history == nullptr || meta->scale == nullptr || meta->scale_inv == nullptr)
        return invalid("%s: incomplete meta", fn);
    if (meta->hist_len < 1) return invalid("%s: hist_len must be >= 1", fn);
    if (idx < 0 || idx >= meta->num_tensors) return invalid("%s: meta index %d out of range", fn, idx);
    return FP8DS_OK;
}

}  // namespace fp8ds

using namespace fp8ds;

extern "C" {

fp8ds_status fp8_quantize(const void *x, fp8ds_dtype x_dtype, int64_t n, fp8ds_format fmt, const float *scale,
                          uint8_t *y, float *amax, float *scale_inv, fp8ds_stream stream) {
    clear_error();
    fp8ds_status st = check_cast("fp8_quantize", x, x_dtype, n, 1, fmt, scale, y);
    if (st != FP8DS_OK) return st;
    return cuda_status(launch_quantize(x, x_dtype, n, fmt, scale, y, amax, scale_inv, stream), "fp8_quantize");
}

fp8ds_status fp8_cast_transpose_amax(const void *x, fp8ds_dtype x_dtype, int64_t rows, int64_t cols,
                                     fp8ds_format fmt, const float *scale, uint8_t *y, uint8_t *yt, float *amax,
                                     float *scale_inv, fp8ds_stream stream) {
    clear_error();
    fp8ds_status st = check_cast("fp8_cast_transpose_amax", x, x_dtype, rows, cols, fmt, scale, y);
    if (st != FP8DS_OK) return st;
    return cuda_status(launch_cast_transpose(x, x_dtype, rows, cols, fmt, scale, y, yt, amax, scale_inv, stream),
                       "fp8_cast_transpose_amax");
}

fp8ds_status fp8_cast_transpose_amax_noop(const void *x, fp8ds_dtype x_dtype, int64_t rows, int64_t cols,
                                          fp8ds_format fmt, const float *scale, uint8_t *y, uint8_t *yt,
                                          float *amax, float *scale_inv, const int32_t *noop_flag,
                                          fp8ds_stream stream) {
    clear_error();
    fp8ds_status st = check_cast("fp8_cast_transpose_amax_noop", x, x_dtype, rows, cols, fmt, scale, y);
    if (st != FP8DS_OK) return st;
    if (noop_flag == nullptr) return invalid("fp8_cast_transpose_amax_noop: noop_flag must not be NULL");
    return cuda_status(
        launch_cast_transpose(x, x_dtype, rows, cols, fmt, scale, y, yt, amax, scale_inv, stream, noop_flag),
        "fp8_cast_transpose_amax_noop");
}

fp8ds_status fp8_cast_transpose_amax_pair(const void *x_a, int64_t rows_a, int64_t cols_a, const float *scale_a,
                                          uint8_t *y_a, uint8_t *yt_a, float *amax_a, float *scale_inv_a,
                                          const void *x_b, int64_t rows_b, int64_t cols_b, const float *scale_b,
                                          uint8_t *y_b, uint8_t *yt_b, float *amax_b, float *scale_inv_b,
                                          const int32_t *noop_b, fp8ds_dtype x_dtype, fp8ds_format fmt,
                                          fp8ds_stream stream) {
    clear_error();
    fp8ds_status st = check_cast("fp8_cast_transpose_amax_pair (a)", x_a, x_dtype, rows_a, cols_a, fmt, scale_a, y_a);
    if (st != FP8DS_OK) return st;
    st = check_cast("fp8_cast_transpose_amax_pair (b)", x_b, x_dtype, rows_b, cols_b, fmt, scale_b, y_b);
    if (st != FP8DS_OK) return st;
    return cuda_status(launch_cast_transpose_pair(x_a, rows_a, cols_a, scale_a, y_a, yt_a, amax_a, scale_inv_a, x_b,
                                                  rows_b, cols_b, scale_b, y_b, yt_b, amax_b, scale_inv_b, noop_b,
                                                  x_dtype, fmt, stream),
                       "fp8_cast_transpose_amax_pair");
}

// Checks of one job of a multi-tensor cast (the message names the job).
static fp8ds_status check_cast_job(const char *fn, const fp8ds_cast_job &j, int32_t i) {
    char what[96];
    snprintf(what, sizeof what, "%s (job %d)", fn, static_cast<int>(i));
    fp8ds_status st = check_cast(what, j.x, j.x_dtype, j.rows, j.cols, j.fmt, j.scale, j.y);
    if (st != FP8DS_OK) return st;
    if (j.yt != nullptr && (j.rows >= (int64_t(1) << 31) || j.cols >= (int64_t(1) << 31)))
        return invalid("%s: rows and cols must be below 2^31 with a transpose", what);
    return FP8DS_OK;
}

fp8ds_status fp8_cast_transpose_amax_multi(const fp8ds_cast_job *jobs, int32_t num_jobs, fp8ds_stream stream) {
    clear_error();
    if (num_jobs < 0) return invalid("fp8_cast_transpose_amax_multi: num_jobs < 0");
    if (num_jobs > 0 && jobs == nullptr) return invalid("fp8_cast_transpose_amax_multi: jobs must not be NULL");
    for (int32_t i = 0; i < num_jobs; ++i) {
        fp8ds_status st = check_cast_job("fp8_cast_transpose_amax_multi", jobs[i], i);
        if (st != FP8DS_OK) return st;
    }
    if (num_jobs == 0) return FP8DS_OK;
    return cuda_status(launch_cast_multi(jobs, num_jobs, stream), "fp8_cast_transpose_amax_multi");
}

fp8ds_status fp8_cast_transpose_amax_dynamic(const void *x, fp8ds_dtype x_dtype, int64_t rows, int64_t cols,
                                             fp8ds_format fmt, float *scale, uint8_t *y, uint8_t *yt, float *amax,
                                             float *scale_inv, fp8ds_stream stream) {
    clear_error();
    fp8ds_status st = check_cast("fp8_cast_transpose_amax_dynamic", x, x_dtype, rows, cols, fmt, scale, y);
    if (st != FP8DS_OK) return st;
    if (amax == nullptr) return invalid("fp8_cast_transpose_amax_dynamic: amax must not be NULL");
    return cuda_status(
        launch_cast_transpose_dynamic(x, x_dtype, rows, cols, fmt, scale, y, yt, amax, scale_inv, stream),
        "fp8_cast_transpose_amax_dynamic");
}

fp8ds_status fp8_transpose(const uint8_t *y, int64_t rows, int64_t cols, uint8_t *yt, fp8ds_stream stream) {
    clear_error();
    if (rows < 0 || cols < 0) return invalid("fp8_transpose: negative size");
    if ((y == nullptr || yt == nullptr) && rows != 0 && cols != 0)
        return invalid("fp8_transpose: y and yt must not be NULL for a non-empty tensor");
    if (y == yt && rows != 0 && cols != 0) return invalid("fp8_transpose: y and yt must not alias");
    return cuda_status(launch_transpose_u8(y, rows, cols, yt, stream), "fp8_transpose");
}

fp8ds_status fp8_update_scales(int64_t num_tensors, int32_t hist_len, float *amax_history, float *scale,
                               float *scale_inv, const uint8_t *formats, fp8ds_amax_algo algo,
                               fp8ds_stream stream) {
    clear_error();
    if (num_tensors < 0) return invalid("fp8_update_scales: num_tensors < 0");
    if (hist_len < 1) return invalid("fp8_update_scales: hist_len must be >= 1");
    if (num_tensors > 0 && (amax_history == nullptr || scale == nullptr || scale_inv == nullptr || formats == nullptr))
        return invalid("fp8_update_scales: NULL pointer");
    if (algo != FP8DS_AMAX_MAX && algo != FP8DS_AMAX_MOST_RECENT) {
        set_error("fp8_update_scales: unknown amax_compute_algo %d", static_cast<int>(algo));
        return FP8DS_ERR_UNSUPPORTED;
    }
    return cuda_status(
        launch_update_scales(num_tensors, hist_len, amax_history, scale, scale_inv, formats, algo, stream),
        "fp8_update_scales");
}

fp8ds_status fp8_gemm(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv, const uint8_t *b,
                      fp8ds_format b_fmt, const float *b_scale_inv, const void *bias, fp8ds_dtype bias_dtype,
                      void *d, fp8ds_dtype d_dtype, int64_t m, int64_t n, int64_t k, fp8ds_stream stream) {
    clear_error();
    fp8ds_status st =
        check_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k);
    if (st != FP8DS_OK) return st;
    return launch_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k, nullptr,
                       0, stream);
}

fp8ds_status fp8_gemm_workspace_size(size_t *bytes) {
    clear_error();
    if (bytes == nullptr) return invalid("fp8_gemm_workspace_size: bytes must not be NULL");
    *bytes = gemm_workspace_bytes();
    return FP8DS_OK;
}

fp8ds_status fp8_gemm_plan(int64_t m, int64_t n, int64_t k, int64_t *info) {
    clear_error();
    if (info == nullptr) return invalid("fp8_gemm_plan: info must not be NULL");
    if (m <= 0 || n <= 0 || k <= 0) return invalid("fp8_gemm_plan: m, n, k must be positive");
    gemm_plan_info(m, n, k, info);
    return FP8DS_OK;
}

fp8ds_status fp8_gemm_ex(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv, const uint8_t *b,
                         fp8ds_format b_fmt, const float *b_scale_inv, const void *bias, fp8ds_dtype bias_dtype,
                         void *d, fp8ds_dtype d_dtype, int64_t m, int64_t n, int64_t k, void *workspace,
                         size_t workspace_bytes, fp8ds_stream stream) {
    clear_error();
    fp8ds_status st =
        check_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k);
    if (st != FP8DS_OK) return st;
    if (workspace != nullptr && !aligned16(workspace)) return invalid("fp8_gemm_ex: workspace must be 16-byte aligned");
    return launch_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k, workspace,
                       workspace_bytes, stream);
}

fp8ds_status fp8_gemm_noalloc(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv, const uint8_t *b,
                              fp8ds_format b_fmt, const float *b_scale_inv, const void *bias, fp8ds_dtype bias_dtype,
                              void *d, fp8ds_dtype d_dtype, int64_t m, int64_t n, int64_t k, fp8ds_stream stream) {
    clear_error();
    fp8ds_status st =
        check_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k);
    if (st != FP8DS_OK) return st;
    return launch_gemm_noalloc(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k,
                               stream);
}

fp8ds_status fp8_gemm_major(const uint8_t *a, fp8ds_format a_fmt, fp8ds_major a_major, const float *a_scale_inv,
                            const uint8_t *b, fp8ds_format b_fmt, fp8ds_major b_major, const float *b_scale_inv,
                            const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype, int64_t m,
                            int64_t n, int64_t k, fp8ds_stream stream) {
    clear_error();
    if ((a_major != FP8DS_K_MAJOR && a_major != FP8DS_MN_MAJOR) ||
        (b_major != FP8DS_K_MAJOR && b_major != FP8DS_MN_MAJOR))
        return invalid("fp8_gemm_major: unknown operand layout");
    const bool a_mn = a_major == FP8DS_MN_MAJOR, b_mn = b_major == FP8DS_MN_MAJOR;
    fp8ds_status st = check_gemm_layout(a, a_fmt, a_scale_inv, a_mn, b, b_fmt, b_scale_inv, b_mn, bias, bias_dtype,
                                        d, d_dtype, m, n, k);
    if (st != FP8DS_OK) return st;
    return launch_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k, nullptr,
                       0, stream, nullptr, a_mn, b_mn);
}

fp8ds_status fp8_gemm_cast(const uint8_t *a, fp8ds_format a_fmt, fp8ds_major a_major, const float *a_scale_inv,
                           const uint8_t *b, fp8ds_format b_fmt, fp8ds_major b_major, const float *b_scale_inv,
                           const void *bias, fp8ds_dtype bias_dtype, int64_t m, int64_t n, int64_t k,
                           fp8ds_format out_fmt, const float *out_scale, uint8_t *d8, uint8_t *d8t, float *out_amax,
                           float *out_scale_inv, fp8ds_stream stream) {
    clear_error();
    if ((a_major != FP8DS_K_MAJOR && a_major != FP8DS_MN_MAJOR) ||
        (b_major != FP8DS_K_MAJOR && b_major != FP8DS_MN_MAJOR))
        return invalid("fp8_gemm_cast: unknown operand layout");
    const bool a_mn = a_major == FP8DS_MN_MAJOR, b_mn = b_major == FP8DS_MN_MAJOR;
    fp8ds_status st = check_gemm_layout(a, a_fmt, a_scale_inv, a_mn, b, b_fmt, b_scale_inv, b_mn, bias, bias_dtype,
                                        d8, FP8DS_BF16, m, n, k);
    if (st != FP8DS_OK) return st;
    if (!valid_fmt(out_fmt)) return invalid("fp8_gemm_cast: unknown output FP8 format %d", out_fmt);
    if ((st = check_cast_out("fp8_gemm_cast", d8, d8t, out_scale, m, n)) != FP8DS_OK) return st;
    const GemmCastOut cast{out_fmt, out_scale, d8t, out_amax, out_scale_inv};
    return launch_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d8, FP8DS_BF16, m, n, k,
                       nullptr, 0, stream, &cast, a_mn, b_mn);
}

// The linear forward and backward, with the options of the _ex forms (NULL:
// none).  io->in_cast: the input (gradient) already sits in x8 / x8t /
// x_scale_inv (dy8 / dy8t / dy_scale_inv).  io->out_meta >= 0: the output
// (dgrad) is cast in the GEMM epilogue with that meta's scale.
static fp8ds_status linear_fwd(const char *fn, fp8ds_linear *lin, const fp8ds_meta *meta, const void *x,
                               fp8ds_dtype x_dtype, int64_t m, void *y, fp8ds_dtype y_dtype,
                               int32_t is_first_microbatch, uint8_t *x8, uint8_t *x8t, float *x_scale_inv,
                               const fp8ds_fp8_io *io, cudaStream_t s) {
    if (lin == nullptr || lin->w == nullptr || lin->w8 == nullptr || lin->w_scale_inv == nullptr)
        return invalid("%s: incomplete linear handle", fn);
    const bool in_cast = io != nullptr && io->in_cast != 0;
    const bool out_cast = io != nullptr && io->out_meta >= 0;
    if ((!in_cast && x == nullptr) || (!out_cast && y == nullptr) || x8 == nullptr || x_scale_inv == nullptr)
        return invalid("%s: x, y, x8 and x_scale_inv must not be NULL", fn);
    if (is_first_microbatch < -1 || is_first_microbatch > 1)
        return invalid("%s: is_first_microbatch must be -1, 0 or 1", fn);
    fp8ds_status st;
    if ((st = check_meta(fn, meta, lin->meta_in)) != FP8DS_OK) return st;
    if ((st = check_meta(fn, meta, lin->meta_w)) != FP8DS_OK) return st;
    if (out_cast && (st = check_meta(fn, meta, io->out_meta)) != FP8DS_OK) return st;
    const int64_t K = lin->in_features, N = lin->out_features;
    if (!in_cast && (st = check_cast(fn, x, x_dtype, m, K, FP8DS_E4M3, meta->scale, x8)) != FP8DS_OK) return st;
    if ((st = check_gemm(x8, FP8DS_E4M3, x_scale_inv, lin->w8, FP8DS_E4M3, lin->w_scale_inv, lin->bias,
                         lin->bias_dtype, out_cast ? static_cast<void *>(io->out8) : y,
                         out_cast ? FP8DS_BF16 : y_dtype, m, N, K)) != FP8DS_OK)
        return st;
    if (out_cast && (st = check_cast_out(fn, io->out8, io->out8t, meta->scale, m, N)) != FP8DS_OK) return st;
    const int32_t hi = lin->meta_in, hw = lin->meta_w;
    // With a device-side flag the weight cast is always enqueued and the GPU
    // decides (a captured graph then serves every microbatch); otherwise the
    // host decides from is_first_microbatch and the cache state.
    const bool refresh = lin->w_noop_flag != nullptr || is_first_microbatch != 0 || !lin->cache_valid;
    if (!in_cast && refresh && x_dtype == FP8DS_F32) {
        // input and weight (both fp32 -> e4m3) in one launch where the
        // shapes allow, else one after the other
        st = cuda_status(launch_cast_transpose_pair(x, m, K, meta->scale + hi, x8, x8t, meta->amax_history + hi,
                                                    x_scale_inv, lin->w, N, K, meta->scale + hw, lin->w8, lin->w8t,
                                                    meta->amax_history + hw, lin->w_scale_inv, lin->w_noop_flag,
                                                    FP8DS_F32, FP8DS_E4M3, s),
                         "fp8_linear_fwd: input and weight cast");
        if (st != FP8DS_OK) return st;
        lin->cache_valid = 1;
    } else {
        if (!in_cast) {
            st = cuda_status(launch_cast_transpose(x, x_dtype, m, K, FP8DS_E4M3, meta->scale + hi, x8, x8t,
                                                   meta->amax_history + hi, x_scale_inv, s),
                             "fp8_linear_fwd: input cast");
            if (st != FP8DS_OK) return st;
        }
        if (refresh) {
            st = cuda_status(launch_cast_transpose(lin->w, FP8DS_F32, N, K, FP8DS_E4M3, meta->scale + hw, lin->w8,
                                                   lin->w8t, meta->amax_history + hw, lin->w_scale_inv, s,
                                                   lin->w_noop_flag),
                             "fp8_linear_fwd: weight cast");
            if (st != FP8DS_OK) return st;
            lin->cache_valid = 1;
        }
    }
    if (out_cast) {
        const int32_t ho = io->out_meta;
        const GemmCastOut cast{FP8DS_E4M3, meta->scale + ho, io->out8t, meta->amax_history + ho, io->out_scale_inv};
        return launch_gemm(x8, FP8DS_E4M3, x_scale_inv, lin->w8, FP8DS_E4M3, lin->w_scale_inv, lin->bias,
                           lin->bias_dtype, io->out8, FP8DS_BF16, m, N, K, lin->workspace, lin->workspace_bytes, s,
                           &cast);
    }
    return launch_gemm(x8, FP8DS_E4M3, x_scale_inv, lin->w8, FP8DS_E4M3, lin->w_scale_inv, lin->bias,
                       lin->bias_dtype, y, y_dtype, m, N, K, lin->workspace, lin->workspace_bytes, s);
}

// Transposes are optional: without w8t the dgrad reads w8 MN-major, without
// dy8t the wgrad reads dy8 MN-major (and the gradient cast writes no
// transpose), without x8t it reads x8 MN-major.
static fp8ds_status linear_bwd(const char *fn, const fp8ds_linear *lin, const fp8ds_meta *meta, const void *dy,
                               fp8ds_dtype dy_dtype, int64_t m, const uint8_t *x8, const uint8_t *x8t,
                               const float *x_scale_inv, void *dx, fp8ds_dtype dx_dtype, float *dw, uint8_t *dy8,
                               uint8_t *dy8t, float *dy_scale_inv, const fp8ds_fp8_io *io, cudaStream_t s) {
    if (lin == nullptr || lin->w8 == nullptr || lin->w_scale_inv == nullptr)
        return invalid("%s: incomplete linear handle", fn);
    if (!lin->cache_valid) return invalid("%s: the weight cache is empty (run the forward first)", fn);
    const bool in_cast = io != nullptr && io->in_cast != 0;
    const bool out_cast = io != nullptr && io->out_meta >= 0;
    if ((!in_cast && dy == nullptr) || (x8t == nullptr && x8 == nullptr) || x_scale_inv == nullptr ||
        dw == nullptr || dy8 == nullptr || dy_scale_inv == nullptr)
        return invalid("%s: NULL pointer argument", fn);
    const bool w_mn = lin->w8t == nullptr, dy_mn = dy8t == nullptr, x_mn = x8t == nullptr;
    const uint8_t *wb = w_mn ? lin->w8 : lin->w8t;         // dgrad B
    const uint8_t *ga = dy_mn ? dy8 : dy8t;                // wgrad A
    const uint8_t *gb = x_mn ? x8 : x8t;                   // wgrad B
    fp8ds_status st;
    if ((st = check_meta(fn, meta, lin->meta_grad)) != FP8DS_OK) return st;
    if (out_cast && (st = check_meta(fn, meta, io->out_meta)) != FP8DS_OK) return st;
    const int64_t K = lin->in_features, N = lin->out_features;
    if (!in_cast && (st = check_cast(fn, dy, dy_dtype, m, N, FP8DS_E5M2, meta->scale, dy8)) != FP8DS_OK) return st;
    if (out_cast) {
        if ((st = check_gemm_layout(dy8, FP8DS_E5M2, dy_scale_inv, false, wb, FP8DS_E4M3, lin->w_scale_inv, w_mn,
                                    nullptr, FP8DS_F32, io->out8, FP8DS_BF16, m, K, N)) != FP8DS_OK)
            return st;
        if ((st = check_cast_out(fn, io->out8, io->out8t, meta->scale, m, K)) != FP8DS_OK) return st;
    } else if (dx != nullptr &&
               (st = check_gemm_layout(dy8, FP8DS_E5M2, dy_scale_inv, false, wb, FP8DS_E4M3, lin->w_scale_inv, w_mn,
                                       nullptr, FP8DS_F32, dx, dx_dtype, m, K, N)) != FP8DS_OK) {
        return st;
    }
    if ((st = check_gemm_layout(ga, FP8DS_E5M2, dy_scale_inv, dy_mn, gb, FP8DS_E4M3, x_scale_inv, x_mn, nullptr,
                                FP8DS_F32, dw, FP8DS_F32, N, K, m)) != FP8DS_OK)
        return st;
    const int32_t hg = lin->meta_grad;
    if (!in_cast) {
        st = cuda_status(launch_cast_transpose(dy, dy_dtype, m, N, FP8DS_E5M2, meta->scale + hg, dy8, dy8t,
                                               meta->amax_history + hg, dy_scale_inv, s),
                         "fp8_linear_bwd: grad cast");
        if (st != FP8DS_OK) return st;
    }
    if (out_cast) {
        const int32_t ho = io->out_meta;
        const GemmCastOut cast{FP8DS_E5M2, meta->scale + ho, io->out8t, meta->amax_history + ho, io->out_scale_inv};
        st = launch_gemm(dy8, FP8DS_E5M2, dy_scale_inv, wb, FP8DS_E4M3, lin->w_scale_inv, nullptr, FP8DS_F32,
                         io->out8, FP8DS_BF16, m, K, N, lin->workspace, lin->workspace_bytes, s, &cast, false, w_mn);
        if (st != FP8DS_OK) return st;
    } else if (dx != nullptr) {
        st = launch_gemm(dy8, FP8DS_E5M2, dy_scale_inv, wb, FP8DS_E4M3, lin->w_scale_inv, nullptr, FP8DS_F32, dx,
                         dx_dtype, m, K, N, lin->workspace, lin->workspace_bytes, s, nullptr, false, w_mn);
        if (st != FP8DS_OK) return st;
    }
    return launch_gemm(ga, FP8DS_E5M2, dy_scale_inv, gb, FP8DS_E4M3, x_scale_inv, nullptr, FP8DS_F32, dw, FP8DS_F32, N,
                       K, m, lin->workspace, lin->workspace_bytes, s, nullptr, dy_mn, x_mn);
}

fp8ds_status fp8_linear_fwd(fp8ds_linear *lin, const fp8ds_meta *meta, const void *x, fp8ds_dtype x_dtype,
                            int64_t m, void *y, fp8ds_dtype y_dtype, int32_t is_first_microbatch, uint8_t *x8,
                            uint8_t *x8t, float *x_scale_inv, fp8ds_stream stream) {
    clear_error();
    return linear_fwd("fp8_linear_fwd", lin, meta, x, x_dtype, m, y, y_dtype, is_first_microbatch, x8, x8t,
                      x_scale_inv, nullptr, stream);
}

fp8ds_status fp8_linear_fwd_ex(fp8ds_linear *lin, const fp8ds_meta *meta, const void *x, fp8ds_dtype x_dtype,
                               int64_t m, void *y, fp8ds_dtype y_dtype, int32_t is_first_microbatch, uint8_t *x8,
                               uint8_t *x8t, float *x_scale_inv, const fp8ds_fp8_io *io, fp8ds_stream stream) {
    clear_error();
    return linear_fwd("fp8_linear_fwd_ex", lin, meta, x, x_dtype, m, y, y_dtype, is_first_microbatch, x8, x8t,
                      x_scale_inv, io, stream);
}

fp8ds_status fp8_linear_refresh_weights(fp8ds_linear *const *lins, int32_t num_lins, const fp8ds_meta *meta,
                                        const fp8ds_cast_job *extra, int32_t num_extra, fp8ds_stream stream) {
    clear_error();
    const char *fn = "fp8_linear_refresh_weights";
    if (num_lins < 0 || num_extra < 0) return invalid("%s: negative count", fn);
    if ((num_lins > 0 && lins == nullptr) || (num_extra > 0 && extra == nullptr))
        return invalid("%s: NULL array", fn);
    std::vector<fp8ds_cast_job> jobs;
    jobs.reserve(static_cast<size_t>(num_lins) + static_cast<size_t>(num_extra));
    for (int32_t i = 0; i < num_lins; ++i) {
        const fp8ds_linear *lin = lins[i];
        if (lin == nullptr || lin->w == nullptr || lin->w8 == nullptr || lin->w_scale_inv == nullptr)
            return invalid("%s: incomplete linear handle %d", fn, static_cast<int>(i));
        fp8ds_status st = check_meta(fn, meta, lin->meta_w);
        if (st != FP8DS_OK) return st;
        fp8ds_cast_job j;
        j.x = lin->w;
        j.x_dtype = FP8DS_F32;
        j.rows = lin->out_features;
        j.cols = lin->in_features;
        j.fmt = FP8DS_E4M3;
        j.scale = meta->scale + lin->meta_w;
        j.y = lin->w8;
        j.yt = lin->w8t;
        j.amax = meta->amax_history + lin->meta_w;
        j.scale_inv = lin->w_scale_inv;
        j.noop_flag = lin->w_noop_flag;
        if ((st = check_cast_job(fn, j, i)) != FP8DS_OK) return st;
        jobs.push_back(j);
    }
    for (int32_t i = 0; i < num_extra; ++i) {
        fp8ds_status st = check_cast_job(fn, extra[i], num_lins + i);
        if (st != FP8DS_OK) return st;
        jobs.push_back(extra[i]);
    }
    if (jobs.empty()) return FP8DS_OK;
    fp8ds_status st = cuda_status(launch_cast_multi(jobs.data(), static_cast<int32_t>(jobs.size()), stream), fn);
    if (st != FP8DS_OK) return st;
    for (int32_t i = 0; i < num_lins; ++i) lins[i]->cache_valid = 1;
    return FP8DS_OK;
}

fp8ds_status fp8_linear_bwd(const fp8ds_linear *lin, const fp8ds_meta *meta, const void *dy, fp8ds_dtype dy_dtype,
                            int64_t m, const uint8_t *x8t, const float *x_scale_inv, void *dx, fp8ds_dtype dx_dtype,
                            float *dw, uint8_t *dy8, uint8_t *dy8t, float *dy_scale_inv, fp8ds_stream stream) {
    clear_error();
    return linear_bwd("fp8_linear_bwd", lin, meta, dy, dy_dtype, m, nullptr, x8t, x_scale_inv, dx, dx_dtype, dw, dy8,
                      dy8t, dy_scale_inv, nullptr, stream);
}

fp8ds_status fp8_linear_bwd_ex(const fp8ds_linear *lin, const fp8ds_meta *meta, const void *dy,
                               fp8ds_dtype dy_dtype, int64_t m, const uint8_t *x8, const uint8_t *x8t,
                               const float *x_scale_inv, void *dx, fp8ds_dtype dx_dtype, float *dw, uint8_t *dy8,
                               uint8_t *dy8t, float *dy_scale_inv, const fp8ds_fp8_io *io, fp8ds_stream stream) {
    clear_error();
    return linear_bwd("fp8_linear_bwd_ex", lin, meta, dy, dy_dtype, m, x8, x8t, x_scale_inv, dx, dx_dtype, dw, dy8, dy8t,
                      dy_scale_inv, io, stream);
}

const char *fp8ds_last_error(void) { return g_msg; }

fp8ds_status fp8ds_device_status(int32_t *code_out, int32_t clear) {
    clear_error();
    if (code_out == nullptr) return invalid("fp8ds_device_status: code_out must not be NULL");
    return cuda_status(read_device_error(code_out, clear != 0), "fp8ds_device_status");
}

fp8ds_status fp8ds_test_stream_k_withhold(int32_t withhold, uint64_t wait_ns) {
    clear_error();
    set_stream_k_withhold(withhold != 0 ? 1 : 0, static_cast<unsigned long long>(wait_ns));
    return FP8DS_OK;
}

const char *fp8ds_version(void) { return "fp8ds 0.1.0 (sm_100a)"; }

}  // extern "C"
