// Internal declarations shared by the translation units of libfp8ds.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "fp8ds.h"

namespace fp8ds {

// Thread-local error message for fp8ds_last_error().
void set_error(const char *fmt, ...);
void clear_error();

// Multiprocessor count of the current device (cached per device).
int num_sms();

// Kernel launchers.  They assume the arguments were validated by the C ABI
// layer and return the launch status.
cudaError_t launch_quantize(const void *x, fp8ds_dtype x_dtype, int64_t n, fp8ds_format fmt,
                            const float *scale, uint8_t *y, float *amax, float *scale_inv,
                            cudaStream_t stream);

// noop (may be NULL): a device int32; when it holds non-zero at run time the
// kernel returns before touching anything (outputs keep their values).
cudaError_t launch_cast_transpose(const void *x, fp8ds_dtype x_dtype, int64_t rows, int64_t cols,
                                  fp8ds_format fmt, const float *scale, uint8_t *y, uint8_t *yt,
                                  float *amax, float *scale_inv, cudaStream_t stream,
                                  const int32_t *noop = nullptr);

// Two casts of one input dtype and format (a: no noop flag; b: noop_b may be
// NULL), in one launch when both suit the TMA kernel and both or neither
// write a transpose, else as two launches.  Results as two calls of
// launch_cast_transpose.
cudaError_t launch_cast_transpose_pair(const void *xa, int64_t rows_a, int64_t cols_a, const float *scale_a,
                                       uint8_t *ya, uint8_t *yta, float *amax_a, float *scale_inv_a, const void *xb,
                                       int64_t rows_b, int64_t cols_b, const float *scale_b, uint8_t *yb,
                                       uint8_t *ytb, float *amax_b, float *scale_inv_b, const int32_t *noop_b,
                                       fp8ds_dtype x_dtype, fp8ds_format fmt, cudaStream_t stream);

// Dynamic scaling: amax = max |x| (written, not accumulated), then
// scale = fp8_max / amax (kept when that is not finite and positive),
// scale_inv = 1 / scale, then the cast with that scale.
cudaError_t launch_cast_transpose_dynamic(const void *x, fp8ds_dtype x_dtype, int64_t rows, int64_t cols,
                                          fp8ds_format fmt, float *scale, uint8_t *y, uint8_t *yt, float *amax,
                                          float *scale_inv, cudaStream_t stream);

// Up to 256 casts per launch (more: consecutive launches); jobs validated by
// the caller (a transpose job needs rows, cols < 2^31).
cudaError_t launch_cast_multi(const fp8ds_cast_job *jobs, int32_t num_jobs, cudaStream_t stream);

// yt[c, r] = y[r, c] for a uint8 tensor [rows, cols].
cudaError_t launch_transpose_u8(const uint8_t *y, int64_t rows, int64_t cols, uint8_t *yt, cudaStream_t stream);

cudaError_t launch_update_scales(int64_t num_tensors, int32_t hist_len, float *amax_history,
                                 float *scale, float *scale_inv, const uint8_t *formats,
                                 fp8ds_amax_algo algo, cudaStream_t stream);

// FP8 output of launch_gemm: the bf16-rounded result cast with the delayed
// scale `*scale` into d (codes [m, n]) and, when d8t is not NULL, its
// transpose [n, m]; amax (may be NULL) receives max |bf16 result|, scale_inv
// (may be NULL) fl32(1 / *scale).
struct GemmCastOut {
    fp8ds_format fmt;
    const float *scale;
    uint8_t *d8t;
    float *amax;
    float *scale_inv;
};

// Returns FP8DS_OK or an error (message set) for tensor-map or launch failures.
// workspace (may be NULL) enables the stream-K schedule when it holds at
// least gemm_workspace_bytes().  With `cast`, d receives FP8 codes and
// d_dtype is ignored.  a_mn / b_mn: the operand is stored MN-major, a as
// [k, m] and b as [k, n] row-major (otherwise a is [m, k] and b [n, k]).
fp8ds_status launch_gemm(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv,
                         const uint8_t *b, fp8ds_format b_fmt, const float *b_scale_inv,
                         const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype,
                         int64_t m, int64_t n, int64_t k, void *workspace, size_t workspace_bytes,
                         cudaStream_t stream, const GemmCastOut *cast = nullptr, bool a_mn = false,
                         bool b_mn = false);

// Workspace bytes the stream-K schedule needs on the current device.
size_t gemm_workspace_bytes();
// The tile schedule of an m x n x k GEMM on the current device (fp8_gemm_plan).
void gemm_plan_info(int64_t m, int64_t n, int64_t k, int64_t info[5]);

// launch_gemm with the library's static device scratch as the workspace.
fp8ds_status launch_gemm_noalloc(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv,
                                 const uint8_t *b, fp8ds_format b_fmt, const float *b_scale_inv,
                                 const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype,
                                 int64_t m, int64_t n, int64_t k, cudaStream_t stream);

// Error-path test setting of the stream-K GEMM (fp8ds_test_stream_k_withhold).
void set_stream_k_withhold(int withhold, unsigned long long wait_ns);

// Device error words written by kernels whose bounded waits give up (one per
// translation unit); read_device_error returns the first non-zero one.
cudaError_t read_device_error(int32_t *out, bool clear);
cudaError_t read_gemm_error(int32_t *out, bool clear);
cudaError_t read_cast_error(int32_t *out, bool clear);

// 2-D tiled tensor map (cuTensorMapEncodeTiled through the runtime's driver
// entry point).  Returns false if the driver rejects the arguments.
bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

// Launches a kernel with programmatic stream serialization (the kernel may
// start before the previous one in the stream completes; it synchronises
// itself with griddepcontrol.wait) and, if cluster_x > 1, thread-block
// clusters of cluster_x CTAs.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       unsigned cluster_x, Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[n].val.programmaticStreamSerializationAllowed = 1;
    ++n;
    if (cluster_x > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster_x;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

}  // namespace fp8ds
