// Internal declarations shared by the translation units of libfp8ds.so.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

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

cudaError_t launch_cast_transpose(const void *x, fp8ds_dtype x_dtype, int64_t rows, int64_t cols,
                                  fp8ds_format fmt, const float *scale, uint8_t *y, uint8_t *yt,
                                  float *amax, float *scale_inv, cudaStream_t stream);

cudaError_t launch_update_scales(int64_t num_tensors, int32_t hist_len, float *amax_history,
                                 float *scale, float *scale_inv, const uint8_t *formats,
                                 cudaStream_t stream);

// Returns FP8DS_OK or an error (message set) for tensor-map or launch failures.
fp8ds_status launch_gemm(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv,
                         const uint8_t *b, fp8ds_format b_fmt, const float *b_scale_inv,
                         const void *bias, fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype,
                         int64_t m, int64_t n, int64_t k, cudaStream_t stream);

// Device error words written by kernels whose bounded waits give up (one per
// translation unit); read_device_error returns the first non-zero one.
cudaError_t read_device_error(int32_t *out, bool clear);
cudaError_t read_gemm_error(int32_t *out, bool clear);
cudaError_t read_cast_error(int32_t *out, bool clear);

// 2-D tiled tensor map (cuTensorMapEncodeTiled through the runtime's driver
// entry point).  Returns false if the driver rejects the arguments.
bool encode_tmap_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
                    uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swizzle);

}  // namespace fp8ds
