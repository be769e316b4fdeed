// Multi-tensor delayed-scaling update for sm_100a: every FP8 meta tensor of a
// model in ONE launch.
//
// What is computed (recipe DelayedScaling(amax_history_len=16,
// amax_compute_algo="max") in "CPU Overhead of te.Linear FP8 Layers"; the
// "FP8 scale update kernel" of "[PyTorch] Refactor FP8 workspaces in linear
// modules"; all linears' amax buffers handled together as in "support delayed
// scaling of weight in float8 all-gather"):
//   a = max over the history window (amax_compute_algo "max"), or the
//   current step's amax alone ("most_recent"); scale = fp8_max / a when a > 0,
//   a finite and the quotient finite, else the scale is kept; scale_inv = 1 / scale;
//   the history rolls by one slot (slot 0 moves to the end) and slot 0 is
//   cleared for the next step's amax.
//
// Layout: amax_history is [hist_len, T] slot-major, so thread t reads and
// writes column t and a warp touches 32 consecutive floats per slot
// (coalesced).  The work is a few tens of KB: the kernel is launch-latency
// bound, which is why all T tensors share one launch.
#include "fp8ds_internal.h"
#include "ptx_sm100.cuh"

namespace fp8ds {
namespace {

constexpr int U_THREADS = 128;

__global__ void __launch_bounds__(U_THREADS)
update_scales_kernel(int64_t T, int H, float *__restrict__ hist, float *__restrict__ scale,
                     float *__restrict__ scale_inv, const uint8_t *__restrict__ formats, int most_recent) {
    ptx::pdl_wait();
    ptx::pdl_launch_dependents();
    const int64_t t = static_cast<int64_t>(blockIdx.x) * U_THREADS + threadIdx.x;
    if (t >= T) return;
    const float first = hist[t];
    float a = first;
    if (!most_recent)
        for (int h = 1; h < H; ++h) a = fmaxf(a, hist[static_cast<int64_t>(h) * T + t]);
    const float fp8_max = formats[t] == FP8DS_E4M3 ? 448.0f : 57344.0f;
    float s = scale[t];
    if (a > 0.0f && isfinite(a)) {
        const float q = __fdiv_rn(fp8_max, a);
        if (isfinite(q)) s = q;
    }
    scale[t] = s;
    scale_inv[t] = __frcp_rn(s);
    for (int h = 0; h < H - 1; ++h)
        hist[static_cast<int64_t>(h) * T + t] = hist[static_cast<int64_t>(h + 1) * T + t];
    hist[static_cast<int64_t>(H - 1) * T + t] = first;
    hist[t] = 0.0f;
}

}  // namespace

cudaError_t launch_update_scales(int64_t num_tensors, int32_t hist_len, float *amax_history,
                                 float *scale, float *scale_inv, const uint8_t *formats,
                                 fp8ds_amax_algo algo, cudaStream_t stream) {
    if (num_tensors == 0) return cudaSuccess;
    const int64_t blocks = (num_tensors + U_THREADS - 1) / U_THREADS;
    return launch_pdl(update_scales_kernel, dim3(static_cast<unsigned>(blocks)), dim3(U_THREADS), 0, stream, 1,
                      num_tensors, static_cast<int>(hist_len), amax_history, scale, scale_inv, formats,
                      algo == FP8DS_AMAX_MOST_RECENT ? 1 : 0);
}

}  // namespace fp8ds
