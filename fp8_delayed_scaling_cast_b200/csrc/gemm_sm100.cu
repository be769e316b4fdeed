// Scaled FP8 GEMM for sm_100a on the 5th-generation tensor cores (tcgen05).
//
// What is computed (torch._scaled_mm as shown on "Accelerating PyTorch
// Training Workloads with FP8 -- Part 2"; HYBRID format of "CPU Overhead of
// te.Linear FP8 Layers": e4m3 x e4m3 forward, e5m2 x e4m3 gradients):
//   D[m,n] = (sum_k A[m,k] B[n,k]) * a_scale_inv * b_scale_inv (+ bias[n])
// with A [M,K] and B [N,K] FP8, both contraction-major ("TN"), fp32
// accumulation in tensor memory, fp32 or bf16 output.
//
// Kernel structure (one persistent CTA per SM, 6 warps):
//   warp 0      TMA producer: 128x128-byte A and 256x128-byte B tiles into a
//               4-stage shared-memory ring (128-byte swizzle), completion
//               signalled on per-stage mbarriers (transaction bytes);
//   warp 1      allocates 512 TMEM columns (two 128x256 fp32 accumulators) and
//               issues tcgen05.mma.kind::f8f6f4 (M=128, N=256, K=32) from one
//               thread; tcgen05.commit frees smem stages and publishes
//               finished accumulators;
//   warps 2..5  epilogue: tcgen05.ld of their 32 TMEM lanes, fp32 fma with the
//               combined scale_inv and bias, conversion, 128-byte-swizzled
//               staging in shared memory and TMA tensor stores.
// Two accumulators let the epilogue of tile i overlap the main loop of tile
// i+1.  No cluster multicast is used anywhere.
//
// Every wait is bounded (wall-clock limit read from %globaltimer).  A wait
// that gives up records FP8DS_ERR_TIMEOUT and its site in the device error
// word, raises a CTA-wide abort flag, and every role then drains what it has
// in flight (outstanding TMA loads, MMAs via a final commit, TMA stores)
// before TMEM is freed and the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "fp8ds_internal.h"

namespace fp8ds {

__device__ int32_t g_device_error = 0;

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes == FP8 elements per k-block (one 128-byte swizzle row)
constexpr int STAGES = 4;
constexpr int UMMA_K = 32;
constexpr int A_STAGE = BM * BK;
constexpr int B_STAGE = BN * BK;
constexpr int THREADS = 192;
constexpr int EPI_WARP0 = 2;
constexpr int TMEM_COLS = 512;
constexpr int EPI_BOX_BYTES = 32 * 128;  // 32 rows x 128 bytes
constexpr int EPI_BUFS = 2;
constexpr int SMEM_ALIGN = 1024;
constexpr int SMEM_BYTES = SMEM_ALIGN + STAGES * (A_STAGE + B_STAGE) + 4 * EPI_BUFS * EPI_BOX_BYTES + 256;
constexpr unsigned long long TIMEOUT_NS = 2000000000ull;  // 2 s
constexpr unsigned long long DRAIN_NS = 200000000ull;     // 0.2 s

enum Site : int32_t {
    SITE_PRODUCER_EMPTY = 1,
    SITE_MMA_FULL = 2,
    SITE_MMA_TMEM_EMPTY = 3,
    SITE_EPI_TMEM_FULL = 4,
};

// ------------------------------------------------------------ PTX helpers --

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t addr, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ void record_error(int32_t site) {
    atomicCAS(&g_device_error, 0, (site << 8) | FP8DS_ERR_TIMEOUT);
}

// Wait for the phase of `bar` with the given parity.  Gives up when another
// role raised the abort flag or after TIMEOUT_NS (then raises it itself).
__device__ __noinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                       int32_t site) {
    const uint32_t addr = smem_u32(bar);
    if (mbar_try_wait(addr, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait(addr, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > TIMEOUT_NS) {
            *abort_flag = 1;
            record_error(site);
            return false;
        }
    }
}

// Drain wait: ignores the abort flag, shorter limit, reports nothing.
__device__ __noinline__ void mbar_wait_drain(uint64_t *bar, uint32_t parity) {
    const uint32_t addr = smem_u32(bar);
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(addr, parity)) {
        if (globaltimer() - t0 > DRAIN_NS) return;
    }
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int32_t x,
                                             int32_t y) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(map),
                 "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void tma_store_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void tma_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void tma_store_wait_all() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with the
// 128-byte swizzle: rows of 128 bytes, 8-row groups 1024 bytes apart.
// Fields: start address >> 4 [0,14), leading byte offset >> 4 [16,30)
// (unused for swizzled K-major, 1 by convention), stride byte offset >> 4
// [32,46), descriptor version 1 [46,48), layout type 2 = 128-byte swizzle
// [61,64).  The tile base must be 1024-byte aligned (base offset 0).
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>(1u) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

__device__ __forceinline__ void umma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Bias value for column n (0 when absent or out of range).
__device__ __forceinline__ float bias_at(const void *bias, int bias_kind, int64_t n, int64_t N) {
    if (bias_kind == 0 || n >= N) return 0.0f;
    if (bias_kind == 1) return __ldg(static_cast<const float *>(bias) + n);
    const uint16_t b = __ldg(static_cast<const uint16_t *>(bias) + n);
    return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

struct Params {
    const float *a_scale_inv;
    const float *b_scale_inv;
    const void *bias;
    int bias_kind;  // 0 none, 1 fp32, 2 bf16
    int32_t M, N, K;
    int32_t tiles_m, tiles_n, num_kb;
    uint32_t idesc;
};

// OUT_BF16: bf16 output (64 columns per 128-byte staging row), else fp32 (32).
template <bool OUT_BF16>
__global__ void __launch_bounds__(THREADS, 1)
fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const __grid_constant__ CUtensorMap tmap_d, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + SMEM_ALIGN - 1) & ~static_cast<uintptr_t>(SMEM_ALIGN - 1));
    uint8_t *smem_a = smem;
    uint8_t *smem_b = smem_a + STAGES * A_STAGE;
    uint8_t *smem_epi = smem_b + STAGES * B_STAGE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem_epi + 4 * EPI_BUFS * EPI_BOX_BYTES);
    uint64_t *full_bar = bars;                   // [STAGES]
    uint64_t *empty_bar = bars + STAGES;         // [STAGES]
    uint64_t *tfull_bar = bars + 2 * STAGES;     // [2]
    uint64_t *tempty_bar = bars + 2 * STAGES + 2;  // [2]
    uint64_t *drain_bar = bars + 2 * STAGES + 4;   // [1]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int num_tiles = p.tiles_m * p.tiles_n;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_bar[s], 1);
            mbar_init(&empty_bar[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tfull_bar[b], 1);
            mbar_init(&tempty_bar[b], 4);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_d);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------ producer --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m_blk = tile % p.tiles_m;
                const int n_blk = tile / p.tiles_m;
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait(&empty_bar[stage], phase ^ 1u, abort_flag, SITE_PRODUCER_EMPTY)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&full_bar[stage], A_STAGE + B_STAGE);
                    tma_load_2d(&tmap_a, &full_bar[stage], smem_a + stage * A_STAGE, kb * BK, m_blk * BM);
                    tma_load_2d(&tmap_b, &full_bar[stage], smem_b + stage * B_STAGE, kb * BK, n_blk * BN);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let every load already issued land before the CTA can exit.
                for (int s = 0; s < STAGES; ++s) {
                    const int64_t n_s = issued > s ? (issued - s + STAGES - 1) / STAGES : 0;
                    if (n_s > 0) mbar_wait_drain(&full_bar[s], static_cast<uint32_t>((n_s - 1) & 1));
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ----------------------------------------------------- MMA issuer --
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
                const int acc = local & 1;
                const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
                if (!mbar_wait(&tempty_bar[acc], acc_phase ^ 1u, abort_flag, SITE_MMA_TMEM_EMPTY)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < p.num_kb; ++kb) {
                    if (!mbar_wait(&full_bar[stage], phase, abort_flag, SITE_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = sw128_kmajor_desc(smem_u32(smem_a + stage * A_STAGE));
                    const uint64_t b_desc = sw128_kmajor_desc(smem_u32(smem_b + stage * B_STAGE));
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        // advance the start address by k * 32 bytes inside the swizzle row
                        const uint64_t adv = static_cast<uint64_t>((k * UMMA_K) >> 4);
                        umma_f8f6f4(d_tmem, a_desc + adv, b_desc + adv, p.idesc, (kb > 0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&empty_bar[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit(&tfull_bar[acc]);
            }
            // Make sure every MMA issued has finished before TMEM can be freed.
            umma_commit(drain_bar);
            mbar_wait_drain(drain_bar, 0);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------- epilogue --
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const int row0 = q * 32;
        uint8_t *bufs = smem_epi + (warp - EPI_WARP0) * EPI_BUFS * EPI_BOX_BYTES;
        const float sab = __fmul_rn(__ldg(p.a_scale_inv), __ldg(p.b_scale_inv));
        constexpr int COLS_PER_BOX = OUT_BF16 ? 64 : 32;
        constexpr int BOXES = BN / COLS_PER_BOX;
        int local = 0;
        int buf = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
            const int m_blk = tile % p.tiles_m;
            const int n_blk = tile / p.tiles_m;
            const int acc = local & 1;
            const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
            if (!mbar_wait(&tfull_bar[acc], acc_phase, abort_flag, SITE_EPI_TMEM_FULL)) break;
            tc_fence_after();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(row0) << 16) + static_cast<uint32_t>(acc * BN);
            const int64_t n_base = static_cast<int64_t>(n_blk) * BN;
            for (int bx = 0; bx < BOXES; ++bx) {
                uint32_t packed[32];
                if (OUT_BF16) {
                    uint32_t r0[32], r1[32];
                    tmem_ld32(t_row + bx * 64, r0);
                    tmem_ld32(t_row + bx * 64 + 32, r1);
                    tmem_ld_wait();
                    if (bx == BOXES - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty_bar[acc]);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t n = n_base + bx * 64 + 2 * j;
                        const float v0 = fmaf(__uint_as_float(r0[2 * j]), sab, bias_at(p.bias, p.bias_kind, n, p.N));
                        const float v1 = fmaf(__uint_as_float(r0[2 * j + 1]), sab, bias_at(p.bias, p.bias_kind, n + 1, p.N));
                        __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
                        packed[j] = *reinterpret_cast<uint32_t *>(&h);
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int64_t n = n_base + bx * 64 + 32 + 2 * j;
                        const float v0 = fmaf(__uint_as_float(r1[2 * j]), sab, bias_at(p.bias, p.bias_kind, n, p.N));
                        const float v1 = fmaf(__uint_as_float(r1[2 * j + 1]), sab, bias_at(p.bias, p.bias_kind, n + 1, p.N));
                        __nv_bfloat162 h = __floats2bfloat162_rn(v0, v1);
                        packed[16 + j] = *reinterpret_cast<uint32_t *>(&h);
                    }
                } else {
                    uint32_t r0[32];
                    tmem_ld32(t_row + bx * 32, r0);
                    tmem_ld_wait();
                    if (bx == BOXES - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&tempty_bar[acc]);
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int64_t n = n_base + bx * 32 + j;
                        packed[j] = __float_as_uint(fmaf(__uint_as_float(r0[j]), sab, bias_at(p.bias, p.bias_kind, n, p.N)));
                    }
                }
                // Staging buffer reuse: the store issued from it two boxes ago
                // must have finished reading shared memory.
                if (lane == 0) tma_store_wait_read<EPI_BUFS - 1>();
                __syncwarp();
                uint8_t *box = bufs + buf * EPI_BOX_BYTES;
                // Row `lane`, 16-byte chunk c goes to chunk c ^ (lane & 7).
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const int pc = c ^ (lane & 7);
                    *reinterpret_cast<uint4 *>(box + lane * 128 + pc * 16) =
                        make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmap_d, box, static_cast<int32_t>(n_base + bx * COLS_PER_BOX),
                                 m_blk * BM + row0);
                    tma_store_commit();
                }
                buf ^= 1;
            }
        }
        if (lane == 0) tma_store_wait_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------- host --

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

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    EncodeTiledFn fn = encode_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {row_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Instruction descriptor of tcgen05.mma.kind::f8f6f4 (dense, K-major A and B):
// [4,6) D format (1 = fp32), [7,10) A format, [10,13) B format (0 = E4M3,
// 1 = E5M2), [15] / [16] A / B major (0 = K), [17,23) N >> 3, [24,29) M >> 4.
uint32_t make_idesc(fp8ds_format fa, fp8ds_format fb) {
    uint32_t d = 0;
    d |= 1u << 4;
    d |= static_cast<uint32_t>(fa == FP8DS_E5M2 ? 1 : 0) << 7;
    d |= static_cast<uint32_t>(fb == FP8DS_E5M2 ? 1 : 0) << 10;
    d |= static_cast<uint32_t>(BN >> 3) << 17;
    d |= static_cast<uint32_t>(BM >> 4) << 24;
    return d;
}

template <bool OUT_BF16>
cudaError_t configure_once() {
    static bool done[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev]) return cudaSuccess;
    e = cudaFuncSetAttribute(fp8_gemm_kernel<OUT_BF16>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev] = true;
    return e;
}

}  // namespace

fp8ds_status launch_gemm(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv, const uint8_t *b,
                         fp8ds_format b_fmt, const float *b_scale_inv, const void *bias, fp8ds_dtype bias_dtype,
                         void *d, fp8ds_dtype d_dtype, int64_t m, int64_t n, int64_t k, cudaStream_t stream) {
    CUtensorMap ta, tb, td;
    const bool out_bf16 = d_dtype == FP8DS_BF16;
    bool ok = encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, k, m, k, BK, BM) &&
              encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, k, n, k, BK, BN) &&
              (out_bf16 ? encode_2d(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d, n, m, n * 2, 64, 32)
                        : encode_2d(&td, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d, n, m, n * 4, 32, 32));
    if (!ok) {
        set_error("fp8_gemm: cuTensorMapEncodeTiled failed (m=%lld n=%lld k=%lld)", (long long)m, (long long)n,
                  (long long)k);
        return FP8DS_ERR_CUDA;
    }
    Params p;
    p.a_scale_inv = a_scale_inv;
    p.b_scale_inv = b_scale_inv;
    p.bias = bias;
    p.bias_kind = bias == nullptr ? 0 : (bias_dtype == FP8DS_F32 ? 1 : 2);
    p.M = static_cast<int32_t>(m);
    p.N = static_cast<int32_t>(n);
    p.K = static_cast<int32_t>(k);
    p.tiles_m = static_cast<int32_t>((m + BM - 1) / BM);
    p.tiles_n = static_cast<int32_t>((n + BN - 1) / BN);
    p.num_kb = static_cast<int32_t>((k + BK - 1) / BK);
    p.idesc = make_idesc(a_fmt, b_fmt);
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    cudaError_t e = out_bf16 ? configure_once<true>() : configure_once<false>();
    if (e == cudaSuccess) {
        if (out_bf16)
            fp8_gemm_kernel<true><<<grid, THREADS, SMEM_BYTES, stream>>>(ta, tb, td, p);
        else
            fp8_gemm_kernel<false><<<grid, THREADS, SMEM_BYTES, stream>>>(ta, tb, td, p);
        e = cudaGetLastError();
    }
    if (e != cudaSuccess) {
        set_error("fp8_gemm: launch failed: %s", cudaGetErrorString(e));
        return FP8DS_ERR_CUDA;
    }
    return FP8DS_OK;
}

cudaError_t read_device_error(int32_t *out, bool clear) {
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return e;
    e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(int32_t));
    if (e != cudaSuccess || !clear) return e;
    const int32_t zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int32_t));
}

}  // namespace fp8ds
