// Scaled FP8 GEMM for sm_100a on the 5th-generation tensor cores (tcgen05).
//
// What is computed (torch._scaled_mm as shown on "Accelerating PyTorch
// Training Workloads with FP8 -- Part 2"; HYBRID format of "CPU Overhead of
// te.Linear FP8 Layers": e4m3 x e4m3 forward, e5m2 x e4m3 gradients):
//   D[m,n] = (sum_k A[m,k] B[n,k]) * a_scale_inv * b_scale_inv (+ bias[n])
// with A [M,K] and B [N,K] FP8, both contraction-major ("TN"), fp32
// accumulation in tensor memory, fp32 or bf16 output.
//
// Two persistent warp-specialised kernels share one structure (10 warps):
//   warp 0      TMA producer: A and B tiles (128-byte rows, 128-byte swizzle)
//               into a shared-memory ring, completion on per-stage mbarriers
//               (transaction bytes);
//   warp 1      allocates 512 TMEM columns (two fp32 accumulators of 256
//               columns) and issues tcgen05.mma.kind::f8f6f4 from one thread;
//               tcgen05.commit frees ring stages and publishes accumulators;
//   warps 2..9  epilogue: each reads 32 TMEM lanes (its lane quarter) of half
//               of the accumulator columns with tcgen05.ld, fp32 fma with the
//               combined scale_inv and the tile's bias (staged once in shared
//               memory), conversion, 128-byte-swizzled staging in shared memory
//               and TMA tensor stores.
// Two accumulators let the epilogue of tile i overlap the main loop of i+1.
//
//   fp8_gemm_1sm_kernel  one CTA per SM, tile 128 x 256, 4 stages of 48 KB
//                        (used when M <= 128).
//   fp8_gemm_2sm_kernel  CTA pairs (cluster of 2), tcgen05.mma.cta_group::2
//                        with a 256 x 256 tile: each CTA loads its 128 rows of
//                        A and its 128 rows of B (32 KB per stage, 6 stages),
//                        the pair's MMA reads both CTAs' shared memory and
//                        leaves rows 0-127 of D in CTA 0's TMEM and rows
//                        128-255 in CTA 1's.  Per SM this halves the B bytes
//                        moved per FLOP.  Both CTAs' loads signal CTA 0's
//                        ring barriers; CTA 0's commits arrive on both CTAs'
//                        barriers; both epilogues report to CTA 0.
// The pair kernel has a second tile mode for long contractions (K >= 4096):
// a 512 x 256 pair tile (each CTA loads two 128-row boxes of A per stage)
// that fills all 512 TMEM columns with one accumulator set.
// Tiles are visited in groups of 8 row-tiles (column index slowest within a
// group) so that concurrently running CTAs share A and B in L2.  With a
// workspace (fp8_gemm_ex, fp8_gemm_noalloc) a ragged last wave is replaced by
// a stream-K split of (tile, k-block) units; partial sums of a split tile go
// through the workspace.  No TMA load uses cluster multicast.
//
// Every wait is bounded (wall-clock limit read from %globaltimer).  A wait
// that gives up records FP8DS_ERR_TIMEOUT and its site in the device error
// word, raises a CTA-wide abort flag, and every role then drains what it has
// in flight (outstanding TMA loads, MMAs via a final commit, TMA stores)
// before TMEM is freed and the CTA exits.
#include <cuda.h>
#include <cuda_bf16.h>

#include <atomic>
#include <mutex>

#include "fp8ds_internal.h"

namespace fp8ds {

__device__ int32_t g_device_error = 0;

namespace {

constexpr int BK = 128;        // bytes == FP8 elements per k-block (one 128-byte swizzle row)
constexpr int UMMA_K = 32;     // K of one kind::f8f6f4 MMA
constexpr int ACC_N = 256;     // accumulator columns (tile N)
constexpr int EPI_WARPS = 8;               // two per TMEM lane quarter
constexpr int THREADS = 64 + 32 * EPI_WARPS; // producer warp, MMA warp, epilogue warps
constexpr int EPI_WARP0 = 2;
constexpr int TMEM_COLS = 512; // two accumulators
// Epilogue shape (compile-time settings): TMEM columns per tcgen05.ld (32 or
// 64) and staging boxes per epilogue warp (1, or 2 so that a box is filled
// while the previous one's TMA store still reads shared memory; the second
// box takes the shared memory of one ring stage).
#ifndef FP8DS_EPI_LD
#define FP8DS_EPI_LD 32
#endif
#ifndef FP8DS_EPI_BOXES
#define FP8DS_EPI_BOXES 1
#endif
// FP8DS_EPI_EARLY: whole-tile bf16 and FP8 epilogues read the accumulator
// into registers and release TMEM before they stage and store D.
#ifndef FP8DS_EPI_EARLY
#define FP8DS_EPI_EARLY 1
#endif
constexpr bool EPI_EARLY = FP8DS_EPI_EARLY != 0;
constexpr int EPI_LD = FP8DS_EPI_LD;
constexpr int EPI_NBOX = FP8DS_EPI_BOXES;
static_assert(EPI_LD == 32 || EPI_LD == 64, "TMEM load width must be 32 or 64 columns");
static_assert(EPI_NBOX == 1 || EPI_NBOX == 2, "one or two staging boxes per epilogue warp");
constexpr int EPI_BOX_BYTES = 32 * 128;  // staging box: 32 rows x 128 bytes
constexpr int EPI_BYTES = EPI_WARPS * EPI_NBOX * EPI_BOX_BYTES + 256 * 4;  // + the tile's bias (fp32 x 256)
constexpr int EPI_THREADS = 32 * EPI_WARPS;
constexpr int SMEM_ALIGN = 1024;
constexpr int GROUP_M = 8;
// Smallest K for which the pair kernel may take the 512-row tile (compile-
// time setting).  On B200 the 512-row tile measured 3-4% faster than the
// 256-row one at 8192 x 8192 x 2048 and at K = 8192, as long as its last
// wave is no emptier (checked at launch).
#ifndef FP8DS_MSUB2_MIN_K
#define FP8DS_MSUB2_MIN_K 2048
#endif
// Output kinds of the epilogue.
constexpr int OUT_F32 = 0;
constexpr int OUT_BF16 = 1;
constexpr int OUT_FP8 = 2;   // bf16-rounded D cast to FP8 with a delayed scale (+ transpose, amax)
constexpr unsigned long long TIMEOUT_NS = 2000000000ull;  // 2 s
constexpr unsigned long long DRAIN_NS = 200000000ull;     // 0.2 s

// 1-SM kernel: tile 128 x 256, 4 stages of 16 KB (A) + 32 KB (B).
constexpr int S1_BM = 128;
constexpr int S1_STAGES = 4 - (EPI_NBOX - 1);
constexpr int S1_A_STAGE = S1_BM * BK;
constexpr int S1_B_STAGE = ACC_N * BK;
constexpr int S1_SMEM = SMEM_ALIGN + S1_STAGES * (S1_A_STAGE + S1_B_STAGE) + EPI_BYTES + 256;

// 2-SM kernel: pair tile (M_SUB x 256) x 256.  Per CTA and stage: M_SUB
// boxes of 128 rows of A and 128 rows of B.  M_SUB = 1: 6 stages of 32 KB,
// two accumulators (double-buffered).  M_SUB = 2: 4 stages of 48 KB, the two
// M halves fill all 512 TMEM columns (one accumulator set) in exchange for
// 25% fewer loaded bytes per FLOP; the halves are released to the next tile
// one at a time, so only the epilogue's first half is not overlapped.
constexpr int S2_BM = 128;           // rows of A (and of D) per CTA and M half
constexpr int S2_BN_HALF = 128;      // rows of B per CTA
constexpr int S2_B_STAGE = S2_BN_HALF * BK;
template <int M_SUB>
struct Pair {
    static constexpr int STAGES = (M_SUB == 1 ? 6 : 4) - (EPI_NBOX - 1);
    static constexpr int A_STAGE = M_SUB * S2_BM * BK;
    static constexpr int ACC_BUFS = M_SUB == 1 ? 2 : 1;
    static constexpr int SMEM = SMEM_ALIGN + STAGES * (A_STAGE + S2_B_STAGE) + EPI_BYTES + 256;
};

static_assert(S1_SMEM <= 232448 && Pair<1>::SMEM <= 232448 && Pair<2>::SMEM <= 232448,
              "shared memory per CTA exceeds 227 KB");

enum Site : int32_t {
    SITE_PRODUCER_EMPTY = 1,
    SITE_MMA_FULL = 2,
    SITE_MMA_TMEM_EMPTY = 3,
    SITE_EPI_TMEM_FULL = 4,
    SITE_EPI_PARTIAL = 5,
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

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t cta_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(cta_addr), "r"(rank));
    return r;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

// Arrive on a barrier given by its shared::cluster address (own CTA or peer).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
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

// The same test, letting the thread sleep until the phase completes or up to
// `hint_ns` have passed (the suspend-time hint of mbarrier.try_wait), so that
// a warp that waits a whole main loop issues almost nothing meanwhile.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t addr, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(addr), "r"(parity), "r"(hint_ns)
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
        // up to 32 x 20 us between looks at the abort flag and the clock
#pragma unroll 1
        for (int i = 0; i < 32; ++i)
            if (mbar_try_wait_sleep(addr, parity, 20000u)) return true;
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

// TMA tile load into this CTA's shared memory, completion on a barrier of
// this CTA.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap *map, uint64_t *bar, void *dst,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// TMA tile load into this CTA's shared memory whose completion is signalled
// on a barrier of the pair's first CTA (bar_cluster_addr, shared::cluster).
__device__ __forceinline__ void tma_load_2d_pair(const CUtensorMap *map, uint32_t bar_cluster_addr, void *dst,
                                                 int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster_addr), "r"(x), "r"(y)
        : "memory");
}

// The same load with an L2 cache-policy hint (createpolicy), for the operand
// that later waves of the launch read again.
__device__ __forceinline__ void tma_load_2d_pair_hint(const CUtensorMap *map, uint32_t bar_cluster_addr, void *dst,
                                                      int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.cta_group::2.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(dst)),
        "l"(map), "r"(bar_cluster_addr), "r"(x), "r"(y), "l"(policy)
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

// MN-major operand tile with the 128-byte swizzle (8-bit elements): each
// K row holds 128 consecutive M (or N) elements, 8 K rows form one 1 KB
// swizzle atom, atoms follow each other along K (SBO = 1 KB), and a second
// group of 128 M (N) elements sits LBO bytes further (the one-CTA kernel's
// 256-column B tile: two TMA boxes 16 KB apart).  The same fields as the
// K-major descriptor otherwise (version 1, layout SWIZZLE_128B).
__device__ __forceinline__ uint64_t sw128_mnmajor_desc(uint32_t smem_addr, uint32_t lbo_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((smem_addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>(1024u >> 4) << 32;
    d |= static_cast<uint64_t>(1u) << 46;
    d |= static_cast<uint64_t>(2u) << 61;
    return d;
}

// Descriptor of a 128 x BK operand tile and its advance (in 16-byte units)
// per K step of UMMA_K elements: 32 bytes along the swizzled row (K-major)
// or 32 rows of 128 bytes (MN-major).
__device__ __forceinline__ uint64_t operand_desc(uint32_t smem_addr, bool mn_major, uint32_t lbo_bytes) {
    return mn_major ? sw128_mnmajor_desc(smem_addr, lbo_bytes) : sw128_kmajor_desc(smem_addr);
}
__device__ __forceinline__ uint64_t operand_kstep(int k, bool mn_major) {
    return static_cast<uint64_t>(mn_major ? (k * UMMA_K * 128) >> 4 : (k * UMMA_K) >> 4);
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

__device__ __forceinline__ void umma_f8f6f4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                 uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// Commit of the pair's MMAs, arriving on the barrier at this offset in every
// CTA of `cta_mask`.
__device__ __forceinline__ void umma_commit_pair_to(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

__device__ __forceinline__ void umma_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
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

__device__ __forceinline__ __attribute__((unused)) void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,"
        "%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,"
        "%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
          "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
          "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
          "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
          "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
        : "r"(taddr));
}

// tcgen05.ld of N = 32 or 64 columns (32 lanes x 32 bits each) into r.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t (&r)[N]) {
    static_assert(N == 32 || N == 64, "TMEM load width");
    if constexpr (N == 32)
        tmem_ld32(taddr, r);
    else
        tmem_ld64(taddr, r);
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

struct Params {
    const float *a_scale_inv;
    const float *b_scale_inv;
    const void *bias;
    int bias_kind;  // 0 none, 1 fp32, 2 bf16
    int32_t M, N, K;
    int32_t tiles_m, tiles_n, num_kb;
    int32_t group_m;      // row tiles per raster group (tile_coords)
    int32_t l2_keep;      // operand loaded with an L2 evict_last hint: 0 none, 1 A, 2 B
    uint32_t idesc;
    int32_t a_mn, b_mn;   // 1: the operand is stored MN-major ([K, M] / [K, N] row-major)
    // stream-K (pair kernel only): 0 = whole tiles per cluster
    int32_t stream_k;
    int32_t sk_pairs;     // clusters the workspace has partial slots for
    uint32_t epoch;       // non-zero per launch; partials are published with it
    int32_t *flags;       // [clusters][2] publication words
    float *partials;      // [clusters][2 CTAs][2 row blocks][128 x 256] fp32
    // OUT_FP8: codes = cast(fl32(bf16(D) * out_scale)), amax of bf16(D)
    const float *out_scale;
    float *out_amax;       // NULL or atomic-max target
    float *out_scale_inv;  // NULL or fl32(1 / out_scale)
    uint8_t *out_d8;       // [M, N] codes
    // limit of the wait for another pair's partial sum, and (tests of the
    // error path only) whether split tiles withhold their publication
    unsigned long long partial_wait_ns;
    int32_t withhold_partials;
    uint8_t *out_d8t;      // [N, M] codes or NULL
    int32_t out_fmt;
};

// Workspace of the stream-K schedule: publication words, then one partial
// accumulator slot per cluster (a pair's two CTAs, up to two row blocks each).
constexpr size_t WS_FLAG_BYTES = 4096;  // room for 1024 clusters
constexpr size_t WS_SLOT_FLOATS = 2 * 2 * 128 * 256;

// Work assignment of a cluster (or CTA).  Whole tiles c, c + C, ... (C
// clusters).  With stream-K, only the tiles of the whole waves go that way
// (the first floor(T / C) * C of the T tiles); the U = R * num_kb (tile,
// k-block) units of the R remaining tiles are shared out afterwards, cluster
// c taking the units [c*U/C, (c+1)*U/C) in tile order as segments (tile,
// kb0, kb1).  A split tile's segments belong to consecutive clusters, the
// one with kb0 = 0 (the last segment of its cluster's range) storing D.
struct Sched {
    int64_t u, u1;
    int t, stride, dp_tiles, num_kb;
    __device__ __forceinline__ Sched(const Params &p, int c, int C) {
        const int num_tiles = p.tiles_m * p.tiles_n;
        num_kb = p.num_kb;
        dp_tiles = p.stream_k != 0 ? (num_tiles / C) * C : num_tiles;
        const int64_t base = static_cast<int64_t>(dp_tiles) * num_kb;
        const int64_t U = static_cast<int64_t>(num_tiles - dp_tiles) * num_kb;
        u = base + U * c / C;
        u1 = base + U * (c + 1) / C;
        t = c;
        stride = C;
    }
    __device__ __forceinline__ bool next(int &tile, int &kb0, int &kb1) {
        if (t < dp_tiles) {
            tile = t;
            kb0 = 0;
            kb1 = num_kb;
            t += stride;
            return true;
        }
        if (u >= u1) return false;
        tile = static_cast<int>(u / num_kb);
        kb0 = static_cast<int>(u % num_kb);
        const int64_t left = u1 - u;
        kb1 = left < num_kb - kb0 ? kb0 + static_cast<int>(left) : num_kb;
        u += kb1 - kb0;
        return true;
    }
};

// Named barrier among the 4 epilogue warps.
__device__ __forceinline__ void epilogue_bar() { asm volatile("bar.sync 1, %0;" ::"n"(EPI_THREADS) : "memory"); }

// Named barrier among the 4 epilogue warps that also returns whether any of
// their threads passed `v` true (so that all of them leave the loop together).
__device__ __forceinline__ bool epilogue_any(bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, 1, %2, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}\n"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(v)), "n"(EPI_THREADS)
        : "memory");
    return r != 0;
}

// The tile's bias, bias[n_base .. n_base+255] (0 when absent or past N), as
// fp32: load_bias reads this thread's values from global memory (issued
// before the epilogue waits for the accumulator, so the load overlaps the
// wait), stage_bias stores them in shared memory once every epilogue warp is
// done with the previous tile's copy.
constexpr int BIAS_PER_THREAD = ACC_N / EPI_THREADS;
__device__ __forceinline__ void load_bias(float (&v)[BIAS_PER_THREAD], const Params &p, int64_t n_base,
                                          int epi_tid) {
#pragma unroll
    for (int i = 0; i < BIAS_PER_THREAD; ++i) {
        const int64_t n = n_base + epi_tid + i * EPI_THREADS;
        v[i] = 0.0f;
        if (p.bias_kind != 0 && n < p.N) {
            if (p.bias_kind == 1) {
                v[i] = __ldg(static_cast<const float *>(p.bias) + n);
            } else {
                const uint16_t b = __ldg(static_cast<const uint16_t *>(p.bias) + n);
                v[i] = __uint_as_float(static_cast<uint32_t>(b) << 16);
            }
        }
    }
}
__device__ __forceinline__ void stage_bias(float *bias_s, const float (&v)[BIAS_PER_THREAD], int epi_tid) {
#pragma unroll
    for (int i = 0; i < BIAS_PER_THREAD; ++i) bias_s[epi_tid + i * EPI_THREADS] = v[i];
}

// Tile order: groups of `group` row-tiles; inside a group the row index runs
// fastest, so CTAs that run together share B columns and a band of A rows
// (group 1: whole rows of tiles, the column index running fastest).
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int group, int &m_blk,
                                            int &n_blk) {
    const int group_size = group * tiles_n;
    const int first_m = (tile / group_size) * group;
    const int rows = min(tiles_m - first_m, group);
    const int in_group = tile % group_size;
    m_blk = first_m + in_group % rows;
    n_blk = in_group / rows;
}

// Epilogue of one accumulator for one warp: 32 rows (this warp's TMEM lane
// quarter) x 256 columns.  t_row addresses the warp's lanes at the
// accumulator's first column; m_row0 is the global row of the warp's first
// row.  After the last TMEM read the warp arrives (lane 0) on the
// accumulator-empty barrier given by its shared::cluster address.
// Partial accumulators of a stream-K split tile, lane-major so that a warp's
// access of 4 consecutive columns of its 32 rows is 512 contiguous bytes:
// element (row block h, lane quarter q, column c, lane l) at
// (((h * 4 + q) * 64 + c / 4) * 32 + l) * 4 + c % 4.
__device__ __forceinline__ float4 *partial_at(float *slot, int h, int q, int col, int lane) {
    return reinterpret_cast<float4 *>(slot) + ((h * 4 + q) * 64 + col / 4) * 32 + lane;
}

// Add the partial of the next cluster (mode bit 2, from `in`), then store
// the sum as this segment's partial (mode bit 1, to `out`), for 32 columns.
constexpr int PART_OUT = 1;
constexpr int PART_IN = 2;
__device__ __forceinline__ void partial_io(int mode, uint32_t *r, const float *in, float *out, int h, int q,
                                           int col0, int lane) {
    if (mode & PART_IN) {
        float4 v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) v[i] = __ldcg(partial_at(const_cast<float *>(in), h, q, col0 + 4 * i, lane));
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            r[4 * i] = __float_as_uint(__uint_as_float(r[4 * i]) + v[i].x);
            r[4 * i + 1] = __float_as_uint(__uint_as_float(r[4 * i + 1]) + v[i].y);
            r[4 * i + 2] = __float_as_uint(__uint_as_float(r[4 * i + 2]) + v[i].z);
            r[4 * i + 3] = __float_as_uint(__uint_as_float(r[4 * i + 3]) + v[i].w);
        }
    }
    if (mode & PART_OUT) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            *partial_at(out, h, q, col0 + 4 * i, lane) =
                make_float4(__uint_as_float(r[4 * i]), __uint_as_float(r[4 * i + 1]), __uint_as_float(r[4 * i + 2]),
                            __uint_as_float(r[4 * i + 3]));
    }
}

// Packed pairs of fp32 (sm_100 f32x2 arithmetic; each lane rounds exactly as
// the scalar fmaf / __fmul_rn).
__device__ __forceinline__ uint64_t pack_f32x2(float lo, float hi) {
    return static_cast<uint64_t>(__float_as_uint(lo)) | (static_cast<uint64_t>(__float_as_uint(hi)) << 32);
}
__device__ __forceinline__ float lo_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v)); }
__device__ __forceinline__ float hi_f32(uint64_t v) { return __uint_as_float(static_cast<uint32_t>(v >> 32)); }
__device__ __forceinline__ uint64_t fma_f32x2(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t mul_f32x2(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// D = acc * sab + bias for two adjacent columns (the raw TMEM words r0, r1).
__device__ __forceinline__ uint64_t scale_bias2(uint32_t r0, uint32_t r1, uint64_t sab2, float b0, float b1) {
    return fma_f32x2(pack_f32x2(__uint_as_float(r0), __uint_as_float(r1)), sab2, pack_f32x2(b0, b1));
}

// Four bias values from the tile's shared-memory copy.  BIAS false: the bias
// is absent and its (zero) copy is not read; the arithmetic is the same fma
// with +0.
template <bool BIAS>
__device__ __forceinline__ float4 bias4(const float *bs) {
    return BIAS ? *reinterpret_cast<const float4 *>(bs) : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
}

// Stream-K modes (bits): 1 = the segment does not end the tile's k-range at
// its start (kb0 > 0), so it stores its raw partial sum for the tile's owner
// instead of D; 2 = the tile's k-range goes on after the segment (kb1 <
// num_kb), so it first adds the partial of the cluster that holds the rest.
// Mode 0 converts and stores D.
// The warp reads its 128 columns as four 32-column TMEM loads (which keeps
// the live registers within the 168 that 10 warps per SM allow).  The load
// of chunk c + 1 is issued as soon as chunk c has been converted, into the
// same registers, so its latency overlaps chunk c's staging and store; the
// loop is fully unrolled so that every load has its own registers.
template <bool OUT_BF16, bool BIAS>
__device__ __forceinline__ void epilogue_tile(uint32_t t_row, int lane, uint8_t *boxes, int &nbox, int half,
                                              const CUtensorMap *tmap_d, int64_t n_base, int32_t m_row0,
                                              float sab, const float *bias_s, uint32_t empty_bar_cluster,
                                              bool arrive, int mode, const float *p_in, float *p_out, int h,
                                              int q) {
    constexpr int SUBS_PER_BOX = OUT_BF16 ? 2 : 1;  // 32-column sub-blocks per staging box
    constexpr int CHUNKS = ACC_N / 2 / EPI_LD;      // TMEM loads per warp and row block
    constexpr int SUBS = EPI_LD / 32;               // 32-column sub-blocks per load
    const uint64_t sab2 = pack_f32x2(sab, sab);
    uint32_t r[EPI_LD];
    tmem_ld(t_row + half * (ACC_N / 2), r);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
        if (arrive && c == CHUNKS - 1) {
            // every TMEM load of this accumulator has completed
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_bar_cluster);
        }
#pragma unroll
        for (int sb = 0; sb < SUBS; ++sb) {
            uint32_t *rr = r + 32 * sb;
            const int col0 = half * (ACC_N / 2) + (c * SUBS + sb) * 32;  // accumulator column
            const int hh = (col0 / 32) % SUBS_PER_BOX;
            const bool last_of_chunk = sb == SUBS - 1;
            if (mode != 0) partial_io(mode, rr, p_in, p_out, h, q, col0, lane);
            if (!(mode & PART_OUT)) {
                uint8_t *box = boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES;
                if (hh == 0) {
                    // Staging buffer reuse: the store issued from this box
                    // EPI_NBOX stores ago must have finished reading it.
                    if (lane == 0) tma_store_wait_read<EPI_NBOX - 1>();
                    __syncwarp();
                }
                const float *bs = bias_s + col0;
                // 32 columns -> 128 bytes (fp32) or 64 bytes (bf16) of row `lane`;
                // 16-byte chunk k of the row goes to chunk k ^ (lane & 7) (the
                // 128-byte swizzle the output tensor map expects).
                if (OUT_BF16) {
                    uint32_t packed[16];
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const float4 b = bias4<BIAS>(bs + 4 * j);
                        const uint64_t v01 = scale_bias2(rr[4 * j], rr[4 * j + 1], sab2, b.x, b.y);
                        const uint64_t v23 = scale_bias2(rr[4 * j + 2], rr[4 * j + 3], sab2, b.z, b.w);
                        __nv_bfloat162 ha = __floats2bfloat162_rn(lo_f32(v01), hi_f32(v01));
                        __nv_bfloat162 hb = __floats2bfloat162_rn(lo_f32(v23), hi_f32(v23));
                        packed[2 * j] = *reinterpret_cast<uint32_t *>(&ha);
                        packed[2 * j + 1] = *reinterpret_cast<uint32_t *>(&hb);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int pc = (hh * 4 + k) ^ (lane & 7);
                        *reinterpret_cast<uint4 *>(box + lane * 128 + pc * 16) =
                            make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
                    }
                } else {
#pragma unroll
                    for (int k = 0; k < 8; ++k) {
                        const int pc = k ^ (lane & 7);
                        const float4 b = bias4<BIAS>(bs + 4 * k);
                        const uint64_t v01 = scale_bias2(rr[4 * k], rr[4 * k + 1], sab2, b.x, b.y);
                        const uint64_t v23 = scale_bias2(rr[4 * k + 2], rr[4 * k + 3], sab2, b.z, b.w);
                        *reinterpret_cast<uint4 *>(box + lane * 128 + pc * 16) =
                            make_uint4(static_cast<uint32_t>(v01), static_cast<uint32_t>(v01 >> 32),
                                       static_cast<uint32_t>(v23), static_cast<uint32_t>(v23 >> 32));
                    }
                }
            }
            // the registers of r are free: start the next chunk's TMEM load
            if (last_of_chunk && c + 1 < CHUNKS) tmem_ld(t_row + half * (ACC_N / 2) + (c + 1) * EPI_LD, r);
            if (!(mode & PART_OUT) && hh == SUBS_PER_BOX - 1) {
                uint8_t *box = boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES;
                fence_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(tmap_d, box, static_cast<int32_t>(n_base + (col0 / (32 * SUBS_PER_BOX)) *
                                                                               (32 * SUBS_PER_BOX)),
                                 m_row0);
                    tma_store_commit();
                }
                ++nbox;
            }
        }
        if (c + 1 < CHUNKS) tmem_ld_wait();
    }
}

// Two FP8 codes (saturating, round to nearest even) packed in 16 bits:
// byte 0 = code(lo), byte 1 = code(hi); NaN becomes 0x7F.
__device__ __forceinline__ uint32_t cvt_fp8x2(float lo, float hi, int fmt) {
    uint16_t r;
    if (fmt == FP8DS_E4M3)
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    else
        asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// FP8-output epilogue of one accumulator for one warp: 32 rows (its TMEM
// lane quarter) x this warp's 128 columns, in chunks of 32 columns.  Each
// value is first rounded to bf16 exactly as the bf16 output would be, then
// cast like fp8_cast_transpose_amax: code = cvt(fl32(h * s_out)), amax over
// |h|.  Lane r holds row r's 32 codes of a chunk and stores them straight to
// global memory (32 contiguous bytes, whole sectors).  For the transpose it
// also writes them into a shared 32 x 32-byte tile whose rows are 48 bytes
// apart (so that both these 16-byte row writes and the byte gathers below are
// free of bank conflicts); lane c then gathers column c (one byte per row)
// and stores it as 32 contiguous bytes of row n0 + c of the transpose.  Two
// tiles per warp alternate between chunks, so one __syncwarp per chunk
// orders the writes and the gathers.  N and M are multiples of 16, so a
// chunk's row (column) segment is whole, half or wholly outside.
constexpr int FP8_TSTRIDE = 48;
constexpr int FP8_TILE_BYTES = 32 * FP8_TSTRIDE;
static_assert(2 * FP8_TILE_BYTES <= EPI_BOX_BYTES, "transpose tiles exceed the warp's staging box");

__device__ __forceinline__ void store_segment(uint8_t *dst, int64_t left, const uint32_t (&w)[8]) {
    if (left >= 32) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4 *>(dst + 16) = make_uint4(w[4], w[5], w[6], w[7]);
    } else if (left >= 16) {
        *reinterpret_cast<uint4 *>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
    }
}

template <bool BIAS>
__device__ __forceinline__ void epilogue_tile_fp8(uint32_t t_row, int lane, uint8_t *boxes, int &nbox, int half,
                                                  uint8_t *d8, uint8_t *d8t, const CUtensorMap *tmap_d,
                                                  int64_t n_base, int32_t m_row0, float sab,
                                                  const float *bias_s, uint32_t empty_bar_cluster, bool arrive,
                                                  int mode, const float *p_in, float *p_out, int h, int q,
                                                  float s_out, int fmt,
                                                  int32_t m_total, int32_t n_total, float &amax) {
    constexpr int CHUNKS = ACC_N / 2 / EPI_LD;  // TMEM loads per warp and row block
    constexpr int SUBS = EPI_LD / 32;           // 32-column sub-blocks per load
    const int32_t m = m_row0 + lane;
    // Without the transpose the warp's 32 rows x 128 code bytes are one
    // 128-byte-swizzled staging box and one TMA store; with it, the codes go
    // out with plain stores beside the transposed ones (in box 0's memory).
    const bool staged = d8t == nullptr;
    uint8_t *box = staged ? boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES : boxes;
    if (staged && !(mode & PART_OUT)) {
        if (lane == 0) tma_store_wait_read<EPI_NBOX - 1>();
        __syncwarp();
    }
    const uint64_t sab2 = pack_f32x2(sab, sab);
    const uint64_t s2 = pack_f32x2(s_out, s_out);
    uint32_t r[EPI_LD];
    tmem_ld(t_row + half * (ACC_N / 2), r);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < CHUNKS; ++c) {
        if (arrive && c == CHUNKS - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_bar_cluster);
        }
#pragma unroll
        for (int sb = 0; sb < SUBS; ++sb) {
            uint32_t *rr = r + 32 * sb;
            const int cs = c * SUBS + sb;              // sub-block within the warp's 128 columns
            const int col0 = half * (ACC_N / 2) + cs * 32;
            if (mode != 0) partial_io(mode, rr, p_in, p_out, h, q, col0, lane);
            uint32_t w[8];
            if (!(mode & PART_OUT)) {
                const float *bs = bias_s + col0;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const float4 b = bias4<BIAS>(bs + 4 * j);
                    const uint64_t v01 = fma_f32x2(
                        pack_f32x2(__uint_as_float(rr[4 * j]), __uint_as_float(rr[4 * j + 1])), sab2,
                        pack_f32x2(b.x, b.y));
                    const uint64_t v23 = fma_f32x2(
                        pack_f32x2(__uint_as_float(rr[4 * j + 2]), __uint_as_float(rr[4 * j + 3])), sab2,
                        pack_f32x2(b.z, b.w));
                    const __nv_bfloat162 ha = __floats2bfloat162_rn(lo_f32(v01), hi_f32(v01));
                    const __nv_bfloat162 hb = __floats2bfloat162_rn(lo_f32(v23), hi_f32(v23));
                    const float h0 = __low2float(ha), h1 = __high2float(ha);
                    const float h2 = __low2float(hb), h3 = __high2float(hb);
                    if (m < m_total)  // rows past M (tile padding) count for no amax
                        amax = fmaxf(amax, fmaxf(fmaxf(fabsf(h0), fabsf(h1)), fmaxf(fabsf(h2), fabsf(h3))));
                    const uint64_t p01 = mul_f32x2(pack_f32x2(h0, h1), s2);
                    const uint64_t p23 = mul_f32x2(pack_f32x2(h2, h3), s2);
                    w[j] = cvt_fp8x2(lo_f32(p01), hi_f32(p01), fmt) |
                           (cvt_fp8x2(lo_f32(p23), hi_f32(p23), fmt) << 16);
                }
            }
            // the registers of r are free: start the next chunk's TMEM load
            if (sb == SUBS - 1 && c + 1 < CHUNKS) tmem_ld(t_row + half * (ACC_N / 2) + (c + 1) * EPI_LD, r);
            if (!(mode & PART_OUT) && staged) {
                // 16-byte chunk k of row `lane` goes to chunk k ^ (lane & 7)
                *reinterpret_cast<uint4 *>(box + lane * 128 + ((2 * cs) ^ (lane & 7)) * 16) =
                    make_uint4(w[0], w[1], w[2], w[3]);
                *reinterpret_cast<uint4 *>(box + lane * 128 + ((2 * cs + 1) ^ (lane & 7)) * 16) =
                    make_uint4(w[4], w[5], w[6], w[7]);
            } else if (!(mode & PART_OUT)) {
                const int64_t n0 = n_base + col0;
                if (m < m_total && n0 < n_total)
                    store_segment(d8 + static_cast<int64_t>(m) * n_total + n0, n_total - n0, w);
                if (d8t != nullptr) {
                    uint8_t *tile = box + (cs & 1) * FP8_TILE_BYTES;
                    *reinterpret_cast<uint4 *>(tile + lane * FP8_TSTRIDE) = make_uint4(w[0], w[1], w[2], w[3]);
                    *reinterpret_cast<uint4 *>(tile + lane * FP8_TSTRIDE + 16) = make_uint4(w[4], w[5], w[6], w[7]);
                    __syncwarp();
                    uint32_t t[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        t[i] = static_cast<uint32_t>(tile[(4 * i) * FP8_TSTRIDE + lane]) |
                               (static_cast<uint32_t>(tile[(4 * i + 1) * FP8_TSTRIDE + lane]) << 8) |
                               (static_cast<uint32_t>(tile[(4 * i + 2) * FP8_TSTRIDE + lane]) << 16) |
                               (static_cast<uint32_t>(tile[(4 * i + 3) * FP8_TSTRIDE + lane]) << 24);
                    }
                    const int64_t n = n0 + lane;
                    if (n < n_total && m_row0 < m_total)
                        store_segment(d8t + n * m_total + m_row0, static_cast<int64_t>(m_total) - m_row0, t);
                }
            }
        }
        if (c + 1 < CHUNKS) tmem_ld_wait();
    }
    if (staged && !(mode & PART_OUT)) {
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmap_d, box, static_cast<int32_t>(n_base + half * (ACC_N / 2)), m_row0);
            tma_store_commit();
        }
        ++nbox;
    }
}

// Whole-tile epilogues that release TMEM before they store (mode 0, staged
// output).  Reading the accumulator out of TMEM is fast (8 warps drain
// 256 bytes per SM cycle); converting, staging and storing D are the slow
// part.  So each half of the accumulator is read and converted into
// registers first and handed back to the MMA warp as soon as its last TMEM
// load has completed; the staging and the TMA stores follow while the next
// tile's MMAs already run.
//
// FP8 output: only the bf16 rounding of D (acc * sa*sb + bias, two columns
// per instruction) happens while a row block's accumulator is read; its 64
// packed bf16 pairs per lane stay in registers and the row block is released
// to the MMA warp right after its last TMEM load.  The delayed-scale
// multiply, the FP8 conversion and the amax (as many conversion instructions
// again, the slow part of this epilogue) are done later: for the first row
// block of the 512-row tile chunk by chunk while the second block is read
// (each chunk's packed words are converted, then replaced by the second
// block's), otherwise after the release, while the next tile's MMAs run.
// The codes go to the warp's staging box and out by TMA.
// The 32 bias values of a chunk from shared memory in one asm block: the
// eight broadcast loads are issued back to back, so their latency is paid
// once per chunk, not once per four columns.
__device__ __forceinline__ void load_bias32(const float *bs, float (&b)[32]) {
    asm volatile(
        "ld.shared.v4.f32 {%0,%1,%2,%3}, [%32];\n\t"
        "ld.shared.v4.f32 {%4,%5,%6,%7}, [%32+16];\n\t"
        "ld.shared.v4.f32 {%8,%9,%10,%11}, [%32+32];\n\t"
        "ld.shared.v4.f32 {%12,%13,%14,%15}, [%32+48];\n\t"
        "ld.shared.v4.f32 {%16,%17,%18,%19}, [%32+64];\n\t"
        "ld.shared.v4.f32 {%20,%21,%22,%23}, [%32+80];\n\t"
        "ld.shared.v4.f32 {%24,%25,%26,%27}, [%32+96];\n\t"
        "ld.shared.v4.f32 {%28,%29,%30,%31}, [%32+112];"
        : "=f"(b[0]), "=f"(b[1]), "=f"(b[2]), "=f"(b[3]), "=f"(b[4]), "=f"(b[5]), "=f"(b[6]), "=f"(b[7]),
          "=f"(b[8]), "=f"(b[9]), "=f"(b[10]), "=f"(b[11]), "=f"(b[12]), "=f"(b[13]), "=f"(b[14]), "=f"(b[15]),
          "=f"(b[16]), "=f"(b[17]), "=f"(b[18]), "=f"(b[19]), "=f"(b[20]), "=f"(b[21]), "=f"(b[22]), "=f"(b[23]),
          "=f"(b[24]), "=f"(b[25]), "=f"(b[26]), "=f"(b[27]), "=f"(b[28]), "=f"(b[29]), "=f"(b[30]), "=f"(b[31])
        : "r"(smem_u32(bs))
        : "memory");
}

template <bool BIAS>
__device__ __forceinline__ void fp8_read_chunk(uint32_t (&pk)[64], int c, const uint32_t (&r)[32], uint64_t sab2,
                                               const float *bs) {
    float bv[32];
    if constexpr (BIAS) load_bias32(bs, bv);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const float4 b = BIAS ? make_float4(bv[4 * j], bv[4 * j + 1], bv[4 * j + 2], bv[4 * j + 3])
                              : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        const uint64_t v01 = scale_bias2(r[4 * j], r[4 * j + 1], sab2, b.x, b.y);
        const uint64_t v23 = scale_bias2(r[4 * j + 2], r[4 * j + 3], sab2, b.z, b.w);
        __nv_bfloat162 ha = __floats2bfloat162_rn(lo_f32(v01), hi_f32(v01));
        __nv_bfloat162 hb = __floats2bfloat162_rn(lo_f32(v23), hi_f32(v23));
        pk[16 * c + 2 * j] = *reinterpret_cast<uint32_t *>(&ha);
        pk[16 * c + 2 * j + 1] = *reinterpret_cast<uint32_t *>(&hb);
    }
}
// Codes of chunk c (32 columns) from its packed bf16 pairs into the box row.
// cmax: running max of |bf16(D)| over the row block's chunks (merged into the
// amax by the caller only for rows below M).
__device__ __forceinline__ void fp8_convert_chunk(const uint32_t (&pk)[64], int c, uint8_t *box, int lane,
                                                  uint64_t s2, int fmt, float &cmax) {
    uint32_t w[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t ua = pk[16 * c + 2 * j], ub = pk[16 * c + 2 * j + 1];
        const float h0 = __uint_as_float(ua << 16), h1 = __uint_as_float(ua & 0xFFFF0000u);
        const float h2 = __uint_as_float(ub << 16), h3 = __uint_as_float(ub & 0xFFFF0000u);
        cmax = fmaxf(cmax, fmaxf(fmaxf(fabsf(h0), fabsf(h1)), fmaxf(fabsf(h2), fabsf(h3))));
        const uint64_t p01 = mul_f32x2(pack_f32x2(h0, h1), s2);
        const uint64_t p23 = mul_f32x2(pack_f32x2(h2, h3), s2);
        w[j] = cvt_fp8x2(lo_f32(p01), hi_f32(p01), fmt) | (cvt_fp8x2(lo_f32(p23), hi_f32(p23), fmt) << 16);
    }
    // 16-byte chunk k of row `lane` goes to chunk k ^ (lane & 7)
    *reinterpret_cast<uint4 *>(box + lane * 128 + ((2 * c) ^ (lane & 7)) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
    *reinterpret_cast<uint4 *>(box + lane * 128 + ((2 * c + 1) ^ (lane & 7)) * 16) =
        make_uint4(w[4], w[5], w[6], w[7]);
}

template <bool BIAS, int MSUB>
__device__ __forceinline__ void epilogue_fp8_regs(uint32_t t_row0, int lane, uint8_t *boxes, int &nbox, int half,
                                                  const CUtensorMap *tmap_d, int64_t n_base, int32_t m_row_h0,
                                                  int32_t rows_per_sub, float sab, const float *bias_s,
                                                  uint32_t empty_base, bool split, float s_out, int fmt,
                                                  int32_t m_total, float &amax) {
    constexpr int CH = ACC_N / 2 / 32;  // chunks of 32 columns per warp and row block
    const uint64_t sab2 = pack_f32x2(sab, sab);
    const uint64_t s2 = pack_f32x2(s_out, s_out);
    const float *bs = bias_s + half * (ACC_N / 2);
    // Rows past M (the last tile's padding: A read as zeros, so D is the bias
    // alone there) are stored by no one and count for no amax.
    float cmax = 0.0f;
    uint32_t pk[CH * 16];               // bf16(D) of a row block, two columns per word
    uint32_t r[32];
    auto release = [&](int h) {
        // every TMEM load of this row block (or of the accumulator) is done
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_cluster(empty_base + static_cast<uint32_t>(split ? h * sizeof(uint64_t) : 0));
    };
    auto store_box = [&](uint8_t *box, int h) {
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
            tma_store_2d(tmap_d, box, static_cast<int32_t>(n_base + half * (ACC_N / 2)), m_row_h0 + h * rows_per_sub);
            tma_store_commit();
        }
        ++nbox;
    };
    // row block 0
    const uint32_t t_h0 = t_row0 + static_cast<uint32_t>(half * (ACC_N / 2));
    tmem_ld32(t_h0, r);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        fp8_read_chunk<BIAS>(pk, c, r, sab2, bs + c * 32);
        if (c + 1 < CH) {
            tmem_ld32(t_h0 + static_cast<uint32_t>((c + 1) * 32), r);
            tmem_ld_wait();
        }
    }
    if (split || MSUB == 1) release(0);
    // the box's last store (the previous tile's) must have finished reading it
    uint8_t *box = boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES;
    if (lane == 0) tma_store_wait_read<EPI_NBOX - 1>();
    __syncwarp();
    if (MSUB > 1) {
        // row block 1 is read while block 0 is converted, chunk by chunk
        const uint32_t t_h1 = t_h0 + static_cast<uint32_t>(ACC_N);
#pragma unroll
        for (int c = 0; c < CH; ++c) {
            tmem_ld32(t_h1 + static_cast<uint32_t>(c * 32), r);
            fp8_convert_chunk(pk, c, box, lane, s2, fmt, cmax);
            tmem_ld_wait();
            fp8_read_chunk<BIAS>(pk, c, r, sab2, bs + c * 32);
        }
        release(1);
        if (m_row_h0 + lane < m_total) amax = fmaxf(amax, cmax);
        cmax = 0.0f;
        store_box(box, 0);
        box = boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES;
        if (lane == 0) tma_store_wait_read<EPI_NBOX - 1>();
        __syncwarp();
    }
#pragma unroll
    for (int c = 0; c < CH; ++c) fp8_convert_chunk(pk, c, box, lane, s2, fmt, cmax);
    if (m_row_h0 + (MSUB - 1) * rows_per_sub + lane < m_total) amax = fmaxf(amax, cmax);
    store_box(box, MSUB - 1);
}

// bf16 output: a half is 128 columns, two staging boxes of 64 columns.  The
// first box is staged in shared memory while the half is read, the second
// box's 32 words per lane stay in registers; the half is released (or, at
// the last half, the accumulator) before the boxes are stored.  Halves are
// read one after the other.
template <bool BIAS>
__device__ __forceinline__ void epilogue_bf16_regs(uint32_t t_h, int lane, uint8_t *boxes, int &nbox, int half,
                                                   const CUtensorMap *tmap_d, int64_t n_base, int32_t m_row0,
                                                   float sab, const float *bias_s, uint32_t empty_addr,
                                                   bool release) {
    constexpr int CH = ACC_N / 2 / 32;   // 4 chunks of 32 columns; 2 per box
    uint32_t packed[16 * (CH / 2)];      // the second box
    const uint64_t sab2 = pack_f32x2(sab, sab);
    uint32_t r[32];
    uint8_t *box = boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES;
    if (lane == 0) tma_store_wait_read<EPI_NBOX - 1>();
    __syncwarp();
    tmem_ld32(t_h + static_cast<uint32_t>(half * (ACC_N / 2)), r);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < CH; ++c) {
        if (release && c == CH - 1) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty_addr);
        }
        const float *bs = bias_s + half * (ACC_N / 2) + c * 32;
        float bv[32];
        if constexpr (BIAS) load_bias32(bs, bv);
        uint32_t w[16];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            const float4 b = BIAS ? make_float4(bv[4 * j], bv[4 * j + 1], bv[4 * j + 2], bv[4 * j + 3])
                                  : make_float4(0.0f, 0.0f, 0.0f, 0.0f);
            const uint64_t v01 = scale_bias2(r[4 * j], r[4 * j + 1], sab2, b.x, b.y);
            const uint64_t v23 = scale_bias2(r[4 * j + 2], r[4 * j + 3], sab2, b.z, b.w);
            __nv_bfloat162 ha = __floats2bfloat162_rn(lo_f32(v01), hi_f32(v01));
            __nv_bfloat162 hb = __floats2bfloat162_rn(lo_f32(v23), hi_f32(v23));
            w[2 * j] = *reinterpret_cast<uint32_t *>(&ha);
            w[2 * j + 1] = *reinterpret_cast<uint32_t *>(&hb);
        }
        if (c + 1 < CH) tmem_ld32(t_h + static_cast<uint32_t>(half * (ACC_N / 2) + (c + 1) * 32), r);
        if (c < CH / 2) {
            // 32 columns = 64 bytes of the box row: 16-byte chunks (c % 2) * 4 + k,
            // swizzled with lane & 7
#pragma unroll
            for (int k = 0; k < 4; ++k)
                *reinterpret_cast<uint4 *>(box + lane * 128 + (((c % 2) * 4 + k) ^ (lane & 7)) * 16) =
                    make_uint4(w[4 * k], w[4 * k + 1], w[4 * k + 2], w[4 * k + 3]);
        } else {
#pragma unroll
            for (int j = 0; j < 16; ++j) packed[16 * (c - CH / 2) + j] = w[j];
        }
        if (c + 1 < CH) tmem_ld_wait();
    }
    // first box (staged during the read), then the second from registers
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_d, box, static_cast<int32_t>(n_base + half * (ACC_N / 2)), m_row0);
        tma_store_commit();
    }
    ++nbox;
    box = boxes + (nbox % EPI_NBOX) * EPI_BOX_BYTES;
    if (lane == 0) tma_store_wait_read<EPI_NBOX - 1>();
    __syncwarp();
#pragma unroll
    for (int k = 0; k < 8; ++k)
        *reinterpret_cast<uint4 *>(box + lane * 128 + (k ^ (lane & 7)) * 16) =
            make_uint4(packed[4 * k], packed[4 * k + 1], packed[4 * k + 2], packed[4 * k + 3]);
    fence_async_smem();
    __syncwarp();
    if (lane == 0) {
        tma_store_2d(tmap_d, box, static_cast<int32_t>(n_base + half * (ACC_N / 2) + 64), m_row0);
        tma_store_commit();
    }
    ++nbox;
}

// Shared-memory carve-up common to both kernels.
struct Smem {
    uint8_t *a, *b, *epi;
    uint64_t *full, *empty, *tfull, *tempty, *drain;
    uint32_t *tmem_slot;
    volatile int *abort_flag;
};

template <int STAGES, int A_STAGE, int B_STAGE>
__device__ __forceinline__ Smem carve(uint8_t *raw) {
    Smem s;
    uint8_t *base = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(raw) + SMEM_ALIGN - 1) & ~static_cast<uintptr_t>(SMEM_ALIGN - 1));
    s.a = base;
    s.b = s.a + STAGES * A_STAGE;
    s.epi = s.b + STAGES * B_STAGE;
    uint64_t *bars = reinterpret_cast<uint64_t *>(s.epi + EPI_BYTES);
    s.full = bars;
    s.empty = bars + STAGES;
    s.tfull = bars + 2 * STAGES;
    s.tempty = bars + 2 * STAGES + 2;
    s.drain = bars + 2 * STAGES + 4;
    s.tmem_slot = reinterpret_cast<uint32_t *>(bars + 2 * STAGES + 5);
    s.abort_flag = reinterpret_cast<volatile int *>(s.tmem_slot + 1);
    return s;
}

__device__ __forceinline__ int32_t ld_acquire(const int32_t *p) {
    int32_t v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int32_t *p, int32_t v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Epilogue loop shared by both kernels.  A tile spans m_sub row blocks of
// rows_per_sub rows (row block h of the tile starts at row h * rows_per_sub,
// and this CTA's rows at row_offset inside it); row block h sits at TMEM
// column h * 256 of the accumulator.  acc_bufs accumulators alternate.
// Stream-K segments: a tail (kb0 > 0, the first segment of this cluster)
// publishes its partial in slot `cluster`; a head (kb0 == 0, kb1 < num_kb,
// the last segment) adds the partial of slot cluster + 1 before storing D.
// BIAS: the launch has a bias (a kernel template parameter, so that each
// kernel holds one epilogue variant and a kernel without a bias does not
// stage one).
template <int OUT, bool BIAS>
__device__ __forceinline__ void epilogue_loop(const Smem &sm, const CUtensorMap *tmap_d, const Params &p,
                                              uint32_t tmem_base, int warp, int lane, int cluster, int clusters,
                                              int m_sub, int rows_per_sub, int row_offset, int acc_bufs,
                                              uint32_t tempty_rank, int rank, bool split) {
    const int q = warp & 3;                  // TMEM lane quarter this warp may access
    const int half = (warp - EPI_WARP0) >> 2;  // which half of the accumulator columns
    uint8_t *boxes = sm.epi + (warp - EPI_WARP0) * EPI_NBOX * EPI_BOX_BYTES;
    int nbox = 0;  // staging boxes this warp has filled (boxes alternate)
    float *bias_s = reinterpret_cast<float *>(sm.epi + EPI_WARPS * EPI_NBOX * EPI_BOX_BYTES);
    const int epi_tid = (warp - EPI_WARP0) * 32 + lane;
    const float sab = __fmul_rn(__ldg(p.a_scale_inv), __ldg(p.b_scale_inv));
    const float s_out = OUT == OUT_FP8 ? __ldg(p.out_scale) : 0.0f;
    float amax = 0.0f;
    Sched sched(p, cluster, clusters);
    int local = 0, tile, kb0, kb1;
    while (sched.next(tile, kb0, kb1)) {
        int m_blk, n_blk;
        tile_coords(tile, p.tiles_m, p.tiles_n, p.group_m, m_blk, n_blk);
        const int acc = acc_bufs == 2 ? (local & 1) : 0;
        const uint32_t acc_phase = static_cast<uint32_t>(acc_bufs == 2 ? (local >> 1) : local) & 1u;
        ++local;
        const int seg = (kb0 > 0 ? PART_OUT : 0) | (kb1 < p.num_kb ? PART_IN : 0);
        const int mode = seg;
        float bias_v[BIAS_PER_THREAD];
        if constexpr (BIAS) load_bias(bias_v, p, static_cast<int64_t>(n_blk) * ACC_N, epi_tid);
        bool ok = mbar_wait(&sm.tfull[acc], acc_phase, sm.abort_flag, SITE_EPI_TMEM_FULL);
        // A cluster's partial slot and publication word (per CTA of the pair):
        // this segment's own (PART_OUT) and the next cluster's (PART_IN).
        float *p_out = nullptr;
        const float *p_in = nullptr;
        int32_t *out_flag = nullptr, *in_flag = nullptr;
        if (seg & PART_OUT) {
            p_out = p.partials + (static_cast<size_t>(cluster) * 2 + rank) * WS_SLOT_FLOATS;
            out_flag = p.flags + cluster * 2 + rank;
        }
        if (seg & PART_IN) {
            p_in = p.partials + (static_cast<size_t>(cluster + 1) * 2 + rank) * WS_SLOT_FLOATS;
            in_flag = p.flags + (cluster + 1) * 2 + rank;
        }
        if ((seg & PART_IN) && ok && epi_tid == 0) {
            // The rest of this tile's k-range is the first segment of the next
            // cluster's range (which, if it does not reach the tile's end
            // either, has added the partial of the cluster after it).
            const uint64_t t0 = globaltimer();
            while (ld_acquire(in_flag) != static_cast<int32_t>(p.epoch)) {
                if (*sm.abort_flag || globaltimer() - t0 > p.partial_wait_ns) {
                    *sm.abort_flag = 1;
                    record_error(SITE_EPI_PARTIAL);
                    ok = false;
                    break;
                }
            }
        }
        // All epilogue warps meet here every tile: they leave together if any
        // wait gave up, and none of them still reads the previous tile's bias
        // (which is then staged and made visible to all of them).
        if (epilogue_any(!ok)) break;
        if constexpr (BIAS) {
            stage_bias(bias_s, bias_v, epi_tid);
            epilogue_bar();
        }
        tc_fence_after();
        // An accumulator is released whole (tempty[acc]) after its last row
        // block, or with `split` (a single accumulator set of two M halves)
        // half by half (tempty[h]), so that the next tile's half-0 MMAs
        // start while half 1 is still being read.
        const uint32_t empty_base = map_to_cta(smem_u32(&sm.tempty[acc]), tempty_rank);
        const int64_t n_tile = static_cast<int64_t>(n_blk) * ACC_N;
        const uint32_t t_acc = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + static_cast<uint32_t>(acc * ACC_N);
        const int32_t m_row_h0 = (m_blk * m_sub) * rows_per_sub + row_offset + q * 32;
        bool done = false;
        if constexpr (EPI_EARLY && OUT == OUT_FP8) {
            if (mode == 0 && p.out_d8t == nullptr) {
                if (m_sub == 2) {
                    if constexpr (BIAS)
                        epilogue_fp8_regs<true, 2>(t_acc, lane, boxes, nbox, half, tmap_d, n_tile, m_row_h0,
                                                   rows_per_sub, sab, bias_s, empty_base, split, s_out, p.out_fmt, p.M, amax);
                    else
                        epilogue_fp8_regs<false, 2>(t_acc, lane, boxes, nbox, half, tmap_d, n_tile, m_row_h0,
                                                    rows_per_sub, sab, bias_s, empty_base, split, s_out, p.out_fmt,
                                                    p.M, amax);
                } else {
                    if constexpr (BIAS)
                        epilogue_fp8_regs<true, 1>(t_acc, lane, boxes, nbox, half, tmap_d, n_tile, m_row_h0,
                                                   rows_per_sub, sab, bias_s, empty_base, split, s_out, p.out_fmt, p.M, amax);
                    else
                        epilogue_fp8_regs<false, 1>(t_acc, lane, boxes, nbox, half, tmap_d, n_tile, m_row_h0,
                                                    rows_per_sub, sab, bias_s, empty_base, split, s_out, p.out_fmt,
                                                    p.M, amax);
                }
                done = true;
            }
        }
        if constexpr (EPI_EARLY && OUT == OUT_BF16) {
            if (mode == 0) {
                for (int h = 0; h < m_sub; ++h) {
                    const uint32_t empty_addr = empty_base + static_cast<uint32_t>(split ? h * sizeof(uint64_t) : 0);
                    const bool release = split || h == m_sub - 1;
                    const uint32_t t_h = t_acc + static_cast<uint32_t>(h * ACC_N);
                    if constexpr (BIAS)
                        epilogue_bf16_regs<true>(t_h, lane, boxes, nbox, half, tmap_d, n_tile,
                                                 m_row_h0 + h * rows_per_sub, sab, bias_s, empty_addr, release);
                    else
                        epilogue_bf16_regs<false>(t_h, lane, boxes, nbox, half, tmap_d, n_tile,
                                                  m_row_h0 + h * rows_per_sub, sab, bias_s, empty_addr, release);
                }
                done = true;
            }
        }
        for (int h = 0; h < m_sub && !done; ++h) {
            const uint32_t empty_addr = empty_base + static_cast<uint32_t>(split ? h * sizeof(uint64_t) : 0);
            const bool release = split || h == m_sub - 1;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                                   static_cast<uint32_t>((acc + h) * ACC_N);
            const int32_t m_row0 = (m_blk * m_sub + h) * rows_per_sub + row_offset + q * 32;
            const int64_t n_base = static_cast<int64_t>(n_blk) * ACC_N;
            if constexpr (OUT == OUT_FP8) {
                if constexpr (BIAS)
                    epilogue_tile_fp8<true>(t_row, lane, boxes, nbox, half, p.out_d8, p.out_d8t, tmap_d, n_base, m_row0, sab,
                                            bias_s, empty_addr, release, mode, p_in, p_out, h, q, s_out, p.out_fmt, p.M,
                                            p.N,
                                            amax);
                else
                    epilogue_tile_fp8<false>(t_row, lane, boxes, nbox, half, p.out_d8, p.out_d8t, tmap_d, n_base, m_row0, sab,
                                             bias_s, empty_addr, release, mode, p_in, p_out, h, q, s_out, p.out_fmt, p.M,
                                            p.N,
                                             amax);
            } else {
                if constexpr (BIAS)
                    epilogue_tile<OUT == OUT_BF16, true>(t_row, lane, boxes, nbox, half, tmap_d, n_base, m_row0, sab, bias_s,
                                                         empty_addr, release, mode, p_in, p_out, h, q);
                else
                    epilogue_tile<OUT == OUT_BF16, false>(t_row, lane, boxes, nbox, half, tmap_d, n_base, m_row0, sab,
                                                          bias_s, empty_addr, release, mode, p_in, p_out, h, q);
            }
        }
        if (seg != 0) {
            // Every epilogue thread is done with the partials: the next
            // cluster's slot is consumed (free for the next launch), and this
            // segment's own partial stores precede its publication.
            epilogue_bar();
            if (epi_tid == 0) {
                if (seg & PART_IN) *in_flag = 0;
                if (seg & PART_OUT) {
                    __threadfence();
                    if (!p.withhold_partials) st_release(out_flag, static_cast<int32_t>(p.epoch));
                }
            }
        }
    }
    if constexpr (OUT == OUT_FP8) {
        // amax of this warp's outputs: one atomic max per warp on the float's
        // bits (non-negative floats order like integers)
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0 && p.out_amax != nullptr && amax > 0.0f)
            atomicMax(reinterpret_cast<int *>(p.out_amax), __float_as_int(amax));
        if (p.out_scale_inv != nullptr && blockIdx.x == 0 && epi_tid == 0) *p.out_scale_inv = __frcp_rn(s_out);
    }
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
}

// ------------------------------------------------------------ 1-SM kernel --

template <int OUT, bool BIAS>
__global__ void __launch_bounds__(THREADS, 1)
fp8_gemm_1sm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_d, const Params p) {
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve<S1_STAGES, S1_A_STAGE, S1_B_STAGE>(smem_raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < S1_STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], EPI_WARPS);
        }
        mbar_init(sm.drain, 1);
        *sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_d);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(sm.tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;
    // Everything above touched only this CTA; global memory waits for the
    // previous kernel in the stream.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            bool ok = true;
            Sched sched(p, blockIdx.x, gridDim.x);
            int tile, kb0, kb1;
            while (ok && sched.next(tile, kb0, kb1)) {
                int m_blk, n_blk;
                tile_coords(tile, p.tiles_m, p.tiles_n, p.group_m, m_blk, n_blk);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&sm.empty[stage], phase ^ 1u, sm.abort_flag, SITE_PRODUCER_EMPTY)) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&sm.full[stage], S1_A_STAGE + S1_B_STAGE);
                    uint8_t *a_dst = sm.a + stage * S1_A_STAGE, *b_dst = sm.b + stage * S1_B_STAGE;
                    if (p.a_mn)
                        tma_load_2d(&tmap_a, &sm.full[stage], a_dst, m_blk * S1_BM, kb * BK);
                    else
                        tma_load_2d(&tmap_a, &sm.full[stage], a_dst, kb * BK, m_blk * S1_BM);
                    if (p.b_mn) {
                        // two 128-column boxes: the tile's column groups, 16 KB apart
                        tma_load_2d(&tmap_b, &sm.full[stage], b_dst, n_blk * ACC_N, kb * BK);
                        tma_load_2d(&tmap_b, &sm.full[stage], b_dst + S1_B_STAGE / 2, n_blk * ACC_N + ACC_N / 2,
                                    kb * BK);
                    } else {
                        tma_load_2d(&tmap_b, &sm.full[stage], b_dst, kb * BK, n_blk * ACC_N);
                    }
                    ++issued;
                    if (++stage == S1_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let every load already issued land before the CTA can exit.
                for (int s = 0; s < S1_STAGES; ++s) {
                    const int64_t n_s = issued > s ? (issued - s + S1_STAGES - 1) / S1_STAGES : 0;
                    if (n_s > 0) mbar_wait_drain(&sm.full[s], static_cast<uint32_t>((n_s - 1) & 1));
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            Sched sched(p, blockIdx.x, gridDim.x);
            int tile, kb0, kb1;
            while (ok && sched.next(tile, kb0, kb1)) {
                const int acc = local & 1;
                const uint32_t acc_phase = static_cast<uint32_t>(local >> 1) & 1u;
                ++local;
                if (!mbar_wait(&sm.tempty[acc], acc_phase ^ 1u, sm.abort_flag, SITE_MMA_TMEM_EMPTY)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * ACC_N);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&sm.full[stage], phase, sm.abort_flag, SITE_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t a_desc = operand_desc(smem_u32(sm.a + stage * S1_A_STAGE), p.a_mn, 0);
                    const uint64_t b_desc = operand_desc(smem_u32(sm.b + stage * S1_B_STAGE), p.b_mn, S1_B_STAGE / 2);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
                        umma_f8f6f4(d_tmem, a_desc + operand_kstep(k, p.a_mn), b_desc + operand_kstep(k, p.b_mn),
                                    p.idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    umma_commit(&sm.empty[stage]);
                    if (++stage == S1_STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit(&sm.tfull[acc]);
            }
            // Every MMA issued must have finished before TMEM can be freed.
            umma_commit(sm.drain);
            mbar_wait_drain(sm.drain, 0);
        }
        __syncwarp();
    } else {
        epilogue_loop<OUT, BIAS>(sm, &tmap_d, p, tmem_base, warp, lane, blockIdx.x, gridDim.x, 1, S1_BM, 0, 2, 0u, 0,
                           false);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------ 2-SM kernel --

// Launched with clusters of 2 CTAs (gridDim.x even).  Cluster c handles pair
// tiles c, c + clusters, ...; a pair tile has M_SUB row blocks of 256 rows
// and 256 columns.  CTA rank r of the pair owns rows r*128..r*128+127 of each
// row block and loads rows r*128.. of the tile's 256 B rows.
template <int OUT, int M_SUB, bool BIAS>
__global__ void __launch_bounds__(THREADS, 1)
fp8_gemm_2sm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_d, const Params p) {
    using PC = Pair<M_SUB>;
    constexpr int STAGES = PC::STAGES;
    constexpr int A_STAGE = PC::A_STAGE;
    constexpr int ACC_BUFS = PC::ACC_BUFS;
    // Half-by-half release of the 512-row tile's accumulator (FP8 output,
    // whose longer epilogue it hides best; measured neutral-to-negative with
    // bf16 and fp32 outputs).
    constexpr bool SPLIT = M_SUB == 2 && OUT == OUT_FP8;
    extern __shared__ uint8_t smem_raw[];
    const Smem sm = carve<STAGES, A_STAGE, S2_B_STAGE>(smem_raw);
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster_id = blockIdx.x >> 1;
    const int num_clusters = gridDim.x >> 1;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sm.tfull[b], 1);
            mbar_init(&sm.tempty[b], 2 * EPI_WARPS);  // epilogue warps of both CTAs (the first CTA's is used)
        }
        mbar_init(sm.drain, 1);
        *sm.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        fence_async_smem();
        prefetch_tmap(&tmap_a);
        prefetch_tmap(&tmap_b);
        prefetch_tmap(&tmap_d);
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(sm.tmem_slot)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *sm.tmem_slot;
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0;
            int64_t issued = 0;
            bool ok = true;
            Sched sched(p, cluster_id, num_clusters);
            int tile, kb0, kb1;
            uint64_t keep_policy;
            asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep_policy));
            const bool keep_a = p.l2_keep == 1, keep_b = p.l2_keep == 2;
            while (ok && sched.next(tile, kb0, kb1)) {
                int m_blk, n_blk;
                tile_coords(tile, p.tiles_m, p.tiles_n, p.group_m, m_blk, n_blk);
                const int32_t a_row = m_blk * M_SUB * 2 * S2_BM + static_cast<int32_t>(rank) * S2_BM;
                const int32_t b_row = n_blk * ACC_N + static_cast<int32_t>(rank) * S2_BN_HALF;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(&sm.empty[stage], phase ^ 1u, sm.abort_flag, SITE_PRODUCER_EMPTY)) {
                        ok = false;
                        break;
                    }
                    // The pair's MMA waits on the first CTA's barrier for the
                    // bytes of both CTAs.
                    if (leader) mbar_arrive_expect_tx(&sm.full[stage], 2 * (A_STAGE + S2_B_STAGE));
                    const uint32_t full_leader = map_to_cta(smem_u32(&sm.full[stage]), 0u);
#pragma unroll
                    for (int h = 0; h < M_SUB; ++h) {
                        uint8_t *a_dst = sm.a + stage * A_STAGE + h * S2_BM * BK;
                        const int32_t ax = p.a_mn ? a_row + h * 2 * S2_BM : kb * BK;
                        const int32_t ay = p.a_mn ? kb * BK : a_row + h * 2 * S2_BM;
                        if (keep_a)
                            tma_load_2d_pair_hint(&tmap_a, full_leader, a_dst, ax, ay, keep_policy);
                        else
                            tma_load_2d_pair(&tmap_a, full_leader, a_dst, ax, ay);
                    }
                    uint8_t *b_dst = sm.b + stage * S2_B_STAGE;
                    const int32_t bx = p.b_mn ? b_row : kb * BK, by = p.b_mn ? kb * BK : b_row;
                    if (keep_b)
                        tma_load_2d_pair_hint(&tmap_b, full_leader, b_dst, bx, by, keep_policy);
                    else
                        tma_load_2d_pair(&tmap_b, full_leader, b_dst, bx, by);
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok && leader) {
                for (int s = 0; s < STAGES; ++s) {
                    const int64_t n_s = issued > s ? (issued - s + STAGES - 1) / STAGES : 0;
                    if (n_s > 0) mbar_wait_drain(&sm.full[s], static_cast<uint32_t>((n_s - 1) & 1));
                }
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int stage = 0;
            uint32_t phase = 0;
            bool ok = true;
            int local = 0;
            Sched sched(p, cluster_id, num_clusters);
            int tile, kb0, kb1;
            while (ok && sched.next(tile, kb0, kb1)) {
                const int acc = ACC_BUFS == 2 ? (local & 1) : 0;
                const uint32_t acc_phase = static_cast<uint32_t>(ACC_BUFS == 2 ? (local >> 1) : local) & 1u;
                ++local;
                if (!mbar_wait(&sm.tempty[acc], acc_phase ^ 1u, sm.abort_flag, SITE_MMA_TMEM_EMPTY)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                int kb = kb0;
                if constexpr (SPLIT) {
                    // The epilogue frees the two M halves one after the other
                    // (tempty[0], then tempty[1]).  The first `pre` k-blocks
                    // run their half-0 MMAs as soon as half 0 is free, holding
                    // their stages; their half-1 MMAs follow once half 1 is
                    // free, and only then are the stages released.  One stage
                    // stays out of this so that the main loop resumes on a
                    // loaded stage while the held ones refill.  Within each
                    // half the accumulation order over (k-block, k) is
                    // unchanged.
                    const int pre = kb1 - kb0 < STAGES - 1 ? kb1 - kb0 : STAGES - 1;
                    int st = stage;
                    uint32_t ph = phase;
                    for (int j = 0; j < pre && ok; ++j) {
                        if (!mbar_wait(&sm.full[st], ph, sm.abort_flag, SITE_MMA_FULL)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint64_t b_desc = operand_desc(smem_u32(sm.b + st * S2_B_STAGE), p.b_mn, 0);
                        const uint64_t a_desc = operand_desc(smem_u32(sm.a + st * A_STAGE), p.a_mn, 0);
#pragma unroll
                        for (int k = 0; k < BK / UMMA_K; ++k)
                            umma_f8f6f4_pair(tmem_base, a_desc + operand_kstep(k, p.a_mn),
                                             b_desc + operand_kstep(k, p.b_mn), p.idesc, (j > 0 || k > 0) ? 1u : 0u);
                        if (++st == STAGES) {
                            st = 0;
                            ph ^= 1u;
                        }
                    }
                    if (!ok || !mbar_wait(&sm.tempty[1], acc_phase ^ 1u, sm.abort_flag, SITE_MMA_TMEM_EMPTY)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    for (int j = 0; j < pre; ++j) {
                        const uint64_t b_desc = operand_desc(smem_u32(sm.b + stage * S2_B_STAGE), p.b_mn, 0);
                        const uint64_t a_desc =
                            operand_desc(smem_u32(sm.a + stage * A_STAGE + S2_BM * BK), p.a_mn, 0);
#pragma unroll
                        for (int k = 0; k < BK / UMMA_K; ++k)
                            umma_f8f6f4_pair(tmem_base + static_cast<uint32_t>(ACC_N),
                                             a_desc + operand_kstep(k, p.a_mn), b_desc + operand_kstep(k, p.b_mn),
                                             p.idesc, (j > 0 || k > 0) ? 1u : 0u);
                        umma_commit_pair_to(&sm.empty[stage], 0x3);
                        if (++stage == STAGES) {
                            stage = 0;
                            phase ^= 1u;
                        }
                    }
                    kb = kb0 + pre;
                }
                for (; kb < kb1; ++kb) {
                    if (!mbar_wait(&sm.full[stage], phase, sm.abort_flag, SITE_MMA_FULL)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t b_desc = operand_desc(smem_u32(sm.b + stage * S2_B_STAGE), p.b_mn, 0);
#pragma unroll
                    for (int k = 0; k < BK / UMMA_K; ++k) {
#pragma unroll
                        for (int h = 0; h < M_SUB; ++h) {
                            const uint64_t a_desc =
                                operand_desc(smem_u32(sm.a + stage * A_STAGE + h * S2_BM * BK), p.a_mn, 0);
                            umma_f8f6f4_pair(tmem_base + static_cast<uint32_t>((acc + h) * ACC_N),
                                             a_desc + operand_kstep(k, p.a_mn), b_desc + operand_kstep(k, p.b_mn),
                                             p.idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                        }
                    }
                    umma_commit_pair_to(&sm.empty[stage], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) umma_commit_pair_to(&sm.tfull[acc], 0x3);
            }
            umma_commit_pair(sm.drain);
            mbar_wait_drain(sm.drain, 0);
        }
        __syncwarp();
    } else {
        epilogue_loop<OUT, BIAS>(sm, &tmap_d, p, tmem_base, warp, lane, cluster_id, num_clusters, M_SUB, 2 * S2_BM,
                           static_cast<int>(rank) * S2_BM, ACC_BUFS, 0u, static_cast<int>(rank), SPLIT);
    }

    tc_fence_before();
    __syncthreads();
    // The peer's MMAs, loads and barrier arrivals target this CTA's memory
    // until both CTAs are here.
    cluster_sync();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                     : "memory");
    }
}

// ------------------------------------------------------------------- host --

bool encode_2d(CUtensorMap *map, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
               uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
    return encode_tmap_2d(map, dt, base, inner, outer, row_bytes, box_inner, box_outer, CU_TENSOR_MAP_SWIZZLE_128B);
}

// Instruction descriptor of tcgen05.mma.kind::f8f6f4 (dense, K-major A and B):
// [4,6) D format (1 = fp32), [7,10) A format, [10,13) B format (0 = E4M3,
// 1 = E5M2), [15] / [16] A / B major (0 = K, 1 = MN), [17,23) N >> 3,
// [24,29) M >> 4.
uint32_t make_idesc(fp8ds_format fa, fp8ds_format fb, int m, int n, bool a_mn, bool b_mn) {
    uint32_t d = 0;
    d |= 1u << 4;
    d |= static_cast<uint32_t>(fa == FP8DS_E5M2 ? 1 : 0) << 7;
    d |= static_cast<uint32_t>(fb == FP8DS_E5M2 ? 1 : 0) << 10;
    d |= static_cast<uint32_t>(a_mn ? 1 : 0) << 15;
    d |= static_cast<uint32_t>(b_mn ? 1 : 0) << 16;
    d |= static_cast<uint32_t>(n >> 3) << 17;
    d |= static_cast<uint32_t>(m >> 4) << 24;
    return d;
}

// Per-device flags and counts below are computed once; concurrent first
// calls may both compute them and store the same value.
template <typename K>
cudaError_t set_smem_once(K kernel, int bytes, std::atomic<bool> (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && done[dev].load(std::memory_order_relaxed)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess && dev >= 0 && dev < 64) done[dev].store(true, std::memory_order_relaxed);
    return e;
}

// Number of CTA pairs of a 2-SM kernel that fit on the device at once.
template <typename K>
int max_pairs(K kernel, int smem_bytes, std::atomic<int> (&cached)[64]) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return num_sms() / 2;
    int n = cached[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
        cfg.blockDim = dim3(THREADS, 1, 1);
        cfg.dynamicSmemBytes = smem_bytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) n = num_sms() / 2;
        cached[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

template <int OUT, int M_SUB, bool BIAS>
cudaError_t launch_2sm(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &td, const Params &p,
                       cudaStream_t stream) {
    static std::atomic<bool> done[64];
    static std::atomic<int> cached_pairs[64];
    auto kernel = fp8_gemm_2sm_kernel<OUT, M_SUB, BIAS>;
    constexpr int smem = Pair<M_SUB>::SMEM;
    cudaError_t e = set_smem_once(kernel, smem, done);
    if (e != cudaSuccess) return e;
    const int tiles = p.tiles_m * p.tiles_n;
    const int cap = max_pairs(kernel, smem, cached_pairs);
    // a stream-K launch shares its remaining tiles' k-blocks among all pairs
    // (as many as the workspace has partial slots for)
    const int pairs = p.stream_k != 0 ? (cap < p.sk_pairs ? cap : p.sk_pairs) : (tiles < cap ? tiles : cap);
    return launch_pdl(kernel, dim3(2 * pairs), dim3(THREADS), smem, stream, 2, ta, tb, td, p);
}

template <int OUT, bool BIAS>
cudaError_t launch_1sm(const CUtensorMap &ta, const CUtensorMap &tb, const CUtensorMap &td, const Params &p,
                       cudaStream_t stream) {
    static std::atomic<bool> done[64];
    auto kernel = fp8_gemm_1sm_kernel<OUT, BIAS>;
    cudaError_t e = set_smem_once(kernel, S1_SMEM, done);
    if (e != cudaSuccess) return e;
    const int tiles = p.tiles_m * p.tiles_n;
    const int grid = tiles < num_sms() ? tiles : num_sms();
    return launch_pdl(kernel, dim3(grid), dim3(THREADS), S1_SMEM, stream, 1, ta, tb, td, p);
}

// The kernel instantiation for an output kind, tile mode and bias presence.
template <bool BIAS>
cudaError_t launch_any(int out, bool pair, int m_sub, const CUtensorMap &ta, const CUtensorMap &tb,
                       const CUtensorMap &td, const Params &p, cudaStream_t stream) {
    if (pair && m_sub == 2)
        return out == OUT_FP8    ? launch_2sm<OUT_FP8, 2, BIAS>(ta, tb, td, p, stream)
               : out == OUT_BF16 ? launch_2sm<OUT_BF16, 2, BIAS>(ta, tb, td, p, stream)
                                 : launch_2sm<OUT_F32, 2, BIAS>(ta, tb, td, p, stream);
    if (pair)
        return out == OUT_FP8    ? launch_2sm<OUT_FP8, 1, BIAS>(ta, tb, td, p, stream)
               : out == OUT_BF16 ? launch_2sm<OUT_BF16, 1, BIAS>(ta, tb, td, p, stream)
                                 : launch_2sm<OUT_F32, 1, BIAS>(ta, tb, td, p, stream);
    return out == OUT_FP8    ? launch_1sm<OUT_FP8, BIAS>(ta, tb, td, p, stream)
           : out == OUT_BF16 ? launch_1sm<OUT_BF16, BIAS>(ta, tb, td, p, stream)
                             : launch_1sm<OUT_F32, BIAS>(ta, tb, td, p, stream);
}

}  // namespace

size_t gemm_workspace_bytes() {
    static std::atomic<int> cached[64];
    const int pairs = max_pairs(fp8_gemm_2sm_kernel<OUT_BF16, 1, false>, Pair<1>::SMEM, cached);
    return WS_FLAG_BYTES + static_cast<size_t>(pairs) * 2 * WS_SLOT_FLOATS * sizeof(float);
}

namespace {

// Error-path test setting (fp8ds_test_stream_k_withhold).
std::atomic<int> g_test_withhold{0};
std::atomic<unsigned long long> g_test_wait_ns{0};

// Tile schedule of a GEMM on the current device: kernel (one CTA or a CTA
// pair), pair-tile rows, tile count, and whether a workspace turns it into
// the stream-K schedule.
struct GemmPlan {
    bool pair;
    int m_sub;
    int64_t tiles;
    int group_m;     // raster group (tile_coords)
    int l2_keep;     // Params::l2_keep
    bool stream_k;   // with a large enough workspace
};

GemmPlan plan_gemm(int64_t m, int64_t n, int64_t k) {
    static std::atomic<int> cached_pairs[64];
    GemmPlan g;
    g.pair = m > S1_BM;
    // Long contractions amortise the partly exposed epilogue of the 512-row
    // pair tile; short ones keep the double-buffered 256-row tile.  The
    // 512-row tile is also declined when its tiles fill the last wave of
    // pairs less well than the 256-row ones (e.g. 4096 x 8192: 256 tiles =
    // 3.46 waves of 74 pairs against 512 = 6.92 waves).
    g.m_sub = 1;
    const int64_t cap = g.pair ? max_pairs(fp8_gemm_2sm_kernel<OUT_BF16, 1, false>, Pair<1>::SMEM, cached_pairs) : 0;
    const int64_t tn = (n + ACC_N - 1) / ACC_N;
    if (g.pair && m > 2 * S2_BM && k >= FP8DS_MSUB2_MIN_K) {
        const int64_t t1 = ((m + 2 * S2_BM - 1) / (2 * S2_BM)) * tn, t2 = ((m + 4 * S2_BM - 1) / (4 * S2_BM)) * tn;
        // wave fill tiles / (waves * cap), compared without division
        const int64_t w1 = (t1 + cap - 1) / cap, w2 = (t2 + cap - 1) / cap;
        if (cap <= 0 || t2 * w1 * 50 >= t1 * w2 * 49) g.m_sub = 2;      // fill(512) >= fill(256) - 2%
    }
    const int64_t tile_m = g.pair ? g.m_sub * 2 * S2_BM : S1_BM;
    const int64_t tm = (m + tile_m - 1) / tile_m;
    g.tiles = tm * tn;
    // Raster: row groups of GROUP_M tiles keep a band of A and the B columns
    // in L2 over many waves.  A pair launch of at most two waves with more
    // row tiles than column tiles takes whole rows of tiles instead, so that
    // each A row block (the larger operand) is streamed by one wave only and
    // the second wave re-reads only the smaller B.
    g.group_m = (g.pair && cap > 0 && g.tiles <= 2 * cap && tm > tn) ? 1 : GROUP_M;
    // An operand that every wave streams whole (B under whole rows of tiles,
    // A when all row tiles fit in one group) is read once per wave; with more
    // than one wave it is loaded with an L2 evict_last hint, if it takes at
    // most a quarter of the 126 MB L2, so that later waves find it there.
    g.l2_keep = 0;
    if (g.pair && cap > 0 && g.tiles > cap) {
        const int64_t a_bytes = tm * tile_m * k, b_bytes = tn * ACC_N * k;
        if (g.group_m == 1 && b_bytes <= (int64_t(32) << 20)) g.l2_keep = 2;
        else if (g.group_m != 1 && tm <= g.group_m && a_bytes <= (int64_t(32) << 20)) g.l2_keep = 1;
    }
    // Stream-K (given a workspace) when whole tiles would leave a ragged
    // last wave worth balancing: R = tiles mod pairs with pairs / 3 <= R <=
    // 7/8 pairs (a split tile then spans at most four clusters, and at
    // least an eighth of a tile's time is saved), fewer than 8 waves, at
    // least 8 k-blocks per tile, and a publication word for every cluster.
    const int64_t rem = cap > 0 ? g.tiles % cap : 0;
    g.stream_k = g.pair && cap > 0 && 3 * rem >= cap && 8 * rem <= 7 * cap && g.tiles < 8 * cap &&
                 (k + BK - 1) / BK >= 8 && cap <= static_cast<int64_t>(WS_FLAG_BYTES / 8);
    return g;
}

}  // namespace

void gemm_plan_info(int64_t m, int64_t n, int64_t k, int64_t info[5]) {
    static std::atomic<int> cached_pairs[64];
    const GemmPlan g = plan_gemm(m, n, k);
    info[0] = g.pair ? 1 : 0;
    info[1] = g.pair ? g.m_sub : 0;
    info[2] = g.tiles;
    info[3] = g.stream_k ? 1 : 0;
    info[4] = g.pair ? max_pairs(fp8_gemm_2sm_kernel<OUT_BF16, 1, false>, Pair<1>::SMEM, cached_pairs) : num_sms();
}

fp8ds_status launch_gemm(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv, const uint8_t *b,
                         fp8ds_format b_fmt, const float *b_scale_inv, const void *bias, fp8ds_dtype bias_dtype,
                         void *d, fp8ds_dtype d_dtype, int64_t m, int64_t n, int64_t k, void *workspace,
                         size_t workspace_bytes, cudaStream_t stream, const GemmCastOut *cast, bool a_mn,
                         bool b_mn) {
    const int out = cast != nullptr ? OUT_FP8 : (d_dtype == FP8DS_BF16 ? OUT_BF16 : OUT_F32);
    const GemmPlan plan = plan_gemm(m, n, k);
    const bool pair = plan.pair;
    const int m_sub = plan.m_sub;
    CUtensorMap ta, tb, td;
    // K-major operands: [rows, k] boxes of BK x rows; MN-major: [k, rows]
    // boxes of 128 columns x BK rows (the one-CTA B tile loads two of them)
    const uint32_t a_rows = pair ? S2_BM : S1_BM, b_rows = pair ? S2_BN_HALF : ACC_N;
    bool ok = (a_mn ? encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, m, k, m, 128, BK)
                    : encode_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_UINT8, a, k, m, k, BK, a_rows)) &&
              (b_mn ? encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, n, k, n, 128, BK)
                    : encode_2d(&tb, CU_TENSOR_MAP_DATA_TYPE_UINT8, b, k, n, k, BK, b_rows));
    if (out == OUT_FP8) {
        // codes [m, n]: 128-byte x 32-row swizzled boxes (the store path
        // without transpose; with it the epilogue uses plain stores)
        ok = ok && encode_2d(&td, CU_TENSOR_MAP_DATA_TYPE_UINT8, d, n, m, n, 128, 32);
    } else {
        ok = ok && (out == OUT_BF16 ? encode_2d(&td, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d, n, m, n * 2, 64, 32)
                                    : encode_2d(&td, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, d, n, m, n * 4, 32, 32));
    }
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
    const int tile_m = pair ? m_sub * 2 * S2_BM : S1_BM;
    p.tiles_m = static_cast<int32_t>((m + tile_m - 1) / tile_m);
    p.tiles_n = static_cast<int32_t>((n + ACC_N - 1) / ACC_N);
    p.num_kb = static_cast<int32_t>((k + BK - 1) / BK);
    p.group_m = plan.group_m;
    p.l2_keep = pair ? plan.l2_keep : 0;
    p.idesc = make_idesc(a_fmt, b_fmt, pair ? 2 * S2_BM : S1_BM, ACC_N, a_mn, b_mn);
    p.a_mn = a_mn ? 1 : 0;
    p.b_mn = b_mn ? 1 : 0;
    p.stream_k = 0;
    p.sk_pairs = 0;
    p.epoch = 0;
    p.flags = nullptr;
    p.partials = nullptr;
    p.out_scale = cast != nullptr ? cast->scale : nullptr;
    p.out_amax = cast != nullptr ? cast->amax : nullptr;
    p.out_scale_inv = cast != nullptr ? cast->scale_inv : nullptr;
    p.out_fmt = cast != nullptr ? static_cast<int32_t>(cast->fmt) : 0;
    p.out_d8 = cast != nullptr ? static_cast<uint8_t *>(d) : nullptr;
    p.out_d8t = cast != nullptr ? cast->d8t : nullptr;
    p.partial_wait_ns = TIMEOUT_NS;
    p.withhold_partials = 0;
    if (g_test_withhold.load(std::memory_order_relaxed) != 0) {
        p.withhold_partials = 1;
        const unsigned long long w = g_test_wait_ns.load(std::memory_order_relaxed);
        if (w != 0) p.partial_wait_ns = w;
    }
    if (plan.stream_k && workspace != nullptr && workspace_bytes >= gemm_workspace_bytes()) {
        static std::atomic<uint32_t> launches{0};
        uint32_t e = ++launches;
        if (e == 0) e = ++launches;
        p.stream_k = 1;
        const size_t slots = (workspace_bytes - WS_FLAG_BYTES) / (2 * WS_SLOT_FLOATS * sizeof(float));
        p.sk_pairs = static_cast<int32_t>(slots < WS_FLAG_BYTES / 8 ? slots : WS_FLAG_BYTES / 8);
        p.epoch = e;
        p.flags = static_cast<int32_t *>(workspace);
        p.partials = reinterpret_cast<float *>(static_cast<uint8_t *>(workspace) + WS_FLAG_BYTES);
    }
    const cudaError_t e = p.bias_kind != 0 ? launch_any<true>(out, pair, m_sub, ta, tb, td, p, stream)
                                           : launch_any<false>(out, pair, m_sub, ta, tb, td, p, stream);
    if (e != cudaSuccess) {
        set_error("fp8_gemm: launch failed: %s", cudaGetErrorString(e));
        return FP8DS_ERR_CUDA;
    }
    return FP8DS_OK;
}

// ------------------------------------------- allocation-free GEMM variant --

// Scratch of fp8_gemm_noalloc: the stream-K workspace (publication words and
// partial-accumulator slots) as a file-scope device array, so that callers
// that may not allocate device memory still get the split-tile schedule.
// Every device that loads the library holds these bytes until the process
// exits.  80 MiB covers the 74 CTA pairs of a B200 (4 KiB of words + 1 MiB
// per pair).
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(80) << 20;
static __device__ __align__(256) uint8_t g_noalloc_scratch[NOALLOC_SCRATCH_BYTES];

fp8ds_status launch_gemm_noalloc(const uint8_t *a, fp8ds_format a_fmt, const float *a_scale_inv, const uint8_t *b,
                                 fp8ds_format b_fmt, const float *b_scale_inv, const void *bias,
                                 fp8ds_dtype bias_dtype, void *d, fp8ds_dtype d_dtype, int64_t m, int64_t n, int64_t k,
                                 cudaStream_t stream) {
    // Device address of the scratch, looked up once per device with that
    // device current (host code cannot use the array's name as an address).
    static void *scratch[64] = {};
    static std::mutex lock;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        set_error("fp8_gemm_noalloc: no usable current device (%s)", cudaGetErrorString(e));
        return FP8DS_ERR_CUDA;
    }
    void *ws = nullptr;
    {
        std::lock_guard<std::mutex> g(lock);
        if (scratch[dev] == nullptr) {
            void *ptr = nullptr;
            e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
            if (e != cudaSuccess || ptr == nullptr) {
                set_error("fp8_gemm_noalloc: cudaGetSymbolAddress of the static scratch failed: %s",
                          cudaGetErrorString(e));
                return FP8DS_ERR_CUDA;
            }
            scratch[dev] = ptr;
        }
        ws = scratch[dev];
    }
    const size_t need = gemm_workspace_bytes();
    if (need > NOALLOC_SCRATCH_BYTES) {
        set_error("fp8_gemm_noalloc: this device needs %zu bytes of stream-K scratch, more than the %zu-byte static "
                  "scratch (use fp8_gemm_ex with a workspace)",
                  need, NOALLOC_SCRATCH_BYTES);
        return FP8DS_ERR_INVALID_ARG;
    }
    // Whole tiles (no ragged last wave, or the one-CTA kernel) need no
    // scratch: the same launch as fp8_gemm, nothing else enqueued.
    if (!plan_gemm(m, n, k).stream_k)
        return launch_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k,
                           nullptr, 0, stream);
    // The array keeps whatever the previous call left.  Each stream-K launch
    // publishes its partials under a fresh non-zero epoch and its consumers
    // clear the words they read, so stale words cannot match; the words are
    // still cleared here so that a launch that ended early (a bounded wait
    // gave up) leaves nothing behind for the next one.
    e = cudaMemsetAsync(ws, 0, WS_FLAG_BYTES, stream);
    if (e != cudaSuccess) {
        set_error("fp8_gemm_noalloc: clearing the scratch failed: %s", cudaGetErrorString(e));
        return FP8DS_ERR_CUDA;
    }
    return launch_gemm(a, a_fmt, a_scale_inv, b, b_fmt, b_scale_inv, bias, bias_dtype, d, d_dtype, m, n, k, ws,
                       NOALLOC_SCRATCH_BYTES, stream);
}

void set_stream_k_withhold(int withhold, unsigned long long wait_ns) {
    g_test_wait_ns.store(wait_ns, std::memory_order_relaxed);
    g_test_withhold.store(withhold, std::memory_order_relaxed);
}

cudaError_t read_gemm_error(int32_t *out, bool clear) {
    cudaError_t e = cudaMemcpyFromSymbol(out, g_device_error, sizeof(int32_t));
    if (e != cudaSuccess || !clear) return e;
    const int32_t zero = 0;
    return cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int32_t));
}

}  // namespace fp8ds
