// common.cuh -- device helpers shared by the libcsla kernels (sm_100a only):
// number formats, bounded mbarrier waits, TMA and tcgen05 (UMMA / TMEM)
// wrappers, and the fixed-order block reductions every kernel uses so that a
// token's result never depends on what else is in the batch.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csla.h"
#include "kernels.h"

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "libcsla kernels target sm_100a only"
#endif

namespace csla {

// Library-wide device error word (CSLA_DEVERR_* bits), one per device.
extern __device__ unsigned int g_dev_err;

__device__ __forceinline__ void set_dev_err(unsigned bits) { atomicOr(&g_dev_err, bits); }

// ------------------------------------------------------------ number formats
// Order-preserving unsigned key of an fp32 score (-0.0 folded onto +0.0):
// a > b as floats exactly when score_key(a) > score_key(b).  The top-k
// selector and the indexer's candidate output compare scores through it.
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
// The score whose key is `key` (key 0, below every score's key: -inf).
__device__ __forceinline__ float key_score(uint32_t key) {
    if (key == 0u) return -__int_as_float(0x7f800000);
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

__device__ __forceinline__ uint16_t f32_to_bf16_bits(float f) {
    return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// E4M3 (satfinite, round to nearest even) via the hardware conversion.
__device__ __forceinline__ uint8_t f32_to_e4m3(float f) {
    return (uint8_t)__nv_cvt_float_to_fp8(f, __NV_SATFINITE, __NV_E4M3);
}

// Two E4M3 codes (low byte = first) -> f16x2 holding the same values, exactly
// (every E4M3 value is an f16 value), by the hardware conversion.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
    const __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)two_codes, __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// Two E4M3 codes (low byte = first) -> bf16x2 holding the same values, exactly.
// The 7 magnitude bits are moved under the bf16 exponent/mantissa fields (the
// E4M3 exponent then reads as a bf16 exponent 120 too small, subnormal codes
// as bf16 subnormals) and one bf16 multiply by 2^120 rebiases both cases.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two_codes) {
    uint32_t x = __byte_perm(two_codes, 0u, 0x1404);   // b1<<24 | b0<<8
    uint32_t b = (x & 0x80008000u) | ((x >> 4) & 0x07F007F0u);
    __nv_bfloat162 v = *reinterpret_cast<__nv_bfloat162 *>(&b);
    const __nv_bfloat162 k = __halves2bfloat162(__ushort_as_bfloat16(0x7B80), __ushort_as_bfloat16(0x7B80));
    v = __hmul2(v, k);                                  // 0x7B80 = 2^120
    return *reinterpret_cast<uint32_t *>(&v);
}

// Exponent of the E4M3 index-key scale: the smallest e (-126 <= e <= 127)
// with 448 * 2^e >= amax (amax >= 0, an fp32 value).  With amax = f * 2^k,
// f in [0.5, 1), 448 * 2^(k-9) = 0.875 * 2^k covers amax iff f <= 0.875,
// i.e. iff amax's mantissa field is at most 0.75 * 2^23; zero and subnormal
// amax take the minimum.
__device__ __forceinline__ int key_exp_e4m3(float amax) {
    const uint32_t bits = __float_as_uint(amax);
    const int E = (int)(bits >> 23);
    if (E == 0) return -126;
    const int e = (bits & 0x7FFFFFu) <= 0x600000u ? E - 135 : E - 134;
    return e < -126 ? -126 : (e > 127 ? 127 : e);
}

// ------------------------------------------------------------ programmatic dependent launch
// Every libcsla kernel is launched with programmatic stream serialization
// (programmatic dependent launch) and calls pdl_trigger() first (kernels that
// allocate TMEM: right after the allocation), so the next kernel on the
// stream can be scheduled while it runs.  pdl_wait() blocks
// until the preceding kernel has completed and its writes are visible; a
// kernel calls it before it reads anything produced on the stream or writes
// global memory (the device error word aside).  Before the wait a kernel
// only reads its call's read-only inputs (activations, weights, slot lists,
// block tables) into registers, shared memory or TMEM, and sets up barriers
// and TMEM.  Every launch has at least one CTA that waits before exiting, so
// kernel completion stays ordered along the stream.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ------------------------------------------------------------ device timeline
// Built with -DCSLA_TIMELINE only (see build.py --timeline): thread 0 of
// every CTA records its kernel id, CTA index and global-timer stamps (start,
// grid-dependency wait passed, exit, and up to eight marks a kernel sets at
// points of interest) into g_timeline, read back with csla_timeline_read().  In normal builds the hooks compile to nothing.
enum TimelineKernel : uint32_t {
    kTlCompress = 1, kTlTailUpdate, kTlIqProject, kTlIqProjectWide, kTlIndexer, kTlTopk, kTlPrepQ, kTlAttend,
    kTlCombine
};
#ifdef CSLA_TIMELINE
constexpr int kTimelineMarks = 8;
struct TimelineRec {
    uint32_t kernel, cta;
    unsigned long long t0, t1, t2, m[kTimelineMarks];
    unsigned long long clk0, clk2;   // SM cycle counter at start and exit
};
constexpr unsigned kTimelineCap = 1u << 16;
extern __device__ TimelineRec g_timeline[kTimelineCap];
extern __device__ unsigned int g_timeline_n;
__device__ __forceinline__ unsigned long long timeline_now() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
static __shared__ unsigned long long tl_marks[kTimelineMarks];   // per CTA; any thread may set a mark
__device__ __forceinline__ void timeline_mark(int i) { tl_marks[i] = timeline_now(); }
__device__ __forceinline__ unsigned long long timeline_clock() {
    unsigned long long c;
    asm volatile("mov.u64 %0, %%clock64;" : "=l"(c));
    return c;
}
struct TimelineScope {
    uint32_t k;
    unsigned long long t0, t1, c0;
    __device__ explicit TimelineScope(uint32_t kernel) : k(kernel), t0(timeline_now()), t1(0), c0(timeline_clock()) {
        if (threadIdx.x == 0)
            for (int i = 0; i < kTimelineMarks; ++i) tl_marks[i] = 0;
    }
    __device__ void waited() { t1 = timeline_now(); }
    __device__ ~TimelineScope() {
        if (threadIdx.x == 0) {
            const unsigned i = atomicAdd(&g_timeline_n, 1u);
            const uint32_t cta = (blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x;
            if (i < kTimelineCap) {
                TimelineRec r{k, cta, t0, t1, timeline_now(), {}, c0, timeline_clock()};
                for (int j = 0; j < kTimelineMarks; ++j) r.m[j] = tl_marks[j];
                g_timeline[i] = r;
            }
        }
    }
};
#define CSLA_TL_SCOPE(kernel) ::csla::TimelineScope csla_tl_scope_(kernel)
#define CSLA_TL_WAITED() csla_tl_scope_.waited()
#define CSLA_TL_MARK(i)                            \
    do {                                           \
        if (threadIdx.x == 0) ::csla::timeline_mark(i); \
    } while (0)
#define CSLA_TL_MARK_ANY(i) ::csla::timeline_mark(i)
#else
#define CSLA_TL_SCOPE(kernel) \
    do {                      \
    } while (0)
#define CSLA_TL_WAITED() \
    do {                 \
    } while (0)
#define CSLA_TL_MARK(i) \
    do {                \
    } while (0)
#define CSLA_TL_MARK_ANY(i) \
    do {                    \
    } while (0)
#endif

// ------------------------------------------------------------ smem / sync
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Bound of every wait on an mbarrier: far above any legitimate wait.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
// Add bytes to the current phase's expected transaction count (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// try_wait that lets the hardware suspend the thread until the phase
// completes or `ns` nanoseconds pass, instead of returning at once: a waiting
// warp then takes no issue slots from the warps doing the work.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}
constexpr uint32_t kWaitSleepNs = 1000000;   // 1 ms: bounds the reaction to an abort

// Wait for phase `parity` of `bar` to complete.  Gives up after limit_ns,
// records CSLA_DEVERR_TIMEOUT and returns false; also returns false at once
// when *abort (shared, may be null) is set by another role of the CTA.
__device__ __forceinline__ bool mbar_wait_limit(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                uint64_t limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint32_t sleep = limit_ns < kWaitSleepNs ? (uint32_t)limit_ns : kWaitSleepNs;
    uint64_t t0 = globaltimer_ns();
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, sleep)) return true;
        if (abort && *abort) return false;
        if (globaltimer_ns() - t0 > limit_ns) {
            set_dev_err(CSLA_DEVERR_TIMEOUT);
            if (abort) *abort = 1;
            return false;
        }
    }
}
// The wait every library kernel uses: limit kWaitLimitNs.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort) {
    return mbar_wait_limit(bar, parity, abort, kWaitLimitNs);
}

// One arrival per warp on an mbarrier initialised with a count of warps:
// every lane's earlier shared-memory (and, after a tcgen05 before-fence,
// TMEM) work is ordered before lane 0's release by the warp barrier.  All
// 32 lanes must call it.  (One arrival per thread costs a shared-memory
// atomic per lane on the same word, which serialises.)
__device__ __forceinline__ void mbar_arrive_warp(uint64_t *bar) {
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
// Warp-uniform outcome of a bounded wait: a lane that gave up makes the whole
// warp give up, so warp-collective instructions after it never see a split warp.
__device__ __forceinline__ bool warp_all(bool v) { return __all_sync(0xffffffffu, v); }

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------ TMA
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int32_t x, int32_t y,
                                            uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ------------------------------------------------------------ tcgen05
// UMMA shared-memory descriptor (sm_100 format: version 1 at bits 46-47,
// layout type at bits 61-63; addresses and offsets in 16-byte units).
constexpr uint32_t kLayoutSW128 = 2;

__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)kLayoutSW128 << 61;
    return d;
}

// Instruction descriptor of kind::f16 with f16 A/B, fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Instruction descriptor of kind::f16 with bf16 A/B, fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((b_mn_major ? 1u : 0u) << 16) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void umma_kind_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// kind::f8f6f4 with E4M3 A and B (K = 32 per instruction), fp32 accumulate.
__host__ __device__ constexpr uint32_t idesc_e4m3(int M, int N) {
    // c_format F32 (bit 4); a_format = b_format = E4M3 (0); both K-major
    return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_kind_f8f6f4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Warp-collective TMEM allocation; the base address lands in *dst (smem).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst)),
                 "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld32x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
                 : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32x16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]) : "memory");
}
__device__ __forceinline__ void tmem_st32x32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};"
                 :: "r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31]) : "memory");
}

// ------------------------------------------------------------ reductions
// Fixed-order reductions: per-thread partials are combined by a xor butterfly
// inside each warp and then warp 0..W-1 in order, so the result is a pure
// function of the inputs (no atomics, no dependence on scheduling).
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
// Block-wide sum / max for blockDim.x == 32*NW; `red` holds >= NW floats.
template <int NW>
__device__ __forceinline__ float block_sum(float v, float *red) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = red[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) s += red[i];
    return s;
}
template <int NW>
__device__ __forceinline__ float block_max(float v, float *red) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) red[w] = v;
    __syncthreads();
    float s = red[0];
#pragma unroll
    for (int i = 1; i < NW; ++i) s = fmaxf(s, red[i]);
    return s;
}

// cos and sin of pos * inv_freq.  The angle (up to ~2^21 rad) is reduced to
// [-pi, pi] first (Cody-Waite style: 2*pi split into a double pair, the
// product k*2pi removed with fused multiply-adds), then evaluated with the
// fp32 sincosf; the reduction keeps the fp32 result accurate for every
// position a 2^20-token context reaches.
__device__ __forceinline__ void rope_cos_sin(long long pos, double inv_freq, float *c, float *s) {
    const double kTwoPiHi = 6.283185307179586232;     // double nearest to 2*pi
    const double kTwoPiLo = 2.4492935982947064e-16;   // 2*pi - kTwoPiHi
    const double ang = (double)pos * inv_freq;
    const double k = rint(ang * 0.15915494309189535);  // 1 / (2*pi)
    double r = fma(-k, kTwoPiHi, ang);
    r = fma(-k, kTwoPiLo, r);
    sincosf((float)r, s, c);
}

}  // namespace csla
