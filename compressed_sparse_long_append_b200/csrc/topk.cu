// topk.cu -- top-k selector (csla_topk_select).
//
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力, CSA part: of all
//   compressed blocks only the k most relevant (512; 1024 for Pro) are kept.
//
// One CTA of 1024 threads per request.  Scores become order-preserving
// uint32 keys (-0.0 folded onto +0.0), staged in shared memory when the
// request's visible entries fit (else re-read from global memory each pass).
// The exact k-th largest key T is found by a radix select over 11/11/10 key
// bits: each pass builds a histogram of the keys matching the prefix so far
// (kCopies private copies, one per group of four warps, so that the
// shared-memory atomics of different groups never contend: scores crowd
// into few bins), sums the copies and picks the bin holding the remaining
// rank.  The first pass's histogram is built while the keys are staged.  The
// output pass keeps every key > T and the lowest-index keys == T: each warp
// owns a contiguous range, per-warp counts give its first slot and ballots
// place the picks, so indices come out ascending.  All counts are integers:
// the selection is exact and independent of thread timing and batch.
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kCopies = 8;                    // histogram copies (4 warps each)
constexpr int kBins = 2048;
constexpr int kSmemKeysMax = 36864;           // keys per request staged in shared memory
constexpr int kBatch = 16;                    // score loads a thread keeps in flight
constexpr size_t kHistBytes = (size_t)kBins * kCopies * sizeof(int);

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Shared {
    int hsum[kBins];           // summed histogram of the current pass
    int warp_a[kWarps], warp_b[kWarps];
    int sel_bin, sel_krem;
};

// Find the bin holding the krem-th largest key of hist[0..nb) (counted from
// the top).  Result in sh->sel_bin / sh->sel_krem.  All threads call it.
__device__ void pick_bin(Shared *sh, const int *hist, int nb, int krem) {
    const int per = nb / kThreads;   // bins per thread, highest first
    int c = 0;
    for (int q = 0; q < per; ++q) c += hist[nb - 1 - (threadIdx.x * per + q)];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int v = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    if (lane == 31) sh->warp_a[warp] = v;
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += sh->warp_a[w];
    const int incl = v + before;
    const int excl = incl - c;
    if (excl < krem && krem <= incl) {
        int run = excl;
        for (int q = 0; q < per; ++q) {
            const int bin = nb - 1 - (threadIdx.x * per + q);
            const int h = hist[bin];
            if (run + h >= krem) {
                sh->sel_bin = bin;
                sh->sel_krem = krem - run;
                break;
            }
            run += h;
        }
    }
    __syncthreads();
}

__device__ __forceinline__ void hist_zero(int *hist) {
    int4 *p = reinterpret_cast<int4 *>(hist);
    for (int i = threadIdx.x; i < kBins * kCopies / 4; i += kThreads) p[i] = make_int4(0, 0, 0, 0);
}

template <bool kSmemKeys>
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
    CSLA_TL_SCOPE(kTlTopk);
    extern __shared__ __align__(16) int dyn[];
    int *hist = dyn;                                                     // [kBins][kCopies]
    uint32_t *keys_s = reinterpret_cast<uint32_t *>(dyn + kBins * kCopies);   // [n] when staged
    __shared__ Shared sh;
    pdl_trigger();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int copy = warp & (kCopies - 1);
    const int slot = __ldg(a.slots + b);
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    hist_zero(hist);
    pdl_wait();
    CSLA_TL_WAITED();
    const int L = slot_ok ? a.len[slot] : 0;
    int n = L / a.m;
    if (!slot_ok || L > a.max_n * a.m) {
        if (threadIdx.x == 0) set_dev_err(CSLA_DEVERR_LEN);
        n = 0;
    }
    const int k = a.k;
    int32_t *out = a.idx + (size_t)b * k;
    const float *sc = a.scores + (size_t)b * a.stride;
    if (n <= k) {
        for (int j = threadIdx.x; j < k; j += kThreads) out[j] = j < n ? j : -1;
        return;
    }
    auto key_at = [&](int i) -> uint32_t { return kSmemKeys ? keys_s[i] : score_key(__ldg(sc + i)); };
    __syncthreads();   // zeroed histogram
    if (kSmemKeys) {
        // stage the keys (kBatch loads in flight per thread) and build the
        // first pass's histogram (top 11 key bits) on the way
        for (int i0 = 0; i0 < n; i0 += kThreads * kBatch) {
            float f[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * kThreads + threadIdx.x;
                f[u] = i < n ? sc[i] : 0.f;
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int i = i0 + u * kThreads + threadIdx.x;
                if (i < n) {
                    const uint32_t key = score_key(f[u]);
                    keys_s[i] = key;
                    atomicAdd(&hist[(key >> 21) * kCopies + copy], 1);
                }
            }
            if (i0 == 0) CSLA_TL_MARK(5);
        }
    }
    CSLA_TL_MARK(0);

    uint32_t prefix = 0, pmask = 0;
    int krem = k;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; ++pass) {
        const int shb = shifts[pass], nb = 1 << widths[pass];
        if (pass > 0 || !kSmemKeys) {
            if (pass > 0) {
                hist_zero(hist);
                __syncthreads();
            }
            for (int i = threadIdx.x; i < n; i += kThreads) {
                const uint32_t key = key_at(i);
                if ((key & pmask) == prefix) atomicAdd(&hist[((key >> shb) & (uint32_t)(nb - 1)) * kCopies + copy], 1);
            }
        }
        __syncthreads();
        for (int bin = threadIdx.x; bin < nb; bin += kThreads) {
            const int4 *h4 = reinterpret_cast<const int4 *>(hist + bin * kCopies);
            int t = 0;
#pragma unroll
            for (int j = 0; j < kCopies / 4; ++j) {
                const int4 v = h4[j];
                t += v.x + v.y + v.z + v.w;
            }
            sh.hsum[bin] = t;
        }
        __syncthreads();
        pick_bin(&sh, sh.hsum, nb, krem);
        prefix |= (uint32_t)sh.sel_bin << shb;
        pmask |= (uint32_t)(nb - 1) << shb;
        krem = sh.sel_krem;
        CSLA_TL_MARK(1 + pass);
    }
    // prefix is now the k-th largest key T; krem = how many keys == T to keep.
    const uint32_t T = prefix;

    // ---- output: warp w owns a contiguous part of the request's range
    const int seg = (n + kWarps - 1) / kWarps;
    const int wlo = min(n, warp * seg), whi = min(n, wlo + seg);
    int gt = 0, eq = 0;
    for (int i0 = wlo; i0 < whi; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < whi ? key_at(i) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, i < whi && key > T));
        eq += __popc(__ballot_sync(0xffffffffu, i < whi && key == T));
    }
    if (lane == 0) {
        sh.warp_a[warp] = gt;
        sh.warp_b[warp] = eq;
    }
    __syncthreads();
    CSLA_TL_MARK(4);
    int gt_before = 0, eq_before = 0;
    for (int w = 0; w < warp; ++w) {
        gt_before += sh.warp_a[w];
        eq_before += sh.warp_b[w];
    }
    int pos = gt_before + min(eq_before, krem);
    int eq_seen = eq_before;
    for (int i0 = wlo; i0 < whi; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < whi ? key_at(i) : 0u;
        const bool is_gt = i < whi && key > T;
        const bool is_eq = i < whi && key == T;
        const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
        const unsigned below = (1u << lane) - 1u;
        const bool take_eq = is_eq && (eq_seen + __popc(meq & below)) < krem;
        const unsigned mtake = __ballot_sync(0xffffffffu, is_gt || take_eq);
        if (is_gt || take_eq) out[pos + __popc(mtake & below)] = i;
        pos += __popc(mtake);
        eq_seen += __popc(meq);
    }
    CSLA_TL_MARK(6);
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)(kHistBytes + kSmemKeysMax * sizeof(uint32_t)));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kHistBytes);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    if (a.max_n <= kSmemKeysMax) {
        const size_t smem = kHistBytes + (size_t)(a.max_n > 0 ? a.max_n : 1) * sizeof(uint32_t);
        return launch_pdl(topk_kernel<true>, dim3(a.B), dim3(kThreads), smem, stream, a);
    }
    return launch_pdl(topk_kernel<false>, dim3(a.B), dim3(kThreads), kHistBytes, stream, a);
}

}  // namespace csla
