// topk.cu -- top-k selector (csla_topk_select).
//
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力, CSA part: of all
//   compressed blocks only the k most relevant (512; 1024 for Pro) are kept.
//
// One 1024-thread CTA per request.  Scores become order-preserving uint32
// keys (-0.0 folded onto +0.0); three histogram passes over 11/11/10 key bits
// find the exact k-th largest key T; a final pass keeps every key > T and the
// lowest-index keys == T, writing indices in ascending order.  All counts are
// integers, so the selection is exact and independent of thread timing.
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kSmemKeysMax = 40960;   // keys staged in shared memory up to this many

__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inclusive prefix sum over the block (thread order); returns this thread's
// inclusive sum, *total gets the block total.  `ws` holds kWarps ints.
__device__ __forceinline__ int block_incl_scan(int v, int *ws, int *total) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += t;
    }
    __syncthreads();
    if (lane == 31) ws[warp] = v;
    __syncthreads();
    if (warp == 0) {
        int w = ws[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += t;
        }
        ws[lane] = w;
    }
    __syncthreads();
    const int before = warp > 0 ? ws[warp - 1] : 0;
    *total = ws[kWarps - 1];
    return v + before;
}

template <bool kSmem>
__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
    extern __shared__ uint32_t keys_s[];
    __shared__ int hist[2048];
    __shared__ int ws[kWarps];
    __shared__ int s_bin, s_krem;

    const int b = blockIdx.x;
    const int slot = __ldg(a.slots + b);
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    const int L = slot_ok ? __ldg(a.len + slot) : 0;
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
    auto key_at = [&](int i) -> uint32_t { return kSmem ? keys_s[i] : score_key(__ldg(sc + i)); };
    if (kSmem) {
        for (int i = threadIdx.x; i < n; i += kThreads) keys_s[i] = score_key(__ldg(sc + i));
    }

    uint32_t prefix = 0, pmask = 0;
    int krem = k;
    const int shifts[3] = {21, 10, 0};
    const int widths[3] = {11, 11, 10};
    for (int pass = 0; pass < 3; ++pass) {
        const int sh = shifts[pass];
        const int nb = 1 << widths[pass];
        for (int i = threadIdx.x; i < 2048; i += kThreads) hist[i] = 0;
        __syncthreads();
        for (int i = threadIdx.x; i < n; i += kThreads) {
            const uint32_t key = key_at(i);
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> sh) & (nb - 1)], 1);
        }
        __syncthreads();
        // counts from the top bin down: thread t owns bins nb-1-2t, nb-2-2t
        const int per = nb / kThreads;   // 2 or 1
        int c = 0;
        for (int q = 0; q < per; ++q) c += hist[nb - 1 - (threadIdx.x * per + q)];
        int total;
        const int incl = block_incl_scan(c, ws, &total);
        const int excl = incl - c;
        if (excl < krem && krem <= incl) {
            int run = excl;
            for (int q = 0; q < per; ++q) {
                const int bin = nb - 1 - (threadIdx.x * per + q);
                if (run + hist[bin] >= krem) {
                    s_bin = bin;
                    s_krem = krem - run;
                    break;
                }
                run += hist[bin];
            }
        }
        __syncthreads();
        prefix |= (uint32_t)s_bin << sh;
        pmask |= (uint32_t)(nb - 1) << sh;
        krem = s_krem;
        __syncthreads();
    }
    // prefix is now the k-th largest key T; krem = how many keys == T to keep.
    const uint32_t T = prefix;
    const int seg = (n + kThreads - 1) / kThreads;
    const int lo = threadIdx.x * seg;
    const int hi = min(n, lo + seg);
    int gt = 0, eq = 0;
    for (int i = lo; i < hi; ++i) {
        const uint32_t key = key_at(i);
        gt += key > T;
        eq += key == T;
    }
    int tot;
    const int gt_before = block_incl_scan(gt, ws, &tot) - gt;
    const int eq_before = block_incl_scan(eq, ws, &tot) - eq;
    int pos = gt_before + min(eq_before, krem);
    int eq_seen = eq_before;
    for (int i = lo; i < hi; ++i) {
        const uint32_t key = key_at(i);
        if (key > T) {
            out[pos++] = i;
        } else if (key == T) {
            if (eq_seen < krem) out[pos++] = i;
            ++eq_seen;
        }
    }
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    if (a.max_n <= kSmemKeysMax) {
        const size_t smem = (size_t)(a.max_n > 0 ? a.max_n : 1) * sizeof(uint32_t);
        static int configured_dev = -1;
        int dev = 0;
        cudaGetDevice(&dev);
        if (configured_dev != dev) {
            cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 kSmemKeysMax * (int)sizeof(uint32_t));
            if (e != cudaSuccess) return e;
            configured_dev = dev;
        }
        topk_kernel<true><<<a.B, kThreads, smem, stream>>>(a);
    } else {
        topk_kernel<false><<<a.B, kThreads, 0, stream>>>(a);
    }
    return cudaGetLastError();
}

}  // namespace csla
