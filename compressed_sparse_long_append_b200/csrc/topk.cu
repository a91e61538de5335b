// topk.cu -- top-k selector (csla_topk_select) and the selection side of
// csla_indexer_topk (thresholds from a score sample, select among the
// candidates the indexer kept).
//
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力, CSA part: of all
//   compressed blocks only the k most relevant (512; 1024 for Pro) are kept.
//
// Scores become order-preserving uint32 keys (-0.0 folded onto +0.0).  The
// output is every key > T and the lowest-index keys == T, T the exact k-th
// largest key, indices ascending: each warp owns a contiguous range (or the
// candidates of one), per-warp counts give its first slot and ballots place
// the picks.  All counts are integers: the selection is exact and
// independent of thread timing and batch.  Two kernels: a cluster of four
// CTAs per request with the scores in registers (up to 36864 visible
// entries: decode), and one CTA per row streaming its scores (longer rows:
// query rows of a long prefill).  Both find T among the candidates above a
// sampled threshold, with a radix select over every key as the fallback.
// The fused call's select kernel applies the same rule to candidates that
// arrive in any order (the picks are marked in a bitmap over the entries).

#include <cooperative_groups.h>
#include <cstddef>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csla {
namespace {

constexpr int kBins = 2048;

// ---------------------------------------------------------------- selection with scores in registers
// The steps, as first written for one CTA of 512 threads (the cluster
// kernel below spreads them over 4 CTAs).  Warp w owns the contiguous
// range [w*seg, (w+1)*seg), seg = ceil(n / 16); lane l holds the scores
// w*seg + 32j + l (j < kPer) in registers, so a warp's ballots walk its
// range in index order.
//  1. Threshold t0 from a sample (no shared-memory pass): every warp sorts
//     32 keys spread over its range, one per lane (bitonic, shuffles), and
//     takes its rw-th largest; t0 is the smallest of these over the warps,
//     so at least 16*rw of the 512 sample keys are >= t0: rw = ceil(48k/n)
//     puts about 1.5k or more keys >= t0 in expectation.
//  2. One sweep converts the scores to keys and compacts the keys >= t0
//     (with their indices) into per-warp regions of shared memory, in index
//     order.  When every region fits and there are at least k of them, the
//     exact k-th largest key T is found among the candidates alone (every
//     key >= T is one of them) and the output is taken from the regions.
//  3. Otherwise (rare) T is found among all keys and the output is taken
//     from the registers.  Either way the output holds the keys > T and the
//     lowest-index keys == T, ascending.
// The radix selects use 11/11/10-bit digits and one shared histogram.
constexpr int kRThreads = 512;
constexpr int kRWarps = kRThreads / 32;
constexpr int kPer = 72;                          // scores per thread
constexpr int kRegMax = kPer * kRThreads;         // 36864
constexpr int kRegion = 512;                      // candidates per warp

// The float whose key is `key` (inverse of score_key; key 0 -> padding NaN).
__device__ __forceinline__ float key_value(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

struct RegShared {
    int hist[kBins];
    uint32_t ckey[kRWarps][kRegion];
    int cidx[kRWarps][kRegion];
    int cnt[kRWarps];
    uint32_t tw[kRWarps];
    int warp_a[kRWarps], warp_b[kRWarps];
    int sel_bin, sel_krem;
    uint32_t small[32];
    int small_n;
    uint32_t small_t;
};

// Exclusive prefix over the kRWarps per-warp values v[] for warp `warp`,
// and their total.  Every thread calls it after a barrier that published v[].
__device__ __forceinline__ int warp_prefix(const int *v, int warp, int *total) {
    const int lane = threadIdx.x & 31;
    const int x = lane < kRWarps ? v[lane] : 0;
    int incl = x;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    *total = __shfl_sync(0xffffffffu, incl, 31);
    return __shfl_sync(0xffffffffu, incl - x, warp);
}

// The bin of sh.hist[0..nb) holding the krem-th largest key (counted from
// the top): sh.sel_bin, and the rank within it: sh.sel_krem.  All threads.
template <typename SH>
__device__ void pick_bin_r(SH &sh, int nb, int krem) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    // thread t covers bins nb-1-t*per .. (highest first); per = 0 for t beyond nb
    const int per = (nb + kRThreads - 1) / kRThreads;
    int c = 0;
    for (int q = 0; q < per; ++q) {
        const int bin = nb - 1 - (threadIdx.x * per + q);
        if (bin >= 0) c += sh.hist[bin];
    }
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sh.warp_a[warp] = incl;
    __syncthreads();
    int total;
    const int before = warp_prefix(sh.warp_a, warp, &total);
    const int excl = before + incl - c;
    if (excl < krem && krem <= excl + c) {
        int run = excl;
        for (int q = 0; q < per; ++q) {
            const int bin = nb - 1 - (threadIdx.x * per + q);
            const int h = bin >= 0 ? sh.hist[bin] : 0;
            if (run + h >= krem) {
                sh.sel_bin = bin;
                sh.sel_krem = krem - run;
                break;
            }
            run += h;
        }
    }
    __syncthreads();
}

// Radix select: the key of rank `rank` (1 = largest) among the non-zero keys
// that each thread passes to the callback given to each(), all of which
// share their top 32 - bits bits with `prefix`; *krem_out = how many keys
// equal to the result are within that rank.  Digits of up to 11 bits, from
// the top of the `bits` low bits down.
template <typename SH, typename Each>
__device__ uint32_t radix_select(SH &sh, const Each &each, int rank, uint32_t prefix, int bits,
                                 int *krem_out) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t pmask = bits >= 32 ? 0u : ~((1u << bits) - 1u);
    prefix &= pmask;
    int krem = rank;
#pragma unroll 1
    for (int left = bits; left > 0;) {
        const int width = left > 11 ? 11 : left;
        const int shb = left - width;
        const int nb = 1 << width;
        left = shb;
        // every thread has read the previous digit's hist[sel] (the small-bin
        // test below) before any thread clears it: without this barrier a
        // fast thread's clearing can flip a slow thread's test, the threads
        // then take different paths through the barriers that follow
        __syncthreads();
        for (int i = threadIdx.x; i < kBins; i += kRThreads) sh.hist[i] = 0;
        __syncthreads();
        each([&](uint32_t key) {
            if (key != 0u && (key & pmask) == prefix) atomicAdd(&sh.hist[(key >> shb) & (uint32_t)(nb - 1)], 1);
        });
        __syncthreads();
        pick_bin_r(sh, nb, krem);
        const int sel = sh.sel_bin;
        prefix |= (uint32_t)sel << shb;
        pmask |= (uint32_t)(nb - 1) << shb;
        krem = sh.sel_krem;
        if (left > 0 && sh.hist[sel] <= 32) {
            // at most 32 keys left in the bin: gather them and let one warp
            // sort them (bitonic, descending) instead of further passes
            if (threadIdx.x == 0) sh.small_n = 0;
            __syncthreads();
            each([&](uint32_t key) {
                if (key != 0u && (key & pmask) == prefix) {
                    const int at = atomicAdd(&sh.small_n, 1);
                    if (at < 32) sh.small[at] = key;
                }
            });
            __syncthreads();
            if (warp == 0) {
                uint32_t v = lane < sh.small_n ? sh.small[lane] : 0u;
#pragma unroll
                for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
                    for (int stride = size >> 1; stride > 0; stride >>= 1) {
                        const uint32_t o = __shfl_xor_sync(0xffffffffu, v, stride);
                        const bool desc = (lane & size) == 0 || size == 32;
                        const bool lower = (lane & stride) == 0;
                        v = (lower == desc) ? max(v, o) : min(v, o);
                    }
                }
                const uint32_t t = __shfl_sync(0xffffffffu, v, krem - 1);
                // keys == t among the first krem of the sorted bin
                const int eqn = __popc(__ballot_sync(0xffffffffu, lane < krem && v == t));
                if (lane == 0) {
                    sh.small_t = t;
                    sh.sel_krem = eqn;
                }
            }
            __syncthreads();
            *krem_out = sh.sel_krem;
            return sh.small_t;
        }
    }
    *krem_out = krem;
    return prefix;
}

// ---------------------------------------------------------------- cluster variant
// For n <= kRegMax: one cluster of kG = 4 CTAs (512 threads each) per
// request; CTA c owns the c-th quarter of the scores, warp w of it a
// contiguous range, lane l the scores 32j + l of that range (18 rows) in
// registers.  The steps above, spread over the cluster:
//  1. every warp sorts a 32-key sample of its range and publishes its
//     2nd-largest key; after a cluster barrier every CTA reads all 64 and
//     takes the j-th largest as the threshold t0 (j = ceil(2048k/n), at
//     most 64), so that about 2k keys or more lie above it;
//  2. each warp compacts its scores >= t0 into its own region (index
//     order) and publishes the count; after a cluster barrier every CTA
//     reads the 64 counts, and when every region fitted and there are at
//     least k candidates, copies its regions into CTA 0's shared memory at
//     their exclusive-prefix offsets (so CTA 0 holds all candidates in
//     index order);
//  3. after a third barrier CTA 0 finds the exact k-th key among the
//     candidates and writes the output, as in the steps above.
// Otherwise (rare: heavy ties, or a sample far off) all four CTAs run the
// radix select over every key with their four histograms summed through
// distributed shared memory, and each writes its own picks.
constexpr int kG = 4;
constexpr int kCPer = kPer / kG;                  // 18 scores per thread
constexpr int kOwn = 128;                         // candidates per warp region

struct ClShared {
    RegShared reg;                                // CTA 0: gathered candidates and select scratch
    uint32_t okey[kRWarps][kOwn];
    int oidx[kRWarps][kOwn];
    int ocnt[kRWarps];
    uint32_t tw[kRWarps], wmax[kRWarps];
    int hist[kBins];                              // fallback: this CTA's histogram
    int fgt[kRWarps], feq[kRWarps];               // fallback: per-warp output counts
};

__global__ void __cluster_dims__(kG, 1, 1) __launch_bounds__(kRThreads, 1) topk_cluster_kernel(TopkArgs a) {
    CSLA_TL_SCOPE(kTlTopk);
    extern __shared__ __align__(16) uint8_t dyn_cl[];
    ClShared &sh = *reinterpret_cast<ClShared *>(dyn_cl);
    pdl_trigger();
    cg::cluster_group cl = cg::this_cluster();
    const int cr = (int)cl.block_rank();
    const int b = blockIdx.x / kG;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    const int slot = __ldg(a.slots + b);
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    pdl_wait();
    CSLA_TL_WAITED();
    const int L = slot_ok ? row_visible_len(a.len, a.q_len, slot, b) : 0;
    int n = L < 0 ? 0 : L / a.m;
    if (!slot_ok || L < 0 || L / a.m > a.max_n) {
        if (threadIdx.x == 0 && cr == 0) set_dev_err(CSLA_DEVERR_LEN);
        n = 0;
    }
    const int k = a.k;
    int32_t *out = a.idx + (size_t)b * k;
    if (a.row_flag && a.row_flag[b] == 0) return;   // the same decision in every CTA of the cluster
    if (n <= k) {   // the same decision in every CTA of the cluster
        if (cr == 0)
            for (int j = threadIdx.x; j < k; j += kRThreads) out[j] = j < n ? j : -1;
        return;
    }
    const float *sc = a.scores + (size_t)b * a.stride;
    const int segc = (n + kG - 1) / kG;
    const int c0 = min(n, cr * segc), cn = min(n, c0 + segc) - c0;
    const int seg = (cn + kRWarps - 1) / kRWarps;
    const int wlo = warp * seg;                   // the warp's range, relative to c0
    const int base = c0 + wlo;
    float f[kCPer];
#pragma unroll
    for (int j = 0; j < kCPer; ++j) {
        const int r = 32 * j + lane;
        f[j] = (r < seg && wlo + r < cn) ? sc[base + r] : __int_as_float(-1);   // the NaN whose key is 0
    }
    CSLA_TL_MARK(0);

    // ---- 1. threshold: per-warp sorted sample, smallest rw-th largest over the cluster
    const int js = (lane * ((seg + 31) >> 5)) >> 5;
    uint32_t smp = 0;
#pragma unroll
    for (int j = 0; j < kCPer; ++j)
        if (j == js) smp = score_key(f[j]);
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xffffffffu, smp, stride);
            const bool desc = (lane & size) == 0 || size == 32;
            const bool lower = (lane & stride) == 0;
            smp = (lower == desc) ? max(smp, o) : min(smp, o);
        }
    }
    // each warp publishes its 2nd-largest sample key; t0 = the j-th largest of
    // the 64 published keys, so that >= 2j samples (1 per n/2048 keys) are
    // >= t0: j = ceil(k * 2048 / n) puts about 2k keys or more above t0
    const uint32_t s_w = __shfl_sync(0xffffffffu, smp, 1);
    if (lane == 0) sh.tw[warp] = s_w;
    cl.sync();
    const int jth = min(2 * kRWarps * kG, max(1, (int)((2048LL * k + n - 1) / n)));
    const uint32_t v0 = cl.map_shared_rank(sh.tw, lane / kRWarps)[lane % kRWarps];
    const uint32_t v1 = cl.map_shared_rank(sh.tw, 2 + lane / kRWarps)[lane % kRWarps];
    // rank of each value (larger first, ties by position) among the 64
    int r0 = 0, r1 = 0;
#pragma unroll 8
    for (int q = 0; q < 32; ++q) {
        const uint32_t w0 = __shfl_sync(0xffffffffu, v0, q), w1 = __shfl_sync(0xffffffffu, v1, q);
        r0 += (w0 > v0 || (w0 == v0 && q < lane)) + (w1 > v0);
        r1 += (w0 > v1 || w0 == v1) + (w1 > v1 || (w1 == v1 && q < lane));
    }
    const unsigned h0 = __ballot_sync(0xffffffffu, r0 == jth - 1), h1 = __ballot_sync(0xffffffffu, r1 == jth - 1);
    const uint32_t t0 = h0 ? __shfl_sync(0xffffffffu, v0, __ffs(h0) - 1) : __shfl_sync(0xffffffffu, v1, __ffs(h1) - 1);
    CSLA_TL_MARK(1);

    // ---- 2. this warp's candidates (scores >= the value of t0) into its region
    const float f0 = t0 == 0u ? -INFINITY : key_value(t0);
    int pos = 0;
    uint32_t cmax = 0;
#pragma unroll
    for (int j = 0; j < kCPer; ++j) {
        const bool q = f[j] >= f0;
        const unsigned mq = __ballot_sync(0xffffffffu, q);
        const int at = pos + __popc(mq & below);
        if (q && at < kOwn) {
            const uint32_t key = score_key(f[j]);
            sh.okey[warp][at] = key;
            sh.oidx[warp][at] = base + 32 * j + lane;
            cmax = max(cmax, key);
        }
        pos += __popc(mq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    if (lane == 0) {
        sh.ocnt[warp] = pos;
        sh.wmax[warp] = cmax;
    }
    cl.sync();
    // the 64 counts in (CTA, warp) order: lane l holds entries l and 32 + l
    const int *rc0 = cl.map_shared_rank(sh.ocnt, lane / kRWarps);
    const int *rc1 = cl.map_shared_rank(sh.ocnt, 2 + lane / kRWarps);
    const int n0 = rc0[lane % kRWarps], n1 = rc1[lane % kRWarps];
    uint32_t kmax = max(cl.map_shared_rank(sh.wmax, lane / kRWarps)[lane % kRWarps],
                        cl.map_shared_rank(sh.wmax, 2 + lane / kRWarps)[lane % kRWarps]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    const bool fits = __all_sync(0xffffffffu, n0 <= kOwn && n1 <= kOwn);
    int i0 = n0, i1 = n1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, i0, o);
        const int u = __shfl_up_sync(0xffffffffu, i1, o);
        if (lane >= o) {
            i0 += t;
            i1 += u;
        }
    }
    const int tot0 = __shfl_sync(0xffffffffu, i0, 31);
    const int n_ge = tot0 + __shfl_sync(0xffffffffu, i1, 31);
    const int e = cr * kRWarps + warp;            // this warp's entry in (CTA, warp) order
    const int off = e < 32 ? __shfl_sync(0xffffffffu, i0 - n0, e)
                           : tot0 + __shfl_sync(0xffffffffu, i1 - n1, e - 32);
    const bool fast = fits && n_ge >= k;
    if (fast) {
        uint32_t *gk = cl.map_shared_rank(&sh.reg.ckey[0][0], 0);
        int *gi = cl.map_shared_rank(&sh.reg.cidx[0][0], 0);
        const int my = sh.ocnt[warp];
        for (int i = lane; i < my; i += 32) {
            gk[off + i] = sh.okey[warp][i];
            gi[off + i] = sh.oidx[warp][i];
        }
    }
    cl.sync();
    CSLA_TL_MARK(2);

    if (fast) {
        if (cr != 0) return;
        // ---- 3. CTA 0: warp w takes the flat candidates [512w, 512w + 512)
        RegShared &rs = sh.reg;
        const int my_n = min(kRegion, max(0, n_ge - warp * kRegion));
        int krem;
        const int bits = 32 - __clz(t0 ^ kmax);
        const uint32_t T = radix_select(rs, [&](auto fn) {
            for (int i = lane; i < my_n; i += 32) fn(rs.ckey[warp][i]);
        }, k, kmax, bits, &krem);
        CSLA_TL_MARK(3);
        int gt = 0, eq = 0;
        for (int i = lane; i < my_n; i += 32) {
            const uint32_t key = rs.ckey[warp][i];
            gt += key > T;
            eq += key == T;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, o);
            eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        if (lane == 0) {
            rs.warp_a[warp] = gt;
            rs.warp_b[warp] = eq;
        }
        __syncthreads();
        int tot;
        const int gt_before = warp_prefix(rs.warp_a, warp, &tot);
        const int eq_before = warp_prefix(rs.warp_b, warp, &tot);
        int opos = gt_before + min(eq_before, krem);
        int eq_seen = eq_before;
        for (int i0 = 0; i0 < my_n; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t key = i < my_n ? rs.ckey[warp][i] : 0u;
            const bool is_gt = i < my_n && key > T;
            const bool is_eq = i < my_n && key == T;
            const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
            const bool take_eq = is_eq && (eq_seen + __popc(meq & below)) < krem;
            const unsigned mtake = __ballot_sync(0xffffffffu, is_gt || take_eq);
            if (is_gt || take_eq) out[opos + __popc(mtake & below)] = rs.cidx[warp][i];
            opos += __popc(mtake);
            eq_seen += __popc(meq);
        }
        CSLA_TL_MARK(4);
        return;
    }

    // ---- fallback: radix select over every key, histograms summed across the cluster
    RegShared &rs = sh.reg;
    uint32_t prefix = 0, pmask = 0;
    int krem = k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shb = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        for (int i = threadIdx.x; i < kBins; i += kRThreads) sh.hist[i] = 0;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kCPer; ++j) {
            const uint32_t key = score_key(f[j]);
            if (key != 0u && (key & pmask) == prefix) atomicAdd(&sh.hist[(key >> shb) & (uint32_t)(nb - 1)], 1);
        }
        cl.sync();
        for (int i = threadIdx.x; i < nb; i += kRThreads) {
            int t = 0;
#pragma unroll
            for (int q = 0; q < kG; ++q) t += cl.map_shared_rank(sh.hist, q)[i];
            rs.hist[i] = t;
        }
        __syncthreads();
        pick_bin_r(rs, nb, krem);
        prefix |= (uint32_t)rs.sel_bin << shb;
        pmask |= (uint32_t)(nb - 1) << shb;
        krem = rs.sel_krem;
        cl.sync();   // every CTA has read every histogram before the next pass clears them
    }
    const uint32_t T = prefix;
    int gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < kCPer; ++j) {
        const uint32_t key = score_key(f[j]);
        gt += __popc(__ballot_sync(0xffffffffu, key > T));
        eq += __popc(__ballot_sync(0xffffffffu, key == T));
    }
    if (lane == 0) {
        sh.fgt[warp] = gt;
        sh.feq[warp] = eq;
    }
    cl.sync();
    // keys before this warp: the lower CTAs' warps, then this CTA's lower warps
    int gt_before = 0, eq_before = 0;
    for (int q = 0; q < cr; ++q) {
        const int *rg = cl.map_shared_rank(sh.fgt, q), *re = cl.map_shared_rank(sh.feq, q);
        gt_before += lane < kRWarps ? rg[lane] : 0;
        eq_before += lane < kRWarps ? re[lane] : 0;
    }
    if (lane < kRWarps && lane < warp) {
        gt_before += sh.fgt[lane];
        eq_before += sh.feq[lane];
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        gt_before += __shfl_xor_sync(0xffffffffu, gt_before, o);
        eq_before += __shfl_xor_sync(0xffffffffu, eq_before, o);
    }
    int opos = gt_before + min(eq_before, krem);
    int eq_seen = eq_before;
#pragma unroll
    for (int j = 0; j < kCPer; ++j) {
        const uint32_t key = score_key(f[j]);
        const bool is_gt = key > T;
        const bool is_eq = key == T;
        const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
        const bool take_eq = is_eq && (eq_seen + __popc(meq & below)) < krem;
        const unsigned mtake = __ballot_sync(0xffffffffu, is_gt || take_eq);
        if (is_gt || take_eq) out[opos + __popc(mtake & below)] = base + 32 * j + lane;
        opos += __popc(mtake);
        eq_seen += __popc(meq);
    }
    cl.sync();   // no CTA leaves while another may still read its counts
}

// ---------------------------------------------------------------- streaming variant
// For n > kRegMax (query rows of a long prefill): one CTA of 512 threads per
// row, the row's scores read from global memory once on the fast path.
// Warp w owns the contiguous range [w*seg, (w+1)*seg), seg = ceil(n / 16).
//  1. Threshold from a sample: every lane takes the largest of S keys
//     spread over its warp's range (S = ceil(n / 6k), at most 64), every
//     warp sorts its 32 and takes the rw-th largest, rw = ceil(48kS / n)
//     (about 8); t0 is the smallest of these, so about 1.5k or more keys
//     lie at or above it whatever the row length, and the warps' regions
//     rarely overflow (a larger sample keeps the smallest of the 16
//     estimates close to the others).
//  2. One streaming sweep (8 loads in flight per lane) compacts the keys
//     >= t0, with their indices, into the warp's region, in index order.
//  3. When every region fitted and there are at least k candidates, the
//     exact k-th largest key T is found among them (every key >= T is one)
//     and the output is written from the regions; otherwise (heavy ties, a
//     sample far off) a radix select over all keys re-reads the row, and
//     the output pass walks it once more.  Either way the output is the
//     keys > T and the lowest-index keys == T, ascending.
constexpr int kSBatch = 8;   // score loads a lane keeps in flight in the sweep

// Row b of the streaming top-k: every thread of the CTA runs it, and every
// barrier inside is taken by all of them or by none.
__device__ void stream_row(const TopkArgs &a, RegShared &sh, int b) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const unsigned below = (1u << lane) - 1u;
    const int slot = __ldg(a.slots + b);
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    const int L = slot_ok ? row_visible_len(a.len, a.q_len, slot, b) : 0;
    int n = L < 0 ? 0 : L / a.m;
    if (!slot_ok || L < 0 || L / a.m > a.max_n) {
        if (threadIdx.x == 0) set_dev_err(CSLA_DEVERR_LEN);
        n = 0;
    }
    const int k = a.k;
    int32_t *out = a.idx + (size_t)b * k;
    if (n <= k) {
        for (int j = threadIdx.x; j < k; j += kRThreads) out[j] = j < n ? j : -1;
        return;
    }
    const float *sc = a.scores + (size_t)b * a.stride;
    const int seg = (n + kRWarps - 1) / kRWarps;
    const int wlo = min(n, warp * seg), whi = min(n, wlo + seg);

    // ---- 1. threshold from a per-warp sample: lane l keeps the largest of
    // its S keys spread over the warp's range
    const int ns = whi - wlo;
    const int S = min(64, max(1, (int)(((long long)n + 6LL * k - 1) / (6LL * k))));
    uint32_t smp = 0;
    if (ns > 0) {
        const long long span = 32LL * S;
        for (int u = 0; u < S; ++u)
            smp = max(smp, score_key(__ldg(sc + wlo + (int)(((long long)(lane * S + u) * ns) / span))));
    }
#pragma unroll
    for (int size = 2; size <= 32; size <<= 1) {
#pragma unroll
        for (int stride = size >> 1; stride > 0; stride >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xffffffffu, smp, stride);
            const bool desc = (lane & size) == 0 || size == 32;
            const bool lower = (lane & stride) == 0;
            smp = (lower == desc) ? max(smp, o) : min(smp, o);
        }
    }
    const int rw = min(32, max(1, (int)((48LL * k * S + n - 1) / n)));
    const uint32_t s_w = __shfl_sync(0xffffffffu, smp, rw - 1);
    if (lane == 0) sh.tw[warp] = ns > 0 ? s_w : 0xFFFFFFFFu;   // an empty range imposes nothing
    __syncthreads();
    uint32_t t0 = lane < kRWarps ? sh.tw[lane] : 0xFFFFFFFFu;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) t0 = min(t0, __shfl_xor_sync(0xffffffffu, t0, o));
    CSLA_TL_MARK(0);

    // ---- 2. this warp's keys >= t0 into its region, in index order
    int pos = 0;
    uint32_t cmax = 0;
    for (int i0 = wlo; i0 < whi; i0 += 32 * kSBatch) {
        float f[kSBatch];
#pragma unroll
        for (int u = 0; u < kSBatch; ++u) {
            const int i = i0 + 32 * u + lane;
            f[u] = i < whi ? __ldg(sc + i) : 0.f;
        }
#pragma unroll
        for (int u = 0; u < kSBatch; ++u) {
            const int i = i0 + 32 * u + lane;
            const uint32_t key = score_key(f[u]);
            const bool q = i < whi && key >= t0;
            const unsigned mq = __ballot_sync(0xffffffffu, q);
            const int at = pos + __popc(mq & below);
            if (q && at < kRegion) {
                sh.ckey[warp][at] = key;
                sh.cidx[warp][at] = i;
            }
            if (q) cmax = max(cmax, key);
            pos += __popc(mq);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cmax = max(cmax, __shfl_xor_sync(0xffffffffu, cmax, o));
    if (lane == 0) {
        sh.cnt[warp] = pos;
        sh.warp_b[warp] = (int)cmax;
    }
    __syncthreads();
    const int cn = lane < kRWarps ? sh.cnt[lane] : 0;
    const bool fits = __all_sync(0xffffffffu, cn <= kRegion);
    int n_ge = cn;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) n_ge += __shfl_xor_sync(0xffffffffu, n_ge, o);
    uint32_t kmax = lane < kRWarps ? (uint32_t)sh.warp_b[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    CSLA_TL_MARK(1);
    __syncthreads();   // warp_b is reused below

    if (fits && n_ge >= k) {
        // ---- 3. the exact k-th key among the candidates, output from the regions
        const int my_n = sh.cnt[warp];
        int krem;
        const int bits = 32 - __clz(t0 ^ kmax);
        const uint32_t T = radix_select(sh, [&](auto fn) {
            for (int i = lane; i < my_n; i += 32) fn(sh.ckey[warp][i]);
        }, k, kmax, bits, &krem);
        CSLA_TL_MARK(2);
        int gt = 0, eq = 0;
        for (int i = lane; i < my_n; i += 32) {
            const uint32_t key = sh.ckey[warp][i];
            gt += key > T;
            eq += key == T;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            gt += __shfl_xor_sync(0xffffffffu, gt, o);
            eq += __shfl_xor_sync(0xffffffffu, eq, o);
        }
        if (lane == 0) {
            sh.warp_a[warp] = gt;
            sh.warp_b[warp] = eq;
        }
        __syncthreads();
        int tot;
        const int gt_before = warp_prefix(sh.warp_a, warp, &tot);
        const int eq_before = warp_prefix(sh.warp_b, warp, &tot);
        int opos = gt_before + min(eq_before, krem);
        int eq_seen = eq_before;
        for (int i0 = 0; i0 < my_n; i0 += 32) {
            const int i = i0 + lane;
            const uint32_t key = i < my_n ? sh.ckey[warp][i] : 0u;
            const bool is_gt = i < my_n && key > T;
            const bool is_eq = i < my_n && key == T;
            const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
            const bool take_eq = is_eq && (eq_seen + __popc(meq & below)) < krem;
            const unsigned mtake = __ballot_sync(0xffffffffu, is_gt || take_eq);
            if (is_gt || take_eq) {
                const int p = opos + __popc(mtake & below);
                if (p >= 0 && p < k) out[p] = sh.cidx[warp][i];
                else set_dev_err(CSLA_DEVERR_INDEX);   // never for a correct selection
            }
            opos += __popc(mtake);
            eq_seen += __popc(meq);
        }
        CSLA_TL_MARK(3);
        return;
    }

    // ---- fallback: radix select over every key, re-read from global memory
    int krem;
    const uint32_t T = radix_select(sh, [&](auto fn) {
        for (int i = wlo + lane; i < whi; i += 32) fn(score_key(__ldg(sc + i)));
    }, k, 0u, 32, &krem);
    int gt = 0, eq = 0;
    for (int i0 = wlo; i0 < whi; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < whi ? score_key(__ldg(sc + i)) : 0u;
        gt += __popc(__ballot_sync(0xffffffffu, i < whi && key > T));
        eq += __popc(__ballot_sync(0xffffffffu, i < whi && key == T));
    }
    if (lane == 0) {
        sh.warp_a[warp] = gt;
        sh.warp_b[warp] = eq;
    }
    __syncthreads();
    int tot;
    const int gt_before = warp_prefix(sh.warp_a, warp, &tot);
    const int eq_before = warp_prefix(sh.warp_b, warp, &tot);
    int opos = gt_before + min(eq_before, krem);
    int eq_seen = eq_before;
    for (int i0 = wlo; i0 < whi; i0 += 32) {
        const int i = i0 + lane;
        const uint32_t key = i < whi ? score_key(__ldg(sc + i)) : 0u;
        const bool is_gt = i < whi && key > T;
        const bool is_eq = i < whi && key == T;
        const unsigned meq = __ballot_sync(0xffffffffu, is_eq);
        const bool take_eq = is_eq && (eq_seen + __popc(meq & below)) < krem;
        const unsigned mtake = __ballot_sync(0xffffffffu, is_gt || take_eq);
        if (is_gt || take_eq) {
            const int p = opos + __popc(mtake & below);
            if (p >= 0 && p < k) out[p] = i;
            else set_dev_err(CSLA_DEVERR_INDEX);   // never for a correct selection
        }
        opos += __popc(mtake);
        eq_seen += __popc(meq);
    }
    CSLA_TL_MARK(4);
}

// One row per CTA; with row flags (the fallback of the fused indexer +
// top-k: most rows unflagged) a grid of two CTAs per SM walks the rows and
// skips the unflagged ones.
__global__ void __launch_bounds__(kRThreads, 2) topk_stream_kernel(TopkArgs a) {
    CSLA_TL_SCOPE(kTlTopk);
    extern __shared__ __align__(16) uint8_t dyn_st[];
    RegShared &sh = *reinterpret_cast<RegShared *>(dyn_st);
    pdl_trigger();
    pdl_wait();
    CSLA_TL_WAITED();
    for (int b = blockIdx.x; b < a.B; b += gridDim.x) {
        if (a.row_flag && a.row_flag[b] == 0) continue;   // the same for every thread
        stream_row(a, sh, b);
        __syncthreads();   // the next row reuses the shared memory
    }
}

// ---------------------------------------------------------------- streaming selection (csla_indexer_topk)
// The indexer scores the long rows without storing their scores.  A sample
// pass scores 32 pages (32 entries each) of each row, spread evenly
// (page_step apart); the threshold kernel takes as t0 the key that about
// cand_target(k) of the row's keys reach (the r-th largest of the valid
// sample keys, r the target scaled by sample size over row length); the
// candidate pass appends every (key, entry) at or above t0; the select
// kernel finds the exact top-k among them when there are at least k and at
// most kSelCap, and otherwise flags the row for the plain path (scores
// stored, then the streaming top-k).  The output never depends on t0: when
// at least k keys reach it, every key at or above the k-th largest is a
// candidate.
struct SelShared {
    int hist[kBins];
    int warp_a[kRWarps];
    int sel_bin, sel_krem;
    uint32_t small[32];
    int small_n;
    uint32_t small_t;
};

// Candidates a select CTA holds: 6144 of the kCandCap a row may keep (three
// CTAs per SM fit; more than 6144 candidates send the row to the fallback).
constexpr int kSelCap = 6144;

// Candidates aimed for per row: 3k, at least 2048 and at most half of
// kCandCap, so that a sample of ~1000 keys rarely lands outside [k, kSelCap].
__device__ __forceinline__ int cand_target(int k) { return min(kCandCap / 2, max(2048, 3 * k)); }

// Entries of row b: n = L/m, 0 (and the LEN bit) for a bad slot or length.
__device__ __forceinline__ int cand_row_n(const TopkArgs &a, int b, int slot, bool report) {
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    const int L = slot_ok ? row_visible_len(a.len, a.q_len, slot, b) : 0;
    if (!slot_ok || L < 0 || L / a.m > a.max_n) {
        if (report && threadIdx.x == 0) set_dev_err(CSLA_DEVERR_LEN);
        return 0;
    }
    return L / a.m;
}

// One warp per row: the r-th largest valid sample key, exactly, by a radix
// select over 8-bit digits (a 256-bin histogram per warp in shared memory,
// four passes).  Lane l holds sample column 32j + l (page j, entry l of the
// page) for every j.
constexpr int kThrWarps = 8;
__global__ void __launch_bounds__(32 * kThrWarps) cand_threshold_kernel(TopkArgs a, CandArgs c) {
    __shared__ int hist_all[kThrWarps][256];
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.x * kThrWarps + warp;
    if (b >= a.B) return;   // warp-uniform; the warps never wait on one another
    const int slot = __ldg(a.slots + b);
    pdl_wait();
    const int n = cand_row_n(a, b, slot, false);
    uint32_t t0 = 0u;   // rows of at most kSelCap entries: every entry is a candidate
    if (n > kSelCap && n > a.k) {
        // sample column 32*j + i holds entry 32*j*Z + i (when below n)
        const int Z = c.page_step;
        const float *sp = c.sample + (size_t)b * kSampleCols;
        uint32_t key[kSampleCols / 32];
        int ns = 0;
#pragma unroll
        for (int j = 0; j < kSampleCols / 32; ++j) {
            key[j] = j * Z * 32 + lane < n ? score_key(sp[32 * j + lane]) : 0u;
            ns += max(0, min(32, n - j * Z * 32));
        }
        if (ns > 0) {
            int r = (int)min((long long)ns, max(1LL, ((long long)cand_target(a.k) * ns + n - 1) / n));
            int *hist = hist_all[warp];
            uint32_t prefix = 0u, pmask = 0u;
            for (int shift = 24; shift >= 0; shift -= 8) {
                for (int i = lane; i < 256; i += 32) hist[i] = 0;
                __syncwarp();
#pragma unroll
                for (int j = 0; j < kSampleCols / 32; ++j)
                    if (key[j] != 0u && (key[j] & pmask) == prefix) atomicAdd(&hist[(key[j] >> shift) & 255u], 1);
                __syncwarp();
                // lane l counts bins 255 - 8l .. 248 - 8l (from the top)
                int cnt[8], sum = 0;
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    cnt[q] = hist[255 - 8 * lane - q];
                    sum += cnt[q];
                }
                int incl = sum;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(0xffffffffu, incl, o);
                    if (lane >= o) incl += t;
                }
                const int excl = incl - sum;
                const bool mine = excl < r && r <= incl;
                const int src = __ffs(__ballot_sync(0xffffffffu, mine)) - 1;
                int sel = 0, rem = 0;
                if (mine) {
                    int run = excl;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        if (sel == 0 && rem == 0 && run + cnt[q] >= r) {
                            sel = 255 - 8 * lane - q;
                            rem = r - run;
                        }
                        run += cnt[q];
                    }
                }
                sel = __shfl_sync(0xffffffffu, sel, src);
                r = __shfl_sync(0xffffffffu, rem, src);
                prefix |= (uint32_t)sel << shift;
                pmask |= 0xFFu << shift;
                __syncwarp();
            }
            t0 = prefix;
        }
    }
    if (lane == 0) c.cand_t0[b] = t0;
    if (lane < kCandSub) c.cand_cnt[b * kCandSub + lane] = 0;
}

struct CandShared {
    SelShared s;
    uint32_t key[kSelCap];
    int ent[kSelCap];
    uint32_t wmax[kRWarps];
    int neq;
    uint32_t bm[1];   // [bm_words]: bitmap of the picked entries (dynamic size)
};
constexpr int kCandFixed = (int)offsetof(CandShared, bm);
constexpr int kCandBmMax = (232448 - kCandFixed) / 4;   // bitmap words that fit the shared memory

// One CTA per row: the exact top-k among the row's candidates (the keys >
// T, then of the keys == T those of lowest entry), marked in a bitmap over
// the row's entries and written in entry order.
__global__ void __launch_bounds__(kRThreads) cand_select_kernel(TopkArgs a, CandArgs c, int bm_words) {
    CSLA_TL_SCOPE(kTlTopk);
    extern __shared__ __align__(16) uint8_t dyn_cs[];
    CandShared &sh = *reinterpret_cast<CandShared *>(dyn_cs);
    pdl_trigger();
    const int b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int slot = __ldg(a.slots + b);
    pdl_wait();
    CSLA_TL_WAITED();
    const int n = cand_row_n(a, b, slot, true);
    const int k = a.k;
    int32_t *out = a.idx + (size_t)b * k;
    if (n <= k) {
        for (int j = threadIdx.x; j < k; j += kRThreads) out[j] = j < n ? j : -1;
        if (threadIdx.x == 0) c.row_flag[b] = 0;
        return;
    }
    // the row's four sub-lists (entries with (entry/32) % 4 = j), each of
    // at most kCandCap/4, taken one after another
    constexpr int kSubCap = kCandCap / kCandSub;
    int sub[kCandSub], cnt = 0;
    bool fits = true;
#pragma unroll
    for (int j = 0; j < kCandSub; ++j) {
        sub[j] = c.cand_cnt[b * kCandSub + j];
        fits = fits && sub[j] <= kSubCap;
        cnt += sub[j];
    }
    const int W = (n + 31) / 32;
    if (cnt < k || cnt > kSelCap || !fits || W > bm_words) {
        if (threadIdx.x == 0) c.row_flag[b] = 1;   // the plain path takes this row
        return;
    }
    if (threadIdx.x == 0) {
        c.row_flag[b] = 0;
        sh.neq = 0;
    }
    uint32_t mx = 0u;
    for (int j = 0, at = 0; j < kCandSub; at += sub[j], ++j) {
        const uint2 *cp = c.cand + ((size_t)b * kCandSub + j) * kSubCap;
        for (int i = threadIdx.x; i < sub[j]; i += kRThreads) {
            const uint2 v = cp[i];
            sh.key[at + i] = v.x;
            sh.ent[at + i] = (int)v.y;
            mx = max(mx, v.x);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    if (lane == 0) sh.wmax[warp] = mx;
    for (int w = threadIdx.x; w < W; w += kRThreads) sh.bm[w] = 0u;
    __syncthreads();
    uint32_t kmax = lane < kRWarps ? sh.wmax[lane] : 0u;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    // every candidate lies in [t0, kmax]: the digits above their highest
    // differing bit are already known
    const uint32_t t0 = c.cand_t0[b];
    const int bits = (t0 ^ kmax) ? 32 - __clz(t0 ^ kmax) : 0;
    int krem;
    const uint32_t T = radix_select(sh.s, [&](auto fn) {
        for (int i = threadIdx.x; i < cnt; i += kRThreads) fn(sh.key[i]);
    }, k, kmax, bits, &krem);
    CSLA_TL_MARK(0);
    for (int i = threadIdx.x; i < cnt; i += kRThreads) {
        const uint32_t key = sh.key[i];
        const int e = sh.ent[i];
        if (key > T && e < n) atomicOr(&sh.bm[e >> 5], 1u << (e & 31));
        else if (key == T) atomicAdd(&sh.neq, 1);
    }
    __syncthreads();
    // of the keys == T, the krem of lowest entry: the entries up to the
    // krem-th smallest (found as the krem-th largest of ~entry)
    uint32_t emax = 0xFFFFFFFFu;
    if (sh.neq > krem) {
        int kr2;
        emax = ~radix_select(sh.s, [&](auto fn) {
            for (int i = threadIdx.x; i < cnt; i += kRThreads)
                if (sh.key[i] == T) fn(~(uint32_t)sh.ent[i]);
        }, krem, 0u, 32, &kr2);
    }
    for (int i = threadIdx.x; i < cnt; i += kRThreads) {
        const int e = sh.ent[i];
        if (sh.key[i] == T && (uint32_t)e <= emax && e < n) atomicOr(&sh.bm[e >> 5], 1u << (e & 31));
    }
    __syncthreads();
    // thread t writes the picks of bitmap words [t*per, (t+1)*per), after
    // those of the threads before it
    const int per = (W + kRThreads - 1) / kRThreads;
    const int w0 = min(W, threadIdx.x * per), w1 = min(W, w0 + per);
    int my = 0;
    for (int w = w0; w < w1; ++w) my += __popc(sh.bm[w]);
    int incl = my;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) sh.s.warp_a[warp] = incl;
    __syncthreads();
    int total;
    int pos = warp_prefix(sh.s.warp_a, warp, &total) + incl - my;
    if (total != k) {   // never for a correct selection
        if (threadIdx.x == 0) set_dev_err(CSLA_DEVERR_INDEX);
        return;
    }
    for (int w = w0; w < w1; ++w) {
        uint32_t m = sh.bm[w];
        while (m) {
            out[pos++] = 32 * w + (__ffs(m) - 1);
            m &= m - 1u;
        }
    }
    CSLA_TL_MARK(1);
}

}  // namespace

cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(ClShared));
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(topk_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)sizeof(RegShared));
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    if (a.max_n <= kRegMax)
        return launch_pdl(topk_cluster_kernel, dim3(a.B * kG), dim3(kRThreads), sizeof(ClShared), stream, a);
    int grid = a.B;
    if (a.row_flag) {
        int sms = 148;
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (grid > 2 * sms) grid = 2 * sms;
    }
    return launch_pdl(topk_stream_kernel, dim3(grid), dim3(kRThreads), sizeof(RegShared), stream, a);
}

cudaError_t launch_cand_threshold(const TopkArgs &t, const CandArgs &c, cudaStream_t stream) {
    return launch_pdl(cand_threshold_kernel, dim3((t.B + kThrWarps - 1) / kThrWarps), dim3(32 * kThrWarps), 0,
                      stream, t, c);
}

cudaError_t launch_cand_select(const TopkArgs &t, const CandArgs &c, cudaStream_t stream) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(cand_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kCandFixed + 4 * kCandBmMax);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    // a bitmap word per 32 entries of the longest row (rows beyond what
    // fits take the plain path)
    long long words = ((long long)t.max_n + 31) / 32;
    if (words < 1) words = 1;
    if (words > kCandBmMax) words = kCandBmMax;
    return launch_pdl(cand_select_kernel, dim3(t.B), dim3(kRThreads), (size_t)kCandFixed + 4 * (size_t)words, stream,
                      t, c, (int)words);
}

}  // namespace csla
