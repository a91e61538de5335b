// compress.cu -- state-cache / classical-cache update (csla_compress_append).
//
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力: token-level compressor
//   (m = 4 for CSA, m' = 128 for HCA), window of 128 raw tokens, RoPE on the
//   last 64 dims, bf16 RoPE dims + fp8 other dims, state cache holding the
//   window and the tail, classical cache in blocks of 128 tokens.
//   haiqwa "DeepSeek-V4" §RMSNorm归一化: RMSNorm on the compressed KV head.
//
// One launch, grid (T + NB, B, J): for request b,
//   x <  T : new token x -> its sliding-window row (if it stays in the ring)
//            and, for single-token calls, its raw row into the tail;
//   x >= T : the (x-T)-th block this call completes -> z = 0: the pooled KV
//            entry (gate softmax, weighted sum, RMSNorm, RoPE at the block's
//            first position, quantisation), z = 1 (CSA): the index key.
// A second small launch stores the raw rows of multi-token calls' open block
// in the tail (after every pooling CTA has read the old tail) and sets len.
// All arithmetic is fp32 with fixed-order reductions; the quantised codes
// are taken with the hardware's round-to-nearest-even conversions.
#include "common.cuh"
#include "kernels.h"

namespace csla {

__device__ unsigned int g_dev_err = 0;

namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;

template <typename T>
__device__ __forceinline__ float load_act(const T *p, size_t i);
template <>
__device__ __forceinline__ float load_act<float>(const float *p, size_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float load_act<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

// RMSNorm(v) * gamma, partial RoPE at `pos`, quantise into one cache row
// (kTwo: also into a second copy `row2`, when not null).  v, gam: smem [D]
// (read only); red: smem scratch.  Thread t works on dims t and t + 256 in
// registers; a RoPE pair (d, d + 1) sits in lanes t, t ^ 1 and is rotated
// through a shuffle.  The rotation angles are taken first so their latency
// overlaps the reductions.  Per dim the same operations, in the same order,
// as the norm, rotation and scaling written out one after the other.
template <bool kTwo = false>
__device__ void norm_rope_quantise(float *v, const float *gam, const CompressArgs &a, long long pos, uint8_t *row,
                                   float *scale_out, float *red, uint8_t *row2 = nullptr,
                                   float *scale2 = nullptr) {
    constexpr int kE = 2;   // dims per thread (D <= 512)
    const int D = a.D, dr = a.d_rope, dn = D - dr;
    float x[kE];
    bool has[kE], rot[kE];
    float c[kE], sn[kE];
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int d = threadIdx.x + kThreads * e;
        has[e] = d < D;
        rot[e] = has[e] && d >= dn;
        c[e] = 1.f;
        sn[e] = 0.f;
        if (rot[e]) rope_cos_sin(pos, a.freq.inv[(d - dn) >> 1], &c[e], &sn[e]);
        x[e] = has[e] ? v[d] : 0.f;
    }
    float ss = 0.f;
#pragma unroll
    for (int e = 0; e < kE; ++e)
        if (has[e]) ss = __fmaf_rn(x[e], x[e], ss);
    ss = block_sum<kWarps>(ss, red);
    const float r = 1.0f / sqrtf(__fdiv_rn(ss, (float)D) + a.eps);
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int d = threadIdx.x + kThreads * e;
        const float y = has[e] ? __fmul_rn(__fmul_rn(x[e], r), gam[d]) : 0.f;
        const float o = __shfl_xor_sync(0xffffffffu, y, 1);   // the other dim of a RoPE pair
        if (rot[e]) {
            x[e] = (d & 1) == 0 ? __fsub_rn(__fmul_rn(y, c[e]), __fmul_rn(o, sn[e]))
                                : __fadd_rn(__fmul_rn(o, sn[e]), __fmul_rn(y, c[e]));
        } else {
            x[e] = y;
            if (has[e]) amax = fmaxf(amax, fabsf(y));
        }
    }
    amax = block_max<kWarps>(amax, red);
    const float scale = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
#pragma unroll
    for (int e = 0; e < kE; ++e) {
        const int d = threadIdx.x + kThreads * e;
        if (!has[e]) continue;
        if (d < dn) {
            const uint8_t q = f32_to_e4m3(__fdiv_rn(x[e], scale));
            row[d] = q;
            if (kTwo && row2) row2[d] = q;
        } else {
            const uint16_t h = f32_to_bf16_bits(x[e]);
            reinterpret_cast<uint16_t *>(row + dn)[d - dn] = h;
            if (kTwo && row2) reinterpret_cast<uint16_t *>(row2 + dn)[d - dn] = h;
        }
    }
    if (threadIdx.x == 0) {
        *scale_out = scale;
        if (kTwo && row2) *scale2 = scale;
    }
}

// Four consecutive activations (16-byte or 8-byte vector load when `vec`).
template <typename T>
__device__ __forceinline__ float4 load4(const T *p, size_t o, bool vec);
template <>
__device__ __forceinline__ float4 load4<float>(const float *p, size_t o, bool vec) {
    if (vec) return __ldg(reinterpret_cast<const float4 *>(p + o));
    return make_float4(__ldg(p + o), __ldg(p + o + 1), __ldg(p + o + 2), __ldg(p + o + 3));
}
template <>
__device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16 *p, size_t o, bool vec) {
    if (vec) {
        const uint2 u = __ldg(reinterpret_cast<const uint2 *>(p + o));
        const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.x));
        const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&u.y));
        return make_float4(lo.x, lo.y, hi.x, hi.y);
    }
    return make_float4(__bfloat162float(p[o]), __bfloat162float(p[o + 1]), __bfloat162float(p[o + 2]),
                       __bfloat162float(p[o + 3]));
}

// One block of m rows (width floats each, width % 4 == 0, width <= 512):
// rows 0..n_tail-1 are the tail's rows, the others rows of `fresh`.
template <typename T>
struct BlockRows {
    const float *tail;
    const T *fresh;
    int n_tail, width;
    bool vec;
    __device__ __forceinline__ float4 get(int i, int c4) const {
        if (i < n_tail) return *reinterpret_cast<const float4 *>(tail + (size_t)i * width + 4 * c4);
        return load4<T>(fresh, (size_t)(i - n_tail) * width + 4 * c4, vec);
    }
};

constexpr int kMaxIdxPerThread = 2;   // index-key inputs (dI <= 512) per thread
constexpr int kStageRows = 32;    // block rows staged in shared memory at a time

// Rows c0 .. c0+R-1 of the block into xs[R][width] (shared memory), one
// float4 per thread and iteration.
template <typename T>
__device__ __forceinline__ void stage_rows(const BlockRows<T> &x, int c0, int R, float *xs) {
    const int nq = x.width >> 2, total = R * nq;
    for (int idx = threadIdx.x; idx < total; idx += kThreads)
        reinterpret_cast<float4 *>(xs)[idx] = x.get(c0 + idx / nq, idx % nq);
}

// Pool the block with softmax weights of the scalar gates g_i = <x_i, w> +
// bias_i.  On entry alpha[i] = bias_i and wsm = w (smem); the pooled row
// (width floats) goes to out (smem).  The rows pass through shared memory
// (xs) kStageRows at a time; a block of at most kStageRows rows is staged
// once for both passes.  Gates: one warp per row, lane l sums columns
// 4(l + 32j) .. +3 in order of j, then a butterfly over the lanes.  Pooled
// sum: G = 256 / (width / 4) row groups; group g sums rows g, g + G, ... in
// order, and the groups are added in order.
template <typename T>
__device__ void pool_block(const BlockRows<T> &x, int m, const float *wsm, float *alpha, float *part, float *xs,
                           float *out, float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int width = x.width, nq = width >> 2;
    const float4 *xs4 = reinterpret_cast<const float4 *>(xs);
    const float4 *w4 = reinterpret_cast<const float4 *>(wsm);
    const bool staged_once = m <= kStageRows;
    for (int c0 = 0; c0 < m; c0 += kStageRows) {
        const int R = min(kStageRows, m - c0);
        __syncthreads();   // the previous chunk is consumed
        stage_rows(x, c0, R, xs);
        __syncthreads();
        if (c0 == 0) CSLA_TL_MARK(3);
        for (int r = warp; r < R; r += kWarps) {
            float acc = 0.f;
            for (int c4 = lane; c4 < nq; c4 += 32) {
                const float4 xv = xs4[r * nq + c4], wv = w4[c4];
                acc = __fmaf_rn(xv.x, wv.x, acc);
                acc = __fmaf_rn(xv.y, wv.y, acc);
                acc = __fmaf_rn(xv.z, wv.z, acc);
                acc = __fmaf_rn(xv.w, wv.w, acc);
            }
            acc = warp_sum(acc);
            if (lane == 0) alpha[c0 + r] = __fadd_rn(acc, alpha[c0 + r]);
        }
    }
    __syncthreads();
    CSLA_TL_MARK(4);
    float gmax = -INFINITY;
    for (int i = threadIdx.x; i < m; i += kThreads) gmax = fmaxf(gmax, alpha[i]);
    gmax = block_max<kWarps>(gmax, red);
    float e = 0.f;
    for (int i = threadIdx.x; i < m; i += kThreads) {
        const float ev = expf(__fsub_rn(alpha[i], gmax));
        alpha[i] = ev;
        e = __fadd_rn(e, ev);
    }
    const float z = block_sum<kWarps>(e, red);   // ends with __syncthreads
    for (int i = threadIdx.x; i < m; i += kThreads) alpha[i] = __fdiv_rn(alpha[i], z);
    __syncthreads();
    CSLA_TL_MARK(5);
    const int G = kThreads / nq;   // nq <= 128, so G >= 2
    const int g = threadIdx.x / nq, c4 = threadIdx.x % nq;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c0 = 0; c0 < m; c0 += kStageRows) {
        const int R = min(kStageRows, m - c0);
        if (!staged_once) {
            __syncthreads();
            stage_rows(x, c0, R, xs);
            __syncthreads();
        }
        if (g < G) {
            for (int r = g; r < R; r += G) {
                const float al = alpha[c0 + r];
                const float4 xv = xs4[r * nq + c4];
                acc.x = __fmaf_rn(al, xv.x, acc.x);
                acc.y = __fmaf_rn(al, xv.y, acc.y);
                acc.z = __fmaf_rn(al, xv.z, acc.z);
                acc.w = __fmaf_rn(al, xv.w, acc.w);
            }
        }
    }
    if (g < G) reinterpret_cast<float4 *>(part)[g * nq + c4] = acc;
    __syncthreads();
    CSLA_TL_MARK(6);
    for (int d = threadIdx.x; d < width; d += kThreads) {
        float t = part[d];
        for (int q = 1; q < G; ++q) t = __fadd_rn(t, part[q * width + d]);
        out[d] = t;
    }
    __syncthreads();
}

// pool_block for blocks of at most kSmallM rows (CSA, m = 4), in registers:
// thread t < width/4 holds columns 4t..4t+3 of every row (one load round
// trip), its partial gate products go through one block reduction (warp
// butterfly, then the warps in order), every thread forms the softmax
// weights itself, and its pooled columns (rows in order) go to out (smem).
// Two barriers instead of the staged path's ten.
constexpr int kSmallM = 4;
template <typename T>
__device__ void pool_small(const BlockRows<T> &x, int m, const float *wsm, const float *bias, float *red8,
                           float *out) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nq = x.width >> 2;
    const bool act = threadIdx.x < nq;
    float4 xv[kSmallM];
#pragma unroll
    for (int i = 0; i < kSmallM; ++i)
        xv[i] = (act && i < m) ? x.get(i, threadIdx.x) : make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 w = act ? reinterpret_cast<const float4 *>(wsm)[threadIdx.x] : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < kSmallM; ++i) {
        float p = __fmul_rn(xv[i].x, w.x);
        p = __fmaf_rn(xv[i].y, w.y, p);
        p = __fmaf_rn(xv[i].z, w.z, p);
        p = __fmaf_rn(xv[i].w, w.w, p);
        p = warp_sum(p);
        if (lane == 0) red8[warp * kSmallM + i] = p;
    }
    __syncthreads();
    CSLA_TL_MARK(4);
    float al[kSmallM];
    float gmax = -INFINITY;
#pragma unroll
    for (int i = 0; i < kSmallM; ++i) {
        float g = 0.f;
#pragma unroll
        for (int q = 0; q < kWarps; ++q) g = __fadd_rn(g, red8[q * kSmallM + i]);
        al[i] = __fadd_rn(g, i < m ? bias[i] : 0.f);
        if (i < m) gmax = fmaxf(gmax, al[i]);
    }
    float zs = 0.f;
#pragma unroll
    for (int i = 0; i < kSmallM; ++i) {
        al[i] = i < m ? expf(__fsub_rn(al[i], gmax)) : 0.f;
        zs = __fadd_rn(zs, al[i]);
    }
    if (act) {
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int i = 0; i < kSmallM; ++i) {
            if (i < m) {
                const float a = __fdiv_rn(al[i], zs);
                o.x = __fmaf_rn(a, xv[i].x, o.x);
                o.y = __fmaf_rn(a, xv[i].y, o.y);
                o.z = __fmaf_rn(a, xv[i].z, o.z);
                o.w = __fmaf_rn(a, xv[i].w, o.w);
            }
        }
        reinterpret_cast<float4 *>(out)[threadIdx.x] = o;
    }
    __syncthreads();
}

// Per-channel gate: channel d of row i has the gate x_id * w_d + b_id, and
// every channel takes its own softmax over the block's rows.  Thread t <
// width/4 owns columns 4t..4t+3; the rows it sees are folded in order into a
// running (max, sum of weights, weighted sum) that is rescaled whenever the
// max rises.  pool_small_channel: one group of rows (m <= kSmallM, every
// row in registers, max first).  pool_block_channel: G = 256 / (width / 4)
// row groups, group g folds rows g, g + G, ...; the groups' states meet in
// shared memory (st, 12 * kThreads floats) and are merged in group order.
// The pooled row (width floats) goes to out (smem).
struct ChanState {
    float4 mx, z, acc;
};
__device__ __forceinline__ void chan_fold1(float &mx, float &z, float &acc, float g, float xv) {
    if (g > mx) {
        const float r = expf(__fsub_rn(mx, g));   // 0 on the first row (mx = -inf)
        z = __fmaf_rn(z, r, 1.f);
        acc = __fmaf_rn(acc, r, xv);
        mx = g;
    } else {
        const float e = g == -INFINITY ? 0.f : expf(__fsub_rn(g, mx));   // a -inf gate weighs 0
        z = __fadd_rn(z, e);
        acc = __fmaf_rn(e, xv, acc);
    }
}
__device__ __forceinline__ void chan_fold(ChanState &s, float4 x, float4 w, float4 b) {
    chan_fold1(s.mx.x, s.z.x, s.acc.x, __fmaf_rn(x.x, w.x, b.x), x.x);
    chan_fold1(s.mx.y, s.z.y, s.acc.y, __fmaf_rn(x.y, w.y, b.y), x.y);
    chan_fold1(s.mx.z, s.z.z, s.acc.z, __fmaf_rn(x.z, w.z, b.z), x.z);
    chan_fold1(s.mx.w, s.z.w, s.acc.w, __fmaf_rn(x.w, w.w, b.w), x.w);
}
// Merge state o into s (o's rows come after s's).
__device__ __forceinline__ void chan_merge1(float &mx, float &z, float &acc, float omx, float oz, float oacc) {
    const float M = fmaxf(mx, omx);
    if (M == -INFINITY) return;
    const float rs = expf(__fsub_rn(mx, M)), ro = expf(__fsub_rn(omx, M));
    z = __fmaf_rn(oz, ro, __fmul_rn(z, rs));
    acc = __fmaf_rn(oacc, ro, __fmul_rn(acc, rs));
    mx = M;
}

template <typename T>
__device__ void pool_small_channel(const BlockRows<T> &x, int m, const float *wsm, const float *bias, float *out) {
    const int nq = x.width >> 2;
    if (threadIdx.x < nq) {
        const float4 w = reinterpret_cast<const float4 *>(wsm)[threadIdx.x];
        ChanState s{make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY), make_float4(0.f, 0.f, 0.f, 0.f),
                    make_float4(0.f, 0.f, 0.f, 0.f)};
#pragma unroll
        for (int i = 0; i < kSmallM; ++i) {
            if (i < m) {
                const float4 b = __ldg(reinterpret_cast<const float4 *>(bias + (size_t)i * x.width) + threadIdx.x);
                chan_fold(s, x.get(i, threadIdx.x), w, b);
            }
        }
        reinterpret_cast<float4 *>(out)[threadIdx.x] =
            make_float4(__fdiv_rn(s.acc.x, s.z.x), __fdiv_rn(s.acc.y, s.z.y), __fdiv_rn(s.acc.z, s.z.z),
                        __fdiv_rn(s.acc.w, s.z.w));
    }
    __syncthreads();
}

template <typename T>
__device__ void pool_block_channel(const BlockRows<T> &x, int m, const float *wsm, const float *bias, float *st,
                                   float *out) {
    const int nq = x.width >> 2;
    const int G = kThreads / nq;   // nq <= 128, so G >= 2
    const int g = threadIdx.x / nq, c4 = threadIdx.x % nq;
    float4 *st4 = reinterpret_cast<float4 *>(st);
    if (g < G) {
        const float4 w = reinterpret_cast<const float4 *>(wsm)[c4];
        ChanState s{make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY), make_float4(0.f, 0.f, 0.f, 0.f),
                    make_float4(0.f, 0.f, 0.f, 0.f)};
#pragma unroll 4
        for (int i = g; i < m; i += G) {
            const float4 b = __ldg(reinterpret_cast<const float4 *>(bias + (size_t)i * x.width) + c4);
            chan_fold(s, x.get(i, c4), w, b);
        }
        st4[(0 * G + g) * nq + c4] = s.mx;
        st4[(1 * G + g) * nq + c4] = s.z;
        st4[(2 * G + g) * nq + c4] = s.acc;
    }
    __syncthreads();
    if (threadIdx.x < nq) {
        ChanState s{st4[threadIdx.x], st4[G * nq + threadIdx.x], st4[2 * G * nq + threadIdx.x]};
        for (int q = 1; q < G; ++q) {
            const float4 omx = st4[q * nq + threadIdx.x], oz = st4[(G + q) * nq + threadIdx.x],
                         oa = st4[(2 * G + q) * nq + threadIdx.x];
            chan_merge1(s.mx.x, s.z.x, s.acc.x, omx.x, oz.x, oa.x);
            chan_merge1(s.mx.y, s.z.y, s.acc.y, omx.y, oz.y, oa.y);
            chan_merge1(s.mx.z, s.z.z, s.acc.z, omx.z, oz.z, oa.z);
            chan_merge1(s.mx.w, s.z.w, s.acc.w, omx.w, oz.w, oa.w);
        }
        reinterpret_cast<float4 *>(out)[threadIdx.x] =
            make_float4(__fdiv_rn(s.acc.x, s.z.x), __fdiv_rn(s.acc.y, s.z.y), __fdiv_rn(s.acc.z, s.z.z),
                        __fdiv_rn(s.acc.w, s.z.w));
    }
    __syncthreads();
}

template <typename T, bool kChannel>
__device__ __forceinline__ void pool_any(const BlockRows<T> &x, int m, const float *wsm, float *alpha,
                                         const float *bias, float *part, float *xs, float *out, float *red) {
    if constexpr (kChannel) {
        if (m <= kSmallM) pool_small_channel<T>(x, m, wsm, bias, out);
        else pool_block_channel<T>(x, m, wsm, bias, xs, out);
    } else if (m <= kSmallM) {
        pool_small<T>(x, m, wsm, alpha, part, out);
    } else {
        pool_block<T>(x, m, wsm, alpha, part, xs, out, red);
    }
}

// kTok: the call also keeps every new token's window row (CompressArgs::tok_rows).
// kChannel: the per-channel gate (a separate instantiation, so that the
// per-token path carries none of its code).
template <typename T, bool kTok, bool kChannel>
__global__ void __launch_bounds__(kThreads) compress_append_kernel(CompressArgs a) {
    CSLA_TL_SCOPE(kTlCompress);
    extern __shared__ __align__(16) float sm[];
    const int D = a.D, m = a.m;
    const int W = D > a.dI ? D : a.dI;  // widest row pooled (KV or index key)
    float *v = sm;                      // [W]
    float *gam = v + W;                 // [D]   gamma_kv
    float *wsm = gam + D;               // [W]   gate weight (wg, or wgi for index keys)
    float *alpha = wsm + W;             // [m]   gate bias, then weights
    float *part = alpha + m;            // [4 * kThreads]
    float *red = part + 4 * kThreads;   // [32]
    float *xs = red + 32;               // [min(m, kStageRows)][W]  staged block rows
    __shared__ int s_old_len;
    pdl_trigger();
    const int x = blockIdx.x, b = blockIdx.y, z = blockIdx.z;
    const bool token = x < a.T;
    if (token && z != 0) return;
    if (!token && z == 1 && a.kidx == nullptr) return;
    const int slot = __ldg(a.slots + b);
    if (slot < 0 || slot >= a.n_slots) {
        if (threadIdx.x == 0 && x == 0 && z == 0) set_dev_err(CSLA_DEVERR_INDEX);
        return;
    }
    // ---- before the wait: only this call's read-only inputs (weights and
    // the new rows), into shared memory and registers
    const bool in_window = token && x >= a.T - a.n_win;   // token stays in the ring
    const bool emit = token && (in_window || kTok);
    float kreg[kMaxIdxPerThread];
    if (z == 0)
        for (int d = threadIdx.x; d < D; d += kThreads) gam[d] = __ldg(a.gamma_kv + d);
    if (token) {
        const T *kv = reinterpret_cast<const T *>(a.kv_new) + ((size_t)b * a.T + x) * D;
        if (a.T == 1 || emit)
            for (int d = threadIdx.x; d < D; d += kThreads) v[d] = load_act<T>(kv, d);
        if (a.T == 1 && a.kidx != nullptr) {
            const T *ki = reinterpret_cast<const T *>(a.kidx_new) + (size_t)b * a.dI;
#pragma unroll
            for (int u = 0; u < kMaxIdxPerThread; ++u) {
                const int e = threadIdx.x + u * kThreads;
                kreg[u] = e < a.dI ? load_act<T>(ki, e) : 0.f;
            }
        }
    } else {
        const int width = z == 0 ? D : a.dI;
        const float *w = z == 0 ? a.wg : a.wgi;
        const float *gb = z == 0 ? a.gb : a.gbi;
        for (int d = threadIdx.x; d < width; d += kThreads) wsm[d] = __ldg(w + d);
        if (!kChannel)
            for (int i = threadIdx.x; i < m; i += kThreads) alpha[i] = __ldg(gb + i);
    }
    pdl_wait();
    CSLA_TL_WAITED();

    if (threadIdx.x == 0) s_old_len = a.len[slot];
    __syncthreads();
    CSLA_TL_MARK(0);
    const long long L0 = s_old_len;
    const long long L1 = L0 + a.T;
    const int rb = (D - a.d_rope) + 2 * a.d_rope;

    if (token) {
        // ---- token x: window row (+ tail row for single-token calls)
        const long long pos = L0 + x;
        if (a.T == 1) {
            // the pooled block never reads this slot: it takes the new row from kv_new
            const int ts = (int)(pos % m);
            for (int d = threadIdx.x; d < D; d += kThreads) a.tail_kv[((size_t)slot * m + ts) * D + d] = v[d];
            if (a.kidx != nullptr) {
#pragma unroll
                for (int u = 0; u < kMaxIdxPerThread; ++u) {
                    const int e = threadIdx.x + u * kThreads;
                    if (e < a.dI) a.tail_idx[((size_t)slot * m + ts) * a.dI + e] = kreg[u];
                }
            }
        }
        CSLA_TL_MARK(1);
        if (!emit) return;
        const size_t ring = (size_t)slot * a.n_win + (size_t)(pos % a.n_win);
        if constexpr (kTok) {
            const size_t t = (size_t)b * a.tok_stride + a.tok_offset + x;
            uint8_t *trow = a.tok_rows + t * rb;
            float *tscale = a.tok_scales + t;
            if (in_window)
                norm_rope_quantise<true>(v, gam, a, pos, a.win_rows + ring * rb, a.win_scales + ring, red, trow,
                                         tscale);
            else
                norm_rope_quantise(v, gam, a, pos, trow, tscale, red);
        } else {
            norm_rope_quantise(v, gam, a, pos, a.win_rows + ring * rb, a.win_scales + ring, red);
        }
        CSLA_TL_MARK(2);
        return;
    }
    // ---- the (x - T)-th block completed by this call
    const long long bk = L0 / m + (x - a.T);
    if ((bk + 1) * m > L1) return;                     // no such block in this call
    const long long p0 = bk * m;
    const int epp = CSLA_PAGE_TOKENS / m;
    const long long col = bk / epp;
    const int page = col < a.bt_stride ? a.block_table[(size_t)slot * a.bt_stride + (size_t)col] : -1;
    if (page < 0 || page >= a.n_pages) {
        if (threadIdx.x == 0) set_dev_err(CSLA_DEVERR_PAGE);
        return;
    }
    const size_t ent = (size_t)page * epp + (size_t)(bk % epp);
    const long long nt = L0 - p0;
    const int n_tail = nt <= 0 ? 0 : (int)(nt < m ? nt : m);
    const size_t f0 = (size_t)(p0 + n_tail - L0);      // kv_new row of the block's first fresh row
    const uintptr_t vec_mask = sizeof(T) == 4 ? 15u : 7u;
    if (z == 0) {
        const T *fresh = reinterpret_cast<const T *>(a.kv_new) + ((size_t)b * a.T + f0) * D;
        const BlockRows<T> rows{a.tail_kv + (size_t)slot * m * D, fresh, n_tail, D,
                                (reinterpret_cast<uintptr_t>(a.kv_new) & vec_mask) == 0};
        pool_any<T, kChannel>(rows, m, wsm, alpha, a.gb, part, xs, v, red);
        CSLA_TL_MARK(1);
        norm_rope_quantise(v, gam, a, p0, a.rows + ent * rb, a.scales + ent, red);
        CSLA_TL_MARK(2);
    } else {
        const int dI = a.dI;
        const T *fresh = reinterpret_cast<const T *>(a.kidx_new) + ((size_t)b * a.T + f0) * dI;
        const BlockRows<T> rows{a.tail_idx + (size_t)slot * m * dI, fresh, n_tail, dI,
                                (reinterpret_cast<uintptr_t>(a.kidx_new) & vec_mask) == 0};
        pool_any<T, kChannel>(rows, m, wsm, alpha, a.gbi, part, xs, v, red);
        CSLA_TL_MARK(1);
        if (a.key_fmt == CSLA_KEY_E4M3) {
            // one power-of-two scale per entry: the smallest 2^e with
            // 448 * 2^e >= max |key dim|, codes E4M3(key / 2^e), on fp32 values
            float am = 0.f;
            for (int e = threadIdx.x; e < dI; e += kThreads) am = fmaxf(am, fabsf(v[e]));
            am = block_max<kThreads / 32>(am, red);
            const int ex = key_exp_e4m3(am);
            const float inv = __uint_as_float((uint32_t)(127 - min(ex, 126)) << 23);   // 2^-ex
            uint8_t *k8 = reinterpret_cast<uint8_t *>(a.kidx) + ent * dI;
            for (int e = threadIdx.x; e < dI; e += kThreads) k8[e] = f32_to_e4m3(__fmul_rn(v[e], inv));
            if (threadIdx.x == 0) a.kscale[ent] = __uint_as_float((uint32_t)(ex + 127) << 23);
        } else {
            uint16_t *k16 = reinterpret_cast<uint16_t *>(a.kidx) + ent * dI;
            for (int e = threadIdx.x; e < dI; e += kThreads) k16[e] = f32_to_bf16_bits(v[e]);
        }
        CSLA_TL_MARK(2);
    }
}

// After the pooling: raw rows of the still-open last block of multi-token
// calls go to the tail; len advances.  grid = B.
template <typename T>
__global__ void __launch_bounds__(kThreads) tail_update_kernel(CompressArgs a) {
    CSLA_TL_SCOPE(kTlTailUpdate);
    pdl_trigger();
    const int b = blockIdx.x;
    const int slot = __ldg(a.slots + b);
    pdl_wait();
    CSLA_TL_WAITED();
    if (slot < 0 || slot >= a.n_slots) return;
    const long long L0 = a.len[slot];
    const long long L1 = L0 + a.T;
    const int m = a.m, D = a.D;
    if (a.T > 1) {
        long long start = (L1 / m) * m;
        if (start < L0) start = L0;
        for (long long p = start; p < L1; ++p) {
            const T *kv = reinterpret_cast<const T *>(a.kv_new) + ((size_t)b * a.T + (size_t)(p - L0)) * D;
            for (int d = threadIdx.x; d < D; d += kThreads)
                a.tail_kv[((size_t)slot * m + (size_t)(p % m)) * D + d] = load_act<T>(kv, d);
            if (a.kidx != nullptr) {
                const T *ki = reinterpret_cast<const T *>(a.kidx_new) + ((size_t)b * a.T + (size_t)(p - L0)) * a.dI;
                for (int e = threadIdx.x; e < a.dI; e += kThreads)
                    a.tail_idx[((size_t)slot * m + (size_t)(p % m)) * a.dI + e] = load_act<T>(ki, e);
            }
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) a.len[slot] = (int32_t)L1;
}

}  // namespace

// Row i of request b = ring row of position len - n + i (a zero row with
// scale 0 where that position is negative).  One CTA per row.
constexpr int kWinThreads = 64;
__global__ void __launch_bounds__(kWinThreads) window_rows_kernel(WindowRowsArgs a) {
    pdl_trigger();
    const int i = blockIdx.x, b = blockIdx.y;
    const int slot = __ldg(a.slots + b);
    uint4 *dst = reinterpret_cast<uint4 *>(a.out_rows + ((size_t)b * a.stride + i) * a.row_bytes);
    float *dscale = a.out_scales + (size_t)b * a.stride + i;
    const int nq = a.row_bytes / 16;
    pdl_wait();
    if (slot < 0 || slot >= a.n_slots) {
        if (threadIdx.x == 0 && i == 0) set_dev_err(CSLA_DEVERR_INDEX);
        return;
    }
    const long long pos = (long long)a.len[slot] - a.n + i;
    if (pos < 0) {
        for (int q = threadIdx.x; q < nq; q += kWinThreads) dst[q] = make_uint4(0u, 0u, 0u, 0u);
        if (threadIdx.x == 0) *dscale = 0.f;
        return;
    }
    const size_t ring = (size_t)slot * a.n_win + (size_t)(pos % a.n_win);
    const uint4 *src = reinterpret_cast<const uint4 *>(a.win_rows + ring * a.row_bytes);
    for (int q = threadIdx.x; q < nq; q += kWinThreads) dst[q] = src[q];
    if (threadIdx.x == 0) *dscale = a.win_scales[ring];
}

cudaError_t launch_window_rows(const WindowRowsArgs &a, cudaStream_t stream) {
    return launch_pdl(window_rows_kernel, dim3(a.n, a.B), dim3(kWinThreads), 0, stream, a);
}

cudaError_t launch_compress_append(const CompressArgs &a, bool bf16, cudaStream_t stream) {
    const int nb = a.T / a.m + 1;   // blocks one call can complete
    const size_t W = (size_t)(a.D > a.dI ? a.D : a.dI);
    const size_t R = (size_t)(a.m < kStageRows ? a.m : kStageRows);
    const size_t smem = (2 * W + (size_t)a.D + (size_t)a.m + 4 * kThreads + 32 + R * W) * sizeof(float);
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        // largest case: W = 512, m = 128
        const int most = (int)((2 * 512 + 512 + 128 + 4 * kThreads + 32 + kStageRows * 512) * sizeof(float));
        cudaError_t e = cudaSuccess;
        for (auto fn : {compress_append_kernel<float, false, false>, compress_append_kernel<float, true, false>,
                        compress_append_kernel<__nv_bfloat16, false, false>,
                        compress_append_kernel<__nv_bfloat16, true, false>,
                        compress_append_kernel<float, false, true>, compress_append_kernel<float, true, true>,
                        compress_append_kernel<__nv_bfloat16, false, true>,
                        compress_append_kernel<__nv_bfloat16, true, true>}) {
            e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
            if (e != cudaSuccess) return e;
        }
        configured_dev = dev;
    }
    const dim3 grid(a.T + nb, a.B, a.kidx ? 2 : 1);
    const bool tok = a.tok_rows != nullptr;
    const bool ch = a.gate == CSLA_GATE_CHANNEL;
    void (*fn)(CompressArgs);
    if (bf16)
        fn = ch ? (tok ? compress_append_kernel<__nv_bfloat16, true, true> : compress_append_kernel<__nv_bfloat16, false, true>)
                : (tok ? compress_append_kernel<__nv_bfloat16, true, false>
                       : compress_append_kernel<__nv_bfloat16, false, false>);
    else
        fn = ch ? (tok ? compress_append_kernel<float, true, true> : compress_append_kernel<float, false, true>)
                : (tok ? compress_append_kernel<float, true, false> : compress_append_kernel<float, false, false>);
    cudaError_t e = launch_pdl(fn, grid, dim3(kThreads), smem, stream, a);
    if (e != cudaSuccess) return e;
    return bf16 ? launch_pdl(tail_update_kernel<__nv_bfloat16>, dim3(a.B), dim3(kThreads), 0, stream, a)
                : launch_pdl(tail_update_kernel<float>, dim3(a.B), dim3(kThreads), 0, stream, a);
}

}  // namespace csla
