// compress.cu -- state-cache / classical-cache update (csla_compress_append).
//
// One CTA per new token (blockIdx.x = token i of the call, blockIdx.y =
// request b).  The CTA writes the token's sliding-window row and, when the
// token closes a block of m positions, pools that block into one compressed
// entry (plus, for CSA, one compressed index key).
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力: token-level compressor
//   (m = 4 for CSA, m' = 128 for HCA), window of 128 raw tokens, RoPE on the
//   last 64 dims, bf16 RoPE dims + fp8 other dims, state cache holding the
//   window and the tail, classical cache in blocks of 128 tokens.
//   haiqwa "DeepSeek-V4" §RMSNorm归一化: RMSNorm on the compressed KV head.
// All arithmetic is fp32 with fixed-order reductions; the quantised codes
// are taken with the hardware's round-to-nearest-even conversions.
#include "common.cuh"
#include "kernels.h"

namespace csla {

__device__ unsigned int g_dev_err = 0;

namespace {

constexpr int kThreads = 128;
constexpr int kWarps = kThreads / 32;

template <typename T>
__device__ __forceinline__ float load_act(const T *p, size_t i);
template <>
__device__ __forceinline__ float load_act<float>(const float *p, size_t i) { return __ldg(p + i); }
template <>
__device__ __forceinline__ float load_act<__nv_bfloat16>(const __nv_bfloat16 *p, size_t i) {
    return __bfloat162float(p[i]);
}

// RMSNorm(v) * gamma, partial RoPE at `pos`, quantise into one cache row.
// v: smem [D] (overwritten), red: smem scratch.
__device__ void norm_rope_quantise(float *v, const CompressArgs &a, long long pos, uint8_t *row,
                                   float *scale_out, float *red) {
    const int D = a.D, dr = a.d_rope, dn = D - dr;
    float ss = 0.f;
    for (int d = threadIdx.x; d < D; d += kThreads) ss += v[d] * v[d];
    ss = block_sum<kWarps>(ss, red);
    const float r = 1.0f / sqrtf(ss / (float)D + a.eps);
    for (int d = threadIdx.x; d < D; d += kThreads) v[d] = v[d] * r * __ldg(a.gamma_kv + d);
    __syncthreads();
    if (threadIdx.x < dr / 2) {
        const int i = threadIdx.x;
        float c, s;
        rope_cos_sin(pos, i, dr, a.theta, &c, &s);
        const float x0 = v[dn + 2 * i], x1 = v[dn + 2 * i + 1];
        v[dn + 2 * i] = x0 * c - x1 * s;
        v[dn + 2 * i + 1] = x0 * s + x1 * c;
    }
    __syncthreads();
    float amax = 0.f;
    for (int d = threadIdx.x; d < dn; d += kThreads) amax = fmaxf(amax, fabsf(v[d]));
    amax = block_max<kWarps>(amax, red);
    const float scale = amax > 0.f ? amax / 448.0f : 1.0f;
    for (int d = threadIdx.x; d < dn; d += kThreads) row[d] = f32_to_e4m3(v[d] / scale);
    uint16_t *rope = reinterpret_cast<uint16_t *>(row + dn);
    for (int d = threadIdx.x; d < dr; d += kThreads) rope[d] = f32_to_bf16_bits(v[dn + d]);
    if (threadIdx.x == 0) *scale_out = scale;
}

// Softmax weights of the block's scalar gates g_i = <x_i, w> + bias[i]
// into alpha[0..m).  Row i of the block comes from row_ptr(i).
template <typename T, typename RowFn>
__device__ void block_gate(RowFn row_ptr, int m, int width, const float *w, const float *bias, float *alpha,
                           float *red) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int i = warp; i < m; i += kWarps) {
        const T *x = nullptr;
        const float *xf = nullptr;
        row_ptr(i, &x, &xf);
        float acc = 0.f;
        for (int d = lane; d < width; d += 32) {
            const float xv = xf ? xf[d] : load_act<T>(x, d);
            acc += xv * __ldg(w + d);
        }
        acc = warp_sum(acc);
        if (lane == 0) alpha[i] = acc + __ldg(bias + i);
    }
    __syncthreads();
    float gmax = -INFINITY;
    for (int i = threadIdx.x; i < m; i += kThreads) gmax = fmaxf(gmax, alpha[i]);
    gmax = block_max<kWarps>(gmax, red);
    float e = 0.f;
    for (int i = threadIdx.x; i < m; i += kThreads) {
        const float ev = expf(alpha[i] - gmax);
        alpha[i] = ev;
        e += ev;
    }
    const float z = block_sum<kWarps>(e, red);   // ends with __syncthreads
    for (int i = threadIdx.x; i < m; i += kThreads) alpha[i] = alpha[i] / z;
    __syncthreads();
}

template <typename T>
__global__ void __launch_bounds__(kThreads) compress_append_kernel(CompressArgs a) {
    extern __shared__ float sm[];
    float *v = sm;                       // [D]
    float *alpha = sm + a.D;             // [m]
    float *red = alpha + a.m;            // [32]
    __shared__ int s_old_len;

    const int tok = blockIdx.x, b = blockIdx.y;
    const int slot = a.slots[b];
    if (slot < 0 || slot >= a.n_slots) {
        if (threadIdx.x == 0 && tok == 0) set_dev_err(CSLA_DEVERR_INDEX);
        return;
    }
    if (threadIdx.x == 0) s_old_len = a.len[slot];
    __syncthreads();
    const long long L0 = s_old_len;
    const long long pos = L0 + tok;
    const long long L1 = L0 + a.T;
    const int D = a.D, m = a.m;
    const int rb = (D - a.d_rope) + 2 * a.d_rope;
    const T *kv = reinterpret_cast<const T *>(a.kv_new) + ((size_t)b * a.T + tok) * D;

    // 1. sliding-window row of this token (only tokens that stay in the ring)
    if (pos >= L1 - a.n_win) {
        for (int d = threadIdx.x; d < D; d += kThreads) v[d] = load_act<T>(kv, d);
        __syncthreads();
        const size_t ring = (size_t)slot * a.n_win + (size_t)(pos % a.n_win);
        norm_rope_quantise(v, a, pos, a.win_rows + ring * rb, a.win_scales + ring, red);
        __syncthreads();
    }

    // 2. block closed by this token -> one compressed entry (+ index key)
    if ((pos + 1) % m == 0) {
        const long long bk = pos / m;
        const long long p0 = bk * m;
        const int epp = CSLA_PAGE_TOKENS / m;
        const long long col = bk / epp;
        const int page = col < a.bt_stride ? a.block_table[(size_t)slot * a.bt_stride + (size_t)col] : -1;
        const bool page_ok = page >= 0 && page < a.n_pages;
        if (!page_ok && threadIdx.x == 0) set_dev_err(CSLA_DEVERR_PAGE);
        const T *kv_b = reinterpret_cast<const T *>(a.kv_new) + (size_t)b * a.T * D;
        const float *tail = a.tail_kv + (size_t)slot * m * D;
        auto row_kv = [&](int i, const T **x, const float **xf) {
            const long long p = p0 + i;
            if (p < L0) *xf = tail + (size_t)(p % m) * D;
            else *x = kv_b + (size_t)(p - L0) * D;
        };
        block_gate<T>(row_kv, m, D, a.wg, a.gb, alpha, red);
        for (int d = threadIdx.x; d < D; d += kThreads) {
            float c = 0.f;
            for (int i = 0; i < m; ++i) {
                const T *x = nullptr;
                const float *xf = nullptr;
                row_kv(i, &x, &xf);
                c += alpha[i] * (xf ? xf[d] : load_act<T>(x, d));
            }
            v[d] = c;
        }
        __syncthreads();
        if (page_ok) {
            const size_t e = (size_t)page * epp + (size_t)(bk % epp);
            norm_rope_quantise(v, a, p0, a.rows + e * rb, a.scales + e, red);
        }
        __syncthreads();
        if (a.kidx != nullptr) {   // CSA: compressed index key
            const int dI = a.dI;
            const T *ki_b = reinterpret_cast<const T *>(a.kidx_new) + (size_t)b * a.T * dI;
            const float *tail_i = a.tail_idx + (size_t)slot * m * dI;
            auto row_ix = [&](int i, const T **x, const float **xf) {
                const long long p = p0 + i;
                if (p < L0) *xf = tail_i + (size_t)(p % m) * dI;
                else *x = ki_b + (size_t)(p - L0) * dI;
            };
            block_gate<T>(row_ix, m, dI, a.wgi, a.gbi, alpha, red);
            for (int e = threadIdx.x; e < dI; e += kThreads) {
                float c = 0.f;
                for (int i = 0; i < m; ++i) {
                    const T *x = nullptr;
                    const float *xf = nullptr;
                    row_ix(i, &x, &xf);
                    c += alpha[i] * (xf ? xf[e] : load_act<T>(x, e));
                }
                if (page_ok)
                    a.kidx[((size_t)page * epp + (size_t)(bk % epp)) * dI + e] = f32_to_bf16_bits(c);
            }
        }
        __syncthreads();
    }

    // 3. single-token calls: push the raw row into the tail and bump len here
    //    (the block read above finished before this overwrite).
    if (a.T == 1) {
        const int ts = (int)(pos % m);
        for (int d = threadIdx.x; d < D; d += kThreads)
            a.tail_kv[((size_t)slot * m + ts) * D + d] = load_act<T>(kv, d);
        if (a.kidx != nullptr) {
            const T *ki = reinterpret_cast<const T *>(a.kidx_new) + (size_t)b * a.dI;
            for (int e = threadIdx.x; e < a.dI; e += kThreads)
                a.tail_idx[((size_t)slot * m + ts) * a.dI + e] = load_act<T>(ki, e);
        }
        if (threadIdx.x == 0) a.len[slot] = (int32_t)L1;
    }
}

// Multi-token calls: after every block read the old tail, store the raw rows
// of the still-open last block and set len.  grid = B.
template <typename T>
__global__ void __launch_bounds__(kThreads) tail_update_kernel(CompressArgs a) {
    const int b = blockIdx.x;
    const int slot = a.slots[b];
    if (slot < 0 || slot >= a.n_slots) return;
    const long long L0 = a.len[slot];
    const long long L1 = L0 + a.T;
    const int m = a.m, D = a.D;
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
    __syncthreads();
    if (threadIdx.x == 0) a.len[slot] = (int32_t)L1;
}

}  // namespace

cudaError_t launch_compress_append(const CompressArgs &a, bool bf16, cudaStream_t stream) {
    const size_t smem = ((size_t)a.D + (size_t)a.m + 32) * sizeof(float);
    dim3 grid(a.T, a.B);
    if (bf16) compress_append_kernel<__nv_bfloat16><<<grid, kThreads, smem, stream>>>(a);
    else compress_append_kernel<float><<<grid, kThreads, smem, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess || a.T == 1) return e;
    if (bf16) tail_update_kernel<__nv_bfloat16><<<a.B, kThreads, 0, stream>>>(a);
    else tail_update_kernel<float><<<a.B, kThreads, 0, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace csla
