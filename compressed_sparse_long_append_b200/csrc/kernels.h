// kernels.h -- launch interfaces between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace csla {

struct CompressArgs {
    int m, D, d_rope, dI, n_win;
    float theta, eps;
    const int32_t *slots;
    int B, T;
    const void *kv_new, *kidx_new;
    const float *gamma_kv, *wg, *gb, *wgi, *gbi;
    uint8_t *win_rows;
    float *win_scales, *tail_kv, *tail_idx;
    int32_t *len;
    uint8_t *rows;
    float *scales;
    uint16_t *kidx;
    const int32_t *block_table;
    int bt_stride, n_pages, n_slots;
};
cudaError_t launch_compress_append(const CompressArgs &a, bool bf16, cudaStream_t stream);

// Lightning indexer.  NQ = rows of the bf16 query operand (hi, mid and lo
// terms of every head, zero padding to a multiple of 16).
struct IndexerArgs {
    int m, HI, dI, dc, NQ;
    const int32_t *slots;
    const int32_t *len;
    const int32_t *block_table;
    int bt_stride, n_pages, n_slots;
    int B, tiles_per_req, max_len;
    const void *cq, *W;
    const float *head_w;
    float *scores;
    int scores_stride;
    uint16_t *q_ws;     // [B][NQ][dI] bf16
};
cudaError_t launch_indexer(const IndexerArgs &a, bool cq_bf16, bool w_bf16, const CUtensorMap &kmap,
                           const CUtensorMap &qmap, int num_sms, cudaStream_t stream);

struct TopkArgs {
    const float *scores;
    int stride;
    const int32_t *slots;
    const int32_t *len;
    int m, k, B, max_n, n_slots;
    int32_t *idx;
};
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream);

// Attention over the canonical row set of each request: compressed entries
// (top-k list or all visible) then the window, reduced in fixed chunks.
struct AttendArgs {
    int m, D, d_rope, H, n_win;
    float theta, eps;
    const int32_t *slots;
    const int32_t *len;
    int B;
    const void *q;
    const int32_t *idx;   // CSA top-k list or null (HCA)
    int k;                // CSA list length
    const float *sink, *gamma_q;
    const uint8_t *rows;
    const float *scales;
    const int32_t *block_table;
    int bt_stride, n_pages, n_slots;
    const uint8_t *win_rows;
    const float *win_scales;
    void *out;
    float *part;          // chunk partials workspace
    int max_chunks;
    int max_len;
};
cudaError_t launch_attend(const AttendArgs &a, bool q_bf16, bool out_bf16, int variant, int num_sms,
                          cudaStream_t stream);

// Canonical chunk length for a set of n rows (a function of n only).
__host__ __device__ inline int attend_chunk_rows(long long n) {
    long long c = (n + 8191) / 8192;
    if (c < 1) c = 1;
    return (int)(256 * c);
}
__host__ __device__ inline int attend_num_chunks(long long n) {
    const int c = attend_chunk_rows(n);
    return (int)((n + c - 1) / c);
}
// Largest chunk count over all set sizes <= n (never above 32).
__host__ __device__ inline int attend_max_chunks(long long n) {
    const long long c = (n + 255) / 256;
    return (int)(c < 1 ? 1 : (c > 32 ? 32 : c));
}

}  // namespace csla
