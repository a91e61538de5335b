// kernels.h -- launch interfaces between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

namespace csla {

// RoPE inverse frequencies theta^(-2i/d_rope), i < d_rope/2, computed on the
// host in double and passed to the kernels.
struct RopeFreq {
    double inv[32];
};

inline RopeFreq rope_freq(float theta, int d_rope) {
    RopeFreq f{};
    for (int i = 0; i < d_rope / 2 && i < 32; ++i) f.inv[i] = pow((double)theta, -(2.0 * i) / (double)d_rope);
    return f;
}

// Launch with programmatic stream serialization (see pdl_wait in common.cuh).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args &&...args) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

struct CompressArgs {
    int m, D, d_rope, dI, n_win;
    float theta, eps;
    RopeFreq freq;
    const int32_t *slots;
    int B, T;
    const void *kv_new, *kidx_new;
    const float *gamma_kv, *wg, *gb, *wgi, *gbi;
    uint8_t *win_rows;
    float *win_scales, *tail_kv, *tail_idx;
    int32_t *len;
    uint8_t *rows;
    float *scales;
    void *kidx;           // bf16 keys, or E4M3 codes (key_fmt)
    float *kscale;        // E4M3 keys: per-entry power-of-two scale
    int key_fmt;
    int gate;             // CSLA_GATE_TOKEN or CSLA_GATE_CHANNEL (gb, gbi [m][width])
    const int32_t *block_table;
    int bt_stride, n_pages, n_slots;
    uint8_t *tok_rows;    // optional: window-format row of every new token
    float *tok_scales;    //   token i of request b -> row b * tok_stride + tok_offset + i
    int tok_stride, tok_offset;
};
cudaError_t launch_compress_append(const CompressArgs &a, bool bf16, cudaStream_t stream);

// Ring rows of the last n positions of each request, in position order.
struct WindowRowsArgs {
    const int32_t *slots;
    const int32_t *len;
    int B, n, n_win, n_slots, row_bytes;
    const uint8_t *win_rows;
    const float *win_scales;
    uint8_t *out_rows;
    float *out_scales;
    int stride;
};
cudaError_t launch_window_rows(const WindowRowsArgs &a, cudaStream_t stream);

// Context-parallel entry records (csla_cp_select / csla_cp_place).
struct CpArgs {
    int place;                   // 0: cache -> records (select), 1: records -> cache (place)
    int slot, epp, bt_stride, n_pages;
    const int32_t *block_table;
    uint8_t *rows;
    float *scales;
    uint8_t *kidx;               // CSA keys (bf16 or E4M3 bytes), else null
    float *kscale;               // E4M3 key scales, else null
    int row_bytes, key_bytes, rec_bytes;
    uint8_t *recs;               // [R][E_max][rec_bytes]
    int R, E_max;
    int b_lo[CSLA_CP_MAX_RANKS];  // first block of rank r's run
    int n[CSLA_CP_MAX_RANKS];     // valid records of rank r
};
cudaError_t launch_cp_move(const CpArgs &a, cudaStream_t stream);

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
    int key_fmt;                // CSLA_KEY_BF16 (keys by TMA tensor map) or CSLA_KEY_E4M3:
    const uint8_t *kidx8;       //   E4M3 key codes [n_pages * 32][dI]
    const float *kscale;        //   and per-entry scales [n_pages * 32]
    const int32_t *q_len;   // optional per-row visible length (else len[slot])
    int rows_per_cta;       // 1, or indexer_rows_per_cta(NQ) when all rows share slots[0]
    int range;              // 0: all visible entries; 1: those below len0[b]/m; 2: those from len0[b]/m on
    const int32_t *len0;    // [B] length of row b's request before the step's append (range 1, 2)
    // Streaming selection (csla_indexer_topk); all zero/null for a plain call.
    int page_step;          // > 1 (range 0, sample): the CTA's pages are the request's pages
                            //   (32x + j)*page_step, j < 32, in 8 tiles of 4; entry i of its j-th
                            //   page goes to score column 32*(32x + j) + i
    int persist;            // > 0 (range 0): `persist` CTAs per row group (grid.x) each walk a
                            //   contiguous run of tiles, page ids read per tile; a CTA whose rows
                            //   are all unflagged (row_flag) exits before it sets anything up
    const uint32_t *cand_t0;   // candidate output: entries whose score_key >= cand_t0[b] are appended,
    uint2 *cand;               //   as (key, entry), to sub-list j = (entry/32) % 4 of row b:
    int32_t *cand_cnt;         //   cand[(4b + j) * cand_cap + ..] (any order), cand_cnt[4b + j] counting
    int cand_cap;              //   them all, also past cand_cap (per sub-list); nothing goes to `scores`
    const int32_t *row_flag;   // rows with row_flag[b] == 0 are not scored
};
// len0[b] = len[slots[b]] (0 for a slot outside the pool).
cudaError_t launch_len_snapshot(const int32_t *slots, const int32_t *len, int B, int n_slots, int32_t *len0,
                                cudaStream_t stream);

// Query rows sharing one key tile per MMA when the rows of a call all belong
// to one request: as many as fit the UMMA N limit of 256 columns.
__host__ __device__ constexpr int indexer_rows_per_cta(int NQ) { return 256 / NQ; }
// Tensor maps of the index-query projection on the tensor cores (bf16 cq
// and W_iq): cq [B][dc] in 128-row boxes, W_iq [HI*dI][dc] in boxes of
// iq_gemm_bn(B) rows, 64 columns (128 bytes) per box, 128-byte swizzle.
struct ProjMaps {
    CUtensorMap cq, w;
};
// Output features per CTA of that projection (the W_iq box height).
// (16 for small batches measured slower at decode: 24.5 against 17.6 us per
// indexer call, the extra CTAs each filling a whole 128-row cq tile.)
inline int iq_gemm_bn(int B) {
    (void)B;
    return 64;
}
cudaError_t launch_indexer(const IndexerArgs &a, bool cq_bf16, bool w_bf16, const CUtensorMap &kmap,
                           const CUtensorMap &qmap, int num_sms, cudaStream_t stream, bool project = true,
                           const ProjMaps *pm = nullptr);

struct TopkArgs {
    const float *scores;
    int stride;
    const int32_t *slots;
    const int32_t *len;
    int m, k, B, max_n, n_slots;
    int32_t *idx;
    const int32_t *q_len;   // optional per-row visible length (else len[slot])
    const int32_t *row_flag;   // rows with row_flag[b] == 0 are left alone (their idx untouched)
};
cudaError_t launch_topk(const TopkArgs &a, cudaStream_t stream);

// Streaming selection (csla_indexer_topk), around the indexer's sample and
// candidate passes.  Per row b of a TopkArgs `t`:
//  threshold: cand_t0[b] from the sample scores (32 pages of 32 entries,
//    page_step apart: 1024 columns per row), cand_cnt[b] = 0;
//  select: the top-k from the cand_cnt[b] candidates when k <= cand_cnt[b]
//    <= cand_cap (row_flag[b] = 0), else row_flag[b] = 1 and idx untouched.
constexpr int kCandCap = 8192;        // candidates kept per row (4 sub-lists of 2048)
constexpr int kCandSub = 4;
constexpr int kSampleCols = 1024;     // sample scores per row (32 pages)
constexpr int kPersistSlices = 2;     // CTAs per row group in the stored-score fallback (few: most
                                      // groups have no flagged row and exit at once)
struct CandArgs {
    const float *sample;
    int page_step;
    uint32_t *cand_t0;
    const uint2 *cand;
    int32_t *cand_cnt;
    int32_t *row_flag;
};
cudaError_t launch_cand_threshold(const TopkArgs &t, const CandArgs &c, cudaStream_t stream);
cudaError_t launch_cand_select(const TopkArgs &t, const CandArgs &c, cudaStream_t stream);

// Attention over the canonical row set of each request: compressed entries
// (top-k list or all visible) then the window, reduced in fixed chunks.
struct AttendArgs {
    int m, D, d_rope, H, n_win;
    float theta, eps;
    RopeFreq freq;
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
    float *part;          // workspace: chunk partials
    int max_chunks;
    int max_len;
    const int32_t *q_len;         // optional per-row visible length (else len[slot])
    const uint8_t *src_rows;      // optional window rows by position:
    const float *src_scales;      //   position p of row b is src row win_base[b] + p
    const int32_t *win_base;
    int n_src;
};

// Visible length of query row b: q_len[b] when given (1 <= q_len[b] <=
// len[slot]), else len[slot].  Returns -1 for a q_len outside that range.
__device__ __forceinline__ int row_visible_len(const int32_t *len, const int32_t *q_len, int slot, int b) {
    const int L = len[slot];
    if (!q_len) return L;
    const int lq = q_len[b];
    return (lq >= 1 && lq <= L) ? lq : -1;
}
cudaError_t launch_attend(const AttendArgs &a, bool q_bf16, bool out_bf16, int variant, int num_sms,
                          cudaStream_t stream);

// Canonical chunk length for a set of n rows (a function of n only):
//   n <= 1024:         64 rows (decode at top-k 512: 10 chunks spread a few
//                      requests over the SMs);
//   1024 < n <= 4096:  320 rows (top-k 1024 + window: 4 chunks, not 18 --
//                      every chunk costs an H*D fp32 partial written and
//                      read back, most of a query row's time when thousands
//                      of rows fill the GPU);
//   n > 4096:          32 * ceil(n / 1024) rows, whole tiles, so that a long
//                      HCA set has close to 32 chunks (8320 rows: 29 chunks
//                      of 288, against 26 of 320 at 64-row granularity).
// A request never has more than 32 chunks.
__host__ __device__ inline int attend_chunk_rows(long long n) {
    if (n <= 1024) return 64;
    if (n <= 4096) return 320;
    return (int)(32 * ((n + 1023) / 1024));
}
__host__ __device__ inline int attend_num_chunks(long long n) {
    const int c = attend_chunk_rows(n);
    return (int)((n + c - 1) / c);
}
// Largest chunk count over all set sizes <= n (never above 32).
__host__ __device__ inline int attend_max_chunks(long long n) {
    const long long c = (n + 63) / 64;
    return (int)(c < 1 ? 1 : (c > 32 ? 32 : c));
}

}  // namespace csla
