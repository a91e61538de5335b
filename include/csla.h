/*
 * csla.h -- C ABI of libcsla, the B200 (sm_100a) implementation of the
 * CSA/HCA hybrid compressed attention decode path.
 *
 * The operation (page title, section):
 *   haiqwa.github.io "DeepSeek-V4" blog, §CSA：压缩稀疏注意力 and §HCA：重度压缩注意力
 *     (every m tokens of KV become one entry; every query attends k entries);
 *     §RMSNorm归一化 (RMSNorm on each query head and on the single KV head);
 *     §Partial RoPE位置编码 (RoPE dims bf16, other dims fp8; sliding window);
 *     §让注意力学会"忽略" (per-head sink logit in the softmax denominator);
 *     §索引可见性处理 (visible compressed range computable by rule).
 *   硅星人 article "DeepSeek V4 ... 让token大降价", §两大压缩注意力: CSA data flow
 *     (compressor m=4, lightning indexer with dc=1024 latent and ReLU scores,
 *     top-k 512/1024, window of 128 raw tokens, MQA), HCA (m'=128, no indexer,
 *     no top-k), RoPE on the last 64 dims, bf16/fp8 cache, the per-request
 *     state cache and the classical cache in blocks of lcm(4,128)=128 tokens.
 *   QbitAI article on DeepSeek V4's batch invariance: outputs bit-identical
 *     whatever the batch; a saturated and a starved attention kernel that
 *     agree bit for bit.
 *
 * Conventions for every entry point
 *   - All array pointers are DEVICE pointers owned by the caller (csla_cfg,
 *     csla_cache and csla_state themselves are host structs holding device
 *     pointers).  The library never allocates device memory; scratch comes
 *     from the caller through `workspace` (size from csla_workspace_size).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = the
 *     legacy default stream).  Host-side argument checks happen before any
 *     launch and return an error without launching anything.
 *   - Return value: CSLA_OK or a CSLA_ERR_* code.  Errors that only the
 *     device can see (a page id outside the pool, an index outside the
 *     visible range, a length above max_len) never trap: the kernel skips
 *     the offending work, records a bit in the library's device error word
 *     and carries on; csla_device_error() reads and clears it.
 *   - A batch is `B` requests given by `slots` (device int32[B], distinct
 *     state-cache slot ids; query rows passed with a csla_queries may share
 *     a slot).  Context length of request b after the call is
 *     st->len[slots[b]].  `max_len` (host) is an upper bound on it, used to
 *     size grids.
 *
 * Data layout (little-endian)
 *   Cache row of one token or compressed entry, D = d_nope + d_rope dims:
 *     bytes [0, d_nope)             E4M3 (OCP FP8 E4M3FN) codes of dims 0..d_nope-1
 *     bytes [d_nope, d_nope+2*dr)   bf16 values of dims d_nope..D-1 (the RoPE dims)
 *   plus one fp32 scale per row: value of dim d < d_nope = e4m3(code)*scale.
 *   Row bytes: 576 for D=512, 192 for D=128.
 *   Classical cache (one layer): pages of CSLA_PAGE_TOKENS=128 raw tokens,
 *   epp = 128/m entries per page (32 for CSA, 1 for HCA):
 *     rows   uint8 [n_pages][epp][row_bytes]
 *     scales f32   [n_pages][epp]
 *     kidx   [n_pages][epp][dI]               (CSA only: compressed index keys),
 *            bf16 values (key_fmt CSLA_KEY_BF16) or E4M3 codes (CSLA_KEY_E4M3)
 *     kscale f32   [n_pages][epp]              (CSLA_KEY_E4M3 only) key scale, a power of two:
 *            key dim e = e4m3(code_e) * kscale
 *     block_table int32 [n_slots][bt_stride]: compressed entry e of slot s is
 *       entry e % epp of page block_table[s][e / epp].
 *   State cache (one layer, per slot):
 *     win_rows   uint8 [n_slots][n_win][row_bytes]  token at position p lives in
 *     win_scales f32   [n_slots][n_win]             ring slot p % n_win
 *     tail_kv    f32   [n_slots][m][D]       raw KV of the not yet compressed block
 *     tail_idx   f32   [n_slots][m][dI]      raw index-key inputs (CSA only)
 *     len        int32 [n_slots]             tokens appended so far
 */
#ifndef CSLA_H
#define CSLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *csla_stream_t; /* same type as cudaStream_t */

enum {
    CSLA_OK = 0,
    CSLA_ERR_ARG = 1,         /* null pointer, bad size, k > supported, workspace too small */
    CSLA_ERR_UNSUPPORTED = 2, /* a shape this build has no kernel for */
    CSLA_ERR_CUDA = 3,        /* a CUDA runtime call or launch failed */
    CSLA_ERR_DEVICE = 4       /* a kernel recorded a bad input (see csla_device_error) */
};

enum { CSLA_F32 = 0, CSLA_BF16 = 1 };

enum { CSLA_VARIANT_AUTO = 0, CSLA_VARIANT_SATURATED = 1, CSLA_VARIANT_STARVED = 2 };

/* Storage of the CSA compressed index keys (haiqwa §FP4精度加速: the
 * indexer's key/query path runs in low precision).  E4M3: one byte per dim
 * plus one power-of-two scale per entry, s = the smallest 2^e (-126 <= e <=
 * 127) with 448 * s >= max |key dim|, codes = E4M3(key / s) rounded to
 * nearest even, both decided on the fp32 pooled key; 132 bytes per entry at
 * dI = 128 instead of 256. */
enum { CSLA_KEY_BF16 = 0, CSLA_KEY_E4M3 = 1 };

/* Gate of the token-level compressor (硅星人 §两大压缩注意力: a token-level
 * compressor turns each block of m tokens into one entry; the pages give no
 * formula).  TOKEN: one scalar gate per token, g_i = <x_i, wg> + gb[i],
 * softmax over the block's tokens, entry = sum_i alpha_i x_i.  CHANNEL: one
 * gate per token and channel, g_id = x_id * wg[d] + gb[i][d], a separate
 * softmax over the block's tokens for every channel d, entry_d =
 * sum_i alpha_id x_id (gb, gbi are then [m][D], [m][dI]). */
enum { CSLA_GATE_TOKEN = 0, CSLA_GATE_CHANNEL = 1 };

enum {
    CSLA_OP_INDEXER = 1,
    CSLA_OP_TOPK = 2,
    CSLA_OP_CSA_ATTEND = 3,
    CSLA_OP_HCA_ATTEND = 4,
    CSLA_OP_CSA_DECODE_STEP = 5, /* ws_step of csla_csa_decode_step; max_len here means k */
    CSLA_OP_INDEXER_TOPK = 6     /* csla_indexer_topk */
};

/* device error word bits */
enum {
    CSLA_DEVERR_PAGE = 1,     /* block-table entry outside [0, n_pages) */
    CSLA_DEVERR_INDEX = 2,    /* top-k index outside [0, visible entries) */
    CSLA_DEVERR_LEN = 4,      /* context length above max_len */
    CSLA_DEVERR_TIMEOUT = 8,  /* a bounded wait inside a kernel gave up */
    CSLA_DEVERR_RANGE = 16    /* a cache row outside the attention operands' range (row masked) */
};

#define CSLA_PAGE_TOKENS 128

/* Layer shape.  Supported: m in {4, 128}; D in {128, 512}; d_rope = 64;
 * 1 <= H <= 64; n_win = 128; CSA (m = 4): dI in {64, 128}, HI in {4, 8, 16},
 * dc a multiple of 8 up to 4096, 1 <= topk <= 2048. */
typedef struct csla_cfg {
    int32_t m;          /* tokens per compressed entry: 4 (CSA) or 128 (HCA) */
    int32_t D;          /* head dim; the last d_rope dims carry RoPE */
    int32_t d_rope;     /* 64 */
    int32_t H;          /* query heads sharing the one KV head */
    int32_t HI;         /* lightning-indexer heads (CSA) */
    int32_t dI;         /* index head dim (CSA) */
    int32_t dc;         /* query latent dim fed to the indexer (CSA) */
    int32_t n_win;      /* sliding window, 128 */
    float rope_theta;   /* RoPE base, 10000 */
    float eps;          /* RMSNorm epsilon, 1e-6 */
    int32_t key_fmt;    /* CSA index-key storage: CSLA_KEY_BF16 (default) or CSLA_KEY_E4M3 (dI = 128) */
    int32_t gate;       /* compressor gate: CSLA_GATE_TOKEN (default) or CSLA_GATE_CHANNEL */
} csla_cfg;

typedef struct csla_cache {
    uint8_t *rows;
    float *scales;
    void *kidx;                /* CSA only, else NULL: bf16 values or E4M3 codes (cfg->key_fmt) */
    const int32_t *block_table;
    int32_t bt_stride;
    int32_t n_pages;
    float *kscale;             /* CSA with CSLA_KEY_E4M3 only, else NULL: per-entry key scale */
} csla_cache;

typedef struct csla_state {
    uint8_t *win_rows;
    float *win_scales;
    float *tail_kv;
    float *tail_idx;           /* CSA only, else NULL */
    int32_t *len;
    int32_t n_slots;
} csla_state;

/* Compressor parameters, device f32 arrays (shapes for CSLA_GATE_TOKEN;
 * with CSLA_GATE_CHANNEL the biases have one value per position and channel
 * and must be 16-byte aligned). */
typedef struct csla_compress_params {
    const float *gamma_kv;     /* [D]  RMSNorm weight of the KV head */
    const float *wg;           /* [D]  gate weight of the KV compressor */
    const float *gb;           /* [m]  gate bias per position in the block ([m][D] per channel) */
    const float *wgi;          /* [dI] gate weight of the index-key compressor (CSA) */
    const float *gbi;          /* [m]  gate bias of the index-key compressor (CSA; [m][dI] per channel) */
} csla_compress_params;

/*
 * Query rows other than each request's latest token (a prefill chunk's
 * queries; several recent positions of one request).  Calls that take a
 * `const csla_queries *qs` treat NULL as plain decode: row b is request
 * slots[b] at its latest position len-1.  With qs:
 *   q_len [B] int32 (device): row b's visible length.  Its query sits at
 *     position q_len[b]-1 and sees what a decode step at that position sees
 *     (haiqwa §百万 token 怎么切分, causal visibility of compressed blocks:
 *     entry e is visible iff (e+1)*m <= q_len[b]; window = the last
 *     min(n_win, q_len[b]) positions before it, inclusive).  Requires
 *     1 <= q_len[b] <= len[slots[b]]: the cache already holds those tokens.
 *     A row outside that range sets CSLA_DEVERR_LEN and is skipped.
 *   win_rows / win_scales / win_base / n_win_rows: where the attention calls
 *     read window rows.  win_rows NULL: from the ring, so each row's window
 *     positions must still be there (q_len[b] - min(q_len[b], n_win) >=
 *     len - n_win, else CSLA_DEVERR_INDEX and the row is skipped).  Else
 *     position p of row b is row win_base[b] + p of win_rows
 *     [n_win_rows][row_bytes] (16-byte aligned) with scale win_scales[...];
 *     a position outside [0, n_win_rows) sets CSLA_DEVERR_INDEX and the row
 *     is masked.  csla_window_rows and the token-row output of
 *     csla_compress_append fill such a buffer for a prefill chunk.
 *   one_request: nonzero promises slots[b] == slots[0] for every row (the
 *     queries of one request's prefill chunk); the indexer then scores
 *     several rows against each key tile it loads.  A row with another slot
 *     sets CSLA_DEVERR_INDEX and is skipped.
 * The indexer and top-k read q_len (and one_request) only.
 */
typedef struct csla_queries {
    const int32_t *q_len;
    const uint8_t *win_rows;
    const float *win_scales;
    const int32_t *win_base;
    int32_t n_win_rows;
    int32_t one_request;
} csla_queries;

/* Optional output of csla_compress_append: the window-format row (the one
 * the ring receives) of every new token, kept for later queries of a prefill
 * chunk.  New token i of request b goes to row b*stride + offset + i. */
typedef struct csla_token_rows {
    uint8_t *rows;       /* [B*stride][row_bytes] */
    float *scales;       /* [B*stride] */
    int32_t stride;      /* rows per request, >= offset + T */
    int32_t offset;      /* row of the call's first new token, >= 0 */
} csla_token_rows;

/*
 * csla_compress_append -- state-cache and classical-cache update
 * (硅星人 §两大压缩注意力, CSA/HCA compressor and cache paragraphs; haiqwa
 * §Partial RoPE位置编码 sliding window; §RMSNorm归一化).
 * Appends T new tokens to each of the B requests.  For every new token at
 * position p (p = old len + i): its window row RoPE(RMSNorm(x)*gamma_kv, p),
 * quantised, goes to ring slot p % n_win; its raw vector joins the tail.
 * When position p closes block b = p/m (p+1 divisible by m), the block's m raw
 * rows are pooled with softmax weights of the scalar gate <x_i,wg> + gb[i],
 * then RMSNorm*gamma_kv, RoPE at position b*m, quantised into compressed entry
 * b; for CSA the index-key inputs are pooled with their own gate (wgi, gbi)
 * and stored as bf16.  Finally len += T.
 *   kv_new   [B][T][D]  dtype kv_dtype (CSLA_F32 or CSLA_BF16)
 *   kidx_new [B][T][dI] dtype kv_dtype, CSA only (NULL for HCA)
 * Requires: the block table maps every page the new tokens reach;
 * st->tail_kv and st->tail_idx 16-byte aligned; CSA: dI a multiple of 4,
 * 4 <= dI <= 512.  kv_new / kidx_new need no alignment (aligned inputs take
 * vector loads).  gamma_kv, wg, gb, wgi, gbi are read before the kernel
 * waits on the grid launched before it on the stream (programmatic
 * dependent launch); write them no later than the kernel before that one.
 * tok: NULL, or where the window-format row of every new token also goes
 * (csla_token_rows; the ring keeps only the last n_win).
 * Errors: CSLA_ERR_ARG on null/bad sizes or misaligned tails;
 * CSLA_ERR_UNSUPPORTED on shapes.
 */
int csla_compress_append(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                         const int32_t *slots, int32_t B, int32_t T, const void *kv_new,
                         const void *kidx_new, int32_t kv_dtype, const csla_compress_params *p,
                         const csla_token_rows *tok, csla_stream_t stream);

/*
 * csla_window_rows -- copy of the ring rows of each request's last n
 * positions, in position order: row b*stride + i = the row of position
 * len - n + i (a zero row with scale 0 where that position is negative).
 * 1 <= n <= n_win.  With the token-row output of csla_compress_append this
 * gives a prefill chunk's queries every window row they need: take the
 * n_win-1 rows before the chunk here, then append the chunk.
 * rows_out 16-byte aligned.  Errors: CSLA_ERR_ARG; CSLA_DEVERR_INDEX for a
 * slot outside [0, n_slots).
 */
int csla_window_rows(const csla_cfg *cfg, const csla_state *st, const int32_t *slots, int32_t B,
                     int32_t n, uint8_t *rows_out, float *scales_out, int32_t stride,
                     csla_stream_t stream);

/*
 * csla_indexer_scores -- lightning indexer (硅星人 §两大压缩注意力, CSA part:
 * the query latent dc is up-projected to HI index heads and scored with ReLU
 * against the compressed index keys).  For row b with N_vis = L/m visible
 * entries (L = len[slots[b]], or q_len[b] with qs; see csla_queries):
 *   qI = W_iq . cq[b]  ([HI*dI] = [HI*dI][dc] . [dc], fp32 accumulation),
 *   scores[b*scores_stride + s] = sum_j head_w[b][j] * max(0, <qI_j, kidx_s>)
 * for s < N_vis (entries beyond N_vis are not written).  qI enters the tensor
 * cores as three bf16 terms (hi, mid, lo), so scores carry fp32-level error.
 *   cq [B][dc] (cq_dtype), W_iq [HI*dI][dc] (w_dtype), head_w [B][HI] f32,
 *   scores f32 [B][scores_stride], scores_stride >= max_len/m.
 * workspace: csla_workspace_size(cfg, CSLA_OP_INDEXER, B, max_len) bytes.
 * qs: NULL (decode) or query rows; with qs->one_request several rows share
 * each key tile.  Errors: CSLA_ERR_ARG (null pointers, stride, workspace,
 * 16-byte alignment of cq, W_iq, kidx and workspace); CSLA_ERR_UNSUPPORTED
 * for HI, dI or dc outside the supported set; device bits PAGE, LEN, INDEX.
 */
int csla_indexer_scores(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                        const int32_t *slots, int32_t B, const csla_queries *qs, int32_t max_len, const void *cq,
                        int32_t cq_dtype, const void *W_iq, int32_t w_dtype, const float *head_w,
                        float *scores, int32_t scores_stride, void *workspace,
                        size_t workspace_bytes, csla_stream_t stream);

/*
 * csla_topk_select -- top-k selector (硅星人 §两大压缩注意力, CSA part).
 * For row b (N_vis = L/m as in csla_indexer_scores): the min(k, N_vis)
 * entries of largest score (ties: lower index first), written to
 * idx[b*k ..] in ascending index order, the rest of the row filled with -1.
 * Exact: integer radix select on the fp32 bits (-0.0 counts as +0.0).
 * scores as produced by csla_indexer_scores.  Errors: CSLA_ERR_ARG (null
 * pointers, k outside 1..2048, stride); device bit LEN (row skipped).
 */
int csla_topk_select(const csla_cfg *cfg, const csla_state *st, const int32_t *slots, int32_t B,
                     const csla_queries *qs, int32_t max_len, const float *scores, int32_t scores_stride, int32_t k,
                     int32_t *idx, csla_stream_t stream);

/*
 * csla_indexer_topk -- csla_indexer_scores then csla_topk_select in one
 * call, without storing the scores of rows that are long (硅星人
 * §两大压缩注意力, CSA part: score every compressed block, keep the k best;
 * "DeepSeek-V4深度拆解" §2: the prefill's KV-cache traffic).  The result,
 * idx [B][k], is bit for bit the one of the two calls.  Steps, all on
 * `stream`: a sample pass scores 32 evenly spaced 32-entry pages of every
 * row; a threshold t0 per row is taken from the sample so that about
 * min(4096, max(2048, 3k)) of the row's scores should reach it (the r-th
 * largest sample score, r scaled from the row to the sample); a candidate
 * pass scores every entry and
 * keeps (score, entry) for those >= t0 only; the exact top-k is selected
 * among the candidates when there are at least k and at most 6144 of them
 * (every score >= the k-th largest is then a candidate).  A row outside that
 * range (heavy ties, a sample far from the row's distribution) is scored
 * again into `scores` and selected there, as by the two calls.  Rows of at
 * most 6144 entries keep every entry as a candidate.
 *   Arguments as for csla_indexer_scores and csla_topk_select (device
 *   pointers owned by the caller; the call keeps none of them); `scores`
 *   [B][scores_stride] f32 is scratch (written only for rows taken by the
 *   fallback; its contents are unspecified afterwards).  workspace:
 *   csla_workspace_size(cfg, CSLA_OP_INDEXER_TOPK, B, max_len) bytes,
 *   16-byte aligned.  Errors: those of the two calls.
 */
int csla_indexer_topk(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                      const int32_t *slots, int32_t B, const csla_queries *qs, int32_t max_len,
                      const void *cq, int32_t cq_dtype, const void *W_iq, int32_t w_dtype,
                      const float *head_w, int32_t k, int32_t *idx, float *scores,
                      int32_t scores_stride, void *workspace, size_t workspace_bytes,
                      csla_stream_t stream);

/*
 * csla_csa_attend -- core MQA of a CSA layer (硅星人 §两大压缩注意力; haiqwa
 * §RMSNorm归一化, §Partial RoPE位置编码, §让注意力学会"忽略").
 * For row b at position t = L-1 (L = len[slots[b]], or q_len[b] with qs)
 * and head h < H:
 *   qh = RoPE(RMSNorm(q[b][h]) * gamma_q, t)
 *   set = compressed entries idx[b][0..k) (entries < 0 skipped), then window
 *         tokens max(0, L-n_win) .. L-1 (from the ring, or from qs's
 *         window rows), each row decoded as above;
 *   s_j = <qh, x_j>/sqrt(D);  o = sum_j e^{s_j} x_j / (e^{sink[h]} + sum_j e^{s_j}).
 * One KV head: K = V = the cached row.  Batch invariant: each request's
 * reduction order is fixed by its own set size, identical for every variant.
 *   q [B][H][D] (q_dtype), idx int32 [B][k], sink f32 [H], gamma_q f32 [D],
 *   out [B][H][D] (out_dtype).
 * variant: CSLA_VARIANT_SATURATED (one CTA walks all chunks of a request),
 *   CSLA_VARIANT_STARVED (one CTA per chunk, then an ordered combine), or AUTO.
 * workspace: csla_workspace_size(cfg, CSLA_OP_CSA_ATTEND, B, max_len) with
 *   max_len here meaning k (the set size is k + n_win).
 * Errors: CSLA_ERR_ARG (null pointers, k, variant, workspace, 16-byte
 * alignment of q, rows, window rows, workspace); CSLA_ERR_UNSUPPORTED when
 * n_pages * (128/m) or n_slots * n_win reaches 2^32; device bits INDEX (an
 * idx entry outside the visible range: row masked), PAGE, LEN, RANGE.
 * Operand range: the tensor cores take each row in f16 as x / (256 * s_eff)
 * with P scaled by 256 * s_eff, s_eff = max(fp8 scale, max|RoPE dim| /
 * 2^23).  A row with s_eff > 15 (fp8 dims above 6720 in magnitude, or RoPE
 * dims above ~1.3e8; rows of RMSNorm-ed vectors stay far below) is masked
 * and sets CSLA_DEVERR_RANGE.  RoPE dims below 2^-24 * 256 * s_eff in
 * magnitude contribute as f16 subnormals or zero.
 */
int csla_csa_attend(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                    const int32_t *slots, int32_t B, const csla_queries *qs, const void *q, int32_t q_dtype,
                    const int32_t *idx, int32_t k, const float *sink, const float *gamma_q,
                    void *out, int32_t out_dtype, int32_t variant, void *workspace,
                    size_t workspace_bytes, csla_stream_t stream);

/*
 * csla_hca_attend -- core MQA of an HCA layer (硅星人 §两大压缩注意力, HCA part:
 * no indexer, no top-k; every compressed entry plus the window).  As
 * csla_csa_attend with set = all N_vis = len/m entries then the window.
 * workspace: csla_workspace_size(cfg, CSLA_OP_HCA_ATTEND, B, max_len).
 */
int csla_hca_attend(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                    const int32_t *slots, int32_t B, const csla_queries *qs, int32_t max_len, const void *q,
                    int32_t q_dtype, const float *sink, const float *gamma_q, void *out,
                    int32_t out_dtype, int32_t variant, void *workspace, size_t workspace_bytes,
                    csla_stream_t stream);

/*
 * csla_csa_decode_step -- one CSA decode step in one call: the same results,
 * bit for bit, as csla_compress_append (T new tokens, no token rows), then
 * csla_indexer_scores, csla_topk_select and csla_csa_attend on `stream`.
 * It differs only in scheduling: the indexer scores the entries that were
 * complete before this append on `stream` while the append runs on a side
 * stream of the calling thread; after the join it scores the entries the
 * append added, then top-k and attention follow.  (The pages' step order is
 * kept for every value: an entry's score does not depend on when it is
 * computed.)  Arguments as in the four calls; ws_indexer as for
 * csla_indexer_scores, ws_step = csla_workspace_size(cfg,
 * CSLA_OP_CSA_DECODE_STEP, B, k) bytes (16-byte aligned).  CSA only (m = 4).
 * The thread's first call on a device creates its side stream and two
 * events; make it before any stream capture (captured calls then fork and
 * join the capture like any two-stream work).
 */
int csla_csa_decode_step(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                         const int32_t *slots, int32_t B, int32_t T, int32_t max_len, const void *kv_new,
                         const void *kidx_new, int32_t kv_dtype, const csla_compress_params *p,
                         const void *cq, int32_t cq_dtype, const void *W_iq, int32_t w_dtype,
                         const float *head_w, float *scores, int32_t scores_stride, int32_t k,
                         int32_t *idx, const void *q, int32_t q_dtype, const float *sink,
                         const float *gamma_q, void *out, int32_t out_dtype, int32_t variant,
                         void *ws_indexer, size_t ws_indexer_bytes, void *ws_step,
                         size_t ws_step_bytes, csla_stream_t stream);

/*
 * csla_indexer_scores_noalloc -- csla_indexer_scores for callers that cannot
 * allocate device memory.  The pages have no counterpart: this is an
 * interface convenience, not a step of the method.
 * Some callers cannot call cudaMalloc at all (a framework that owns and has
 * reserved the whole memory pool, code running inside an allocator hook or
 * a host callback, an embedding restricted to the buffers it was given).
 * This entry point takes the same inputs and outputs as csla_indexer_scores
 * but no workspace: its scratch is one fixed array of
 * CSLA_NOALLOC_INDEXER_SCRATCH_BYTES inside the library, present on every
 * GPU that loads libcsla until the process exits.  Limit: B * NQ * dI * 2
 * bytes <= CSLA_NOALLOC_INDEXER_SCRATCH_BYTES, NQ = 3*HI rounded up to 16
 * (64 requests at HI = 16, dI = 128); larger batches return CSLA_ERR_ARG
 * without launching.  The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress, with that device current); make that first
 * call before any stream capture.  The address is cached for the life of the
 * process and not looked up again after a cudaDeviceReset of that device.  Every call shares the array: calls that
 * overlap on the GPU race on it, calls ordered on one stream do not.  It
 * calls no allocation routine.
 */
#define CSLA_NOALLOC_INDEXER_SCRATCH_BYTES 786432
int csla_indexer_scores_noalloc(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                                const int32_t *slots, int32_t B, const csla_queries *qs,
                                int32_t max_len, const void *cq,
                                int32_t cq_dtype, const void *W_iq, int32_t w_dtype,
                                const float *head_w, float *scores, int32_t scores_stride,
                                csla_stream_t stream);

/* Scratch bytes an entry point needs for B requests (0 for ops with none).
 * `max_len`: context bound (INDEXER, HCA_ATTEND) or k (CSA_ATTEND). */
size_t csla_workspace_size(const csla_cfg *cfg, int32_t op, int32_t B, int32_t max_len);

/* Synchronise `stream`, then read and clear the device error word of the
 * current device.  Returns CSLA_OK, or CSLA_ERR_DEVICE with the CSLA_DEVERR_*
 * bits in *bits (bits may be NULL), or CSLA_ERR_CUDA. */
int csla_device_error(csla_stream_t stream, uint32_t *bits);

/*
 * csla_check_wait_timeout -- exercise of the failure path every kernel's
 * bounded waits share (the pages have no counterpart: an operational check).
 * Launches one CTA on `stream` whose thread waits, with the library's own
 * bounded mbarrier wait, on a barrier that nobody arrives at, for at most
 * limit_us microseconds (1 .. 2000000); the wait gives up, sets
 * CSLA_DEVERR_TIMEOUT in the device error word and the kernel returns, so
 * csla_device_error() afterwards reports CSLA_ERR_DEVICE with that bit and
 * the context stays usable.  (The kernels' own waits give up after 2 s.)
 * Errors: CSLA_ERR_ARG for a limit outside the range; CSLA_ERR_CUDA if the
 * launch fails.
 */
int csla_check_wait_timeout(uint32_t limit_us, csla_stream_t stream);

/*
 * Context-parallel prefill (haiqwa "DeepSeek-V4" blog, §百万 token
 * 怎么切分到多张卡: the compressed KV of one long request is built by R ranks,
 * each compressing the blocks that close inside its own token range, then
 * exchanged by one all-gather and reassembled by a select-and-pad step).
 * Every rank holds a full copy of the request's paged cache (same block
 * table shape; page ids may differ per rank).  These two calls are the
 * data movement on either side of the all-gather; the exchange itself is
 * the caller's collective (NCCL all-gather of equal-sized buffers).
 *
 * Entry record (csla_cp_record_bytes(cfg) bytes, a multiple of 16):
 *   [row_bytes: the entry's row][key: dI*2 bytes bf16 or dI bytes E4M3, CSA
 *   only][f32 row scale][f32 key scale, 0 for bf16 keys][zero pad].
 *
 * csla_cp_select: records 0..n-1 of `recs` = entries b_lo..b_lo+n-1 of
 *   request `slot` (in block order); records n..E_max-1 are zero (padding).
 *   recs [E_max][record] device, 16-byte aligned; 0 <= n <= E_max.
 * csla_cp_place: for every rank r < R and j < n[r], record r*E_max + j of
 *   `recs` becomes entry b_lo[r] + j of request `slot`; padding records are
 *   skipped.  b_lo, n: HOST arrays of R int32 (copied at the call);
 *   1 <= R <= CSLA_CP_MAX_RANKS.
 * slot: the request's row of the block table (0 <= slot < st->n_slots;
 * only st->n_slots is read).  A block whose page the block table does not
 * map sets CSLA_DEVERR_PAGE and is skipped.  Errors: CSLA_ERR_ARG on null/bad sizes or misalignment;
 * CSLA_ERR_UNSUPPORTED on shapes.
 */
#define CSLA_CP_MAX_RANKS 64
int32_t csla_cp_record_bytes(const csla_cfg *cfg);
int csla_cp_select(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, int32_t slot,
                   int32_t b_lo, int32_t n, int32_t E_max, uint8_t *recs, csla_stream_t stream);
int csla_cp_place(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, int32_t slot,
                  const uint8_t *recs, int32_t R, int32_t E_max, const int32_t *b_lo, const int32_t *n,
                  csla_stream_t stream);

/* Static text for a status code. */
const char *csla_strerror(int status);

/* Library version as major*10000 + minor*100 + patch. */
int csla_version(void);

/*
 * Device timeline (libraries built with -DCSLA_TIMELINE only, e.g.
 * `build.py --timeline OUT.so`; absent from normal builds).  Thread 0 of
 * every CTA of every library kernel appends one record
 *   { uint32 kernel id, uint32 linear CTA index, uint64 t_start,
 *     uint64 t_waited (0 if the CTA exited before its grid-dependency wait),
 *     uint64 t_exit, uint64 marks[8] (kernel-specific points, 0 if unset),
 *     uint64 clock_start, uint64 clock_exit (SM cycle counter) }
 *   (global-timer nanoseconds, 112 bytes)
 * to a device buffer of 65536 records.  csla_timeline_read synchronises the
 * device and copies up to `bytes` of records to host memory `records`,
 * storing how many in *count; csla_timeline_clear synchronises and empties
 * the buffer.  Kernel ids: 1 compress, 2 tail update, 3 index-query
 * projection, 4 wide projection, 5 indexer, 6 top-k, (7 unused),
 * 8 attention, 9 chunk combine.
 */
#ifdef CSLA_TIMELINE
int csla_timeline_read(void *records, size_t bytes, uint32_t *count);
int csla_timeline_clear(void);
#endif

#ifdef __cplusplus
}
#endif

#endif /* CSLA_H */
