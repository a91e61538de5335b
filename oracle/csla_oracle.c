/*
 * csla_oracle.c -- plain, slow, fp64 CPU definition of the CSA/HCA compressed
 * attention hot path.  TEST INFRASTRUCTURE ONLY: nothing in the product path
 * may link, load or call this file.  Only tests/, the smoke check and the
 * CPU-baseline leg of bench.py use it.  It shares no code, header, table or
 * constant with the CUDA library; the cache byte format is re-derived here
 * from its written definition.
 *
 * Sources (page title, section):
 *   [haiqwa]  haiqwa.github.io "DeepSeek-V4" blog
 *             §CSA：压缩稀疏注意力, §HCA：重度压缩注意力, §RMSNorm归一化,
 *             §Partial RoPE位置编码, §让注意力学会"忽略", §索引可见性处理
 *   [silicon] 硅星人 article "DeepSeek V4 ... 让token大降价" (bjxrzxf.com),
 *             §两大压缩注意力 (sub-sections CSA / HCA and the cache paragraphs)
 *   [aieng]   "DeepSeek-V4深度拆解：一篇论文同时做了五件大事", §2 CSA/HCA混合注意力
 *   OCP 8-bit Floating Point Specification (OFP8) rev 1.0, E4M3 encoding.
 *
 * Where the pages are silent the reading used is stated at the function.
 * Every arithmetic step is fp64 except the two places where a float value
 * decides an integer code (fp8 / bf16 quantisation): there the decision is
 * taken on the fp32 value, the precision the kernels decide in.
 *
 * Parity status: every function below is pinned by tests under
 * tests/test_oracle_*.py (closed forms, invariants, brute force, library
 * routines, a second numpy transcription).  None is "parity unpinned".
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------ */
/* Number formats                                                      */
/* ------------------------------------------------------------------ */

/* E4M3 (OCP OFP8 "E4M3FN"): sign, 4 exponent bits (bias 7), 3 mantissa bits,
 * no infinities, S.1111.111 is NaN, largest finite 448, subnormals m*2^-9. */
double csla_orc_e4m3_value(unsigned code)
{
    unsigned s = (code >> 7) & 1u, e = (code >> 3) & 15u, m = code & 7u;
    double mag;
    if (e == 15u && m == 7u) return NAN;
    if (e == 0u) mag = ldexp((double)m, -9);
    else mag = ldexp(1.0 + (double)m / 8.0, (int)e - 7);
    return s ? -mag : mag;
}

/* Round an fp32 value to the nearest E4M3 value, ties to even mantissa,
 * values beyond 448 clamp to +-448 (the "satfinite" convention), NaN -> 0x7F.
 * Works on the exact value of the float in double arithmetic. */
unsigned csla_orc_e4m3_from_f32(float vf)
{
    double v = (double)vf, a;
    unsigned s;
    int e;
    double step, q, r, fl;
    if (isnan(v)) return 0x7Fu;
    s = signbit(v) ? 0x80u : 0u;
    a = fabs(v);
    if (a >= 448.0) return s | 0x7Eu;
    if (a == 0.0) return s;
    e = (int)floor(log2(a));
    /* guard against log2 rounding at exact powers of two */
    if (ldexp(1.0, e) > a) e -= 1;
    if (ldexp(1.0, e + 1) <= a) e += 1;
    if (e < -6) step = ldexp(1.0, -9);          /* subnormal grid */
    else step = ldexp(1.0, e - 3);              /* 3 mantissa bits */
    q = a / step;                               /* exact: step is 2^k */
    fl = floor(q);
    r = q - fl;
    if (r > 0.5) fl += 1.0;
    else if (r == 0.5 && fmod(fl, 2.0) != 0.0) fl += 1.0;
    a = fl * step;                              /* rounded magnitude */
    if (a > 448.0) a = 448.0;
    if (a == 0.0) return s;
    if (a < ldexp(1.0, -6)) return s | (unsigned)(a / ldexp(1.0, -9));
    e = (int)floor(log2(a));
    if (ldexp(1.0, e) > a) e -= 1;
    if (ldexp(1.0, e + 1) <= a) e += 1;
    return s | ((unsigned)(e + 7) << 3) | (unsigned)((a / ldexp(1.0, e) - 1.0) * 8.0);
}

/* bfloat16: the upper 16 bits of an IEEE binary32. */
double csla_orc_bf16_value(unsigned h)
{
    uint32_t u = (uint32_t)(h & 0xFFFFu) << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* fp32 -> bf16, round to nearest even on the dropped 16 bits; NaN stays NaN. */
unsigned csla_orc_bf16_from_f32(float f)
{
    uint32_t u;
    memcpy(&u, &f, 4);
    if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (u >> 16) | 0x0040u;
    u += 0x7FFFu + ((u >> 16) & 1u);
    return u >> 16;
}

/* ------------------------------------------------------------------ */
/* Row primitives                                                      */
/* ------------------------------------------------------------------ */

/* RMSNorm ([haiqwa] §RMSNorm归一化: an extra RMSNorm on every query head and on
 * the single compressed-KV head before core attention).
 * y = x / sqrt(mean(x^2) + eps) * gamma. */
void csla_orc_rmsnorm(const double *x, const double *gamma, int D, double eps, double *y)
{
    double ss = 0.0, r;
    int d;
    for (d = 0; d < D; ++d) ss += x[d] * x[d];
    r = 1.0 / sqrt(ss / (double)D + eps);
    for (d = 0; d < D; ++d) y[d] = x[d] * r * (gamma ? gamma[d] : 1.0);
}

/* Partial RoPE ([silicon] §两大压缩注意力, last paragraph of the HCA part:
 * RoPE on the last 64 dims of q and KV only; [haiqwa] §Partial RoPE位置编码).
 * Reading: interleaved pairs (D-dr+2i, D-dr+2i+1), angle pos * theta^(-2i/dr). */
void csla_orc_rope(double *y, int D, int d_rope, long long pos, double theta)
{
    int i, base = D - d_rope;
    for (i = 0; i < d_rope / 2; ++i) {
        double inv = pow(theta, -(2.0 * i) / (double)d_rope);
        double ang = (double)pos * inv;
        double c = cos(ang), s = sin(ang);
        double a = y[base + 2 * i], b = y[base + 2 * i + 1];
        y[base + 2 * i] = a * c - b * s;
        y[base + 2 * i + 1] = a * s + b * c;
    }
}

/* Mixed-precision cache row ([haiqwa] §Partial RoPE位置编码, the mixed-precision storage paragraph;
 * [silicon] same paragraph: RoPE dims bf16, the other dims fp8).
 * Row bytes: [0, D-dr) = E4M3 codes of dims 0..D-dr-1, then dr little-endian
 * bf16 values of dims D-dr..D-1.  One fp32 scale per row for the fp8 part:
 * scale = amax/448 (1 when amax == 0), code = E4M3(y/scale).
 * The scale, the division and both roundings are taken on fp32(y). */
void csla_orc_quantize(const double *y, int D, int d_rope, uint8_t *row, float *scale_out)
{
    int dn = D - d_rope, d;
    float amax = 0.0f, scale;
    for (d = 0; d < dn; ++d) {
        float v = fabsf((float)y[d]);
        if (v > amax) amax = v;
    }
    scale = (amax > 0.0f) ? amax / 448.0f : 1.0f;
    for (d = 0; d < dn; ++d) row[d] = (uint8_t)csla_orc_e4m3_from_f32((float)y[d] / scale);
    for (d = 0; d < d_rope; ++d) {
        unsigned h = csla_orc_bf16_from_f32((float)y[dn + d]);
        row[dn + 2 * d] = (uint8_t)(h & 0xFFu);
        row[dn + 2 * d + 1] = (uint8_t)(h >> 8);
    }
    *scale_out = scale;
}

/* The value a cache row stands for: code * scale for the fp8 dims, the bf16
 * value for the RoPE dims (fp64, exact). */
void csla_orc_dequantize(const uint8_t *row, float scale, int D, int d_rope, double *x)
{
    int dn = D - d_rope, d;
    for (d = 0; d < dn; ++d) x[d] = csla_orc_e4m3_value(row[d]) * (double)scale;
    for (d = 0; d < d_rope; ++d)
        x[dn + d] = csla_orc_bf16_value((unsigned)row[dn + 2 * d] | ((unsigned)row[dn + 2 * d + 1] << 8));
}

/* Token-level compressor ([haiqwa] §CSA：压缩稀疏注意力: one cache entry per block
 * of m tokens; [silicon] §CSA: Token-Level Compressor, m=4; §HCA: m'=128).
 * The pages give no formula.  Reading: one scalar gate per token,
 * g_i = <x_i, wg> + gb[i]; alpha = softmax_i(g); out = sum_i alpha_i x_i. */
void csla_orc_gate_pool(const double *xs, int m, int width, const double *wg, const double *gb,
                        double *out, double *alpha)
{
    int i, d;
    double gmax = -INFINITY, z = 0.0;
    double *g = (double *)malloc(sizeof(double) * (size_t)m);
    for (i = 0; i < m; ++i) {
        double acc = gb ? gb[i] : 0.0;
        for (d = 0; d < width; ++d) acc += xs[(size_t)i * width + d] * wg[d];
        g[i] = acc;
        if (acc > gmax) gmax = acc;
    }
    for (i = 0; i < m; ++i) { g[i] = exp(g[i] - gmax); z += g[i]; }
    for (d = 0; d < width; ++d) out[d] = 0.0;
    for (i = 0; i < m; ++i) {
        double a = g[i] / z;
        if (alpha) alpha[i] = a;
        for (d = 0; d < width; ++d) out[d] += a * xs[(size_t)i * width + d];
    }
    free(g);
}

/* Per-channel gated pooling (the compressor variant with a gate per
 * channel; the pages give no compressor formula at all, see gate_pool).
 * Reading: channel d of token i has the gate g_id = x_id * w_d + b_id
 * (b is [m][width]); alpha_id = softmax over the m tokens of g_.d, per
 * channel; out_d = sum_i alpha_id x_id.  With w = 0 and b_id = beta_i for
 * every d it is gate_pool with wg = 0, gb = beta. */
void csla_orc_gate_pool_channel(const double *xs, int m, int width, const double *w, const double *b,
                                double *out)
{
    int i, d;
    for (d = 0; d < width; ++d) {
        double gmax = -INFINITY, z = 0.0, acc = 0.0;
        for (i = 0; i < m; ++i) {
            double g = xs[(size_t)i * width + d] * w[d] + b[(size_t)i * width + d];
            if (g > gmax) gmax = g;
        }
        for (i = 0; i < m; ++i) z += exp(xs[(size_t)i * width + d] * w[d] + b[(size_t)i * width + d] - gmax);
        for (i = 0; i < m; ++i) {
            double a = exp(xs[(size_t)i * width + d] * w[d] + b[(size_t)i * width + d] - gmax) / z;
            acc += a * xs[(size_t)i * width + d];
        }
        out[d] = acc;
    }
}

/* Sliding-window row of token `pos` ([haiqwa] §Partial RoPE位置编码, sliding-window paragraph;
 * [silicon] §两大压缩注意力: the last 128 raw tokens kept uncompressed).
 * Reading: the row gets the same RMSNorm (gamma_kv), RoPE at its own position
 * and the same mixed-precision format as a compressed entry. */
void csla_orc_window_row(const double *x, const double *gamma, int D, int d_rope, double eps,
                         double theta, long long pos, uint8_t *row, float *scale)
{
    double *y = (double *)malloc(sizeof(double) * (size_t)D);
    csla_orc_rmsnorm(x, gamma, D, eps, y);
    csla_orc_rope(y, D, d_rope, pos, theta);
    csla_orc_quantize(y, D, d_rope, row, scale);
    free(y);
}

/* Compressed entry of block bk ([silicon] §CSA/§HCA): pool the m raw rows of
 * the block, RMSNorm, RoPE at the block's first position bk*m, quantise. */
void csla_orc_compressed_row(const double *xs, int m, const double *wg, const double *gb,
                             const double *gamma, int D, int d_rope, double eps, double theta,
                             long long bk, uint8_t *row, float *scale)
{
    double *c = (double *)malloc(sizeof(double) * (size_t)D);
    double *y = (double *)malloc(sizeof(double) * (size_t)D);
    csla_orc_gate_pool(xs, m, D, wg, gb, c, NULL);
    csla_orc_rmsnorm(c, gamma, D, eps, y);
    csla_orc_rope(y, D, d_rope, bk * (long long)m, theta);
    csla_orc_quantize(y, D, d_rope, row, scale);
    free(c);
    free(y);
}

void csla_orc_key_bf16(const double *c, int dI, uint16_t *key);

/* Compressed index key of a CSA block ([silicon] §CSA: the indexer derives its own
 * compressed keys from the same KV hidden states and scores queries against them).
 * Reading: its own scalar gate (wgi, gbi), no norm, no RoPE, stored bf16
 * (rounded from fp32). */
void csla_orc_index_key(const double *xis, int m, const double *wgi, const double *gbi, int dI,
                        uint16_t *key)
{
    int e;
    double *c = (double *)malloc(sizeof(double) * (size_t)dI);
    csla_orc_gate_pool(xis, m, dI, wgi, gbi, c, NULL);
    csla_orc_key_bf16(c, dI, key);
    free(c);
}

/* Storage of a pooled index key c (dI values): bf16 rounded from fp32. */
void csla_orc_key_bf16(const double *c, int dI, uint16_t *key)
{
    int e;
    for (e = 0; e < dI; ++e) key[e] = (uint16_t)csla_orc_bf16_from_f32((float)c[e]);
}

/* E4M3 storage of an index key ([haiqwa] §FP4精度加速: the indexer's key /
 * query path runs in low precision).  The pages fix neither the format nor
 * the scale.  Reading: one power-of-two scale per entry, the smallest
 * s = 2^e (-126 <= e <= 127) with 448 * s >= amax, amax = max |key dim| of
 * the fp32 key; each dim's code is E4M3(fp32 key / s), round to nearest
 * even, saturating (the division by a power of two is exact).  The key dim
 * then reads e4m3(code) * s.  This is the definition written out: e is
 * found by counting up from -126. */
double csla_orc_key_scale_e4m3(double amax)
{
    int e = -126;
    while (e < 127 && 448.0 * ldexp(1.0, e) < amax) ++e;
    return ldexp(1.0, e);
}

void csla_orc_key_e4m3(const double *c, int dI, uint8_t *codes, float *scale_out)
{
    int e;
    double amax = 0.0, s;
    for (e = 0; e < dI; ++e) {
        double v = fabs((double)(float)c[e]);
        if (v > amax) amax = v;
    }
    s = csla_orc_key_scale_e4m3(amax);
    for (e = 0; e < dI; ++e) codes[e] = (uint8_t)csla_orc_e4m3_from_f32((float)((double)(float)c[e] / s));
    *scale_out = (float)s;
}

void csla_orc_index_key_e4m3(const double *xis, int m, const double *wgi, const double *gbi, int dI,
                             uint8_t *codes, float *scale_out)
{
    double *c = (double *)malloc(sizeof(double) * (size_t)dI);
    csla_orc_gate_pool(xis, m, dI, wgi, gbi, c, NULL);
    csla_orc_key_e4m3(c, dI, codes, scale_out);
    free(c);
}

/* ------------------------------------------------------------------ */
/* Lightning indexer, top-k, attention                                 */
/* ------------------------------------------------------------------ */

/* Index query: up-projection of the latent cq (dc) to HI heads of dI
 * ([silicon] §CSA: the query is first reduced to a dc=1024 latent, then
 * expanded to the index heads).
 * W is [HI*dI][dc] (row r = output feature r).  qI[j*dI+e] = sum_c W[j*dI+e][c] cq[c]. */
void csla_orc_index_query(const double *cq, const double *W, int HI, int dI, int dc, double *qI)
{
    int r, c;
    for (r = 0; r < HI * dI; ++r) {
        double acc = 0.0;
        for (c = 0; c < dc; ++c) acc += W[(size_t)r * dc + c] * cq[c];
        qI[r] = acc;
    }
}

/* Index scores ([silicon] §CSA: ReLU activation, scores against the compressed
 * index keys).  Reading: score_s = sum_j w_j * max(0, <qI_j, k_s>). */
void csla_orc_index_scores(const double *qI, const double *w, int HI, int dI, const double *keys,
                           long long N, double *scores)
{
    long long s;
    for (s = 0; s < N; ++s) {
        double acc = 0.0;
        int j, e;
        for (j = 0; j < HI; ++j) {
            double dot = 0.0;
            for (e = 0; e < dI; ++e) dot += qI[(size_t)j * dI + e] * keys[(size_t)s * dI + e];
            acc += w[j] * (dot > 0.0 ? dot : 0.0);
        }
        scores[s] = acc;
    }
}

/* Top-k selector ([silicon] §CSA: picks the 512 (Pro: 1024) most relevant
 * compressed blocks).  Reading: total order (score descending, index
 * ascending); take min(k, n); return them in ascending index order; pad -1. */
/* Sort key: the score travels with its index, so the comparator needs no
 * shared state (requests are sorted concurrently under OpenMP). */
typedef struct {
    double score;
    int32_t index;
} orc_ranked;
static int cmp_rank(const void *pa, const void *pb)
{
    const orc_ranked *a = (const orc_ranked *)pa, *b = (const orc_ranked *)pb;
    if (a->score > b->score) return -1;
    if (a->score < b->score) return 1;
    return (a->index < b->index) ? -1 : (a->index > b->index);
}
static int cmp_int(const void *pa, const void *pb)
{
    int32_t a = *(const int32_t *)pa, b = *(const int32_t *)pb;
    return (a < b) ? -1 : (a > b);
}
void csla_orc_topk(const double *scores, int n, int k, int32_t *idx)
{
    int i, take = n < k ? n : k;
    orc_ranked *order = (orc_ranked *)malloc(sizeof(orc_ranked) * (size_t)(n > 0 ? n : 1));
    int32_t *picked = (int32_t *)malloc(sizeof(int32_t) * (size_t)(take > 0 ? take : 1));
    for (i = 0; i < n; ++i) {
        order[i].score = scores[i];
        order[i].index = i;
    }
    qsort(order, (size_t)n, sizeof(orc_ranked), cmp_rank);
    for (i = 0; i < take; ++i) picked[i] = order[i].index;
    qsort(picked, (size_t)take, sizeof(int32_t), cmp_int);
    for (i = 0; i < k; ++i) idx[i] = (i < take) ? picked[i] : -1;
    free(order);
    free(picked);
}

/* Core MQA with sink ([silicon] §CSA: top-k entries concatenated with the 128
 * window tokens, multi-query attention; §两大压缩注意力: a learnable sink logit
 * per head added to the softmax denominator; [haiqwa] §让注意力学会"忽略").
 * For every head h: qh = RoPE(RMSNorm(q_h) * gamma_q, t);
 *   s_j = <qh, x_j> / sqrt(D);  M = max(z_h, max_j s_j);
 *   p_j = e^(s_j - M) / (e^(z_h - M) + sum_j e^(s_j - M));  o_h = sum_j p_j x_j.
 * Reading: K = V = the cached row (one shared KV head, no de-rotation);
 * the sink carries no value vector.  rows: [n][D] fp64 values. */
void csla_orc_attend(const double *q, const double *gamma_q, long long t, const double *rows, int n,
                     const double *sink, int H, int D, int d_rope, double eps, double theta,
                     double *out, double *sink_share)
{
    int h, j, d;
    double *qh = (double *)malloc(sizeof(double) * (size_t)D);
    double *s = (double *)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
    double inv_sqrt_d = 1.0 / sqrt((double)D);
    for (h = 0; h < H; ++h) {
        double mx = sink[h], den, ez;
        csla_orc_rmsnorm(q + (size_t)h * D, gamma_q, D, eps, qh);
        csla_orc_rope(qh, D, d_rope, t, theta);
        for (j = 0; j < n; ++j) {
            double acc = 0.0;
            for (d = 0; d < D; ++d) acc += qh[d] * rows[(size_t)j * D + d];
            s[j] = acc * inv_sqrt_d;
            if (s[j] > mx) mx = s[j];
        }
        ez = exp(sink[h] - mx);
        den = ez;
        for (j = 0; j < n; ++j) { s[j] = exp(s[j] - mx); den += s[j]; }
        for (d = 0; d < D; ++d) out[(size_t)h * D + d] = 0.0;
        for (j = 0; j < n; ++j) {
            double p = s[j] / den;
            for (d = 0; d < D; ++d) out[(size_t)h * D + d] += p * rows[(size_t)j * D + d];
        }
        if (sink_share) sink_share[h] = ez / den;
    }
    free(qh);
    free(s);
}

/* ------------------------------------------------------------------ */
/* Cache addressing ([silicon] last cache paragraph: a classical-cache block   */
/* covers lcm(4,128) = 128 raw tokens -> 32 CSA entries or 1 HCA entry;        */
/* the state cache holds the window and the tail).                             */
/* ------------------------------------------------------------------ */

#define ORC_PAGE_TOKENS 128

/* Number of compressed entries visible at context length L ([haiqwa]
 * §索引可见性处理: visibility computable by rule).  Reading: block b is
 * visible to the query at t = L-1 iff its last token (b+1)m-1 <= t. */
long long csla_orc_n_visible(long long L, int m) { return L / m; }

/* Row pointer of compressed entry b of request slot `slot`. */
static const uint8_t *orc_entry_row(const uint8_t *rows, const int32_t *block_table, int bt_stride,
                                    int slot, long long b, int m, int row_bytes)
{
    int epp = ORC_PAGE_TOKENS / m;
    long long page = block_table[(size_t)slot * bt_stride + b / epp];
    return rows + ((size_t)page * epp + (size_t)(b % epp)) * row_bytes;
}
static float orc_entry_scale(const float *scales, const int32_t *block_table, int bt_stride, int slot,
                             long long b, int m)
{
    int epp = ORC_PAGE_TOKENS / m;
    long long page = block_table[(size_t)slot * bt_stride + b / epp];
    return scales[(size_t)page * epp + (size_t)(b % epp)];
}

/* Decode the attention set of one request: the selected (or all) compressed
 * entries in ascending order, then the window tokens max(0,L-n_win)..L-1 in
 * ascending position.  sel == NULL means every visible entry (HCA).
 * Returns the number of rows written to out ([n][D]). */
int csla_orc_gather_set(const uint8_t *rows, const float *scales, const int32_t *block_table,
                        int bt_stride, const uint8_t *win_rows, const float *win_scales, int n_win,
                        int slot, long long L, int m, int D, int d_rope, const int32_t *sel, int k,
                        double *out)
{
    int row_bytes = (D - d_rope) + 2 * d_rope;
    long long nv = csla_orc_n_visible(L, m), b, p, p0;
    int n = 0, i;
    if (sel) {
        for (i = 0; i < k; ++i) {
            if (sel[i] < 0) continue;
            b = sel[i];
            csla_orc_dequantize(orc_entry_row(rows, block_table, bt_stride, slot, b, m, row_bytes),
                                orc_entry_scale(scales, block_table, bt_stride, slot, b, m), D, d_rope,
                                out + (size_t)n * D);
            ++n;
        }
    } else {
        for (b = 0; b < nv; ++b) {
            csla_orc_dequantize(orc_entry_row(rows, block_table, bt_stride, slot, b, m, row_bytes),
                                orc_entry_scale(scales, block_table, bt_stride, slot, b, m), D, d_rope,
                                out + (size_t)n * D);
            ++n;
        }
    }
    p0 = L - n_win;
    if (p0 < 0) p0 = 0;
    for (p = p0; p < L; ++p) {
        size_t ring = (size_t)slot * n_win + (size_t)(p % n_win);
        csla_orc_dequantize(win_rows + ring * row_bytes, win_scales[ring], D, d_rope, out + (size_t)n * D);
        ++n;
    }
    return n;
}

/* Decoded index keys of the first N compressed entries of a request. */
/* Decoded index keys of entries 0..N-1 of `slot`: bf16 values, or (kscale
 * not NULL) E4M3 codes times the entry's scale. */
void csla_orc_gather_keys(const void *kidx, const float *kscale, const int32_t *block_table, int bt_stride,
                          int slot, long long N, int m, int dI, double *keys)
{
    int epp = ORC_PAGE_TOKENS / m, e;
    long long b;
    for (b = 0; b < N; ++b) {
        long long page = block_table[(size_t)slot * bt_stride + b / epp];
        size_t ent = (size_t)page * epp + (size_t)(b % epp);
        if (kscale) {
            const uint8_t *k = (const uint8_t *)kidx + ent * dI;
            for (e = 0; e < dI; ++e) keys[(size_t)b * dI + e] = csla_orc_e4m3_value(k[e]) * (double)kscale[ent];
        } else {
            const uint16_t *k = (const uint16_t *)kidx + ent * dI;
            for (e = 0; e < dI; ++e) keys[(size_t)b * dI + e] = csla_orc_bf16_value(k[e]);
        }
    }
}

/* One whole decode step of a CSA layer (indexer -> top-k -> attention) for
 * B requests, straight from the cache bytes.  Used for sampled parity checks
 * and, timed, as the CPU baseline.  q: [B][H][D]; cq: [B][dc]; W: [HI*dI][dc];
 * head_w: [B][HI]; idx_out: [B][k]; out: [B][H][D].  OpenMP over requests. */
void csla_orc_csa_decode(const uint8_t *rows, const float *scales, const void *kidx, const float *kscale,
                         const int32_t *block_table, int bt_stride, const uint8_t *win_rows,
                         const float *win_scales, int n_win, const int32_t *slots,
                         const int32_t *lens, int B, int m, int H, int D, int d_rope, int HI, int dI,
                         int dc, int k, double eps, double theta, const double *q,
                         const double *gamma_q, const double *cq, const double *W,
                         const double *head_w, const double *sink, int32_t *idx_out, double *out)
{
    int b;
#pragma omp parallel for schedule(dynamic, 1)
    for (b = 0; b < B; ++b) {
        long long L = lens[b], nv = csla_orc_n_visible(L, m);
        double *qI = (double *)malloc(sizeof(double) * (size_t)HI * dI);
        double *keys = (double *)malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1) * dI);
        double *sc = (double *)malloc(sizeof(double) * (size_t)(nv > 0 ? nv : 1));
        double *set = (double *)malloc(sizeof(double) * (size_t)(k + n_win) * D);
        int n;
        csla_orc_index_query(cq + (size_t)b * dc, W, HI, dI, dc, qI);
        csla_orc_gather_keys(kidx, kscale, block_table, bt_stride, slots[b], nv, m, dI, keys);
        csla_orc_index_scores(qI, head_w + (size_t)b * HI, HI, dI, keys, nv, sc);
        csla_orc_topk(sc, (int)nv, k, idx_out + (size_t)b * k);
        n = csla_orc_gather_set(rows, scales, block_table, bt_stride, win_rows, win_scales, n_win,
                                slots[b], L, m, D, d_rope, idx_out + (size_t)b * k, k, set);
        csla_orc_attend(q + (size_t)b * H * D, gamma_q, L - 1, set, n, sink, H, D, d_rope, eps, theta,
                        out + (size_t)b * H * D, NULL);
        free(qI);
        free(keys);
        free(sc);
        free(set);
    }
}

/* One decode step of an HCA layer: attention over every visible compressed
 * entry plus the window ([silicon] §HCA: no indexer, no top-k selector). */
void csla_orc_hca_decode(const uint8_t *rows, const float *scales, const int32_t *block_table,
                         int bt_stride, const uint8_t *win_rows, const float *win_scales, int n_win,
                         const int32_t *slots, const int32_t *lens, int B, int m, int H, int D,
                         int d_rope, double eps, double theta, const double *q, const double *gamma_q,
                         const double *sink, double *out)
{
    int b;
#pragma omp parallel for schedule(dynamic, 1)
    for (b = 0; b < B; ++b) {
        long long L = lens[b], nv = csla_orc_n_visible(L, m);
        double *set = (double *)malloc(sizeof(double) * (size_t)(nv + n_win) * D);
        int n = csla_orc_gather_set(rows, scales, block_table, bt_stride, win_rows, win_scales, n_win,
                                    slots[b], L, m, D, d_rope, NULL, 0, set);
        csla_orc_attend(q + (size_t)b * H * D, gamma_q, L - 1, set, n, sink, H, D, d_rope, eps, theta,
                        out + (size_t)b * H * D, NULL);
        free(set);
    }
}

int csla_orc_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
