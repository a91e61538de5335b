// api.cu -- the C ABI of libcsla (declared in include/csla.h): host-side
// argument checks, TMA descriptor encoding and kernel launches.
#include <math.h>
#include <string.h>

#include "../../include/csla.h"
#include "common.cuh"
#include "kernels.h"

namespace {

using namespace csla;

int num_sms_current() {
    static int cached[64];
    static bool init[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (dev >= 0 && dev < 64 && init[dev]) return cached[dev];
    int n = 148;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (dev >= 0 && dev < 64) {
        cached[dev] = n;
        init[dev] = true;
    }
    return n;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 2-D bf16 tensor [rows][cols] (cols contiguous), box = 64 cols x box_rows, 128B swizzle.
bool encode_bf16_2d(CUtensorMap *map, const void *ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// 2-D byte tensor [rows][cols] (cols contiguous, cols <= 128), box = cols x
// box_rows, 128B swizzle: the E4M3 index keys.
bool encode_u8_2d(CUtensorMap *map, const void *ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    EncodeTiledFn f = encode_fn();
    if (!f) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols};
    cuuint32_t box[2] = {(cuuint32_t)cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = f(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_cfg(const csla_cfg *c) {
    if (!c) return CSLA_ERR_ARG;
    if (c->d_rope != 64 || (c->D != 128 && c->D != 512) || (c->m != 4 && c->m != 128) || c->n_win != 128)
        return CSLA_ERR_UNSUPPORTED;
    if (c->H < 1 || c->H > 64) return CSLA_ERR_UNSUPPORTED;
    if (!(c->eps >= 0.f) || !(c->rope_theta > 0.f)) return CSLA_ERR_ARG;
    if (c->key_fmt != CSLA_KEY_BF16 && c->key_fmt != CSLA_KEY_E4M3) return CSLA_ERR_UNSUPPORTED;
    if (c->key_fmt == CSLA_KEY_E4M3 && c->m == 4 && c->dI != 128) return CSLA_ERR_UNSUPPORTED;
    if (c->gate != CSLA_GATE_TOKEN && c->gate != CSLA_GATE_CHANNEL) return CSLA_ERR_UNSUPPORTED;
    return CSLA_OK;
}

int check_csa_indexer_shape(const csla_cfg *c) {
    if (c->m != 4) return CSLA_ERR_UNSUPPORTED;
    if (c->dI != 64 && c->dI != 128) return CSLA_ERR_UNSUPPORTED;
    if (c->HI != 4 && c->HI != 8 && c->HI != 16) return CSLA_ERR_UNSUPPORTED;
    if (c->dc < 8 || c->dc > 4096 || c->dc % 8) return CSLA_ERR_UNSUPPORTED;
    return CSLA_OK;
}

int nq_of(int HI) { return (3 * HI + 15) / 16 * 16; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? CSLA_OK : CSLA_ERR_CUDA; }

int row_bytes_of(const csla_cfg *c) { return (c->D - c->d_rope) + 2 * c->d_rope; }

// Query rows: q_len required; a window source needs its scales and bases.
int check_queries(const csla_queries *qs) {
    if (!qs) return CSLA_OK;
    if (!qs->q_len) return CSLA_ERR_ARG;
    if (qs->win_rows && (!qs->win_scales || !qs->win_base || qs->n_win_rows < 1 || !aligned16(qs->win_rows)))
        return CSLA_ERR_ARG;
    return CSLA_OK;
}

// Attention workspace: the chunk partials (H*D + 2H floats per chunk).
size_t attend_ws(const csla_cfg *c, int B, long long max_rows) {
    const size_t per = ((size_t)c->H * c->D + 2 * (size_t)c->H) * sizeof(float);
    return (size_t)B * attend_max_chunks(max_rows) * per;
}

}  // namespace

#ifdef CSLA_TIMELINE
namespace csla {
__device__ TimelineRec g_timeline[kTimelineCap];
__device__ unsigned int g_timeline_n = 0;
}  // namespace csla
#endif

namespace csla {
namespace {
// One thread waits, with the library's bounded wait, on an mbarrier that
// expects one arrival nobody makes; the wait gives up after limit_ns and
// records CSLA_DEVERR_TIMEOUT.
__global__ void __launch_bounds__(32) wait_check_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        mbar_wait_limit(&bar, 0, nullptr, limit_ns);
    }
}
}  // namespace
}  // namespace csla

extern "C" {

int csla_version(void) { return 100; }

int csla_check_wait_timeout(uint32_t limit_us, csla_stream_t stream) {
    if (limit_us < 1 || limit_us > 2000000) return CSLA_ERR_ARG;
    csla::wait_check_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>((uint64_t)limit_us * 1000ull);
    return cudaGetLastError() == cudaSuccess ? CSLA_OK : CSLA_ERR_CUDA;
}

#ifdef CSLA_TIMELINE
int csla_timeline_read(void *records, size_t bytes, uint32_t *count) {
    unsigned int n = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return CSLA_ERR_CUDA;
    if (cudaMemcpyFromSymbol(&n, csla::g_timeline_n, sizeof(n)) != cudaSuccess) return CSLA_ERR_CUDA;
    if (n > csla::kTimelineCap) n = csla::kTimelineCap;
    size_t want = (size_t)n * sizeof(csla::TimelineRec);
    if (want > bytes) want = bytes / sizeof(csla::TimelineRec) * sizeof(csla::TimelineRec);
    if (want && cudaMemcpyFromSymbol(records, csla::g_timeline, want) != cudaSuccess) return CSLA_ERR_CUDA;
    if (count) *count = (uint32_t)(want / sizeof(csla::TimelineRec));
    return CSLA_OK;
}
int csla_timeline_clear(void) {
    unsigned int zero = 0;
    if (cudaDeviceSynchronize() != cudaSuccess) return CSLA_ERR_CUDA;
    return cudaMemcpyToSymbol(csla::g_timeline_n, &zero, sizeof(zero)) == cudaSuccess ? CSLA_OK : CSLA_ERR_CUDA;
}
#endif

const char *csla_strerror(int s) {
    switch (s) {
        case CSLA_OK: return "ok";
        case CSLA_ERR_ARG: return "invalid argument";
        case CSLA_ERR_UNSUPPORTED: return "unsupported shape";
        case CSLA_ERR_CUDA: return "CUDA error";
        case CSLA_ERR_DEVICE: return "device-side input error";
        default: return "unknown status";
    }
}

// csla_indexer_topk workspace: the indexer's query terms, then sample
// scores [B][kSampleCols], thresholds [B], candidate counts [B][kCandSub],
// row flags [B] and candidates [B][kCandCap] (key, entry), each part
// 16-byte aligned.
struct ItkLayout {
    size_t sample, t0, cnt, flag, cand, total;
};
static size_t up16(size_t x) { return (x + 15) / 16 * 16; }
static ItkLayout itk_layout(int B, int NQ, int dI) {
    ItkLayout l;
    l.sample = up16((size_t)B * NQ * dI * 2);
    l.t0 = l.sample + up16((size_t)B * kSampleCols * 4);
    l.cnt = l.t0 + up16((size_t)B * 4);
    l.flag = l.cnt + up16((size_t)B * kCandSub * 4);
    l.cand = l.flag + up16((size_t)B * 4);
    l.total = l.cand + (size_t)B * kCandCap * 8;
    return l;
}

size_t csla_workspace_size(const csla_cfg *cfg, int32_t op, int32_t B, int32_t max_len) {
    if (check_cfg(cfg) != CSLA_OK || B < 1 || max_len < 0) return 0;
    switch (op) {
        case CSLA_OP_INDEXER:
            if (check_csa_indexer_shape(cfg) != CSLA_OK) return 0;
            return (size_t)B * nq_of(cfg->HI) * cfg->dI * 2;
        case CSLA_OP_TOPK: return 0;
        case CSLA_OP_CSA_ATTEND: return attend_ws(cfg, B, (long long)max_len + cfg->n_win);
        case CSLA_OP_HCA_ATTEND: return attend_ws(cfg, B, (long long)max_len / cfg->m + cfg->n_win);
        case CSLA_OP_CSA_DECODE_STEP:
            return attend_ws(cfg, B, (long long)max_len + cfg->n_win) + ((size_t)B * 4 + 15) / 16 * 16;
        case CSLA_OP_INDEXER_TOPK:
            if (check_csa_indexer_shape(cfg) != CSLA_OK) return 0;
            return itk_layout(B, nq_of(cfg->HI), cfg->dI).total;
        default: return 0;
    }
}

int csla_device_error(csla_stream_t stream, uint32_t *bits) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return CSLA_ERR_CUDA;
    unsigned int v = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&v, csla::g_dev_err, sizeof(v)) != cudaSuccess) return CSLA_ERR_CUDA;
    if (v && cudaMemcpyToSymbol(csla::g_dev_err, &zero, sizeof(zero)) != cudaSuccess) return CSLA_ERR_CUDA;
    if (bits) *bits = v;
    return v ? CSLA_ERR_DEVICE : CSLA_OK;
}

static int prep_compress(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                         int32_t B, int32_t T, const void *kv_new, const void *kidx_new, int32_t kv_dtype,
                         const csla_compress_params *p, const csla_token_rows *tok, CompressArgs *out) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!st || !cache || !slots || !kv_new || !p || B < 1 || T < 1 || T > 65535) return CSLA_ERR_ARG;
    if (st->n_slots < 1 || B > 65535) return CSLA_ERR_ARG;
    if (kv_dtype != CSLA_F32 && kv_dtype != CSLA_BF16) return CSLA_ERR_ARG;
    if (!st->win_rows || !st->win_scales || !st->tail_kv || !st->len || !cache->rows || !cache->scales ||
        !cache->block_table || cache->bt_stride < 1 || cache->n_pages < 1)
        return CSLA_ERR_ARG;
    if (!p->gamma_kv || !p->wg || !p->gb) return CSLA_ERR_ARG;
    const bool per_channel = cfg->gate == CSLA_GATE_CHANNEL;
    if (per_channel && (!aligned16(p->gb) || (p->gbi && !aligned16(p->gbi)))) return CSLA_ERR_ARG;
    if (!aligned16(st->tail_kv)) return CSLA_ERR_ARG;
    if (tok && (!tok->rows || !tok->scales || tok->offset < 0 || (long long)tok->offset + T > tok->stride))
        return CSLA_ERR_ARG;
    const bool csa = cfg->m == 4;
    if (csa) {
        if (cfg->dI < 4 || cfg->dI > 512 || cfg->dI % 4 || !kidx_new || !cache->kidx || !st->tail_idx || !p->wgi ||
            !p->gbi)
            return CSLA_ERR_ARG;
        if (!aligned16(st->tail_idx)) return CSLA_ERR_ARG;
        if (cfg->key_fmt == CSLA_KEY_E4M3 && !cache->kscale) return CSLA_ERR_ARG;
    }
    CompressArgs a{};
    a.m = cfg->m; a.D = cfg->D; a.d_rope = cfg->d_rope; a.dI = csa ? cfg->dI : 0; a.n_win = cfg->n_win;
    a.theta = cfg->rope_theta; a.eps = cfg->eps;
    a.freq = rope_freq(cfg->rope_theta, cfg->d_rope);
    a.slots = slots; a.B = B; a.T = T;
    a.kv_new = kv_new; a.kidx_new = csa ? kidx_new : nullptr;
    a.gamma_kv = p->gamma_kv; a.wg = p->wg; a.gb = p->gb; a.wgi = p->wgi; a.gbi = p->gbi;
    a.win_rows = st->win_rows; a.win_scales = st->win_scales; a.tail_kv = st->tail_kv;
    a.tail_idx = csa ? st->tail_idx : nullptr; a.len = st->len;
    a.rows = cache->rows; a.scales = cache->scales; a.kidx = csa ? cache->kidx : nullptr;
    a.key_fmt = csa ? cfg->key_fmt : CSLA_KEY_BF16;
    a.gate = cfg->gate;
    a.kscale = csa ? cache->kscale : nullptr;
    a.block_table = cache->block_table; a.bt_stride = cache->bt_stride; a.n_pages = cache->n_pages;
    a.n_slots = st->n_slots;
    if (tok) {
        a.tok_rows = tok->rows; a.tok_scales = tok->scales; a.tok_stride = tok->stride; a.tok_offset = tok->offset;
    }
    *out = a;
    return CSLA_OK;
}

int csla_compress_append(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                         int32_t B, int32_t T, const void *kv_new, const void *kidx_new, int32_t kv_dtype,
                         const csla_compress_params *p, const csla_token_rows *tok, csla_stream_t stream) {
    CompressArgs a;
    const int rc = prep_compress(cfg, st, cache, slots, B, T, kv_new, kidx_new, kv_dtype, p, tok, &a);
    if (rc) return rc;
    return cuda_status(launch_compress_append(a, kv_dtype == CSLA_BF16, reinterpret_cast<cudaStream_t>(stream)));
}

int csla_window_rows(const csla_cfg *cfg, const csla_state *st, const int32_t *slots, int32_t B, int32_t n,
                     uint8_t *rows_out, float *scales_out, int32_t stride, csla_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!st || !st->len || !st->win_rows || !st->win_scales || st->n_slots < 1 || !slots || !rows_out ||
        !scales_out || B < 1 || B > 65535 || n < 1 || n > cfg->n_win || stride < n)
        return CSLA_ERR_ARG;
    if (!aligned16(rows_out) || !aligned16(st->win_rows)) return CSLA_ERR_ARG;
    WindowRowsArgs a{};
    a.slots = slots; a.len = st->len; a.B = B; a.n = n; a.n_win = cfg->n_win; a.n_slots = st->n_slots;
    a.row_bytes = row_bytes_of(cfg); a.win_rows = st->win_rows; a.win_scales = st->win_scales;
    a.out_rows = rows_out; a.out_scales = scales_out; a.stride = stride;
    return cuda_status(launch_window_rows(a, reinterpret_cast<cudaStream_t>(stream)));
}

struct IndexerLaunch {
    IndexerArgs a;
    CUtensorMap kmap, qmap;
    ProjMaps pm;
    bool gemm;   // the projection runs on the tensor cores (bf16 cq and W_iq)
    bool cq_bf16, w_bf16;
};

static int prep_indexer(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                        int32_t B, const csla_queries *qs, int32_t max_len, const void *cq, int32_t cq_dtype,
                        const void *W_iq, int32_t w_dtype, const float *head_w, float *scores, int32_t scores_stride,
                        void *workspace, size_t workspace_bytes, IndexerLaunch *L) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    rc = check_csa_indexer_shape(cfg);
    if (rc) return rc;
    if (!st || !st->len || !cache || !cache->kidx || !cache->block_table || !slots || !cq || !W_iq || !head_w ||
        !scores || !workspace || B < 1 || max_len < 1)
        return CSLA_ERR_ARG;
    if ((cq_dtype != CSLA_F32 && cq_dtype != CSLA_BF16) || (w_dtype != CSLA_F32 && w_dtype != CSLA_BF16))
        return CSLA_ERR_ARG;
    if (scores_stride < max_len / cfg->m || check_queries(qs)) return CSLA_ERR_ARG;
    if (workspace_bytes < csla_workspace_size(cfg, CSLA_OP_INDEXER, B, max_len)) return CSLA_ERR_ARG;
    if (!aligned16(cq) || !aligned16(W_iq) || !aligned16(cache->kidx) || !aligned16(workspace)) return CSLA_ERR_ARG;
    const bool e4m3 = cfg->key_fmt == CSLA_KEY_E4M3;
    if (e4m3 && !cache->kscale) return CSLA_ERR_ARG;
    const int NQ = nq_of(cfg->HI);
    CUtensorMap kmap, qmap;
    memset(&qmap, 0, sizeof(qmap));
    if (e4m3) {
        // E4M3 keys: one 128-byte box per entry row; the kernel builds its
        // four-term E4M3 query operand from the projection's bf16 terms
        if (!encode_u8_2d(&kmap, cache->kidx, (uint64_t)cfg->dI, (uint64_t)cache->n_pages * 32, 32))
            return CSLA_ERR_CUDA;
    } else if (!encode_bf16_2d(&kmap, cache->kidx, (uint64_t)cfg->dI, (uint64_t)cache->n_pages * 32, 32)) {
        return CSLA_ERR_CUDA;
    }
    const int G = (qs && qs->one_request) ? indexer_rows_per_cta(e4m3 ? 4 * cfg->HI : NQ) : 1;
    if (!e4m3 && !encode_bf16_2d(&qmap, workspace, (uint64_t)cfg->dI, (uint64_t)B * NQ, (uint32_t)(G * NQ)))
        return CSLA_ERR_CUDA;
    L->kmap = kmap;
    L->qmap = qmap;
    L->cq_bf16 = cq_dtype == CSLA_BF16;
    L->w_bf16 = w_dtype == CSLA_BF16;
    L->gemm = L->cq_bf16 && L->w_bf16;
    if (L->gemm && (!encode_bf16_2d(&L->pm.cq, cq, (uint64_t)cfg->dc, (uint64_t)B, 128) ||
                    !encode_bf16_2d(&L->pm.w, W_iq, (uint64_t)cfg->dc, (uint64_t)cfg->HI * cfg->dI,
                                    (uint32_t)iq_gemm_bn(B))))
        return CSLA_ERR_CUDA;
    IndexerArgs a{};
    a.m = cfg->m; a.HI = cfg->HI; a.dI = cfg->dI; a.dc = cfg->dc; a.NQ = NQ;
    a.slots = slots; a.len = st->len; a.block_table = cache->block_table; a.bt_stride = cache->bt_stride;
    a.n_pages = cache->n_pages; a.n_slots = st->n_slots; a.B = B;
    const int nvmax = max_len / cfg->m;
    a.tiles_per_req = (nvmax + 127) / 128;
    if (a.tiles_per_req < 1) a.tiles_per_req = 1;
    a.max_len = max_len;
    a.cq = cq; a.W = W_iq; a.head_w = head_w; a.scores = scores; a.scores_stride = scores_stride;
    a.q_ws = reinterpret_cast<uint16_t *>(workspace);
    a.key_fmt = cfg->key_fmt;
    a.kidx8 = e4m3 ? reinterpret_cast<const uint8_t *>(cache->kidx) : nullptr;
    a.kscale = e4m3 ? cache->kscale : nullptr;
    a.q_len = qs ? qs->q_len : nullptr;
    a.rows_per_cta = G;
    L->a = a;
    return CSLA_OK;
}

int csla_indexer_scores(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                        int32_t B, const csla_queries *qs, int32_t max_len, const void *cq, int32_t cq_dtype, const void *W_iq,
                        int32_t w_dtype, const float *head_w, float *scores, int32_t scores_stride, void *workspace,
                        size_t workspace_bytes, csla_stream_t stream) {
    IndexerLaunch L;
    const int rc = prep_indexer(cfg, st, cache, slots, B, qs, max_len, cq, cq_dtype, W_iq, w_dtype, head_w, scores,
                                scores_stride, workspace, workspace_bytes, &L);
    if (rc) return rc;
    return cuda_status(launch_indexer(L.a, L.cq_bf16, L.w_bf16, L.kmap, L.qmap, num_sms_current(),
                                      reinterpret_cast<cudaStream_t>(stream), true, L.gemm ? &L.pm : nullptr));
}

static int prep_topk(const csla_cfg *cfg, const csla_state *st, const int32_t *slots, int32_t B,
                     const csla_queries *qs, int32_t max_len,
                     const float *scores, int32_t scores_stride, int32_t k, int32_t *idx, TopkArgs *out) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!st || !st->len || !slots || !scores || !idx || B < 1 || max_len < 0 || k < 1 || k > 2048)
        return CSLA_ERR_ARG;
    if (scores_stride < max_len / cfg->m || check_queries(qs)) return CSLA_ERR_ARG;
    TopkArgs a{};
    a.scores = scores; a.stride = scores_stride; a.slots = slots; a.len = st->len;
    a.m = cfg->m; a.k = k; a.B = B; a.max_n = max_len / cfg->m; a.idx = idx; a.n_slots = st->n_slots;
    a.q_len = qs ? qs->q_len : nullptr;
    *out = a;
    return CSLA_OK;
}

int csla_topk_select(const csla_cfg *cfg, const csla_state *st, const int32_t *slots, int32_t B,
                     const csla_queries *qs, int32_t max_len, const float *scores, int32_t scores_stride, int32_t k,
                     int32_t *idx, csla_stream_t stream) {
    TopkArgs a;
    const int rc = prep_topk(cfg, st, slots, B, qs, max_len, scores, scores_stride, k, idx, &a);
    if (rc) return rc;
    return cuda_status(launch_topk(a, reinterpret_cast<cudaStream_t>(stream)));
}

int csla_indexer_topk(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                      int32_t B, const csla_queries *qs, int32_t max_len, const void *cq, int32_t cq_dtype,
                      const void *W_iq, int32_t w_dtype, const float *head_w, int32_t k, int32_t *idx,
                      float *scores, int32_t scores_stride, void *workspace, size_t workspace_bytes,
                      csla_stream_t stream) {
    if (k < 1 || k > 2048) return CSLA_ERR_ARG;
    if (workspace_bytes < csla_workspace_size(cfg, CSLA_OP_INDEXER_TOPK, B, max_len)) return CSLA_ERR_ARG;
    TopkArgs t;
    int rc = prep_topk(cfg, st, slots, B, qs, max_len, scores, scores_stride, k, idx, &t);
    if (rc) return rc;
    IndexerLaunch L;
    rc = prep_indexer(cfg, st, cache, slots, B, qs, max_len, cq, cq_dtype, W_iq, w_dtype, head_w, scores,
                      scores_stride, workspace, workspace_bytes, &L);
    if (rc) return rc;
    const ItkLayout l = itk_layout(B, L.a.NQ, cfg->dI);
    uint8_t *w = reinterpret_cast<uint8_t *>(workspace);
    CandArgs c{};
    c.sample = reinterpret_cast<const float *>(w + l.sample);
    c.page_step = (L.a.tiles_per_req * 4 + 31) / 32;   // 32 sample pages spread over the longest row
    if (c.page_step < 1) c.page_step = 1;
    c.cand_t0 = reinterpret_cast<uint32_t *>(w + l.t0);
    c.cand_cnt = reinterpret_cast<int32_t *>(w + l.cnt);
    c.row_flag = reinterpret_cast<int32_t *>(w + l.flag);
    c.cand = reinterpret_cast<const uint2 *>(w + l.cand);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int nsm = num_sms_current();
    // 1. projection, then the sample pass (scores of the sample tiles only)
    IndexerArgs as = L.a;
    as.page_step = c.page_step;
    as.scores = reinterpret_cast<float *>(w + l.sample);
    as.scores_stride = kSampleCols;
    cudaError_t e = launch_indexer(as, L.cq_bf16, L.w_bf16, L.kmap, L.qmap, nsm, s, true, L.gemm ? &L.pm : nullptr);
    // 2. thresholds; 3. candidate pass; 4. selection among the candidates
    if (e == cudaSuccess) e = launch_cand_threshold(t, c, s);
    IndexerArgs ac = L.a;
    ac.cand_t0 = c.cand_t0;
    ac.cand = reinterpret_cast<uint2 *>(w + l.cand);
    ac.cand_cnt = c.cand_cnt;
    ac.cand_cap = kCandCap / kCandSub;
    if (e == cudaSuccess) e = launch_indexer(ac, L.cq_bf16, L.w_bf16, L.kmap, L.qmap, nsm, s, false);
    if (e == cudaSuccess) e = launch_cand_select(t, c, s);
    // 5. flagged rows: scores stored (kPersistSlices CTAs per row group,
    //    each a run of tiles; groups without a flagged row exit at once),
    //    then the top-k on them
    IndexerArgs af = L.a;
    af.persist = kPersistSlices;
    af.row_flag = c.row_flag;
    if (e == cudaSuccess) e = launch_indexer(af, L.cq_bf16, L.w_bf16, L.kmap, L.qmap, nsm, s, false);
    TopkArgs tf = t;
    tf.row_flag = c.row_flag;
    if (e == cudaSuccess) e = launch_topk(tf, s);
    return cuda_status(e);
}

static int prep_attend(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                       int32_t B, const csla_queries *qs, int32_t max_len, const void *q, int32_t q_dtype,
                       const int32_t *idx, int32_t k, const float *sink, const float *gamma_q, void *out,
                       int32_t out_dtype, int32_t variant, void *workspace, size_t workspace_bytes,
                       AttendArgs *res) {
    if (!st || !st->len || !st->win_rows || !st->win_scales || !cache || !cache->rows || !cache->scales ||
        !cache->block_table || !slots || !q || !sink || !gamma_q || !out || !workspace || B < 1)
        return CSLA_ERR_ARG;
    if ((q_dtype != CSLA_F32 && q_dtype != CSLA_BF16) || (out_dtype != CSLA_F32 && out_dtype != CSLA_BF16))
        return CSLA_ERR_ARG;
    if (variant < CSLA_VARIANT_AUTO || variant > CSLA_VARIANT_STARVED || check_queries(qs)) return CSLA_ERR_ARG;
    if (!aligned16(q) || !aligned16(cache->rows) || !aligned16(st->win_rows) || !aligned16(workspace))
        return CSLA_ERR_ARG;
    // row locations are 32-bit indices into the cache, the ring and the window-row buffer
    if ((long long)cache->n_pages * (CSLA_PAGE_TOKENS / cfg->m) > 0xFFFFFFFFll ||
        (long long)st->n_slots * cfg->n_win > 0xFFFFFFFFll)
        return CSLA_ERR_UNSUPPORTED;
    AttendArgs a{};
    a.m = cfg->m; a.D = cfg->D; a.d_rope = cfg->d_rope; a.H = cfg->H; a.n_win = cfg->n_win;
    a.theta = cfg->rope_theta; a.eps = cfg->eps;
    a.freq = rope_freq(cfg->rope_theta, cfg->d_rope);
    a.slots = slots; a.len = st->len; a.B = B; a.q = q; a.idx = idx; a.k = idx ? k : 0;
    a.sink = sink; a.gamma_q = gamma_q;
    a.rows = cache->rows; a.scales = cache->scales; a.block_table = cache->block_table;
    a.bt_stride = cache->bt_stride; a.n_pages = cache->n_pages; a.n_slots = st->n_slots;
    a.win_rows = st->win_rows; a.win_scales = st->win_scales; a.out = out;
    a.part = reinterpret_cast<float *>(workspace);
    const long long max_rows = idx ? (long long)k + cfg->n_win : (long long)max_len / cfg->m + cfg->n_win;
    a.max_chunks = attend_max_chunks(max_rows);
    a.max_len = max_len;
    if (qs) {
        a.q_len = qs->q_len;
        a.src_rows = qs->win_rows; a.src_scales = qs->win_scales; a.win_base = qs->win_base;
        a.n_src = qs->n_win_rows;
    }
    if (workspace_bytes < attend_ws(cfg, B, max_rows)) return CSLA_ERR_ARG;
    *res = a;
    return CSLA_OK;
}

static int attend_common(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                         int32_t B, const csla_queries *qs, int32_t max_len, const void *q, int32_t q_dtype,
                         const int32_t *idx, int32_t k, const float *sink, const float *gamma_q, void *out,
                         int32_t out_dtype, int32_t variant, void *workspace, size_t workspace_bytes,
                         csla_stream_t stream) {
    AttendArgs a;
    const int rc = prep_attend(cfg, st, cache, slots, B, qs, max_len, q, q_dtype, idx, k, sink, gamma_q, out, out_dtype,
                               variant, workspace, workspace_bytes, &a);
    if (rc) return rc;
    return cuda_status(launch_attend(a, q_dtype == CSLA_BF16, out_dtype == CSLA_BF16, variant, num_sms_current(),
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int csla_csa_attend(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                    int32_t B, const csla_queries *qs, const void *q, int32_t q_dtype, const int32_t *idx, int32_t k, const float *sink,
                    const float *gamma_q, void *out, int32_t out_dtype, int32_t variant, void *workspace,
                    size_t workspace_bytes, csla_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!idx || k < 1 || k > 2048) return CSLA_ERR_ARG;
    // Without max_len the bound on the context is the int32 range.
    return attend_common(cfg, st, cache, slots, B, qs, 0x7FFFFFFF, q, q_dtype, idx, k, sink, gamma_q, out, out_dtype,
                         variant, workspace, workspace_bytes, stream);
}

int csla_hca_attend(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                    int32_t B, const csla_queries *qs, int32_t max_len, const void *q, int32_t q_dtype, const float *sink,
                    const float *gamma_q, void *out, int32_t out_dtype, int32_t variant, void *workspace,
                    size_t workspace_bytes, csla_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (max_len < 1) return CSLA_ERR_ARG;
    return attend_common(cfg, st, cache, slots, B, qs, max_len, q, q_dtype, nullptr, 0, sink, gamma_q, out, out_dtype,
                         variant, workspace, workspace_bytes, stream);
}

// Side stream and fork/join events of the calling thread on each device
// (created on the thread's first decode-step call on that device).
struct SideStream {
    cudaStream_t s = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
static thread_local SideStream tl_side[64];

static int side_stream(SideStream **out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return CSLA_ERR_CUDA;
    SideStream &x = tl_side[dev];
    if (!x.s) {
        if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
            cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess)
            return CSLA_ERR_CUDA;
    }
    *out = &x;
    return CSLA_OK;
}

int csla_csa_decode_step(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, const int32_t *slots,
                         int32_t B, int32_t T, int32_t max_len, const void *kv_new, const void *kidx_new,
                         int32_t kv_dtype, const csla_compress_params *p, const void *cq, int32_t cq_dtype,
                         const void *W_iq, int32_t w_dtype, const float *head_w, float *scores,
                         int32_t scores_stride, int32_t k, int32_t *idx, const void *q, int32_t q_dtype,
                         const float *sink, const float *gamma_q, void *out, int32_t out_dtype, int32_t variant,
                         void *ws_indexer, size_t ws_indexer_bytes, void *ws_step, size_t ws_step_bytes,
                         csla_stream_t stream) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (cfg->m != 4) return CSLA_ERR_UNSUPPORTED;
    if (!idx || k < 1 || k > 2048 || !ws_step || !aligned16(ws_step)) return CSLA_ERR_ARG;
    CompressArgs ca;
    IndexerLaunch il;
    TopkArgs ta;
    AttendArgs aa;
    rc = prep_compress(cfg, st, cache, slots, B, T, kv_new, kidx_new, kv_dtype, p, nullptr, &ca);
    if (rc) return rc;
    rc = prep_indexer(cfg, st, cache, slots, B, nullptr, max_len, cq, cq_dtype, W_iq, w_dtype, head_w, scores,
                      scores_stride, ws_indexer, ws_indexer_bytes, &il);
    if (rc) return rc;
    rc = prep_topk(cfg, st, slots, B, nullptr, max_len, scores, scores_stride, k, idx, &ta);
    if (rc) return rc;
    const size_t att_bytes = attend_ws(cfg, B, (long long)k + cfg->n_win);
    if (ws_step_bytes < csla_workspace_size(cfg, CSLA_OP_CSA_DECODE_STEP, B, k)) return CSLA_ERR_ARG;
    rc = prep_attend(cfg, st, cache, slots, B, nullptr, 0x7FFFFFFF, q, q_dtype, idx, k, sink, gamma_q, out,
                     out_dtype, variant, ws_step, att_bytes, &aa);
    if (rc) return rc;
    int32_t *len0 = reinterpret_cast<int32_t *>(reinterpret_cast<uint8_t *>(ws_step) + att_bytes);
    SideStream *side = nullptr;
    rc = side_stream(&side);
    if (rc) return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // old entries (complete before this append) on the caller's stream while
    // the append runs on the side stream; then the entries it added
    IndexerArgs old_a = il.a, new_a = il.a;
    old_a.range = 1;
    old_a.len0 = len0;
    new_a.range = 2;
    new_a.len0 = len0;
    new_a.tiles_per_req = ((T / cfg->m + 2) + 127) / 128 + 1;
    cudaError_t e = launch_len_snapshot(slots, st->len, B, st->n_slots, len0, s);
    if (e == cudaSuccess) e = cudaEventRecord(side->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(side->s, side->fork, 0);
    if (e == cudaSuccess) {
        // forked: from here on the side stream is always joined back into the
        // caller's stream, also when a launch fails (an unjoined fork would
        // invalidate a stream capture), and the first error is returned
        e = launch_compress_append(ca, kv_dtype == CSLA_BF16, side->s);
        cudaError_t ej = cudaEventRecord(side->join, side->s);
        if (e == cudaSuccess) e = launch_indexer(old_a, il.cq_bf16, il.w_bf16, il.kmap, il.qmap, num_sms_current(), s, true,
                                                 il.gemm ? &il.pm : nullptr);
        if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, side->join, 0);
        if (e == cudaSuccess) e = ej;
    }
    if (e == cudaSuccess)
        e = launch_indexer(new_a, il.cq_bf16, il.w_bf16, il.kmap, il.qmap, num_sms_current(), s, false);
    if (e == cudaSuccess) e = launch_topk(ta, s);
    if (e == cudaSuccess)
        e = launch_attend(aa, q_dtype == CSLA_BF16, out_dtype == CSLA_BF16, variant, num_sms_current(), s);
    return cuda_status(e);
}

// ---- context-parallel entry records

static int cp_key_bytes(const csla_cfg *cfg) {
    if (cfg->m != 4) return 0;
    return cfg->key_fmt == CSLA_KEY_E4M3 ? cfg->dI : 2 * cfg->dI;
}

int32_t csla_cp_record_bytes(const csla_cfg *cfg) {
    if (check_cfg(cfg) != CSLA_OK) return 0;
    return (row_bytes_of(cfg) + cp_key_bytes(cfg) + 8 + 15) / 16 * 16;
}

static int prep_cp(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, int32_t slot,
                   const void *recs, int32_t E_max, CpArgs *a) {
    int rc = check_cfg(cfg);
    if (rc) return rc;
    if (!st || slot >= st->n_slots) return CSLA_ERR_ARG;
    if (!cache || !cache->rows || !cache->scales || !cache->block_table || cache->bt_stride < 1 ||
        cache->n_pages < 1 || !recs || slot < 0 || E_max < 0)
        return CSLA_ERR_ARG;
    const bool csa = cfg->m == 4;
    if (csa && (!cache->kidx || (cfg->key_fmt == CSLA_KEY_E4M3 && !cache->kscale))) return CSLA_ERR_ARG;
    if (!aligned16(recs) || !aligned16(cache->rows) || (csa && !aligned16(cache->kidx))) return CSLA_ERR_ARG;
    *a = CpArgs{};
    a->slot = slot; a->epp = CSLA_PAGE_TOKENS / cfg->m; a->bt_stride = cache->bt_stride; a->n_pages = cache->n_pages;
    a->block_table = cache->block_table; a->rows = cache->rows; a->scales = cache->scales;
    a->kidx = csa ? static_cast<uint8_t *>(cache->kidx) : nullptr;
    a->kscale = csa && cfg->key_fmt == CSLA_KEY_E4M3 ? cache->kscale : nullptr;
    a->row_bytes = row_bytes_of(cfg); a->key_bytes = cp_key_bytes(cfg); a->rec_bytes = csla_cp_record_bytes(cfg);
    a->E_max = E_max;
    return CSLA_OK;
}

int csla_cp_select(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, int32_t slot,
                   int32_t b_lo, int32_t n, int32_t E_max, uint8_t *recs, csla_stream_t stream) {
    CpArgs a;
    int rc = prep_cp(cfg, st, cache, slot, recs, E_max, &a);
    if (rc) return rc;
    if (b_lo < 0 || n < 0 || n > E_max) return CSLA_ERR_ARG;
    a.place = 0; a.R = 1; a.b_lo[0] = b_lo; a.n[0] = n;
    a.recs = recs;
    return cuda_status(launch_cp_move(a, reinterpret_cast<cudaStream_t>(stream)));
}

int csla_cp_place(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache, int32_t slot,
                  const uint8_t *recs, int32_t R, int32_t E_max, const int32_t *b_lo, const int32_t *n,
                  csla_stream_t stream) {
    CpArgs a;
    int rc = prep_cp(cfg, st, cache, slot, recs, E_max, &a);
    if (rc) return rc;
    if (R < 1 || R > CSLA_CP_MAX_RANKS || !b_lo || !n) return CSLA_ERR_ARG;
    for (int r = 0; r < R; ++r) {
        if (b_lo[r] < 0 || n[r] < 0 || n[r] > E_max) return CSLA_ERR_ARG;
        a.b_lo[r] = b_lo[r];
        a.n[r] = n[r];
    }
    a.place = 1; a.R = R;
    a.recs = const_cast<uint8_t *>(recs);
    return cuda_status(launch_cp_move(a, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
