// indexer.cu -- lightning indexer (csla_indexer_scores).
//
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力, CSA part: the query
//   latent (dc = 1024) is up-projected to multi-head index queries; with a
//   ReLU they are scored against the compressed index keys, and the top-k
//   selector consumes the scores.
//
// Two kernels:
//  1. iq_project: qI = W_iq . cq for every request, one warp per output
//     feature, W read once per launch for the whole batch; each dot product
//     has a fixed summation order.  qI is stored as three bf16 terms
//     (hi = bf16(qI), mid = bf16(qI - hi), lo = bf16(qI - hi - mid)), so the
//     bf16 tensor-core products carry the full fp32 value of qI.
//  2. indexer: warp-specialised tcgen05 kernel; a CTA owns 8 consecutive
//     tiles of one request, a tile being 128 compressed entries (4 pages of
//     32).  Warp 0 loads the request's query operand once and streams key
//     tiles with TMA into a 3-stage ring (page ids fetched up front, one
//     lane per page); warp 1 issues UMMA (M=128 entries, N=NQ query rows,
//     K=dI) into one of two TMEM accumulators; warps 2-5 read the
//     accumulator (one entry per thread) and reduce
//       score = sum_j w_j * relu((acc[j] + acc[HI + j]) + acc[2HI + j])
//     in head order.  Every score depends only on its own entry and request.
//     Query rows of one request: G rows share each key tile, and a few CTAs
//     per row group each walk a run of tiles (page ids read per tile).
//     For csla_indexer_topk (separate instantiations): a sample mode (32
//     spread pages per row, scores into a small buffer), a candidate mode
//     (only the entries at or above a per-row threshold leave the kernel,
//     as (key, entry) pairs) and a row-flag mode for the rows that fall
//     back to stored scores.
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kProjThreads = 256;

template <typename T>
__device__ __forceinline__ void load8(const T *p, float (&v)[8]);
template <>
__device__ __forceinline__ void load8<float>(const float *p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
template <>
__device__ __forceinline__ void load8<__nv_bfloat16>(const __nv_bfloat16 *p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p));
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = bf16_bits_to_f32(w[i] & 0xFFFFu);
        v[2 * i + 1] = bf16_bits_to_f32(w[i] >> 16);
    }
}

constexpr int kProjWarps = kProjThreads / 32;   // output features per CTA
constexpr int kProjChunkB = 8;                   // requests' cq rows staged in shared memory at a time
constexpr int kProjKeepB = 128;                  // requests whose results are held before the wait

// One warp per output feature r; lane l covers 8-element chunks l, l+32, ...
// of the dc inputs.  The W row is read once into registers; the cq rows of
// the CTA's kProjKeepB requests (blockIdx.y) are staged in shared memory
// kProjChunkB requests at a time, split into two planes of 4-element halves
// so that a warp's 16-byte reads are contiguous (no bank conflicts).  Each
// request's value is one chain of fused multiply-adds over chunks then
// elements, then the warp's xor tree (the chains of a chunk's requests run
// interleaved): the same arithmetic whatever the batch.  The products are
// formed before the grid-dependency wait (W and cq are inputs of the call)
// and held in shared memory; the stores into the workspace follow the wait.
template <typename TC, typename TW>
__global__ void __launch_bounds__(kProjThreads, 2) iq_project_kernel(IndexerArgs a) {
    CSLA_TL_SCOPE(kTlIqProject);
    constexpr int kMaxCh = 4;   // dc <= 32 * 8 * kMaxCh = 1024 on this path
    __shared__ __align__(16) float4 cs[kProjChunkB][2][32 * kMaxCh];
    __shared__ uint16_t res[kProjKeepB][kProjWarps][3];
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.x * kProjWarps;
    const int r = r0 + warp;
    const bool active = r < a.HI * a.dI;
    const TW *w = reinterpret_cast<const TW *>(a.W) + (size_t)(active ? r : 0) * a.dc;
    const int nch = a.dc / 8;
    float wv[kMaxCh][8];
#pragma unroll
    for (int q = 0; q < kMaxCh; ++q) {
        const int ch = lane + 32 * q;
        if (active && ch < nch) load8<TW>(w + ch * 8, wv[q]);
        else
#pragma unroll
            for (int i = 0; i < 8; ++i) wv[q][i] = 0.f;
    }
    bool waited = false;
    const int b_begin = blockIdx.y * kProjKeepB, b_end = min(a.B, b_begin + kProjKeepB);
    int held0 = b_begin;   // first request whose results sit in res
    for (int b0 = b_begin; b0 < b_end; b0 += kProjChunkB) {
        const int nb = min(kProjChunkB, b_end - b0);
        __syncthreads();   // the previous chunk's cq rows are consumed
        for (int i = threadIdx.x; i < nb * nch; i += kProjThreads) {
            const int u = i / nch, ch = i % nch;
            float t[8];
            load8<TC>(reinterpret_cast<const TC *>(a.cq) + (size_t)(b0 + u) * a.dc + ch * 8, t);
            cs[u][0][ch] = make_float4(t[0], t[1], t[2], t[3]);
            cs[u][1][ch] = make_float4(t[4], t[5], t[6], t[7]);
        }
        __syncthreads();
        if (b0 == b_begin) CSLA_TL_MARK(0);
        if (active) {
            float acc[kProjChunkB];
#pragma unroll
            for (int u = 0; u < kProjChunkB; ++u) acc[u] = 0.f;
#pragma unroll
            for (int q = 0; q < kMaxCh; ++q) {
                const int ch = lane + 32 * q;
                if (ch < nch) {
#pragma unroll
                    for (int u = 0; u < kProjChunkB; ++u) {
                        if (u < nb) {
                            const float4 c0 = cs[u][0][ch], c1 = cs[u][1][ch];
                            const float cv[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
                            for (int i = 0; i < 8; ++i) acc[u] = __fmaf_rn(wv[q][i], cv[i], acc[u]);
                        }
                    }
                }
            }
#pragma unroll
            for (int u = 0; u < kProjChunkB; ++u) acc[u] = warp_sum(acc[u]);
            if (lane == 0) {
#pragma unroll
                for (int u = 0; u < kProjChunkB; ++u) {
                    if (u < nb) {
                        const uint16_t hi = f32_to_bf16_bits(acc[u]);
                        const float r1 = __fsub_rn(acc[u], bf16_bits_to_f32(hi));
                        const uint16_t mid = f32_to_bf16_bits(r1);
                        const uint16_t lo = f32_to_bf16_bits(__fsub_rn(r1, bf16_bits_to_f32(mid)));
                        uint16_t *o = res[(b0 + u) - held0][warp];
                        o[0] = hi;
                        o[1] = mid;
                        o[2] = lo;
                    }
                }
            }
        }
        const int held = b0 + nb - held0;
        if (b0 == b_begin) CSLA_TL_MARK(1);
        if (held == kProjKeepB || b0 + nb == b_end) {
            __syncthreads();
            CSLA_TL_MARK(2);
            if (!waited) {
                pdl_wait();
                CSLA_TL_WAITED();
                waited = true;
            }
            const int nf = min(kProjWarps, a.HI * a.dI - r0);
            for (int i = threadIdx.x; i < held * nf * 3; i += kProjThreads) {
                const int f = i % nf, t = (i / nf) % 3, bb = i / (3 * nf);
                const int rr = r0 + f, j = rr / a.dI, e = rr % a.dI;
                a.q_ws[((size_t)(held0 + bb) * a.NQ + t * a.HI + j) * a.dI + e] = res[bb][f][t];
            }
            held0 = b0 + nb;
        }
    }
    if (!waited) {
        pdl_wait();
        CSLA_TL_WAITED();
    }
}

// Same product for latents wider than 1024 (W row re-read per request).
template <typename TC, typename TW>
__global__ void __launch_bounds__(kProjThreads) iq_project_wide_kernel(IndexerArgs a) {
    CSLA_TL_SCOPE(kTlIqProjectWide);
    pdl_trigger();
    pdl_wait();
    CSLA_TL_WAITED();
    const int r = blockIdx.x * (kProjThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= a.HI * a.dI) return;
    const int j = r / a.dI, e = r % a.dI;
    const TW *w = reinterpret_cast<const TW *>(a.W) + (size_t)r * a.dc;
    const int nch = a.dc / 8;
    const int b_end = min(a.B, (int)(blockIdx.y + 1) * kProjKeepB);
    for (int b = blockIdx.y * kProjKeepB; b < b_end; ++b) {
        const TC *c = reinterpret_cast<const TC *>(a.cq) + (size_t)b * a.dc;
        float acc = 0.f;
        for (int ch = lane; ch < nch; ch += 32) {
            float wv[8], cv[8];
            load8<TW>(w + ch * 8, wv);
            load8<TC>(c + ch * 8, cv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc = __fmaf_rn(wv[i], cv[i], acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) {
            const uint16_t hi = f32_to_bf16_bits(acc);
            const float r1 = __fsub_rn(acc, bf16_bits_to_f32(hi));
            const uint16_t mid = f32_to_bf16_bits(r1);
            const uint16_t lo = f32_to_bf16_bits(__fsub_rn(r1, bf16_bits_to_f32(mid)));
            a.q_ws[((size_t)b * a.NQ + j) * a.dI + e] = hi;
            a.q_ws[((size_t)b * a.NQ + a.HI + j) * a.dI + e] = mid;
            a.q_ws[((size_t)b * a.NQ + 2 * a.HI + j) * a.dI + e] = lo;
        }
    }
}

constexpr int kTileE = 128;          // entries per tile
constexpr int kPageE = 32;           // CSA entries per 128-token page
constexpr int kTPC = 8;              // tiles per CTA (consecutive, one request)
// warp 0: TMA, warp 1: MMA, then 4 epilogue warps per set of query rows
// (set s takes the group's rows s, s + sets, ...): one set for G = 1, one
// per row up to 7 rows (balanced: 5 at 16 index heads), else four.
template <int G>
constexpr int idx_epi_sets() { return G == 1 ? 1 : (G <= 7 ? G : 4); }
template <int G>
constexpr int idx_threads() { return 64 + 128 * idx_epi_sets<G>(); }
// Query operand rows per query row: bf16 keys take three bf16 terms of every
// head (NQ = 3*HI rounded up to 16); E4M3 keys take four E4M3 terms (4*HI).
template <int HI>
constexpr int nq_e4m3() { return 4 * HI; }

// Key tiles arrive by TMA into a 3-stage ring: bf16 (2-D map, 64-dim boxes)
// or E4M3 codes (2-D map over bytes, one 128-byte box per entry row).
template <int DI, int NQ, int G, bool kE4M3>
struct IdxSmem {
    static constexpr int kStages = 3;
    static constexpr int kElt = kE4M3 ? 1 : 2;
    static constexpr int kKeyBytes = kTileE * DI * kElt;
    static constexpr int kQBytes = G * NQ * DI * kElt;
    // candidate staging (query rows of one request, G > 1): 64 (key, entry)
    // pairs per epilogue warp; none for decode rows (shared memory for two
    // CTAs per SM)
    static constexpr int kStageBytes = G > 1 ? 4 * idx_epi_sets<G>() * 64 * 8 : 0;
    static constexpr int kBytes = kStages * kKeyBytes + kQBytes + kStageBytes + 1024 /*align*/ +
                                  2048 /*barriers, pages, weights, term scales*/;
};

// Two accumulators of G*NQ columns, rounded up to a power of two >= 32.
template <int N>
constexpr uint32_t kTmemCols() {
    return 2 * N <= 32 ? 32 : (2 * N <= 64 ? 64 : (2 * N <= 128 ? 128 : (2 * N <= 256 ? 256 : 512)));
}

// E4M3 query operand of one (row, head): q (the fp32 sum of the projection's
// three bf16 terms, 4 dims per lane) split into four E4M3 terms with
// power-of-two scales, q ~ sum_t 2^(e_t) code_t: e_t as for index keys (the
// smallest 2^e with 448 * 2^e >= max |residual|), codes rounded to nearest
// even, each residual formed exactly.  After four terms the residual is
// below ~2^-19 of max |q|.  Warp-collective; lane l writes dims 4l..4l+3 of
// operand rows n_t = base + t*HI (SW128 K-major, 128 bytes per row) and lane
// 0 the scales sig[t*HI].
__device__ __forceinline__ void split_q_e4m3(float (&q)[4], uint8_t *qb, int base, int HI, float *sig) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
        float am = fmaxf(fmaxf(fabsf(q[0]), fabsf(q[1])), fmaxf(fabsf(q[2]), fabsf(q[3])));
        am = warp_max(am);
        const int ex = key_exp_e4m3(am);
        const float inv = __uint_as_float((uint32_t)(127 - min(ex, 126)) << 23);
        const float sc = __uint_as_float((uint32_t)(ex + 127) << 23);
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint8_t c = f32_to_e4m3(__fmul_rn(q[i], inv));
            const __half_raw h = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3);
            const float cv = __half2float(__half(h));
            q[i] = __fsub_rn(q[i], __fmul_rn(cv, sc));   // exact: the rounding residual
            word |= (uint32_t)c << (8 * i);
        }
        const int n = base + t * HI;
        *reinterpret_cast<uint32_t *>(qb + (n >> 3) * 1024 + (n & 7) * 128 + ((((lane >> 2) ^ (n & 7))) << 4) +
                                      4 * (lane & 3)) = word;
        if (lane == 0) sig[t * HI] = sc;
    }
}

// A warp's candidates of one (row, tile) whose list places are still to be
// read from the row counter (lane 0's `at`).
constexpr int kStageCands = 64;   // staged candidates per epilogue warp

struct Pending {
    unsigned mq = 0u;
    bool q = false;
    uint32_t key = 0u;
    int e = 0, row = 0, at = 0;
};

// CTA (blockIdx.x, blockIdx.y) scores tiles [blockIdx.x*kTPC, +kTPC) (128
// entries each) of the query rows r0 = blockIdx.y*G .. r0+G-1, which all
// read the keys of request slots[r0]: one key tile feeds one MMA of N = G*NQ
// query columns (decode: G = 1; query rows of one request: G > 1).
// kE4M3: keys are E4M3 codes with a power-of-two scale per entry, scored by
// kind::f8f6f4 MMAs against the four-term E4M3 query operand that the
// epilogue warps build before they start (NQ = 4*HI); the epilogue forms
// each head's dot product from its four terms and applies the entry scale.
template <int DI, int NQ, int HI, int G, bool kE4M3, bool kSel>
// decode rows (G = 1): two CTAs per SM (registers for 2 x 192 threads)
__global__ void __launch_bounds__(idx_threads<G>(), G == 1 ? 2 : 1)
    indexer_kernel(IndexerArgs a, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap qmap) {
    CSLA_TL_SCOPE(kTlIndexer);
    using S = IdxSmem<DI, NQ, G, kE4M3>;
    constexpr int kStages = S::kStages;
    constexpr int N = G * NQ;
    static_assert(N % 16 == 0 && N <= 256, "UMMA N for M = 128");
    static_assert(!kE4M3 || (DI == 128 && NQ == 4 * HI), "E4M3 keys: dI = 128, four query terms");
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *qbuf = base + kStages * S::kKeyBytes;
    uint2 *stage_all = reinterpret_cast<uint2 *>(qbuf + S::kQBytes);   // [epilogue warp][64] candidates
    uint64_t *bars = reinterpret_cast<uint64_t *>(qbuf + S::kQBytes + S::kStageBytes);
    uint64_t *full = bars, *empty = bars + kStages, *tfull = bars + 2 * kStages, *tempty = tfull + 2;
    uint64_t *qfull = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(qfull + 1);
    int *pages = reinterpret_cast<int *>(tmem_holder + 1);      // [kTPC * 4]
    int *row_nv = pages + kTPC * 4;                              // [G] entries scored below this (-1: skip)
    int *row_lo = row_nv + G;                                    // [G] first entry scored
    float *hw = reinterpret_cast<float *>(row_lo + G);           // [G][HI] head weights
    float *sig = hw + G * HI;                                    // [G][NQ] E4M3 query-term scales
    float *row_t0 = sig + G * NQ;                                // [G] candidate thresholds (scores)
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r0 = blockIdx.y * G;
    // the streaming-selection modes (sample, candidates, row flags) exist in
    // the kSel instantiations only; runs of tiles also for grouped rows
    const int persist = (kSel || G > 1) ? a.persist : 0;
    const int page_step = kSel ? a.page_step : 0;
    const int32_t *row_flag = kSel ? a.row_flag : nullptr;
    const uint32_t *cand_t0 = kSel ? a.cand_t0 : nullptr;
    if (persist && row_flag) {
        // the fallback of a streaming selection: most row groups have no
        // flagged row, so look before taking barriers and TMEM
        pdl_wait();
        int any = 0;
        if (threadIdx.x < G && r0 + threadIdx.x < a.B) any = row_flag[r0 + threadIdx.x] != 0;
        if (!__syncthreads_or(any)) return;
    }
    const int slot = __ldg(a.slots + r0);
    const bool slot_ok = slot >= 0 && slot < a.n_slots;
    __shared__ int s_t0;   // range 2: first tile of the request's new entries

    // ---- before the wait: barriers, TMEM, page ids, head weights
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull + i, 1);
            mbar_init(tempty + i, 4 * idx_epi_sets<G>());   // one arrival per epilogue warp
        }
        // the query operand: one TMA (bf16), or one arrival per epilogue warp (E4M3)
        mbar_init(qfull, kE4M3 ? 4 * idx_epi_sets<G>() : 1);
        fence_mbar_init();
    }
    // page j of this CTA (j < 4*kTPC) is page (4*kTPC*x + j)*Z of the request
    const int Z = page_step > 1 ? page_step : 1;
    int pg = -1;   // warp 0: page id of this CTA's page `lane`
    if (warp == 0) {
        const int col = (blockIdx.x * kTPC * 4 + lane) * Z;
        if (!persist && a.range != 2 && slot_ok && lane < kTPC * 4 && col < a.bt_stride)
            pg = __ldg(a.block_table + (size_t)slot * a.bt_stride + col);
        if (lane == 0) {
            tma_prefetch_desc(&kmap);
            if (!kE4M3) tma_prefetch_desc(&qmap);
        }
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols<N>());
        tmem_relinquish();
    }
    for (int i = threadIdx.x; i < G * HI; i += idx_threads<G>()) {
        const int r = r0 + i / HI;
        hw[i] = r < a.B ? __ldg(a.head_w + (size_t)r * HI + i % HI) : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // the next kernel may start only once this CTA holds its TMEM: a later
    // kernel's CTA allocating first and then waiting on this grid could
    // otherwise keep this CTA from ever getting its columns
    pdl_trigger();
    pdl_wait();
    CSLA_TL_WAITED();


    // ---- entries of each row scored here; the CTA streams the tiles of the longest.
    // range 0: [0, visible); 1: [0, len0/m) (entries complete before an append
    // that may still be running); 2: [len0/m, visible) (the ones it added).
    if (threadIdx.x < G) {
        const int r = r0 + threadIdx.x;
        int nv = -1, lo = 0;
        if (r < a.B) {
            const int sr = __ldg(a.slots + r);
            if (!slot_ok || sr != slot) {
                if (blockIdx.x == 0) set_dev_err(CSLA_DEVERR_INDEX);
            } else {
                const int L = a.range == 1 ? a.len0[r] : row_visible_len(a.len, a.q_len, slot, r);
                if (L < 0 || L > a.max_len) {
                    if (blockIdx.x == 0) set_dev_err(CSLA_DEVERR_LEN);
                } else {
                    nv = L / a.m;
                    if (a.range == 2) {
                        lo = a.len0[r] / a.m;
                        if (lo >= nv) nv = -1;
                    }
                    if (row_flag && row_flag[r] == 0) nv = -1;
                }
            }
        }
        row_nv[threadIdx.x] = nv;
        row_lo[threadIdx.x] = lo;
        row_t0[threadIdx.x] = key_score((cand_t0 && r < a.B) ? cand_t0[r] : 0u);
        if (threadIdx.x == 0) s_t0 = a.range == 2 ? lo / kTileE : 0;
    }
    __syncthreads();
    // persist: CTA x walks tiles [x*run, (x+1)*run) of the request
    const int run = persist ? (a.tiles_per_req + persist - 1) / persist : kTPC;
    const int t_begin = persist ? blockIdx.x * run : blockIdx.x * kTPC + s_t0;
    int nv_max = 0;
#pragma unroll
    for (int g = 0; g < G; ++g) nv_max = max(nv_max, row_nv[g]);
    const int pages_row = (nv_max + kPageE - 1) / kPageE;
    // tiles with an entry to score: of 4 consecutive pages, or (sample) of 4 pages Z apart
    const int n_tiles = min(run, ((pages_row + Z - 1) / Z + 3) / 4 - t_begin);
    if (a.range == 2 && warp == 0) {
        const int col = (t_begin * kTileE + lane * kPageE) / kPageE;
        if (slot_ok && lane < kTPC * 4 && col < a.bt_stride)
            pg = __ldg(a.block_table + (size_t)slot * a.bt_stride + col);
    }
    if (!persist && warp == 0 && lane < kTPC * 4) {
        const int e0 = ((t_begin * 4 + lane) * Z) * kPageE;
        if (e0 < nv_max && (pg < 0 || pg >= a.n_pages)) {
            set_dev_err(CSLA_DEVERR_PAGE);
            pg = -1;
        }
        pages[lane] = e0 < nv_max ? pg : -1;
    }
    __syncthreads();   // the epilogue warps read pages[] too (entries of a bad page stay unscored)
    // Page id of page p (< 4) of this CTA's tile t, -1 when it holds no
    // entry to score or lies outside the pool: from pages[] for the kTPC
    // tiles of a CTA, read from the block table per tile when a CTA walks a
    // longer run (persist: Z = 1).
    auto page_id = [&](int t, int p, bool report) -> int {
        if (!persist) return pages[t * 4 + p];
        const int e0 = (t_begin + t) * kTileE + p * kPageE;
        if (e0 >= nv_max) return -1;
        const int col = e0 / kPageE;
        const int q = col < a.bt_stride ? __ldg(a.block_table + (size_t)slot * a.bt_stride + col) : -1;
        if (q < 0 || q >= a.n_pages) {
            if (report) set_dev_err(CSLA_DEVERR_PAGE);
            return -1;
        }
        return q;
    };

    if (n_tiles <= 0) {
        // nothing to score: fall through to the teardown
    } else if (warp == 0) {
        if (lane == 0) {
            if (!kE4M3) {
                mbar_arrive_expect_tx(qfull, (uint32_t)S::kQBytes);
#pragma unroll
                for (int h = 0; h < DI / 64; ++h) tma_load_2d(qbuf + h * N * 128, &qmap, h * 64, r0 * NQ, qfull);
            }
            int n = 0;
            for (int t = 0; t < n_tiles; ++t, ++n) {
                const int s = n % kStages;
                if (n >= kStages && !mbar_wait(empty + s, ((n / kStages) - 1) & 1, &abort_flag)) break;
                uint8_t *kb = base + s * S::kKeyBytes;
                int tp[4], np = 0;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    tp[p] = page_id(t, p, true);
                    np += tp[p] >= 0;
                }
                mbar_arrive_expect_tx(full + s, (uint32_t)(np * kPageE * DI * S::kElt));
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int pg = tp[p];
                    if (pg < 0) continue;
                    if constexpr (kE4M3) {
                        // one 128-byte box per entry row (the whole E4M3 key)
                        tma_load_2d(kb + p * (kPageE * 128), &kmap, 0, pg * kPageE, full + s);
                    } else {
#pragma unroll
                        for (int h = 0; h < DI / 64; ++h)
                            tma_load_2d(kb + h * (kTileE * 128) + p * (kPageE * 128), &kmap, h * 64, pg * kPageE,
                                        full + s);
                    }
                }
            }
            // every issued copy must land before the CTA may exit
            for (int i = (n > kStages ? n - kStages : 0); i < n; ++i)
                mbar_wait(full + (i % kStages), (i / kStages) & 1, nullptr);
            mbar_wait(qfull, 0, nullptr);
            CSLA_TL_MARK_ANY(4);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = kE4M3 ? idesc_e4m3(128, N) : idesc_bf16(128, N, false, false);
            int n = 0;
            if (mbar_wait(qfull, 0, &abort_flag)) {
                const uint32_t qb = smem_u32(qbuf);
                for (int t = 0; t < n_tiles; ++t, ++n) {
                    const int s = n % kStages;
                    const int acc = n & 1;
                    if (!mbar_wait(full + s, (n / kStages) & 1, &abort_flag)) break;
                    if (t == 0) CSLA_TL_MARK_ANY(0);
                    if (t == kTPC - 1) CSLA_TL_MARK_ANY(1);
                    if (n >= 2 && !mbar_wait(tempty + acc, ((n / 2) - 1) & 1, &abort_flag)) break;
                    tc_fence_after();
                    const uint32_t kb = smem_u32(base + s * S::kKeyBytes);
                    if constexpr (kE4M3) {
                        // K = 32 codes (32 bytes) per instruction
#pragma unroll
                        for (int k = 0; k < DI / 32; ++k)
                            umma_kind_f8f6f4(tmem + acc * N, sdesc(kb + k * 32, 16, 1024), sdesc(qb + k * 32, 16, 1024),
                                             idesc, k > 0 ? 1u : 0u);
                    } else {
#pragma unroll
                        for (int k = 0; k < DI / 16; ++k) {
                            const uint32_t half = k / 4, ko = (k % 4) * 32;
                            const uint64_t ad = sdesc(kb + half * (kTileE * 128) + ko, 16, 1024);
                            const uint64_t bd = sdesc(qb + half * (N * 128) + ko, 16, 1024);
                            umma_kind_f16(tmem + acc * N, ad, bd, idesc, k > 0 ? 1u : 0u);
                        }
                    }
                    umma_commit(empty + s);
                    umma_commit(tfull + acc);
                }
            }
            if (n > 0) mbar_wait(tfull + ((n - 1) & 1), ((n - 1) / 2) & 1, nullptr);
        }
    } else {
        // TMEM lanes 32*(warp%4).. are this warp's key rows; set `es` takes
        // the group's rows es, es + sets, ...
        constexpr int kSets = idx_epi_sets<G>();
        const int lane_base = 32 * (warp & 3);
        const int es = (warp - 2) / 4;
        const int row = lane_base + lane;
        if constexpr (kE4M3) {
            // the E4M3 query operand: (query row g, head j) per warp task,
            // from the projection's three bf16 terms (their fp32 sum is q)
            for (int task = warp - 2; task < G * HI; task += 4 * kSets) {
                const int g = task / HI, j = task % HI, r = r0 + g;
                float q[4] = {0.f, 0.f, 0.f, 0.f};
                if (r < a.B) {
                    const uint16_t *qw = a.q_ws + (size_t)r * a.NQ * DI + 4 * lane;
                    const uint2 h = *reinterpret_cast<const uint2 *>(qw + (size_t)j * DI);
                    const uint2 m = *reinterpret_cast<const uint2 *>(qw + (size_t)(HI + j) * DI);
                    const uint2 l = *reinterpret_cast<const uint2 *>(qw + (size_t)(2 * HI + j) * DI);
                    const uint32_t hv[4] = {h.x & 0xFFFFu, h.x >> 16, h.y & 0xFFFFu, h.y >> 16};
                    const uint32_t mv[4] = {m.x & 0xFFFFu, m.x >> 16, m.y & 0xFFFFu, m.y >> 16};
                    const uint32_t lv[4] = {l.x & 0xFFFFu, l.x >> 16, l.y & 0xFFFFu, l.y >> 16};
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        q[i] = __fadd_rn(__fadd_rn(bf16_bits_to_f32(hv[i]), bf16_bits_to_f32(mv[i])),
                                         bf16_bits_to_f32(lv[i]));
                }
                split_q_e4m3(q, qbuf, g * NQ + j, HI, sig + g * NQ + j);
            }
            fence_proxy_async_smem();
            mbar_arrive_warp(qfull);
            // the term scales are read by every epilogue warp
            asm volatile("bar.sync 1, %0;" ::"r"(128 * kSets) : "memory");
        }
        // Candidate output, into the row's sub-list of this warp's entries
        // ((entry/32) % 4 = warp % 4).  When a set scores one of several
        // rows (kStaged),
        // the warp gathers its candidates in shared memory (ballot order)
        // and moves them out once more than 32 are staged, and after its
        // last tile: one counter update per ~32 candidates.  Otherwise each
        // (row, tile) takes its places from one counter update.
        constexpr bool kStaged = kSel && kSets >= G && G > 1;
        uint2 *stage = stage_all + (warp - 2) * kStageCands;
        int staged = 0;
        int stage_row = 0;
        auto stage_out = [&]() {
            if (staged > 0) {
                int at = 0;
                if (lane == 0) at = atomicAdd(a.cand_cnt + stage_row, staged);
                at = __shfl_sync(0xffffffffu, at, 0);
                __syncwarp();
                for (int i = lane; i < staged; i += 32)
                    if (at + i < a.cand_cap) a.cand[(size_t)stage_row * a.cand_cap + at + i] = stage[i];
                __syncwarp();
                staged = 0;
            }
        };
        Pending pend;
        auto flush = [&]() {
            if (pend.mq) {
                const int at = __shfl_sync(0xffffffffu, pend.at, 0) + __popc(pend.mq & ((1u << lane) - 1u));
                if (pend.q && at < a.cand_cap)
                    a.cand[(size_t)pend.row * a.cand_cap + at] = make_uint2(pend.key, (uint32_t)pend.e);
                pend.mq = 0u;
            }
        };
        for (int t = 0, n = 0; t < n_tiles; ++t, ++n) {
            const int acc = n & 1;
            float ksc = 0.f;   // E4M3: this row's entry scale, loaded before the accumulator wait
            const int pgr = page_id(t, row / kPageE, false);
            if constexpr (kE4M3) {
                if (pgr >= 0) ksc = __ldg(a.kscale + (size_t)pgr * kPageE + row % kPageE);
            }
            if (!warp_all(mbar_wait(tfull + acc, (n / 2) & 1, &abort_flag))) break;
            tc_fence_after();
            const int tile_e0 = (t_begin + t) * 4 * Z * kPageE;          // the tile's first entry
            const int e = (((t_begin + t) * 4 + row / kPageE) * Z) * kPageE + row % kPageE;
            const int col_out = (t_begin + t) * kTileE + row;            // its score column (e unless sampling)
            int last = -1;   // this set's last row with entries in the tile (warp-uniform)
            for (int g = es; g < G; g += kSets)
                if (row_nv[g] > tile_e0) last = g;
            if (last < 0) {
                tc_fence_before();
                mbar_arrive_warp(tempty + acc);
            }
#pragma unroll 1
            for (int g = es; g <= last; g += kSets) {
                const int nv = row_nv[g];
                if (nv <= tile_e0) continue;   // the whole tile is past this row (warp-uniform)
                uint32_t r[NQ];
                const uint32_t ta = tmem + ((uint32_t)lane_base << 16) + acc * N + g * NQ;
                if constexpr (NQ == 16) {
                    tmem_ld32x16(ta, r);
                } else if constexpr (NQ == 32) {
                    tmem_ld32x32(ta, r);
                } else if constexpr (NQ == 64) {
                    uint32_t (&r0_)[32] = *reinterpret_cast<uint32_t (*)[32]>(r);
                    uint32_t (&r1_)[32] = *reinterpret_cast<uint32_t (*)[32]>(r + 32);
                    tmem_ld32x32(ta, r0_);
                    tmem_ld32x32(ta + 32, r1_);
                } else {
                    static_assert(NQ == 48, "query operand rows");
                    uint32_t (&r0_)[32] = *reinterpret_cast<uint32_t (*)[32]>(r);
                    uint32_t (&r1_)[16] = *reinterpret_cast<uint32_t (*)[16]>(r + 32);
                    tmem_ld32x32(ta, r0_);
                    tmem_ld32x16(ta + 32, r1_);
                }
                tmem_wait_ld();
                if (g == last) {
                    // every column this set reads is in registers: the MMA may reuse the accumulator
                    tc_fence_before();
                    mbar_arrive_warp(tempty + acc);
                }
                // entries of a page outside the pool were not loaded: leave them unscored
                const bool valid = e < nv && e >= row_lo[g] && pgr >= 0;
                float sc = 0.f;
                if (valid) {
                    if constexpr (kE4M3) {
                        // head j: sum_t sig_t * acc_t (terms in order), then
                        // the entry's power-of-two key scale (ReLU commutes with it)
                        const float *sg = sig + g * NQ;
#pragma unroll
                        for (int j = 0; j < HI; ++j) {
                            float dot = __fmul_rn(sg[j], __uint_as_float(r[j]));
#pragma unroll
                            for (int tt = 1; tt < 4; ++tt)
                                dot = __fmaf_rn(sg[tt * HI + j], __uint_as_float(r[tt * HI + j]), dot);
                            sc = __fmaf_rn(hw[g * HI + j], fmaxf(dot, 0.f), sc);
                        }
                        sc = __fmul_rn(sc, ksc);
                    } else {
#pragma unroll
                        for (int j = 0; j < HI; ++j) {
                            const float dot = __fadd_rn(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(r[HI + j])),
                                                        __uint_as_float(r[2 * HI + j]));
                            sc = __fmaf_rn(hw[g * HI + j], fmaxf(dot, 0.f), sc);
                        }
                    }
                }
                if (cand_t0) {
                    // the entries at or above the row's threshold (warp-uniform
                    // mask; the float order is the key order, -0 == +0)
                    const bool q = valid && sc >= row_t0[g];
                    const unsigned mq = __ballot_sync(0xffffffffu, q);
                    if constexpr (kStaged) {
                        if (mq) {
                            stage_row = (r0 + g) * kCandSub + (warp & 3);   // the set's one row
                            if (q) stage[staged + __popc(mq & ((1u << lane) - 1u))] = make_uint2(score_key(sc), (uint32_t)e);
                            staged += __popc(mq);
                            if (staged > kStageCands - 32) stage_out();
                        }
                    } else {
                        pend.mq = mq;
                        pend.q = q;
                        pend.key = score_key(sc);
                        pend.e = e;
                        pend.row = (r0 + g) * kCandSub + (warp & 3);
                        if (mq && lane == 0) pend.at = atomicAdd(a.cand_cnt + pend.row, __popc(mq));
                        flush();
                    }
                } else if (valid) {
                    a.scores[(size_t)(r0 + g) * a.scores_stride + col_out] = sc;
                }
            }
            if (threadIdx.x == 64 && t == 0) CSLA_TL_MARK_ANY(2);
            if (threadIdx.x == 64 && t == kTPC - 1) CSLA_TL_MARK_ANY(3);
        }
        if constexpr (kStaged) stage_out();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols<N>());
    }
}


template <int DI, int NQ, int HI, int G, bool kE4M3, bool kSel>
cudaError_t launch_indexer_t(const IndexerArgs &a, const CUtensorMap &kmap, const CUtensorMap &qmap,
                             cudaStream_t stream) {
    using S = IdxSmem<DI, NQ, G, kE4M3>;
    static_assert(S::kBytes <= 232448, "shared memory budget");
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(indexer_kernel<DI, NQ, HI, G, kE4M3, kSel>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    // tiles a row group walks: all of the request's, or (sample) tiles of 4
    // pages page_step apart; persist: `persist` CTAs per row group
    const int Z = kSel && a.page_step > 1 ? a.page_step : 1;
    const int persist = (kSel || G > 1) ? a.persist : 0;   // as the kernel reads it
    const int groups = persist ? persist : (((a.tiles_per_req * 4 + Z - 1) / Z + 3) / 4 + kTPC - 1) / kTPC;
    return launch_pdl(indexer_kernel<DI, NQ, HI, G, kE4M3, kSel>, dim3(groups, (a.B + G - 1) / G),
                      dim3(idx_threads<G>()), S::kBytes, stream, a, kmap, qmap);
}

template <int DI, int NQ, int HI, bool kE4M3>
cudaError_t launch_indexer_g(const IndexerArgs &a, const CUtensorMap &kmap, const CUtensorMap &qmap,
                             cudaStream_t stream) {
    // the plain scoring kernels carry none of the streaming-selection code
    const bool sel = a.page_step > 1 || a.cand_t0 != nullptr || a.row_flag != nullptr;
    constexpr int GR = indexer_rows_per_cta(NQ);
    if (a.rows_per_cta == 1)
        return sel ? launch_indexer_t<DI, NQ, HI, 1, kE4M3, true>(a, kmap, qmap, stream)
                   : launch_indexer_t<DI, NQ, HI, 1, kE4M3, false>(a, kmap, qmap, stream);
    if (a.rows_per_cta == GR)
        return sel ? launch_indexer_t<DI, NQ, HI, GR, kE4M3, true>(a, kmap, qmap, stream)
                   : launch_indexer_t<DI, NQ, HI, GR, kE4M3, false>(a, kmap, qmap, stream);
    return cudaErrorInvalidValue;
}

// NQ: rows of the bf16 query operand; E4M3 keys (dI = 128 only) score
// against four E4M3 terms per head instead.
template <int DI, int NQ, int HI>
cudaError_t launch_indexer_k(const IndexerArgs &a, const CUtensorMap &kmap, const CUtensorMap &qmap,
                             cudaStream_t stream) {
    if (a.key_fmt == CSLA_KEY_E4M3) {
        if constexpr (DI == 128) return launch_indexer_g<DI, nq_e4m3<HI>(), HI, true>(a, kmap, qmap, stream);
        return cudaErrorInvalidValue;
    }
    return launch_indexer_g<DI, NQ, HI, false>(a, kmap, qmap, stream);
}

// len0[b] = len[slots[b]], read after the grid wait (0 for a bad slot).
__global__ void __launch_bounds__(256) len_snapshot_kernel(const int32_t *slots, const int32_t *len, int B,
                                                           int n_slots, int32_t *len0) {
    pdl_trigger();
    pdl_wait();
    const int b = blockIdx.x * 256 + threadIdx.x;
    if (b >= B) return;
    const int slot = slots[b];
    len0[b] = (slot >= 0 && slot < n_slots) ? len[slot] : 0;
}

// ---- index-query projection on the tensor cores (bf16 cq and W_iq)
//
// q_I = cq . W_iq^T as a tcgen05 GEMM: a CTA owns 128 query rows x 64
// output features; warp 0 streams 64-column (128-byte) slabs of both
// operands by TMA into a 4-stage ring (128-byte swizzle, K-major), warp 1
// issues one M=128 N=64 K=16 bf16 MMA per 32 bytes of a slab into a 64-column
// fp32 TMEM accumulator, warps 2-5 read it back (one row per thread) and
// store each value as its three bf16 terms (hi, mid, lo: their fp32 sum is
// the value) in the workspace.  Every output is one accumulation over the
// slabs in order: the same arithmetic whatever the batch.  Slabs past dc
// and rows past B read as zeros (TMA fill).  The loads and products come
// before the grid-dependency wait (cq and W_iq are inputs of the call);
// the stores follow it.
constexpr int kGemmBM = 128, kGemmStages = 4, kGemmThreads = 192;
constexpr int kGemmABytes = kGemmBM * 128;
template <int BN>
constexpr int gemm_smem() { return 1024 + kGemmStages * (kGemmABytes + BN * 128) + 256; }

// BN: output features per CTA (iq_gemm_bn).  An output's value does not
// depend on it, nor on the output's tile or lane: each is its own dot
// product over the K slabs, in order.
template <int BN>
__global__ void __launch_bounds__(kGemmThreads) iq_gemm_kernel(IndexerArgs a, const __grid_constant__ CUtensorMap cqmap,
                                                                const __grid_constant__ CUtensorMap wmap) {
    CSLA_TL_SCOPE(kTlIqProject);
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t *As = base;
    uint8_t *Bs = base + kGemmStages * kGemmABytes;
    uint64_t *full = reinterpret_cast<uint64_t *>(Bs + kGemmStages * (BN * 128));
    uint64_t *empty = full + kGemmStages, *done = empty + kGemmStages;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(done + 1);
    __shared__ volatile int abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int m0 = blockIdx.x * kGemmBM, n0 = blockIdx.y * BN;
    const int nk = (a.dc + 63) / 64;
    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kGemmStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        mbar_init(done, 1);
        fence_mbar_init();
        tma_prefetch_desc(&cqmap);
        tma_prefetch_desc(&wmap);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, 64);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    pdl_trigger();   // after the TMEM allocation (see indexer_kernel)

    if (warp == 0) {
        if (lane == 0) {
            int k = 0;
            for (; k < nk; ++k) {
                const int s = k % kGemmStages;
                if (k >= kGemmStages && !mbar_wait(empty + s, ((k / kGemmStages) - 1) & 1, &abort_flag)) break;
                mbar_arrive_expect_tx(full + s, (uint32_t)(kGemmABytes + (BN * 128)));
                tma_load_2d(As + s * kGemmABytes, &cqmap, k * 64, m0, full + s);
                tma_load_2d(Bs + s * (BN * 128), &wmap, k * 64, n0, full + s);
            }
            // every issued copy must land before the CTA may exit
            for (int i = (k > kGemmStages ? k - kGemmStages : 0); i < k; ++i)
                mbar_wait(full + (i % kGemmStages), (i / kGemmStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(kGemmBM, BN, false, false);
            int k = 0;
            for (; k < nk; ++k) {
                const int s = k % kGemmStages;
                if (!mbar_wait(full + s, (k / kGemmStages) & 1, &abort_flag)) break;
                tc_fence_after();
                const uint32_t ab = smem_u32(As + s * kGemmABytes), bb = smem_u32(Bs + s * (BN * 128));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    umma_kind_f16(tmem, sdesc(ab + kk * 32, 16, 1024), sdesc(bb + kk * 32, 16, 1024), idesc,
                                  (k | kk) > 0 ? 1u : 0u);
                umma_commit(empty + s);
            }
            if (k == nk) umma_commit(done);
            else abort_flag = 1;
        }
    } else {
        const int lane_base = 32 * (warp & 3);
        const int row = m0 + lane_base + lane;
        const bool ok = warp_all(mbar_wait(done, 0, &abort_flag));
        pdl_wait();
        CSLA_TL_WAITED();
        if (ok) {
            tc_fence_after();
            const int j = n0 / a.dI, e0 = n0 % a.dI;
            uint16_t *dst = a.q_ws + (size_t)(row < a.B ? row : 0) * a.NQ * a.dI + (size_t)j * a.dI + e0;
            const size_t tstride = (size_t)a.HI * a.dI;   // hi, mid, lo term rows are HI rows apart
#pragma unroll 1
            for (int c16 = 0; c16 < BN / 16; ++c16) {
                uint32_t r[16];
                tmem_ld32x16(tmem + ((uint32_t)lane_base << 16) + 16 * c16, r);
                tmem_wait_ld();
                if (row < a.B) {
#pragma unroll
                    for (int c8 = 0; c8 < 2; ++c8) {
                        uint32_t h[4], md[4], lo[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t hh[2], mm[2], ll[2];
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                const float v = __uint_as_float(r[c8 * 8 + 2 * i + u]);
                                const uint16_t vh = f32_to_bf16_bits(v);
                                const float rem = __fsub_rn(v, bf16_bits_to_f32(vh));
                                const uint16_t vm = f32_to_bf16_bits(rem);
                                hh[u] = vh;
                                mm[u] = vm;
                                ll[u] = f32_to_bf16_bits(__fsub_rn(rem, bf16_bits_to_f32(vm)));
                            }
                            h[i] = hh[0] | (hh[1] << 16);
                            md[i] = mm[0] | (mm[1] << 16);
                            lo[i] = ll[0] | (ll[1] << 16);
                        }
                        uint16_t *o = dst + 16 * c16 + c8 * 8;
                        *reinterpret_cast<uint4 *>(o) = make_uint4(h[0], h[1], h[2], h[3]);
                        *reinterpret_cast<uint4 *>(o + tstride) = make_uint4(md[0], md[1], md[2], md[3]);
                        *reinterpret_cast<uint4 *>(o + 2 * tstride) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 64);
    }
}

cudaError_t launch_iq_gemm(const IndexerArgs &a, const ProjMaps &pm, cudaStream_t stream) {
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(iq_gemm_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             gemm_smem<64>());
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    if (iq_gemm_bn(a.B) != 64) return cudaErrorInvalidValue;
    const dim3 grid((a.B + kGemmBM - 1) / kGemmBM, (a.HI * a.dI) / 64);
    return launch_pdl(iq_gemm_kernel<64>, grid, dim3(kGemmThreads), (size_t)gemm_smem<64>(), stream, a, pm.cq, pm.w);
}

// Rows of one request (G > 1, all entries): instead of one CTA per 8
// tiles, S CTAs per row group each walk a run of ceil(tiles/S) tiles (page
// ids read per tile), which saves most CTA set-ups and pipeline drains
// (prefill, 4096 rows at 65536 entries: 3.69 against 4.03 ms).  S minimises
// waves x run length, the waves counted as whole multiples of the SMs.
int persist_slices(int groups, int tiles, int num_sms) {
    int best = 1;
    long long best_cost = -1;
    for (int S = 1; S <= 16; ++S) {
        const long long waves = ((long long)groups * S + num_sms - 1) / num_sms;
        const long long cost = waves * ((tiles + S - 1) / S + 1);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = S;
        }
    }
    return best;
}

cudaError_t launch_scoring(const IndexerArgs &a0, const CUtensorMap &kmap, const CUtensorMap &qmap, int num_sms,
                           cudaStream_t stream) {
    IndexerArgs a = a0;
    if (a.rows_per_cta > 1 && a.range == 0 && a.page_step <= 1 && a.persist == 0)
        a.persist = persist_slices((a.B + a.rows_per_cta - 1) / a.rows_per_cta, a.tiles_per_req,
                                   num_sms > 0 ? num_sms : 148);
    // HI is a template parameter so the epilogue's head loop is unrolled.
    if (a.dI == 128) {
        switch (a.HI) {
            case 16: return launch_indexer_k<128, 48, 16>(a, kmap, qmap, stream);
            case 8: return launch_indexer_k<128, 32, 8>(a, kmap, qmap, stream);
            case 4: return launch_indexer_k<128, 16, 4>(a, kmap, qmap, stream);
            default: break;
        }
    } else if (a.dI == 64) {
        switch (a.HI) {
            case 16: return launch_indexer_k<64, 48, 16>(a, kmap, qmap, stream);
            case 8: return launch_indexer_k<64, 32, 8>(a, kmap, qmap, stream);
            case 4: return launch_indexer_k<64, 16, 4>(a, kmap, qmap, stream);
            default: break;
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_indexer(const IndexerArgs &a, bool cq_bf16, bool w_bf16, const CUtensorMap &kmap,
                           const CUtensorMap &qmap, int num_sms, cudaStream_t stream, bool project,
                           const ProjMaps *pm) {
    if (project) {
        if (a.NQ > 3 * a.HI) {
            cudaError_t e = cudaMemsetAsync(a.q_ws, 0, (size_t)a.B * a.NQ * a.dI * 2, stream);
            if (e != cudaSuccess) return e;
        }
        if (pm != nullptr && cq_bf16 && w_bf16) {
            cudaError_t e = launch_iq_gemm(a, *pm, stream);
            if (e != cudaSuccess) return e;
            return launch_scoring(a, kmap, qmap, num_sms, stream);
        }
        const int pblocks = (a.HI * a.dI + kProjThreads / 32 - 1) / (kProjThreads / 32);
        const dim3 pg(pblocks, (a.B + kProjKeepB - 1) / kProjKeepB), pb(kProjThreads);
        cudaError_t e;
        if (a.dc <= 1024) {
            if (cq_bf16 && w_bf16) e = launch_pdl(iq_project_kernel<__nv_bfloat16, __nv_bfloat16>, pg, pb, 0, stream, a);
            else if (cq_bf16) e = launch_pdl(iq_project_kernel<__nv_bfloat16, float>, pg, pb, 0, stream, a);
            else if (w_bf16) e = launch_pdl(iq_project_kernel<float, __nv_bfloat16>, pg, pb, 0, stream, a);
            else e = launch_pdl(iq_project_kernel<float, float>, pg, pb, 0, stream, a);
        } else {
            if (cq_bf16 && w_bf16) e = launch_pdl(iq_project_wide_kernel<__nv_bfloat16, __nv_bfloat16>, pg, pb, 0, stream, a);
            else if (cq_bf16) e = launch_pdl(iq_project_wide_kernel<__nv_bfloat16, float>, pg, pb, 0, stream, a);
            else if (w_bf16) e = launch_pdl(iq_project_wide_kernel<float, __nv_bfloat16>, pg, pb, 0, stream, a);
            else e = launch_pdl(iq_project_wide_kernel<float, float>, pg, pb, 0, stream, a);
        }
        if (e != cudaSuccess) return e;
    }
    return launch_scoring(a, kmap, qmap, num_sms, stream);
}

cudaError_t launch_len_snapshot(const int32_t *slots, const int32_t *len, int B, int n_slots, int32_t *len0,
                                cudaStream_t stream) {
    return launch_pdl(len_snapshot_kernel, dim3((B + 255) / 256), dim3(256), 0, stream, slots, len, B, n_slots,
                      len0);
}

}  // namespace csla
