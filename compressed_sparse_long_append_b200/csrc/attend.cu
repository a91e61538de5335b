// attend.cu -- core MQA of CSA and HCA layers (csla_csa_attend, csla_hca_attend).
//
//   硅星人 "DeepSeek V4 ... 让token大降价" §两大压缩注意力: the selected
//   compressed entries (CSA: top-k; HCA: all) concatenated with the 128
//   window tokens feed a multi-query attention (one shared KV head); each
//   head has a learnable sink logit in the softmax denominator; RoPE on the
//   last 64 dims.  haiqwa "DeepSeek-V4" §RMSNorm归一化: RMSNorm on each query
//   head.  QbitAI article on batch invariance: a token's output must not
//   depend on the batch, and the saturated / starved kernels agree bit for bit.
//
// Canonical reduction.  A request's attention set (n rows: compressed
// entries, then window tokens, in that order) is cut into chunks of
// attend_chunk_rows(n) rows -- a function of n alone.  Each chunk yields a
// partial (running max m, sum l, unnormalised O); fold_weights()/fold_dim()
// combine them with the sink in chunk order.  The saturated kernel walks
// all chunks of a request in one CTA and folds at the end; the starved kernel
// gives every chunk its own CTA and a combine kernel folds.  Both run the
// same code on the same data, so their outputs are identical bit for bit,
// and nothing depends on which other requests share the launch.
//
// One CTA = three roles over a stream of 64-row tiles:
//   warps 4-7 (loader)  resolve the 64 row addresses of a tile (one thread
//                       per row) and fetch the raw cache rows with 1-D bulk
//                       copies into one of two staging buffers (tiles t+1 and
//                       t+2 are in flight while tile t is converted); widen
//                       fp8 codes to f16 (exact; the RoPE dims stay bf16)
//                       into the SW128 K-major X tile once the previous
//                       tile's PV product is done;
//   warp 8 (MMA)        S = Qhat . X^T   tcgen05 M=64 (heads) N=64 (rows),
//                                        nope and RoPE dims in separate TMEM
//                                        accumulators: s = scale*S_nope + S_rope
//                       O^T += X^T . P^T tcgen05 M=128 (dims) N=64 (heads);
//   warps 0-3 (softmax) build Qhat = RoPE(RMSNorm(q)*gamma_q, t) in smem
//                       (the norm before the grid-dependency wait, the
//                       rotation after it); per tile read S, P = 2^(s - m)
//                       (lanes 0-15 of each warp own one head),
//                       P_nope = f16(P*scale), P_rope = bf16(P); lazy
//                       rescale of O^T when a head's max grows by more than 8
//                       (log2 units); at chunk end read O^T out as the partial.
// mbarriers hand tiles between roles; every wait is bounded.
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kSoftWarps = 4, kLoadWarps = 4;
constexpr int kThreads = 32 * (kSoftWarps + kLoadWarps + 1);   // 288
constexpr int kLoadThreads = 32 * kLoadWarps;
constexpr int kMmaWarp = kSoftWarps + kLoadWarps;               // warp 8
constexpr int kHP = 64;          // heads padded to the UMMA M of the S product
constexpr int kTile = 64;        // rows per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;
constexpr int kBarLoad = 1;   // named barrier of the loader warps (0 = __syncthreads)
// K blocks widened per proxy fence: 1 measured fastest (2 and 8 were 1.4
// and 2.5 us slower per step: the S products then start later)
constexpr int kWidenGroup = 1;

template <int D>
struct Cfg {
    static constexpr int kRB = D + 64;                 // row bytes
    static constexpr int kCH = kRB / 16;               // 16-byte chunks per row
    static constexpr int kNopeCH = (D - 64) / 16;      // chunks holding fp8 codes
    static constexpr int kKB = D / 64;                 // 64-dim K blocks
    static constexpr int kKBN = (D - 64) / 64;         // nope K blocks
    static constexpr int kMB = D / 128;                // 128-dim O^T blocks
    static constexpr int kKBBytes = kTile * 128;       // one K block of X (64 rows x 128 B)
    static constexpr int kXBytes = kKB * kKBBytes;
    static constexpr int kQKB = kHP * 128;             // one K block of Qhat
    static constexpr int kQBytes = kKB * kQKB;
    static constexpr int kPBytes = kHP * kTile * 2;
    static constexpr int kTasks = kTile * kCH;         // 16-byte chunks per tile
    static_assert(kTasks % kLoadThreads == 0, "tile split");
    static constexpr int kRawBytes = kTile * kRB;      // one staged tile of raw rows
    // TMEM columns
    static constexpr int kColSN = 0, kColSR = 64, kColO = 128;
    static constexpr int kColOR = 128 + 64 * kMB;
    static constexpr int kTmemCols = (kColOR + 64) <= 256 ? 256 : 512;
    // smem offsets (from a 1024-aligned base)
    static constexpr int kOffQ = 0;
    static constexpr int kOffX = kOffQ + kQBytes;
    static constexpr int kOffRaw0 = kOffX + kXBytes;
    static constexpr int kOffRaw1 = kOffRaw0 + kRawBytes;
    static constexpr int kOffPn = kOffRaw1 + kRawBytes;
    static constexpr int kOffPr = kOffPn + kPBytes;
    static constexpr int kOffMisc = kOffPr + kPBytes;
};

struct Misc {
    float rawscale[2][kTile];          // loader-private, per staging buffer: fp8 scale of each row
    int rawvalid[2][kTile];
    float tscale[2][kTile];            // per tile parity: fp8 scale of each row (0 = masked)
    int tvalid[2][kTile];
    float fac[2][kHP];                 // per tile parity: O^T column factors (1 = none)
    uint64_t raw_full[2], x_full[2], x_empty[2], s_full, s_free, p_full, pv_done, o_free, q_ready, fac_ready;
    uint64_t kb_full[8];               // per K block of X: widened (one phase per tile)
    int go[2];                         // loader: keep fetching (per tile parity)
    uint32_t tmem;
    int abort;
};

template <int D>
constexpr int smem_bytes() {
    return Cfg<D>::kOffMisc + (int)sizeof(Misc) + 1024;
}

// Request-level facts both variants derive the same way.
struct Req {
    int slot, L, nv, n_cmp, win_len, n_rows, chunk, n_chunks, wbase;
    bool ok;
};
__device__ __forceinline__ Req request(const AttendArgs &a, int b) {
    Req r;
    r.slot = __ldg(a.slots + b);
    const bool slot_ok = r.slot >= 0 && r.slot < a.n_slots;
    r.L = slot_ok ? row_visible_len(a.len, a.q_len, r.slot, b) : 0;
    r.ok = slot_ok && r.L >= 1 && r.L <= a.max_len;
    if (!r.ok) r.L = 0;
    r.nv = r.L / a.m;
    r.n_cmp = a.idx ? a.k : r.nv;
    r.win_len = r.L < a.n_win ? r.L : a.n_win;
    r.wbase = 0;
    if (r.ok && a.src_rows) {
        r.wbase = a.win_base[b];
    } else if (r.ok && a.q_len && r.L - r.win_len < a.len[r.slot] - a.n_win) {
        // an earlier query's window rows have left the ring
        if (threadIdx.x == 0) set_dev_err(CSLA_DEVERR_INDEX);
        r.ok = false;
        r.L = r.nv = r.n_cmp = r.win_len = 0;
    }
    r.n_rows = r.ok ? r.n_cmp + r.win_len : 0;
    r.chunk = attend_chunk_rows(r.n_rows);
    r.n_chunks = r.ok ? attend_num_chunks(r.n_rows) : 0;
    return r;
}

__device__ __forceinline__ void named_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// Byte offset of 8-element group g (dims 8g..8g+7) of row r in a SW128
// K-major tile whose K blocks are `kb_bytes` apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int g, int kb_bytes) {
    return (uint32_t)((g >> 3) * kb_bytes + (r >> 3) * 1024 + (r & 7) * 128 + (((g & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// ---------------------------------------------------------------- query preparation
// Qhat = RoPE(RMSNorm(q_h) * gamma_q, t) for the 64 (padded) heads of the
// request, built in shared memory by the softmax warps in two steps.
// Before the grid-dependency wait (q and gamma_q are inputs of the call):
// warp w normalises heads 16w .. 16w+15, lane l owning dims l*D/32 ..; the
// non-RoPE dims go to the SW128 K-major Qhat image as f16, the RoPE dims
// stay fp32 in the P area (64 heads x 64 dims x 4 B, unused until the first
// tile's softmax).  After the wait, when the position t = len - 1 is known,
// lane i rotates pair i of its warp's 16 heads and writes them as bf16.
template <int D>
__device__ void build_q_normed(const AttendArgs &a, int b, uint8_t *smem, int q_bf16) {
    using C = Cfg<D>;
    constexpr int DPL = D / 32;              // dims per lane (16 or 4)
    constexpr int kBatch = 4;                // heads whose loads are in flight together
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float *ropef = reinterpret_cast<float *>(smem + C::kOffPn);   // [64 heads][64 dims]
    const int d0 = lane * DPL;
    float gam[DPL];
#pragma unroll
    for (int e = 0; e < DPL; ++e) gam[e] = __ldg(a.gamma_q + d0 + e);
    for (int h0 = 16 * warp; h0 < 16 * warp + 16; h0 += kBatch) {
        float x[kBatch][DPL];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            // padding heads (h >= H) load head H-1 (in bounds); their values are zeroed below
            const int h = min(h0 + u, a.H - 1);
            const size_t off = ((size_t)b * a.H + h) * D + d0;
#pragma unroll
            for (int e0 = 0; e0 < DPL; e0 += 8 > DPL ? DPL : 8) {
                if (q_bf16) {
                    if constexpr (DPL >= 8) {
                        const uint4 w4 = __ldg(reinterpret_cast<const uint4 *>(
                            reinterpret_cast<const __nv_bfloat16 *>(a.q) + off + e0));
                        const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            x[u][e0 + 2 * e] = bf16_bits_to_f32(w[e] & 0xFFFFu);
                            x[u][e0 + 2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
                        }
                    } else {
                        const uint2 w2 = __ldg(reinterpret_cast<const uint2 *>(
                            reinterpret_cast<const __nv_bfloat16 *>(a.q) + off + e0));
                        x[u][e0] = bf16_bits_to_f32(w2.x & 0xFFFFu);
                        x[u][e0 + 1] = bf16_bits_to_f32(w2.x >> 16);
                        x[u][e0 + 2] = bf16_bits_to_f32(w2.y & 0xFFFFu);
                        x[u][e0 + 3] = bf16_bits_to_f32(w2.y >> 16);
                    }
                } else {
                    const float4 *p4 = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.q) + off + e0);
#pragma unroll
                    for (int e = 0; e < (8 > DPL ? DPL : 8); e += 4) {
                        const float4 f4 = __ldg(p4 + e / 4);
                        x[u][e0 + e] = f4.x;
                        x[u][e0 + e + 1] = f4.y;
                        x[u][e0 + e + 2] = f4.z;
                        x[u][e0 + e + 3] = f4.w;
                    }
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int h = h0 + u;
            float ss = 0.f;
#pragma unroll
            for (int e = 0; e < DPL; ++e) ss = __fmaf_rn(x[u][e], x[u][e], ss);
            ss = warp_sum(ss);
            const float r = 1.0f / sqrtf(__fdiv_rn(ss, (float)D) + a.eps);
            float y[DPL];   // padding heads (h >= H) are zero
#pragma unroll
            for (int e = 0; e < DPL; ++e) y[e] = h < a.H ? __fmul_rn(__fmul_rn(x[u][e], r), gam[e]) : 0.f;
            if (d0 >= D - 64) {
#pragma unroll
                for (int e = 0; e < DPL; ++e) ropef[h * 64 + (d0 - (D - 64)) + e] = y[e];
            } else {
#pragma unroll
                for (int e0 = 0; e0 < DPL; e0 += 8 > DPL ? DPL : 8) {
                    const int d = d0 + e0;
                    if constexpr (DPL >= 8) {
                        uint4 o;
                        o.x = pack_f16x2(y[e0], y[e0 + 1]);
                        o.y = pack_f16x2(y[e0 + 2], y[e0 + 3]);
                        o.z = pack_f16x2(y[e0 + 4], y[e0 + 5]);
                        o.w = pack_f16x2(y[e0 + 6], y[e0 + 7]);
                        *reinterpret_cast<uint4 *>(smem + C::kOffQ + sw128_off(h, d >> 3, C::kQKB)) = o;
                    } else {
                        uint2 o;
                        o.x = pack_f16x2(y[e0], y[e0 + 1]);
                        o.y = pack_f16x2(y[e0 + 2], y[e0 + 3]);
                        *reinterpret_cast<uint2 *>(smem + C::kOffQ + sw128_off(h, d >> 3, C::kQKB) + (d & 7) * 2) = o;
                    }
                }
            }
        }
    }
}

// After the wait: rotate the RoPE dims by position t and publish Qhat.
template <int D>
__device__ void build_q_rope(const AttendArgs &a, long long t, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const float *ropef = reinterpret_cast<const float *>(smem + C::kOffPn);
    float c, sn;
    rope_cos_sin(t, a.freq.inv[lane], &c, &sn);
    const int dim = (D - 64) + 2 * lane;
    for (int h = 16 * warp; h < 16 * warp + 16; ++h) {
        const float y0 = ropef[h * 64 + 2 * lane], y1 = ropef[h * 64 + 2 * lane + 1];
        const float r0 = __fsub_rn(__fmul_rn(y0, c), __fmul_rn(y1, sn));
        const float r1 = __fadd_rn(__fmul_rn(y0, sn), __fmul_rn(y1, c));
        *reinterpret_cast<uint32_t *>(smem + C::kOffQ + sw128_off(h, dim >> 3, C::kQKB) + (dim & 7) * 2) =
            pack_bf16x2(r0, r1);
    }
    fence_proxy_async_smem();
    mbar_arrive(&ms->q_ready);
}

// ---------------------------------------------------------------- loader role helpers
// Source row (nullptr = masked) and fp8 scale of row r of the request's set.
__device__ __forceinline__ const uint8_t *row_source(const AttendArgs &a, int b, const Req &rq, int r, int rb,
                                                     float *scale) {
    *scale = 0.f;
    if (r < rq.n_cmp) {
        const int e = a.idx ? __ldg(a.idx + (size_t)b * a.k + r) : r;
        if (e < 0) return nullptr;
        if (e >= rq.nv) {
            set_dev_err(CSLA_DEVERR_INDEX);
            return nullptr;
        }
        const int epp = CSLA_PAGE_TOKENS / a.m;
        const int col = e / epp;
        const int pg = col < a.bt_stride ? __ldg(a.block_table + (size_t)rq.slot * a.bt_stride + col) : -1;
        if (pg < 0 || pg >= a.n_pages) {
            set_dev_err(CSLA_DEVERR_PAGE);
            return nullptr;
        }
        const size_t ent = (size_t)pg * epp + (size_t)(e % epp);
        *scale = __ldg(a.scales + ent);
        return a.rows + ent * rb;
    }
    if (r < rq.n_rows) {
        const int w = r - rq.n_cmp;
        const int pos = rq.L - rq.win_len + w;
        if (a.src_rows) {
            const long long i = (long long)rq.wbase + pos;
            if (i < 0 || i >= a.n_src) {
                set_dev_err(CSLA_DEVERR_INDEX);
                return nullptr;
            }
            *scale = __ldg(a.src_scales + i);
            return a.src_rows + (size_t)i * rb;
        }
        const size_t ring = (size_t)rq.slot * a.n_win + (size_t)(pos % a.n_win);
        *scale = __ldg(a.win_scales + ring);
        return a.win_rows + ring * rb;
    }
    return nullptr;
}

// Widen one 16-byte chunk of a cache row into the X tile: fp8 codes become
// f16 (exact), the RoPE dims stay bf16.
template <int D>
__device__ __forceinline__ void store_chunk(uint8_t *xs, int r, int c, const uint4 v) {
    using C = Cfg<D>;
    if (c < C::kNopeCH) {
        const int g0 = c * 2;   // 16 codes = two 8-dim groups
        uint4 lo, hi;
        lo.x = e4m3x2_to_f16x2(v.x & 0xFFFFu);
        lo.y = e4m3x2_to_f16x2(v.x >> 16);
        lo.z = e4m3x2_to_f16x2(v.y & 0xFFFFu);
        lo.w = e4m3x2_to_f16x2(v.y >> 16);
        hi.x = e4m3x2_to_f16x2(v.z & 0xFFFFu);
        hi.y = e4m3x2_to_f16x2(v.z >> 16);
        hi.z = e4m3x2_to_f16x2(v.w & 0xFFFFu);
        hi.w = e4m3x2_to_f16x2(v.w >> 16);
        *reinterpret_cast<uint4 *>(xs + sw128_off(r, g0, C::kKBBytes)) = lo;
        *reinterpret_cast<uint4 *>(xs + sw128_off(r, g0 + 1, C::kKBBytes)) = hi;
    } else {
        const int g = (D - 64) / 8 + (c - C::kNopeCH);
        *reinterpret_cast<uint4 *>(xs + sw128_off(r, g, C::kKBBytes)) = v;
    }
}

// The chunk range a CTA works on, and where chunk c's partial lives.
struct Span {
    int c0, c1;
};

// Chunk partial record: O[H][D], then m[H] and l[H], all f32.
__device__ __forceinline__ size_t partial_floats(int H, int D) { return (size_t)H * D + 2 * (size_t)H; }
__device__ __forceinline__ float *partial_ptr(const AttendArgs &a, int b, int c, int D) {
    return a.part + ((size_t)b * a.max_chunks + c) * partial_floats(a.H, D);
}

// ---------------------------------------------------------------- the three roles
template <int D>
__device__ void loader_role(const AttendArgs &a, int b, const Req &rq, Span sp, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    const int lt = threadIdx.x - 32 * kSoftWarps;
    // the span's rows, in 64-row tiles (chunk boundaries are tile boundaries)
    const int r_begin = sp.c0 * rq.chunk;
    const int r_end = min(rq.n_rows, sp.c1 * rq.chunk);
    const int n_tiles = (r_end - r_begin + kTile - 1) / kTile;
    // Bulk-copy tile t's rows into staging buffer t & 1.  Every thread that
    // issues a copy first adds its bytes to the buffer's transaction count;
    // one arrival after the loader barrier closes the phase's bookkeeping.
    // Called uniformly by all loader threads (each reaches the barrier).
    auto issue = [&](int t) {
        const int buf = t & 1;
        if (lt < kTile) {
            float sc;
            const int r = r_begin + t * kTile + lt;
            const uint8_t *p = r < r_end ? row_source(a, b, rq, r, C::kRB, &sc) : nullptr;
            if (p) {
                mbar_expect_tx(&ms->raw_full[buf], (uint32_t)C::kRB);
                bulk_load(smem + (buf ? C::kOffRaw1 : C::kOffRaw0) + lt * C::kRB, p, (uint32_t)C::kRB,
                          &ms->raw_full[buf]);
            }
            ms->rawscale[buf][lt] = p ? sc : 0.f;   // the scale load completes while the copy runs
            ms->rawvalid[buf][lt] = p ? 1 : 0;
        }
        named_sync(kBarLoad, kLoadThreads);
        if (lt == 0) mbar_arrive(&ms->raw_full[buf]);
    };
    int issued = 0, first_fail = n_tiles;
    if (n_tiles > 0) issue(issued++);
    if (n_tiles > 1) issue(issued++);
    CSLA_TL_MARK_ANY(6);
    for (int t = 0; t < n_tiles; ++t) {
        const int buf = t & 1;
        // the staged rows, and the X tile free again (PV of the previous tile done)
        bool ok = t < issued && mbar_wait(&ms->raw_full[buf], (t >> 1) & 1, &ms->abort);
        if (lt == 0 && t == 0) CSLA_TL_MARK_ANY(7);
        if (!ok && t < first_fail) first_fail = t;
        if (ok && t > 0) ok = mbar_wait(&ms->x_empty[(t - 1) & 1], ((t - 1) >> 1) & 1, &ms->abort);
        const uint8_t *raw = smem + (buf ? C::kOffRaw1 : C::kOffRaw0);
        uint8_t *xs = smem + C::kOffX;
        // widen kWidenGroup K blocks at a time (one proxy fence per group);
        // the MMA warp starts on a block as soon as every loader thread has
        // arrived on its barrier
#pragma unroll 1
        for (int kb0 = 0; kb0 < C::kKB; kb0 += kWidenGroup) {
            if (ok) {
#pragma unroll 1
                for (int kb = kb0; kb < kb0 + kWidenGroup && kb < C::kKB; ++kb) {
                    // source chunks of this block: 4 fp8 chunks per row (nope)
                    // or 8 bf16 chunks per row (RoPE block)
                    const int cpr = kb < C::kKBN ? 4 : 8;
                    const int ch0 = kb < C::kKBN ? 4 * kb : C::kNopeCH;
#pragma unroll 4
                    for (int id = lt; id < kTile * cpr; id += kLoadThreads) {
                        const int r = id / cpr, ch = ch0 + id % cpr;
                        const uint4 v = ms->rawvalid[buf][r]
                                            ? *reinterpret_cast<const uint4 *>(raw + r * C::kRB + ch * 16)
                                            : make_uint4(0u, 0u, 0u, 0u);
                        store_chunk<D>(xs, r, ch, v);
                    }
                }
                fence_proxy_async_smem();
            }
            for (int kb = kb0; kb < kb0 + kWidenGroup && kb < C::kKB; ++kb) mbar_arrive(&ms->kb_full[kb]);
        }
        if (ok) {
            if (lt < kTile) {
                ms->tscale[buf][lt] = ms->rawscale[buf][lt];
                ms->tvalid[buf][lt] = ms->rawvalid[buf][lt];
            }
            if (lt == 0 && t == 0) CSLA_TL_MARK_ANY(4);
        }
        mbar_arrive(&ms->x_full[buf]);
        // staging buffer `buf` is consumed: fetch tile t + 2 into it, unless
        // the CTA is aborting (one decision for all loader threads)
        if (lt == 0) ms->go[t & 1] = ms->abort ? 0 : 1;
        named_sync(kBarLoad, kLoadThreads);
        if (t + 2 < n_tiles && ms->go[t & 1]) issue(issued++);
    }
    // copies still in flight after an abort must land before the CTA exits
    for (int t = first_fail; t < issued; ++t) mbar_wait(&ms->raw_full[t & 1], (t >> 1) & 1, nullptr);
}

template <int D>
__device__ void mma_role(const Req &rq, Span sp, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    // f16 operands for the fp8-coded dims, bf16 for the RoPE dims.  The PV
    // blocks are 128 dims tall, so the last non-RoPE block also spans the
    // RoPE dims (and the RoPE block the last 64 non-RoPE dims) read as the
    // other type: those O^T rows are never read out.
    constexpr uint32_t kIdescSN = idesc_f16(64, 64, false, false);
    constexpr uint32_t kIdescSR = idesc_bf16(64, 64, false, false);
    constexpr uint32_t kIdescON = idesc_f16(128, 64, true, false);
    constexpr uint32_t kIdescOR = idesc_bf16(128, 64, true, false);
    const uint32_t tmem = ms->tmem;
    const uint32_t q0 = smem_u32(smem + C::kOffQ);
    const uint32_t p0n = smem_u32(smem + C::kOffPn), p0r = smem_u32(smem + C::kOffPr);
    if (!mbar_wait(&ms->q_ready, 0, &ms->abort)) return;
    CSLA_TL_MARK_ANY(5);
    int g = 0;
    for (int c = sp.c0; c < sp.c1; ++c) {
        const int lo = c * rq.chunk;
        const int hi = min(rq.n_rows, lo + rq.chunk);
        for (int r0 = lo, ti = 0; r0 < hi; r0 += kTile, ++ti, ++g) {
            const int buf = g & 1;
            if (g > 0 && !mbar_wait(&ms->s_free, (g - 1) & 1, &ms->abort)) return;
            const uint32_t x0 = smem_u32(smem + C::kOffX);
#pragma unroll 1
            for (int kb = 0; kb < C::kKBN; ++kb) {
                if (!mbar_wait(&ms->kb_full[kb], g & 1, &ms->abort)) return;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_kind_f16(tmem + C::kColSN, sdesc(q0 + kb * C::kQKB + ks * 32, 16, 1024),
                                  sdesc(x0 + kb * C::kKBBytes + ks * 32, 16, 1024), kIdescSN, (kb | ks) ? 1u : 0u);
            }
            if (!mbar_wait(&ms->kb_full[C::kKBN], g & 1, &ms->abort)) return;
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_kind_f16(tmem + C::kColSR, sdesc(q0 + C::kKBN * C::kQKB + ks * 32, 16, 1024),
                              sdesc(x0 + C::kKBN * C::kKBBytes + ks * 32, 16, 1024), kIdescSR, ks ? 1u : 0u);
            if (g == 0) CSLA_TL_MARK_ANY(0);
            umma_commit(&ms->s_full);
            if (!mbar_wait(&ms->p_full, g & 1, &ms->abort)) return;
            if (ti == 0 && c > sp.c0 && !mbar_wait(&ms->o_free, (c - sp.c0 - 1) & 1, &ms->abort)) return;
            tc_fence_after();
#pragma unroll
            for (int mb = 0; mb < C::kMB; ++mb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_kind_f16(tmem + C::kColO + 64 * mb,
                              sdesc(x0 + 2 * mb * C::kKBBytes + 2 * ks * 1024, C::kKBBytes, 1024),
                              sdesc(p0n + ks * 32, 16, 1024), kIdescON, (ti > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_kind_f16(tmem + C::kColOR,
                          sdesc(x0 + 2 * (C::kMB - 1) * C::kKBBytes + 2 * ks * 1024, C::kKBBytes, 1024),
                          sdesc(p0r + ks * 32, 16, 1024), kIdescOR, (ti > 0 || ks > 0) ? 1u : 0u);
            umma_commit(&ms->x_empty[buf]);
            umma_commit(&ms->pv_done);
        }
    }
}

template <int D>
__device__ void softmax_role(const AttendArgs &a, int b, const Req &rq, Span sp, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const int h = 16 * warp + lane;       // head owned by lanes 0..15 (M=64 TMEM layout)
    const bool head_thread = lane < 16;
    const float cscale = kLog2e / sqrtf((float)D);
    const uint32_t tmem = ms->tmem;
    uint8_t *pn = smem + C::kOffPn;
    uint8_t *pr = smem + C::kOffPr;

    build_q_rope<D>(a, (long long)rq.L - 1, smem, ms);

    int g = 0, nfac = 0;
    for (int c = sp.c0; c < sp.c1; ++c) {
        const int lo = c * rq.chunk;
        const int hi = min(rq.n_rows, lo + rq.chunk);
        float m_run = -INFINITY, l_run = 0.f;
        for (int r0 = lo, ti = 0; r0 < hi; r0 += kTile, ++ti, ++g) {
            const int buf = g & 1;
            if (!mbar_wait(&ms->x_full[buf], (g >> 1) & 1, &ms->abort)) return;
            if (!mbar_wait(&ms->s_full, g & 1, &ms->abort)) return;
            if (threadIdx.x == 0 && g == 0) CSLA_TL_MARK(1);
            tc_fence_after();
            float s[kTile];
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t rn[32], rr[32];
                tmem_ld32x32(tmem + lane_base + C::kColSN + 32 * half, rn);
                tmem_ld32x32(tmem + lane_base + C::kColSR + 32 * half, rr);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int jj = 32 * half + j;
                    const float v = __fmul_rn(
                        __fmaf_rn(ms->tscale[buf][jj], __uint_as_float(rn[j]), __uint_as_float(rr[j])), cscale);
                    s[jj] = ms->tvalid[buf][jj] ? v : -INFINITY;
                }
            }
            tc_fence_before();
            mbar_arrive(&ms->s_free);        // S may be overwritten by the next tile's MMA
            float mt = -INFINITY;
#pragma unroll
            for (int j = 0; j < kTile; ++j) mt = fmaxf(mt, s[j]);
            // PV of the previous tile must be done before P and O^T are touched.
            if (g > 0 && !mbar_wait(&ms->pv_done, (g - 1) & 1, &ms->abort)) return;
            tc_fence_after();
            float f = 1.f;
            if (head_thread) {
                float mnew = m_run;
                if (ti == 0) {
                    mnew = mt;
                } else if (mt > m_run + kRescaleThresh || (m_run == -INFINITY && mt > -INFINITY)) {
                    mnew = mt;
                    f = exp2f(__fsub_rn(m_run, mnew));
                }
                const float muse = mnew == -INFINITY ? 0.f : mnew;
                float lsum = 0.f;
#pragma unroll
                for (int c8 = 0; c8 < kTile / 8; ++c8) {
                    float p[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        p[e] = exp2f(__fsub_rn(s[c8 * 8 + e], muse));
                        lsum = __fadd_rn(lsum, p[e]);
                    }
                    const float *sc = &ms->tscale[buf][c8 * 8];
                    uint4 un, ur;
                    un.x = pack_f16x2(__fmul_rn(p[0], sc[0]), __fmul_rn(p[1], sc[1]));
                    un.y = pack_f16x2(__fmul_rn(p[2], sc[2]), __fmul_rn(p[3], sc[3]));
                    un.z = pack_f16x2(__fmul_rn(p[4], sc[4]), __fmul_rn(p[5], sc[5]));
                    un.w = pack_f16x2(__fmul_rn(p[6], sc[6]), __fmul_rn(p[7], sc[7]));
                    ur.x = pack_bf16x2(p[0], p[1]);
                    ur.y = pack_bf16x2(p[2], p[3]);
                    ur.z = pack_bf16x2(p[4], p[5]);
                    ur.w = pack_bf16x2(p[6], p[7]);
                    const uint32_t off = (uint32_t)((h >> 3) * 1024 + (h & 7) * 128 + ((c8 ^ (h & 7)) << 4));
                    *reinterpret_cast<uint4 *>(pn + off) = un;
                    *reinterpret_cast<uint4 *>(pr + off) = ur;
                }
                l_run = (ti == 0) ? lsum : __fadd_rn(__fmul_rn(l_run, f), lsum);
                m_run = mnew;
                ms->fac[g & 1][h] = f;
            }
            // every head's factor is needed by every thread (each owns one O^T
            // row); a chunk's first tile has none (every factor is 1)
            bool any_rescale = false;
            if (ti > 0) {
                mbar_arrive(&ms->fac_ready);
                if (!mbar_wait(&ms->fac_ready, nfac & 1, &ms->abort)) return;
                ++nfac;
#pragma unroll 8
                for (int j = 0; j < kHP; ++j) any_rescale |= ms->fac[g & 1][j] != 1.f;
            }
            if (any_rescale) {
                // O^T columns are heads: every thread scales its own dim lane.
#pragma unroll 1
                for (int blk = 0; blk <= C::kMB; ++blk) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        uint32_t v[32];
                        const uint32_t addr = tmem + lane_base + C::kColO + 64 * blk + 32 * half;
                        tmem_ld32x32(addr, v);
                        tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            v[j] = __float_as_uint(__fmul_rn(__uint_as_float(v[j]), ms->fac[g & 1][32 * half + j]));
                        tmem_st32x32(addr, v);
                    }
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&ms->p_full);
        }
        // chunk done: drain its last PV and read O^T out as the partial
        if (!mbar_wait(&ms->pv_done, (g - 1) & 1, &ms->abort)) return;
        if (threadIdx.x == 0) CSLA_TL_MARK(2);
        tc_fence_after();
        float *part = partial_ptr(a, b, c, D);
        float *ml = part + (size_t)a.H * D;
#pragma unroll 1
        for (int blk = 0; blk <= C::kMB; ++blk) {
            const bool rope_blk = blk == C::kMB;
            const int dim = (rope_blk ? (D - 128) : 128 * blk) + 32 * warp + lane;
            const bool write = rope_blk ? (dim >= D - 64) : (dim < D - 64);
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32x32(tmem + lane_base + C::kColO + 64 * blk + 32 * half, v);
                tmem_wait_ld();
                if (write) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) {
                        const int hh = 32 * half + j;
                        if (hh < a.H) part[(size_t)hh * D + dim] = __uint_as_float(v[j]);
                    }
                }
            }
        }
        if (head_thread && h < a.H) {
            ml[h] = m_run;
            ml[a.H + h] = l_run;
        }
        if (threadIdx.x == 0) CSLA_TL_MARK(3);
        tc_fence_before();
        mbar_arrive(&ms->o_free);
    }
}

// Fold of the chunk partials of request b, head h (sink first):
//   M = max(sink*log2e, m_0 .. m_{n-1})                (exact, order-free)
//   w_c = 2^(m_c - M);  l = 2^(sink*log2e - M) + sum_c l_c w_c;  o_d = sum_c O_c[d] w_c
// with both sums taken in chunk order; out = o / l.  The saturated and the
// starved kernels both use these functions.
// fold_weights is warp-collective (lane c loads chunk c, n_chunks <= 32);
// on return every lane holds w_c of its own chunk c in *w_lane and l in *l_out.
__device__ __forceinline__ void fold_weights(const AttendArgs &a, int b, int n_chunks, int h, int D, float *w_lane,
                                             float *l_out) {
    const size_t stride = partial_floats(a.H, D);
    const float *p = a.part + (size_t)b * a.max_chunks * stride + (size_t)a.H * D;
    const int lane = threadIdx.x & 31;
    const float z = __fmul_rn(__ldg(a.sink + h), kLog2e);
    const float mc = lane < n_chunks ? p[lane * stride + h] : -INFINITY;
    const float lc = lane < n_chunks ? p[lane * stride + a.H + h] : 0.f;
    const float M = fmaxf(z, warp_max(mc));
    const float wc = lane < n_chunks ? exp2f(__fsub_rn(mc, M)) : 0.f;
    float l = exp2f(__fsub_rn(z, M));
    for (int c = 0; c < n_chunks; ++c)
        l = __fmaf_rn(__shfl_sync(0xffffffffu, lc, c), __shfl_sync(0xffffffffu, wc, c), l);
    *w_lane = wc;
    *l_out = l;
}
// O_c[d] of head h, chunk c.
__device__ __forceinline__ float partial_o(const AttendArgs &a, int b, int c, int h, int d, int D) {
    return partial_ptr(a, b, c, D)[(size_t)h * D + d];
}
// o_d = sum_c O_c[d] w_c in chunk order, w[] the per-chunk weights.
__device__ __forceinline__ float fold_dim(const AttendArgs &a, int b, int n_chunks, int h, int d, int D,
                                          const float *w, float l) {
    float v[32];
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = partial_o(a, b, min(c, n_chunks - 1), h, d, D);
    float o = 0.f;
#pragma unroll
    for (int c = 0; c < 32; ++c)
        if (c < n_chunks) o = __fmaf_rn(v[c], w[c], o);
    return __fdiv_rn(o, l);
}

__device__ __forceinline__ void store_out(const AttendArgs &a, bool out_bf16, size_t i, float v) {
    if (out_bf16) reinterpret_cast<__nv_bfloat16 *>(a.out)[i] = __float2bfloat16_rn(v);
    else reinterpret_cast<float *>(a.out)[i] = v;
}

template <int D, bool kSaturated>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(AttendArgs a, int q_bf16, int out_bf16) {
    CSLA_TL_SCOPE(kTlAttend);
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Misc *ms = reinterpret_cast<Misc *>(smem + C::kOffMisc);
    const int b = kSaturated ? blockIdx.x : blockIdx.y;
    const int warp = threadIdx.x >> 5;

    // ---- before the wait: barriers and TMEM
    if (threadIdx.x == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ms->raw_full[i], 1);
            mbar_init(&ms->x_full[i], kLoadThreads);
            mbar_init(&ms->x_empty[i], 1);
        }
        for (int i = 0; i < C::kKB; ++i) mbar_init(&ms->kb_full[i], kLoadThreads);
        mbar_init(&ms->s_full, 1);
        mbar_init(&ms->s_free, 32 * kSoftWarps);
        mbar_init(&ms->p_full, 32 * kSoftWarps);
        mbar_init(&ms->pv_done, 1);
        mbar_init(&ms->o_free, 32 * kSoftWarps);
        mbar_init(&ms->q_ready, 32 * kSoftWarps);
        mbar_init(&ms->fac_ready, 32 * kSoftWarps);
        ms->abort = 0;
        fence_mbar_init();
    }
    if (warp == kMmaWarp) {
        tmem_alloc(&ms->tmem, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    pdl_trigger();   // after the TMEM allocation (see the indexer kernel)
    if (warp < kSoftWarps) build_q_normed<D>(a, b, smem, q_bf16);
    pdl_wait();
    CSLA_TL_WAITED();

    const Req rq = request(a, b);
    if (!rq.ok && threadIdx.x == 0 && (kSaturated || blockIdx.x == 0)) set_dev_err(CSLA_DEVERR_LEN);
    const bool run = rq.ok && (kSaturated || (int)blockIdx.x < rq.n_chunks);
    const Span sp = kSaturated ? Span{0, rq.n_chunks} : Span{(int)blockIdx.x, (int)blockIdx.x + 1};
    if (!run) {
        // nothing to do: fall through to the teardown
    } else if (warp < kSoftWarps) {
        softmax_role<D>(a, b, rq, sp, smem, ms);
    } else if (warp < kSoftWarps + kLoadWarps) {
        loader_role<D>(a, b, rq, sp, smem, ms);
    } else if ((threadIdx.x & 31) == 0) {
        mma_role<D>(rq, sp, smem, ms);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(ms->tmem, C::kTmemCols);
    }
    if (!run) return;
    if (kSaturated) {
        // partials written by this CTA are visible to it after the barrier
        // above.  Every head's chunk weights first (warp-collective per head),
        // into the staging area the loader no longer uses.
        float *wall = reinterpret_cast<float *>(smem + C::kOffRaw0);   // [H][33]: w_0..w_31, l
        const int lane = threadIdx.x & 31;
        const int n = rq.n_chunks;
        for (int hh = warp; hh < a.H; hh += kThreads / 32) {
            float wl, l;
            fold_weights(a, b, n, hh, D, &wl, &l);
            wall[hh * 33 + lane] = wl;
            if (lane == 0) wall[hh * 33 + 32] = l;
        }
        __syncthreads();
        if (partial_floats(a.H, D) % 4 == 0) {
            // (head, 128 dims) per warp, 4 consecutive dims per lane: 16-byte
            // partial loads, 8 chunks in flight; each dim folded in chunk
            // order exactly like fold_dim()
            constexpr int kQ = D / 128;
            for (int it = warp; it < a.H * kQ; it += kThreads / 32) {
                const int hh = it / kQ, d = (it % kQ) * 128 + 4 * lane;
                const float *w = wall + hh * 33;
                float o0 = 0.f, o1 = 0.f, o2 = 0.f, o3 = 0.f;
                for (int c0 = 0; c0 < n; c0 += 8) {
                    float4 v[8];
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        v[j] = *reinterpret_cast<const float4 *>(partial_ptr(a, b, min(c0 + j, n - 1), D) +
                                                                 (size_t)hh * D + d);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (c0 + j < n) {
                            const float wc = w[c0 + j];
                            o0 = __fmaf_rn(v[j].x, wc, o0);
                            o1 = __fmaf_rn(v[j].y, wc, o1);
                            o2 = __fmaf_rn(v[j].z, wc, o2);
                            o3 = __fmaf_rn(v[j].w, wc, o3);
                        }
                    }
                }
                const float l = w[32];
                const size_t base = ((size_t)b * a.H + hh) * D + d;
                store_out(a, out_bf16 != 0, base, __fdiv_rn(o0, l));
                store_out(a, out_bf16 != 0, base + 1, __fdiv_rn(o1, l));
                store_out(a, out_bf16 != 0, base + 2, __fdiv_rn(o2, l));
                store_out(a, out_bf16 != 0, base + 3, __fdiv_rn(o3, l));
            }
        } else {
            // odd head counts: partial records are not 16-byte multiples
            for (int hh = warp; hh < a.H; hh += kThreads / 32)
                for (int d = lane; d < D; d += 32)
                    store_out(a, out_bf16 != 0, ((size_t)b * a.H + hh) * D + d,
                              fold_dim(a, b, n, hh, d, D, wall + hh * 33, wall[hh * 33 + 32]));
        }
    }
}

// One CTA of 128 threads per (head, request); thread t folds dims t, t+128,
// ... (D/128 of them).  All of a thread's partial loads are issued before
// the chunk weights are known (warp 0 forms them meanwhile); each dim is
// then folded in chunk order exactly like fold_dim().  kMaxC bounds the
// chunk count (it sizes the register array).
template <int D, int kMaxC>
__global__ void __launch_bounds__(128) combine_kernel(AttendArgs a, int out_bf16) {
    CSLA_TL_SCOPE(kTlCombine);
    constexpr int kDPT = D / 128;   // dims per thread
    __shared__ float wts[33];
    pdl_trigger();
    const int h = blockIdx.x, b = blockIdx.y;
    pdl_wait();
    CSLA_TL_WAITED();
    const Req rq = request(a, b);
    if (!rq.ok) return;
    const int n_chunks = rq.n_chunks;
    // unconditional loads (chunks past the last reread the last one; unused)
    float v[kDPT][kMaxC];
#pragma unroll
    for (int c = 0; c < kMaxC; ++c)
#pragma unroll
        for (int j = 0; j < kDPT; ++j) v[j][c] = partial_o(a, b, min(c, n_chunks - 1), h, threadIdx.x + 128 * j, D);
    if (threadIdx.x < 32) {
        float wl, l;
        fold_weights(a, b, n_chunks, h, D, &wl, &l);
        wts[threadIdx.x] = wl;
        if (threadIdx.x == 0) wts[32] = l;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kDPT; ++j) {
        float o = 0.f;
#pragma unroll
        for (int c = 0; c < kMaxC; ++c)
            if (c < n_chunks) o = __fmaf_rn(v[j][c], wts[c], o);
        store_out(a, out_bf16 != 0, ((size_t)b * a.H + h) * D + threadIdx.x + 128 * j, __fdiv_rn(o, wts[32]));
    }
}

template <int D>
cudaError_t launch_attend_t(const AttendArgs &a, bool q_bf16, bool out_bf16, int variant, int num_sms,
                            cudaStream_t stream) {
    constexpr int kSmem = smem_bytes<D>();
    static_assert(kSmem <= 232448, "shared memory budget");
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmem);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(attend_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    bool saturated;
    if (variant == CSLA_VARIANT_SATURATED) saturated = true;
    else if (variant == CSLA_VARIANT_STARVED) saturated = false;
    else saturated = a.B >= num_sms || a.max_chunks <= 1;
    if (saturated)
        return launch_pdl(attend_kernel<D, true>, dim3(a.B), dim3(kThreads), kSmem, stream, a, (int)q_bf16,
                          (int)out_bf16);
    cudaError_t e =
        launch_pdl(attend_kernel<D, false>, dim3(a.max_chunks, a.B), dim3(kThreads), kSmem, stream, a, (int)q_bf16,
                   (int)out_bf16);
    if (e != cudaSuccess) return e;
    if (a.max_chunks <= 16)
        return launch_pdl(combine_kernel<D, 16>, dim3(a.H, a.B), dim3(128), 0, stream, a, (int)out_bf16);
    return launch_pdl(combine_kernel<D, 32>, dim3(a.H, a.B), dim3(128), 0, stream, a, (int)out_bf16);
}

}  // namespace

cudaError_t launch_attend(const AttendArgs &a, bool q_bf16, bool out_bf16, int variant, int num_sms,
                          cudaStream_t stream) {
    if (a.D == 512) return launch_attend_t<512>(a, q_bf16, out_bf16, variant, num_sms, stream);
    if (a.D == 128) return launch_attend_t<128>(a, q_bf16, out_bf16, variant, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace csla
