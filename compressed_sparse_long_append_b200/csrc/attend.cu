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
// partial (running max m, sum l, unnormalised O) computed by chunk_pass();
// the partials are folded left to right, starting from the sink, by
// fold_store().  The saturated kernel walks all chunks of a request in one
// CTA and folds at the end; the starved kernel gives every chunk its own CTA
// and a combine kernel folds.  Both run the same two functions on the same
// data, so their outputs are identical bit for bit, and nothing depends on
// which other requests share the launch.
//
// Per 64-row tile of a chunk (one CTA = 128 threads, warp 0 lane 0 issues UMMA):
//   X  [64 rows x D] bf16 in smem (fp8 codes widened exactly, bf16 RoPE dims)
//   S  = Qhat . X^T      tcgen05 M=64 (heads) N=64 (rows), nope and RoPE dims
//                        into separate TMEM accumulators: s = scale*S_nope + S_rope
//   P  = 2^(s - m)       one thread per head; P_nope = P*scale, P_rope = P (bf16)
//   O^T += X^T . P^T     tcgen05 M=128 (dims) N=64 (heads), accumulated in TMEM
// Lazy rescale: the running max moves only when a tile's max exceeds it by
// more than 8 (log2 units); then O^T columns and l are rescaled in place.
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kThreads = 128;
constexpr int kHP = 64;          // heads padded to the UMMA M of the S product
constexpr int kTile = 64;        // rows per tile
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 8.0f;

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
    // TMEM columns
    static constexpr int kColSN = 0, kColSR = 64, kColO = 128;
    static constexpr int kColOR = 128 + 64 * kMB;
    static constexpr int kTmemCols = (kColOR + 64) <= 256 ? 256 : 512;
    // smem offsets (from a 1024-aligned base)
    static constexpr int kOffQ = 0;
    static constexpr int kOffX0 = kOffQ + kQBytes;
    static constexpr int kOffX1 = kOffX0 + kXBytes;
    static constexpr int kOffPn = kOffX1 + kXBytes;
    static constexpr int kOffPr = kOffPn + kPBytes;
    static constexpr int kOffMisc = kOffPr + kPBytes;
    static constexpr int kSmemBytes = kOffMisc + 4096 + 1024;
};

struct Misc {
    const uint8_t *rowptr[kTile];
    float rscale[kTile];
    int rvalid[kTile];
    float fac[kHP];
    float cs[32][2];
    uint64_t bar_s, bar_o;
    uint32_t tmem;
    int any_rescale;
    int abort;
};

// Request-level facts both variants derive the same way.
struct Req {
    int slot, L, nv, n_cmp, win_len, n_rows, chunk, n_chunks;
    bool ok;
};
__device__ __forceinline__ Req request(const AttendArgs &a, int b) {
    Req r;
    r.slot = __ldg(a.slots + b);
    const bool slot_ok = r.slot >= 0 && r.slot < a.n_slots;
    r.L = slot_ok ? __ldg(a.len + r.slot) : 0;
    r.ok = slot_ok && r.L >= 1 && r.L <= a.max_len;
    if (!r.ok) r.L = 0;
    r.nv = r.L / a.m;
    r.n_cmp = a.idx ? a.k : r.nv;
    r.win_len = r.L < a.n_win ? r.L : a.n_win;
    r.n_rows = r.ok ? r.n_cmp + r.win_len : 0;
    r.chunk = attend_chunk_rows(r.n_rows);
    r.n_chunks = r.ok ? attend_num_chunks(r.n_rows) : 0;
    return r;
}

__device__ __forceinline__ uint4 ld_nc_v4(const void *p) {
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Byte offset of 8-element group g (dims 8g..8g+7) of row r in a SW128
// K-major tile whose K blocks are `kb_bytes` apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int g, int kb_bytes) {
    return (uint32_t)((g >> 3) * kb_bytes + (r >> 3) * 1024 + (r & 7) * 128 + (((g & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    return (uint32_t)f32_to_bf16_bits(lo) | ((uint32_t)f32_to_bf16_bits(hi) << 16);
}

// qhat = RoPE(RMSNorm(q_h) * gamma_q, t) for the 64 (padded) heads -> smem.
template <int D>
__device__ void prepare_q(const AttendArgs &a, int b, long long t, bool q_bf16, uint8_t *qs, Misc *ms) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x < 32) {
        float c, s;
        rope_cos_sin(t, threadIdx.x, 64, a.theta, &c, &s);
        ms->cs[threadIdx.x][0] = c;
        ms->cs[threadIdx.x][1] = s;
    }
    __syncthreads();
    constexpr int NG = D / 8;                   // 8-dim groups per head
    constexpr int GPL = (NG + 31) / 32;         // groups per lane
    for (int h = warp; h < kHP; h += 4) {
        float x[GPL][8];
        float ss = 0.f;
#pragma unroll
        for (int i = 0; i < GPL; ++i) {
            const int g = lane + 32 * i;
#pragma unroll
            for (int e = 0; e < 8; ++e) x[i][e] = 0.f;
            if (g < NG && h < a.H) {
                const size_t off = ((size_t)b * a.H + h) * D + (size_t)g * 8;
                if (q_bf16) {
                    const uint4 u = __ldg(reinterpret_cast<const uint4 *>(
                        reinterpret_cast<const __nv_bfloat16 *>(a.q) + off));
                    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        x[i][2 * e] = bf16_bits_to_f32(w[e] & 0xFFFFu);
                        x[i][2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
                    }
                } else {
                    const float4 *p = reinterpret_cast<const float4 *>(reinterpret_cast<const float *>(a.q) + off);
                    const float4 u0 = __ldg(p), u1 = __ldg(p + 1);
                    x[i][0] = u0.x; x[i][1] = u0.y; x[i][2] = u0.z; x[i][3] = u0.w;
                    x[i][4] = u1.x; x[i][5] = u1.y; x[i][6] = u1.z; x[i][7] = u1.w;
                }
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) ss = __fmaf_rn(x[i][e], x[i][e], ss);
        }
        ss = warp_sum(ss);
        const float r = 1.0f / sqrtf(__fdiv_rn(ss, (float)D) + a.eps);
#pragma unroll
        for (int i = 0; i < GPL; ++i) {
            const int g = lane + 32 * i;
            if (g >= NG) continue;
            float y[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) y[e] = __fmul_rn(__fmul_rn(x[i][e], r), __ldg(a.gamma_q + g * 8 + e));
            if (g * 8 >= D - 64) {
#pragma unroll
                for (int e = 0; e < 8; e += 2) {
                    const int pi = (g * 8 + e - (D - 64)) >> 1;
                    const float c = ms->cs[pi][0], s = ms->cs[pi][1];
                    const float y0 = y[e], y1 = y[e + 1];
                    y[e] = __fsub_rn(__fmul_rn(y0, c), __fmul_rn(y1, s));
                    y[e + 1] = __fadd_rn(__fmul_rn(y0, s), __fmul_rn(y1, c));
                }
            }
            uint4 o;
            o.x = pack_bf16x2(y[0], y[1]);
            o.y = pack_bf16x2(y[2], y[3]);
            o.z = pack_bf16x2(y[4], y[5]);
            o.w = pack_bf16x2(y[6], y[7]);
            *reinterpret_cast<uint4 *>(qs + sw128_off(h, g, Cfg<D>::kQKB)) = o;
        }
    }
}

// Sources of the tile's rows [r0, r0+64) restricted to [lo, hi).
__device__ void tile_sources(const AttendArgs &a, int b, const Req &rq, int r0, int hi, int rb, Misc *ms) {
    const int t = threadIdx.x;
    if (t >= kTile) return;
    const int r = r0 + t;
    const uint8_t *p = nullptr;
    float sc = 0.f;
    int ok = 0;
    if (r < hi) {
        if (r < rq.n_cmp) {
            const int e = a.idx ? __ldg(a.idx + (size_t)b * a.k + r) : r;
            if (e >= 0) {
                if (e >= rq.nv) {
                    set_dev_err(CSLA_DEVERR_INDEX);
                } else {
                    const int epp = CSLA_PAGE_TOKENS / a.m;
                    const int col = e / epp;
                    const int pg = col < a.bt_stride ? __ldg(a.block_table + (size_t)rq.slot * a.bt_stride + col) : -1;
                    if (pg < 0 || pg >= a.n_pages) {
                        set_dev_err(CSLA_DEVERR_PAGE);
                    } else {
                        const size_t ent = (size_t)pg * epp + (size_t)(e % epp);
                        p = a.rows + ent * rb;
                        sc = __ldg(a.scales + ent);
                        ok = 1;
                    }
                }
            }
        } else {
            const int w = r - rq.n_cmp;
            const int pos = rq.L - rq.win_len + w;
            const size_t ring = (size_t)rq.slot * a.n_win + (size_t)(pos % a.n_win);
            p = a.win_rows + ring * rb;
            sc = __ldg(a.win_scales + ring);
            ok = 1;
        }
    }
    ms->rowptr[t] = p;
    ms->rscale[t] = sc;
    ms->rvalid[t] = ok;
}

// Widen the tile's cache rows into the bf16 SW128 K-major X tile.
template <int D>
__device__ void load_tile(uint8_t *xs, const Misc *ms) {
    using C = Cfg<D>;
    constexpr int kTasks = kTile * C::kCH;
    constexpr int kU = 6;
    static_assert(kTasks % (kThreads * kU) == 0 || kTasks < kThreads * kU, "task split");
    for (int base = 0; base < kTasks; base += kThreads * kU) {
        uint4 v[kU];
        int rr[kU], cc[kU];
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int id = base + u * kThreads + threadIdx.x;
            rr[u] = id / C::kCH;
            cc[u] = id % C::kCH;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (id < kTasks && ms->rvalid[rr[u]]) v[u] = ld_nc_v4(ms->rowptr[rr[u]] + cc[u] * 16);
        }
#pragma unroll
        for (int u = 0; u < kU; ++u) {
            const int id = base + u * kThreads + threadIdx.x;
            if (id >= kTasks) continue;
            const int r = rr[u], c = cc[u];
            if (c < C::kNopeCH) {
                const int g0 = c * 2;   // 16 codes = two 8-dim groups
                uint4 lo, hi;
                lo.x = e4m3x2_to_bf16x2(v[u].x & 0xFFFFu);
                lo.y = e4m3x2_to_bf16x2(v[u].x >> 16);
                lo.z = e4m3x2_to_bf16x2(v[u].y & 0xFFFFu);
                lo.w = e4m3x2_to_bf16x2(v[u].y >> 16);
                hi.x = e4m3x2_to_bf16x2(v[u].z & 0xFFFFu);
                hi.y = e4m3x2_to_bf16x2(v[u].z >> 16);
                hi.z = e4m3x2_to_bf16x2(v[u].w & 0xFFFFu);
                hi.w = e4m3x2_to_bf16x2(v[u].w >> 16);
                *reinterpret_cast<uint4 *>(xs + sw128_off(r, g0, C::kKBBytes)) = lo;
                *reinterpret_cast<uint4 *>(xs + sw128_off(r, g0 + 1, C::kKBBytes)) = hi;
            } else {
                const int g = (D - 64) / 8 + (c - C::kNopeCH);
                *reinterpret_cast<uint4 *>(xs + sw128_off(r, g, C::kKBBytes)) = v[u];
            }
        }
    }
}

struct HeadState {
    float m, l;
};

// One chunk of request b: rows [lo, hi) of its attention set.  Writes the
// chunk partial (O [H][D], m [H], l [H]) to `part`.  Ends with every thread
// past a __syncthreads and no UMMA in flight.
template <int D>
__device__ void chunk_pass(const AttendArgs &a, int b, const Req &rq, int lo, int hi, uint8_t *smem, Misc *ms,
                           uint32_t &ph_s, uint32_t &ph_o, float *part) {
    using C = Cfg<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    const int h = 16 * warp + lane;       // head owned by lanes 0..15 (M=64 TMEM layout)
    const bool head_thread = lane < 16;
    const float cscale = kLog2e / sqrtf((float)D);
    constexpr uint32_t kIdescS = idesc_bf16(64, 64, false, false);
    constexpr uint32_t kIdescO = idesc_bf16(128, 64, true, false);
    uint8_t *qs = smem + C::kOffQ;
    uint8_t *pn = smem + C::kOffPn;
    uint8_t *pr = smem + C::kOffPr;
    const uint32_t tmem = ms->tmem;
    HeadState hs{-INFINITY, 0.f};
    int buf = 0;

    for (int r0 = lo, ti = 0; r0 < hi; r0 += kTile, ++ti, buf ^= 1) {
        uint8_t *xs = smem + (buf ? C::kOffX1 : C::kOffX0);
        tile_sources(a, b, rq, r0, hi, C::kRB, ms);
        __syncthreads();
        load_tile<D>(xs, ms);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint32_t q0 = smem_u32(qs), x0 = smem_u32(xs);
#pragma unroll
            for (int kb = 0; kb < C::kKBN; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + C::kColSN, sdesc(q0 + kb * C::kQKB + ks * 32, 16, 1024),
                              sdesc(x0 + kb * C::kKBBytes + ks * 32, 16, 1024), kIdescS, (kb | ks) ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tmem + C::kColSR, sdesc(q0 + C::kKBN * C::kQKB + ks * 32, 16, 1024),
                          sdesc(x0 + C::kKBN * C::kKBBytes + ks * 32, 16, 1024), kIdescS, ks ? 1u : 0u);
            umma_commit(&ms->bar_s);
        }
        mbar_wait(&ms->bar_s, ph_s, &ms->abort);
        ph_s ^= 1;
        tc_fence_after();

        // ---- scores of this tile: lanes 0..15 hold head rows
        float s[kTile];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            uint32_t rn[32], rrp[32];
            tmem_ld32x32(tmem + lane_base + C::kColSN + 32 * half, rn);
            tmem_ld32x32(tmem + lane_base + C::kColSR + 32 * half, rrp);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j) {
                const int jj = 32 * half + j;
                const float v = __fmul_rn(__fmaf_rn(ms->rscale[jj], __uint_as_float(rn[j]), __uint_as_float(rrp[j])),
                                          cscale);
                s[jj] = ms->rvalid[jj] ? v : -INFINITY;
            }
        }
        float mt = -INFINITY;
#pragma unroll
        for (int j = 0; j < kTile; ++j) mt = fmaxf(mt, s[j]);

        // PV of the previous tile must be done before P and O^T are touched.
        if (ti > 0) {
            mbar_wait(&ms->bar_o, ph_o, &ms->abort);
            ph_o ^= 1;
            tc_fence_after();
        }
        if (threadIdx.x == 0) ms->any_rescale = 0;
        __syncthreads();
        float f = 1.f;
        if (head_thread) {
            float mnew = hs.m;
            if (ti == 0) {
                mnew = mt;
            } else if (mt > hs.m + kRescaleThresh || (hs.m == -INFINITY && mt > -INFINITY)) {
                mnew = mt;
                f = exp2f(__fsub_rn(hs.m, mnew));
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
                uint4 un, ur;
                un.x = pack_bf16x2(__fmul_rn(p[0], ms->rscale[c8 * 8 + 0]), __fmul_rn(p[1], ms->rscale[c8 * 8 + 1]));
                un.y = pack_bf16x2(__fmul_rn(p[2], ms->rscale[c8 * 8 + 2]), __fmul_rn(p[3], ms->rscale[c8 * 8 + 3]));
                un.z = pack_bf16x2(__fmul_rn(p[4], ms->rscale[c8 * 8 + 4]), __fmul_rn(p[5], ms->rscale[c8 * 8 + 5]));
                un.w = pack_bf16x2(__fmul_rn(p[6], ms->rscale[c8 * 8 + 6]), __fmul_rn(p[7], ms->rscale[c8 * 8 + 7]));
                ur.x = pack_bf16x2(p[0], p[1]);
                ur.y = pack_bf16x2(p[2], p[3]);
                ur.z = pack_bf16x2(p[4], p[5]);
                ur.w = pack_bf16x2(p[6], p[7]);
                const uint32_t off = (uint32_t)((h >> 3) * 1024 + (h & 7) * 128 + ((c8 ^ (h & 7)) << 4));
                *reinterpret_cast<uint4 *>(pn + off) = un;
                *reinterpret_cast<uint4 *>(pr + off) = ur;
            }
            hs.l = (ti == 0) ? lsum : __fadd_rn(__fmul_rn(hs.l, f), lsum);
            hs.m = mnew;
            ms->fac[h] = f;
            if (ti > 0 && f != 1.f) ms->any_rescale = 1;
        }
        __syncthreads();
        if (ms->any_rescale) {
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
                        v[j] = __float_as_uint(__fmul_rn(__uint_as_float(v[j]), ms->fac[32 * half + j]));
                    tmem_st32x32(addr, v);
                }
            }
            tmem_wait_st();
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncthreads();
        if (threadIdx.x == 0) {
            tc_fence_after();
            const uint32_t x0 = smem_u32(xs), p0n = smem_u32(pn), p0r = smem_u32(pr);
#pragma unroll
            for (int mb = 0; mb < C::kMB; ++mb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_bf16(tmem + C::kColO + 64 * mb, sdesc(x0 + 2 * mb * C::kKBBytes + 2 * ks * 1024, C::kKBBytes, 1024),
                              sdesc(p0n + ks * 32, 16, 1024), kIdescO, (ti > 0 || ks > 0) ? 1u : 0u);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
                umma_bf16(tmem + C::kColOR, sdesc(x0 + 2 * (C::kMB - 1) * C::kKBBytes + 2 * ks * 1024, C::kKBBytes, 1024),
                          sdesc(p0r + ks * 32, 16, 1024), kIdescO, (ti > 0 || ks > 0) ? 1u : 0u);
            umma_commit(&ms->bar_o);
        }
    }
    // drain the last PV, then read O^T out of TMEM
    mbar_wait(&ms->bar_o, ph_o, &ms->abort);
    ph_o ^= 1;
    tc_fence_after();
    const size_t HD = (size_t)a.H * D;
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
        part[HD + h] = hs.m;
        part[HD + a.H + h] = hs.l;
    }
    tc_fence_before();
    __syncthreads();
}

// Ordered fold of the chunk partials of request b, head h, dim d (sink first).
__device__ __forceinline__ float fold_one(const AttendArgs &a, int b, int n_chunks, int h, int d, int D,
                                          float *l_out) {
    const size_t stride = (size_t)a.H * D + 2 * (size_t)a.H;
    const float *p = a.part + (size_t)b * a.max_chunks * stride;
    float m = __fmul_rn(__ldg(a.sink + h), kLog2e);
    float l = 1.f, o = 0.f;
    for (int c = 0; c < n_chunks; ++c, p += stride) {
        const float mc = p[(size_t)a.H * D + h];
        const float lc = p[(size_t)a.H * D + a.H + h];
        const float mn = fmaxf(m, mc);
        const float fa = exp2f(__fsub_rn(m, mn));
        const float fb = exp2f(__fsub_rn(mc, mn));
        l = __fmaf_rn(l, fa, __fmul_rn(lc, fb));
        o = __fmaf_rn(o, fa, __fmul_rn(p[(size_t)h * D + d], fb));
        m = mn;
    }
    *l_out = l;
    return __fdiv_rn(o, l);
}

__device__ __forceinline__ void store_out(const AttendArgs &a, bool out_bf16, size_t i, float v) {
    if (out_bf16) reinterpret_cast<__nv_bfloat16 *>(a.out)[i] = __float2bfloat16_rn(v);
    else reinterpret_cast<float *>(a.out)[i] = v;
}

template <int D, bool kSaturated>
__global__ void __launch_bounds__(kThreads, 1) attend_kernel(AttendArgs a, int q_bf16, int out_bf16) {
    using C = Cfg<D>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Misc *ms = reinterpret_cast<Misc *>(smem + C::kOffMisc);

    const int b = kSaturated ? blockIdx.x : blockIdx.y;
    const Req rq = request(a, b);
    if (!rq.ok) {
        if (threadIdx.x == 0 && (kSaturated || blockIdx.x == 0)) set_dev_err(CSLA_DEVERR_LEN);
        return;
    }
    if (!kSaturated && (int)blockIdx.x >= rq.n_chunks) return;

    if (threadIdx.x == 0) {
        mbar_init(&ms->bar_s, 1);
        mbar_init(&ms->bar_o, 1);
        ms->abort = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < 32) {
        tmem_alloc(&ms->tmem, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();

    prepare_q<D>(a, b, (long long)rq.L - 1, q_bf16 != 0, smem + C::kOffQ, ms);
    fence_proxy_async_smem();
    __syncthreads();

    uint32_t ph_s = 0, ph_o = 0;
    const size_t stride = (size_t)a.H * D + 2 * (size_t)a.H;
    const int c0 = kSaturated ? 0 : (int)blockIdx.x;
    const int c1 = kSaturated ? rq.n_chunks : c0 + 1;
    for (int c = c0; c < c1; ++c) {
        const int lo = c * rq.chunk;
        const int hi = min(rq.n_rows, lo + rq.chunk);
        float *part = a.part + ((size_t)b * a.max_chunks + c) * stride;
        chunk_pass<D>(a, b, rq, lo, hi, smem, ms, ph_s, ph_o, part);
    }
    if (threadIdx.x < 32) {
        tc_fence_after();
        tmem_dealloc(ms->tmem, C::kTmemCols);
    }
    if (kSaturated) {
        __syncthreads();   // partials written by this CTA are visible to it
        for (int i = threadIdx.x; i < a.H * D; i += kThreads) {
            const int hh = i / D, d = i % D;
            float l;
            const float v = fold_one(a, b, rq.n_chunks, hh, d, D, &l);
            store_out(a, out_bf16 != 0, ((size_t)b * a.H + hh) * D + d, v);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(kThreads) combine_kernel(AttendArgs a, int out_bf16) {
    const int h = blockIdx.x, b = blockIdx.y;
    const Req rq = request(a, b);
    if (!rq.ok) return;
    for (int d = threadIdx.x; d < D; d += kThreads) {
        float l;
        const float v = fold_one(a, b, rq.n_chunks, h, d, D, &l);
        store_out(a, out_bf16 != 0, ((size_t)b * a.H + h) * D + d, v);
    }
}

template <int D>
cudaError_t launch_attend_t(const AttendArgs &a, bool q_bf16, bool out_bf16, int variant, int num_sms,
                            cudaStream_t stream) {
    using C = Cfg<D>;
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(attend_kernel<D, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             C::kSmemBytes);
        if (e != cudaSuccess) return e;
        e = cudaFuncSetAttribute(attend_kernel<D, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 C::kSmemBytes);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    bool saturated;
    if (variant == CSLA_VARIANT_SATURATED) saturated = true;
    else if (variant == CSLA_VARIANT_STARVED) saturated = false;
    else saturated = a.B >= num_sms || a.max_chunks <= 1;
    if (saturated) {
        attend_kernel<D, true><<<a.B, kThreads, C::kSmemBytes, stream>>>(a, q_bf16, out_bf16);
        return cudaGetLastError();
    }
    attend_kernel<D, false><<<dim3(a.max_chunks, a.B), kThreads, C::kSmemBytes, stream>>>(a, q_bf16, out_bf16);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    combine_kernel<D><<<dim3(a.H, a.B), kThreads, 0, stream>>>(a, out_bf16);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend(const AttendArgs &a, bool q_bf16, bool out_bf16, int variant, int num_sms,
                          cudaStream_t stream) {
    if (a.D == 512) return launch_attend_t<512>(a, q_bf16, out_bf16, variant, num_sms, stream);
    if (a.D == 128) return launch_attend_t<128>(a, q_bf16, out_bf16, variant, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace csla
