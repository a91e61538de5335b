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
// Operands.  A cache row holds fp8 (E4M3) codes c_d with one scale s per row
// for the first D-64 dims and bf16 values for the 64 RoPE dims.  Every row
// enters the tensor cores as one f16 vector X' of D dims:
//   X'_d = e4m3(c_d) / 256            (exact: a move of the code's bits)
//   X'_d = x_d / (256 s)              (RoPE dims, rounded to f16)
// so that x_d = 256 s X'_d for every dim.  With Qhat in f16,
//   s_j = 256 s_j^row * <Qhat, X'_j> / sqrt(D)        (one accumulator),
//   O  += X'^T . P',   P'_hj = f16(p_hj * 256 s_j^row).
// A row whose RoPE dims would leave the f16 range this way (|x_d| > 2^15 *
// 256 s, which needs a row whose fp8 part is ~10^5 times smaller than its
// RoPE part) takes a larger effective scale on a slow path.  A row whose
// effective scale exceeds kScaleMax (fp8 dims beyond 448 * 15 = 6720, or
// RoPE dims beyond ~1.3e8: never a row of a normalised vector) would
// overflow P'; it is masked and sets CSLA_DEVERR_RANGE.
//
// One CTA = three roles over a stream of 64-row tiles:
//   warps 4-11 (loader)  resolve row addresses eight tiles ahead (a ring of
//                        16 tiles in shared memory; the three dependent
//                        lookups -- top-k index, block table, scale -- run
//                        on separate lane groups for three future tiles
//                        each step), convert tile t's raw rows from
//                        registers into X'[t & 1], then load tile t+1
//                        (bulk-prefetched into L2 a step earlier) and
//                        prefetch tile t+2;
//   warp 12 (MMA)        S[t&1] = Qhat . X'^T  tcgen05 M=64 (heads) N=64 (rows)
//                        O^T   += X'^T . P'^T  tcgen05 M=128 (dims) N=64 (heads),
//                        issuing S of tile t+1 before PV of tile t;
//   warps 0-3 (softmax)  build Qhat = RoPE(RMSNorm(q)*gamma_q, t) from a bulk
//                        copy of q (the norm before the grid-dependency wait,
//                        the rotation after it); per tile read S, P = 2^(s - m)
//                        (lanes 0-15 of each warp own one head), lazy rescale
//                        of O^T when a head's max grows by more than 4 (log2
//                        units); at chunk end read O^T out as the partial.
// mbarriers hand tiles between roles; every wait is bounded.
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kSoftWarps = 4, kLoadWarps = 8;
constexpr int kThreads = 32 * (kSoftWarps + kLoadWarps + 1);   // 416
constexpr int kMmaWarp = kSoftWarps + kLoadWarps;               // warp 12
constexpr int kHP = 64;          // heads padded to the UMMA M of the S product
constexpr int kTile = 32;        // rows per tile
constexpr int kRowsPerWarp = kTile / kLoadWarps;                // 4 rows of each tile per loader warp
constexpr int kRing = 16;        // tiles of resolved row addresses
constexpr int kAhead = 8;        // tiles resolved before the first conversion
constexpr int kNR = 2;           // raw-row buffers (tiles of bulk copies in flight)
// X' buffers.  Converting tile t needs X'[t % kNX] back from the PV of tile
// t - kNX; with two buffers that PV is issued only after S of tile t - 1, so
// every conversion waited on the tensor cores and softmax of the tile before
// (half of a loader's time); with three the conversions run back to back.
constexpr int kNX = 3;
// X' buffer of tile t.  q is staged from X'[0] on, so tile 0 goes to the last
// buffer: when q fits in the first two, tile 0 is converted while Qhat is
// still being built.
__device__ __forceinline__ int xbuf(int t) { return (t + kNX - 1) % kNX; }
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleThresh = 4.0f;
constexpr float kRopeMax = 32768.0f;   // largest |X'| taken for a RoPE dim at the row's own scale
// Largest effective row scale: P' = p * 256 * scale stays below the f16
// maximum for p <= 2^kRescaleThresh.  Rows beyond it are masked and flagged.
constexpr float kScaleMax = 15.0f;

template <int D>
struct Cfg {
    static constexpr int kRB = D + 64;                 // row bytes
    static constexpr int kNopeCH = (D - 64) / 16;      // 16-byte chunks of fp8 codes per row
    static constexpr int kKB = D / 64;                 // 64-dim K blocks
    static constexpr int kMB = D / 128;                // 128-dim O^T blocks
    static constexpr int kKBBytes = kTile * 128;       // one K block of X' (32 rows x 128 B)
    static constexpr int kXBytes = kKB * kKBBytes;
    static constexpr int kQKB = kHP * 128;             // one K block of Qhat
    static constexpr int kQBytes = kKB * kQKB;
    static constexpr int kPBytes = kHP * 64 * 2;        // P [64 heads][64 cols], cols 0..kTile-1 used
    static constexpr int kRawBytes = kTile * kRB;       // one raw buffer (bulk-copied cache rows)
    static constexpr int kNopeIt = (kRowsPerWarp * kNopeCH + 31) / 32;   // fp8 chunk rounds per loader lane
    static_assert(kRowsPerWarp * 8 == 32, "one RoPE chunk per loader lane");
    // TMEM columns: two S buffers of kTile columns, then O^T
    static constexpr int kColS = 0, kColO = 2 * kTile;
    static constexpr int kTmemCols = (kColO + 64 * kMB) <= 128 ? 128 : ((kColO + 64 * kMB) <= 256 ? 256 : 512);
    // smem offsets (from a 1024-aligned base); q is staged from X'[0] on at
    // the start (into the raw buffers too when it is larger than the X' buffers)
    static constexpr int kOffQ = 0;
    static constexpr int kOffX = kOffQ + kQBytes;      // X'[0 .. kNX)
    static constexpr int kOffRaw = kOffX + kNX * kXBytes;
    static constexpr int kOffP = kOffRaw + kNR * kRawBytes;
    static constexpr int kOffMisc = kOffP + kPBytes;
};

// Kinds of row locations in the loader ring.
enum : uint8_t { kLocNone = 0, kLocCache = 1, kLocRing = 2, kLocSrc = 3 };

struct Misc {
    float tscale[kNX][kTile];          // per X' buffer: 256 * effective fp8 scale of each row (0 = masked)
    float fac[2][kHP];                 // per tile parity: O^T column factors (1 = none)
    // loader ring, per tile slot (t % kRing) and row of the tile
    int ent[kRing][kTile];             // stage 1: compressed entry index (or the set row for window rows)
    uint32_t loc[kRing][kTile];        // stage 2: row index in its array
    float scl[kRing][kTile];           // stage 3: fp8 scale (0 = masked)
    uint8_t kind[kRing][kTile];        // stage 2: kLoc*
    uint64_t q_staged, q_ready, x_full[kNX], x_empty[kNX], s_full[2], s_free[2], p_full, pv_done, o_free, fac_ready,
        drain, raw_full[kLoadWarps][kNR];   // raw_full[w][j]: warp w's rows of raw buffer j landed
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

// Byte offset of 8-element group g (dims 8g..8g+7) of row r in a SW128
// K-major tile whose K blocks are `kb_bytes` apart.
__device__ __forceinline__ uint32_t sw128_off(int r, int g, int kb_bytes) {
    return (uint32_t)((g >> 3) * kb_bytes + (r >> 3) * 1024 + (r & 7) * 128 + (((g & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t *>(&h);
}

// Two E4M3 codes (bytes kLo and kLo+1 of w) -> f16x2 of their values / 256,
// exactly: the 7 magnitude bits go under the f16 exponent/mantissa fields,
// which places E4M3 normals and subnormals alike 8 binades low, and the
// sign bit moves to bit 15.  (The NaN codes 0x7F/0xFF, which the quantiser
// never writes, read as 480/256.)
template <int kLo>
__device__ __forceinline__ uint32_t e4m3x2_f16x2_div256(uint32_t w) {
    constexpr uint32_t kSel = kLo == 0 ? 0x1404u : 0x3424u;   // code kLo+1 -> byte 3, code kLo -> byte 1
    const uint32_t x = __byte_perm(w, 0u, kSel);
    return (x & 0x80008000u) | ((x >> 1) & 0x3F803F80u);
}

// ---------------------------------------------------------------- query preparation
// Qhat = RoPE(RMSNorm(q_h) * gamma_q, t) for the 64 (padded) heads of the
// request, built in shared memory by the softmax warps in two steps from a
// bulk copy of the request's q rows (`stage`, H*D elements).
// Before the grid-dependency wait (q and gamma_q are inputs of the call):
// gamma_q is loaded while the copy is in flight, then warp w normalises heads
// 16w .. 16w+15, two heads at a time (false if the copy's wait gave up);
// lane l owns the
// 8-dim groups l and l+32 (D = 512) or the 4 dims 4l.. (D = 128), so the
// staged reads are consecutive per lane (no bank conflicts).  Non-RoPE dims
// go to the SW128 K-major Qhat image as f16; the RoPE dims are kept in fp32
// at the start of the head's own staged row (already read).  After the
// wait, when the position t = len - 1 is known, lane i rotates pair i of its
// warp's 16 heads and writes them as f16.
template <int D>
__device__ bool build_q_normed(const AttendArgs &a, uint8_t *smem, uint8_t *stage, int q_bf16, Misc *ms) {
    using C = Cfg<D>;
    constexpr int kG = D == 512 ? 2 : 1;       // element groups per lane
    constexpr int kE = D == 512 ? 8 : 4;       // elements per group
    constexpr int kStride = D == 512 ? 256 : 0; // dims between a lane's two groups
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = D * (q_bf16 ? 2 : 4);       // staged bytes per head
    float gam[kG][kE];
#pragma unroll
    for (int g = 0; g < kG; ++g)
#pragma unroll
        for (int e = 0; e < kE; ++e) gam[g][e] = __ldg(a.gamma_q + g * kStride + kE * lane + e);
    // gamma_q is in registers before q's rows are waited for
    if (!warp_all(mbar_wait(&ms->q_staged, 0, &ms->abort))) return false;
    // two heads at a time: their loads, reductions and square roots are
    // independent chains that overlap
    constexpr int kHB = 2;
    for (int h0 = 16 * warp; h0 < 16 * warp + 16; h0 += kHB) {
        float x[kHB][kG][kE];
#pragma unroll
        for (int u = 0; u < kHB; ++u) {
            const int h = h0 + u;
            const uint8_t *src = stage + h * rb;
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                const int d = g * kStride + kE * lane;
                if (h >= a.H) {
#pragma unroll
                    for (int e = 0; e < kE; ++e) x[u][g][e] = 0.f;
                } else if (q_bf16) {
                    if constexpr (kE == 8) {
                        const uint4 w = *reinterpret_cast<const uint4 *>(src + 2 * d);
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            x[u][g][2 * e] = bf16_bits_to_f32(ww[e] & 0xFFFFu);
                            x[u][g][2 * e + 1] = bf16_bits_to_f32(ww[e] >> 16);
                        }
                    } else {
                        const uint2 w = *reinterpret_cast<const uint2 *>(src + 2 * d);
                        x[u][g][0] = bf16_bits_to_f32(w.x & 0xFFFFu);
                        x[u][g][1] = bf16_bits_to_f32(w.x >> 16);
                        x[u][g][2] = bf16_bits_to_f32(w.y & 0xFFFFu);
                        x[u][g][3] = bf16_bits_to_f32(w.y >> 16);
                    }
                } else {
#pragma unroll
                    for (int e0 = 0; e0 < kE; e0 += 4) {
                        const float4 f4 = *reinterpret_cast<const float4 *>(src + 4 * (d + e0));
                        x[u][g][e0] = f4.x;
                        x[u][g][e0 + 1] = f4.y;
                        x[u][g][e0 + 2] = f4.z;
                        x[u][g][e0 + 3] = f4.w;
                    }
                }
            }
        }
        float r[kHB];
#pragma unroll
        for (int u = 0; u < kHB; ++u) {
            float ss = 0.f;
#pragma unroll
            for (int g = 0; g < kG; ++g)
#pragma unroll
                for (int e = 0; e < kE; ++e) ss = __fmaf_rn(x[u][g][e], x[u][g][e], ss);
            r[u] = ss;
        }
        // every lane has read both heads' rows before anything is written back
#pragma unroll
        for (int o = 16; o > 0; o >>= 1)
#pragma unroll
            for (int u = 0; u < kHB; ++u) r[u] += __shfl_xor_sync(0xffffffffu, r[u], o);
#pragma unroll
        for (int u = 0; u < kHB; ++u) r[u] = 1.0f / sqrtf(__fdiv_rn(r[u], (float)D) + a.eps);
#pragma unroll
        for (int u = 0; u < kHB; ++u) {
            const int h = h0 + u;
#pragma unroll
            for (int g = 0; g < kG; ++g) {
                const int d = g * kStride + kE * lane;
                float y[kE];
#pragma unroll
                for (int e = 0; e < kE; ++e) y[e] = __fmul_rn(__fmul_rn(x[u][g][e], r[u]), gam[g][e]);
                if (h >= a.H) {
                    // padding head: zero Qhat row (the RoPE dims are written zero after the wait)
                    if (d < D - 64) {
                        if constexpr (kE == 8)
                            *reinterpret_cast<uint4 *>(smem + C::kOffQ + sw128_off(h, d >> 3, C::kQKB)) =
                                make_uint4(0u, 0u, 0u, 0u);
                        else
                            *reinterpret_cast<uint2 *>(smem + C::kOffQ + sw128_off(h, d >> 3, C::kQKB) + (d & 7) * 2) =
                                make_uint2(0u, 0u);
                    }
                } else if (d >= D - 64) {
                    float *rf = reinterpret_cast<float *>(stage + h * rb);
#pragma unroll
                    for (int e = 0; e < kE; ++e) rf[(d - (D - 64)) + e] = y[e];
                } else if constexpr (kE == 8) {
                    uint4 o;
                    o.x = pack_f16x2(y[0], y[1]);
                    o.y = pack_f16x2(y[2], y[3]);
                    o.z = pack_f16x2(y[4], y[5]);
                    o.w = pack_f16x2(y[6], y[7]);
                    *reinterpret_cast<uint4 *>(smem + C::kOffQ + sw128_off(h, d >> 3, C::kQKB)) = o;
                } else {
                    uint2 o;
                    o.x = pack_f16x2(y[0], y[1]);
                    o.y = pack_f16x2(y[2], y[3]);
                    *reinterpret_cast<uint2 *>(smem + C::kOffQ + sw128_off(h, d >> 3, C::kQKB) + (d & 7) * 2) = o;
                }
            }
        }
    }
    __syncwarp();   // the fp32 RoPE dims written by some lanes are read by all in build_q_rope
    return true;
}

// After the wait: rotate the RoPE dims by position t and publish Qhat.
template <int D>
__device__ void build_q_rope(const AttendArgs &a, long long t, uint8_t *smem, const uint8_t *stage, int q_bf16,
                             Misc *ms) {
    using C = Cfg<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = D * (q_bf16 ? 2 : 4);
    float c, sn;
    rope_cos_sin(t, a.freq.inv[lane], &c, &sn);
    const int dim = (D - 64) + 2 * lane;
    for (int h = 16 * warp; h < 16 * warp + 16; ++h) {
        float y0 = 0.f, y1 = 0.f;
        if (h < a.H) {
            const float *rf = reinterpret_cast<const float *>(stage + h * rb);
            y0 = rf[2 * lane];
            y1 = rf[2 * lane + 1];
        }
        const float r0 = __fsub_rn(__fmul_rn(y0, c), __fmul_rn(y1, sn));
        const float r1 = __fadd_rn(__fmul_rn(y0, sn), __fmul_rn(y1, c));
        *reinterpret_cast<uint32_t *>(smem + C::kOffQ + sw128_off(h, dim >> 3, C::kQKB) + (dim & 7) * 2) =
            pack_f16x2(r0, r1);
    }
    fence_proxy_async_smem();
    mbar_arrive_warp(&ms->q_ready);
}

// ---------------------------------------------------------------- row resolution (loader)
// Row r of request b's set: stage 1 -> compressed entry index (a load of the
// top-k list for CSA); stage 2 -> location (a load of the block table for
// compressed entries; ring slot or chunk-buffer row for window rows);
// stage 3 -> fp8 scale.  Bad indices and pages set the device error word and
// mask the row.
__device__ __forceinline__ int resolve_s1(const AttendArgs &a, int b, const Req &rq, int r) {
    if (r < rq.n_cmp && a.idx) return __ldg(a.idx + (size_t)b * a.k + r);
    return r;
}
__device__ __forceinline__ uint8_t resolve_s2(const AttendArgs &a, const Req &rq, int r, int e, uint32_t *loc) {
    *loc = 0;
    if (r >= rq.n_rows) return kLocNone;
    if (r < rq.n_cmp) {
        if (e < 0) return kLocNone;
        if (e >= rq.nv) {
            set_dev_err(CSLA_DEVERR_INDEX);
            return kLocNone;
        }
        const int epp = CSLA_PAGE_TOKENS / a.m;
        const int col = e / epp;
        const int pg = col < a.bt_stride ? __ldg(a.block_table + (size_t)rq.slot * a.bt_stride + col) : -1;
        if (pg < 0 || pg >= a.n_pages) {
            set_dev_err(CSLA_DEVERR_PAGE);
            return kLocNone;
        }
        *loc = (uint32_t)pg * (uint32_t)epp + (uint32_t)(e % epp);
        return kLocCache;
    }
    const int w = r - rq.n_cmp;
    const int pos = rq.L - rq.win_len + w;
    if (a.src_rows) {
        const long long i = (long long)rq.wbase + pos;
        if (i < 0 || i >= a.n_src) {
            set_dev_err(CSLA_DEVERR_INDEX);
            return kLocNone;
        }
        *loc = (uint32_t)i;
        return kLocSrc;
    }
    *loc = (uint32_t)rq.slot * (uint32_t)a.n_win + (uint32_t)(pos % a.n_win);
    return kLocRing;
}
__device__ __forceinline__ float resolve_s3(const AttendArgs &a, uint8_t kind, uint32_t loc) {
    if (kind == kLocCache) return __ldg(a.scales + loc);
    if (kind == kLocRing) return __ldg(a.win_scales + loc);
    if (kind == kLocSrc) return __ldg(a.src_scales + loc);
    return 0.f;
}
__device__ __forceinline__ const uint8_t *row_ptr(const AttendArgs &a, uint8_t kind, uint32_t loc, int rb) {
    if (kind == kLocCache) return a.rows + (size_t)loc * rb;
    if (kind == kLocRing) return a.win_rows + (size_t)loc * rb;
    if (kind == kLocSrc) return a.src_rows + (size_t)loc * rb;
    return nullptr;
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

// ---------------------------------------------------------------- loader role
// Loader warp lw owns rows 4*lw .. 4*lw+3 of every tile: it resolves them,
// bulk-copies them from the cache into its slots of the raw buffers (the
// copy engine, no registers and no load/store-unit traffic), converts them
// into X' and re-issues copies into the slots it has just consumed.
struct LoadCtx {
    int b, lw, lane, r_begin, r_end, n_tiles;
};

// Bulk copies of this warp's rows of tile t into raw buffer t % kNR: lanes
// 0-3 add their row's bytes to the warp's barrier of that buffer and start
// the copy; lane 0 then arrives on it.  Masked rows copy nothing.
template <int D>
__device__ __forceinline__ void issue_rows(const AttendArgs &a, const LoadCtx &L, int t, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    uint64_t *bar = &ms->raw_full[L.lw][t % kNR];
    if (L.lane < kRowsPerWarp) {
        const int i = kRowsPerWarp * L.lw + L.lane;
        const uint8_t *p = row_ptr(a, ms->kind[t % kRing][i], ms->loc[t % kRing][i], C::kRB);
        if (p) {
            mbar_expect_tx(bar, (uint32_t)C::kRB);
            bulk_load(smem + C::kOffRaw + (t % kNR) * C::kRawBytes + i * C::kRB, p, (uint32_t)C::kRB, bar);
        }
    }
    __syncwarp();
    if (L.lane == 0) mbar_arrive(bar);
}

// Eight bf16 RoPE values (one 16-byte chunk) -> f16 of x * inv; true if one
// leaves the range the f16 operand takes at this scale.
__device__ __forceinline__ bool rope_chunk(const uint4 v, float inv, uint4 *o) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t out[4];
    float mx = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float y0 = __fmul_rn(bf16_bits_to_f32(w[e] & 0xFFFFu), inv);
        const float y1 = __fmul_rn(bf16_bits_to_f32(w[e] >> 16), inv);
        mx = fmaxf(mx, fmaxf(fabsf(y0), fabsf(y1)));
        out[e] = pack_f16x2(y0, y1);
    }
    *o = make_uint4(out[0], out[1], out[2], out[3]);
    return !(mx <= kRopeMax);
}

// Rows whose RoPE dims exceed the f16 range at 256 * their own scale (or
// whose scale is beyond kScaleMax): the warp re-reads each such row from its
// raw slot and writes it with the effective scale
// es = max(s, max|x_rope| / (256 * kRopeMax)): fp8 dims e4m3(c) * (s / es) / 256
// and RoPE dims x / (256 es), both rounded to f16; a row with es beyond
// kScaleMax is masked and flagged.  Rare (never for rows of normalised
// vectors); correctness, not speed, matters here.
template <int D>
__device__ void wide_rows(const LoadCtx &L, int t, uint32_t rows, const uint8_t *raw, uint8_t *xs, Misc *ms,
                          int buf) {
    using C = Cfg<D>;
    const int slot = t % kRing;
    while (rows) {
        const int i4 = __ffs(rows) - 1;
        rows &= rows - 1;
        const int i = kRowsPerWarp * L.lw + i4;
        const uint8_t *p = raw + i * C::kRB;
        const float s = ms->scl[slot][i];
        float mx = 0.f;
        if (L.lane < 8) {
            const uint4 v = *reinterpret_cast<const uint4 *>(p + 16 * (C::kNopeCH + L.lane));
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                mx = fmaxf(mx, fmaxf(fabsf(bf16_bits_to_f32(w[e] & 0xFFFFu)), fabsf(bf16_bits_to_f32(w[e] >> 16))));
        }
        mx = warp_max(mx);
        const float es = fmaxf(s, __fdiv_rn(mx, 256.0f * kRopeMax));
        const bool masked = !(es <= kScaleMax);
        const float ratio = masked ? 0.f : __fdiv_rn(s, es);
        const float inv = masked ? 0.f : __fdiv_rn(1.0f, __fmul_rn(256.0f, es));
        for (int c = L.lane; c < C::kNopeCH + 8; c += 32) {
            const uint4 v = *reinterpret_cast<const uint4 *>(p + 16 * c);
            if (c < C::kNopeCH) {
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
                uint32_t o[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const uint32_t lo = e4m3x2_f16x2_div256<0>(w[e]), hi = e4m3x2_f16x2_div256<2>(w[e]);
                    const __half2 hl = *reinterpret_cast<const __half2 *>(&lo);
                    const __half2 hh = *reinterpret_cast<const __half2 *>(&hi);
                    o[e] = pack_f16x2(__fmul_rn(__low2float(hl), ratio), __fmul_rn(__high2float(hl), ratio));
                    o[4 + e] = pack_f16x2(__fmul_rn(__low2float(hh), ratio), __fmul_rn(__high2float(hh), ratio));
                }
                // o[e] holds dims 4e, 4e+1 of the chunk; o[4+e] dims 4e+2, 4e+3
                *reinterpret_cast<uint4 *>(xs + sw128_off(i, 2 * c, C::kKBBytes)) = make_uint4(o[0], o[4], o[1], o[5]);
                *reinterpret_cast<uint4 *>(xs + sw128_off(i, 2 * c + 1, C::kKBBytes)) =
                    make_uint4(o[2], o[6], o[3], o[7]);
            } else {
                uint4 o;
                rope_chunk(v, inv, &o);
                *reinterpret_cast<uint4 *>(xs + sw128_off(i, (D - 64) / 8 + (c - C::kNopeCH), C::kKBBytes)) = o;
            }
        }
        if (L.lane == 0) {
            ms->tscale[buf][i] = masked ? 0.f : __fmul_rn(256.0f, es);
            if (masked) set_dev_err(CSLA_DEVERR_RANGE);
        }
        __syncwarp();
    }
}

// Convert this warp's rows of tile t from its raw slots into X'[buf];
// returns the rows (bit i4 = row 4*lw + i4) that need the wide-range path
// (warp-uniform).  Masked rows (nothing was copied) become zeros.
template <int D>
__device__ __forceinline__ uint32_t convert_rows(const LoadCtx &L, int t, const uint8_t *raw, uint8_t *xs, Misc *ms,
                                                 int buf) {
    using C = Cfg<D>;
    const int slot = t % kRing;
    constexpr int kNope = kRowsPerWarp * C::kNopeCH;   // this warp's fp8 chunks per tile
    // every shared-memory read first (the row kinds of this warp's 4 rows in
    // one word, then all raw chunks), so that the loads overlap instead of
    // each waiting behind the previous chunk's stores
    static_assert(kRowsPerWarp == 4, "one 32-bit word of row kinds per warp");
    const uint32_t kinds = *reinterpret_cast<const uint32_t *>(&ms->kind[slot][kRowsPerWarp * L.lw]);
    uint4 v[C::kNopeIt];
#pragma unroll
    for (int k = 0; k < C::kNopeIt; ++k) {
        const int f = L.lane + 32 * k;
        const int r = f / C::kNopeCH, c = f % C::kNopeCH;
        const bool live = (kNope % 32 == 0 || f < kNope) && ((kinds >> (8 * (r & 3))) & 0xFFu) != kLocNone;
        v[k] = live ? *reinterpret_cast<const uint4 *>(raw + (kRowsPerWarp * L.lw + r) * C::kRB + 16 * c)
                    : make_uint4(0u, 0u, 0u, 0u);
    }
    const int i4 = L.lane >> 3, cr = L.lane & 7;
    const int ir = kRowsPerWarp * L.lw + i4;
    const float s = ms->scl[slot][ir];
    const uint4 vr = ((kinds >> (8 * i4)) & 0xFFu) != kLocNone
                         ? *reinterpret_cast<const uint4 *>(raw + ir * C::kRB + 16 * (C::kNopeCH + cr))
                         : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int k = 0; k < C::kNopeIt; ++k) {
        const int f = L.lane + 32 * k;
        if (kNope % 32 == 0 || f < kNope) {
            const int i = kRowsPerWarp * L.lw + f / C::kNopeCH, c = f % C::kNopeCH;
            uint4 lo, hi;
            lo.x = e4m3x2_f16x2_div256<0>(v[k].x);
            lo.y = e4m3x2_f16x2_div256<2>(v[k].x);
            lo.z = e4m3x2_f16x2_div256<0>(v[k].y);
            lo.w = e4m3x2_f16x2_div256<2>(v[k].y);
            hi.x = e4m3x2_f16x2_div256<0>(v[k].z);
            hi.y = e4m3x2_f16x2_div256<2>(v[k].z);
            hi.z = e4m3x2_f16x2_div256<0>(v[k].w);
            hi.w = e4m3x2_f16x2_div256<2>(v[k].w);
            *reinterpret_cast<uint4 *>(xs + sw128_off(i, 2 * c, C::kKBBytes)) = lo;
            *reinterpret_cast<uint4 *>(xs + sw128_off(i, 2 * c + 1, C::kKBBytes)) = hi;
        }
    }
    uint32_t wide = 0;
    {
        // 1 / (256 s), correctly rounded (the same value as a division)
        const float inv = s > 0.f ? __frcp_rn(__fmul_rn(256.0f, s)) : 0.f;
        uint4 o;
        if (rope_chunk(vr, inv, &o) || s > kScaleMax) wide = 1u << i4;
        *reinterpret_cast<uint4 *>(xs + sw128_off(ir, (D - 64) / 8 + cr, C::kKBBytes)) = o;
    }
    if (L.lane < kRowsPerWarp) {
        const int i = kRowsPerWarp * L.lw + L.lane;
        ms->tscale[buf][i] = __fmul_rn(256.0f, ms->scl[slot][i]);
    }
    // OR of every lane's rows
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) wide |= __shfl_xor_sync(0xffffffffu, wide, o);
    return wide;
}

// One resolution step for three future tiles on three lane groups: lanes
// 0-3 stage 3 of tile t3, lanes 4-7 stage 2 of tile t3+1, lanes 8-11 stage
// 1 of tile t3+2.  Loads are issued now; results are stored by
// resolve_store at the start of the next step, so their latency overlaps a
// whole step (each stage reads what the previous step stored).
struct ResolveRegs {
    int e;
    uint32_t loc;
    uint8_t kind;
    float s;
};
__device__ __forceinline__ ResolveRegs resolve_issue(const AttendArgs &a, const Req &rq, const LoadCtx &L, int t3,
                                                     const Misc *ms) {
    ResolveRegs x{0, 0u, kLocNone, 0.f};
    const int grp = L.lane / kRowsPerWarp, i = kRowsPerWarp * L.lw + L.lane % kRowsPerWarp;
    const int t = t3 + grp;
    if (grp > 2 || t >= L.n_tiles) return x;
    const int r = L.r_begin + t * kTile + i;
    const int slot = t % kRing;
    if (grp == 0) {
        x.kind = ms->kind[slot][i];
        x.loc = ms->loc[slot][i];
        x.s = resolve_s3(a, x.kind, x.loc);
    } else if (grp == 1) {
        x.kind = r < L.r_end ? resolve_s2(a, rq, r, ms->ent[slot][i], &x.loc) : kLocNone;
    } else {
        x.e = r < L.r_end ? resolve_s1(a, L.b, rq, r) : 0;
    }
    return x;
}
__device__ __forceinline__ void resolve_store(const LoadCtx &L, int t3, const ResolveRegs &x, Misc *ms) {
    const int grp = L.lane / kRowsPerWarp, i = kRowsPerWarp * L.lw + L.lane % kRowsPerWarp;
    const int t = t3 + grp;
    if (grp > 2 || t >= L.n_tiles) return;
    const int slot = t % kRing;
    if (grp == 0) {
        ms->scl[slot][i] = x.s;
    } else if (grp == 1) {
        ms->kind[slot][i] = x.kind;
        ms->loc[slot][i] = x.loc;
    } else {
        ms->ent[slot][i] = x.e;
    }
}

// Tile t: store the previous step's resolution results and issue this
// step's; wait for this warp's rows of tile t and for X'[t & 1]; convert
// them and hand X' over; then copy tile t + kNR into the slots just read.
// *landed is the last tile whose copies this warp has seen land, *issued the
// last tile whose copies it has started.
template <int D>
__device__ __forceinline__ bool loader_step(const AttendArgs &a, const Req &rq, const LoadCtx &L, int t,
                                            uint8_t *smem, Misc *ms, ResolveRegs &rr, int *landed, int *issued) {
    using C = Cfg<D>;
    if (t > 0) {
        resolve_store(L, t - 1 + kAhead, rr, ms);
        __syncwarp();
    }
    rr = resolve_issue(a, rq, L, t + kAhead, ms);
    const int buf = xbuf(t);
    if (!warp_all(mbar_wait(&ms->raw_full[L.lw][t % kNR], (t / kNR) & 1, &ms->abort))) return false;
    *landed = t;
    if (t >= kNX && !warp_all(mbar_wait(&ms->x_empty[buf], ((t - kNX) / kNX) & 1, &ms->abort))) return false;
    const uint8_t *raw = smem + C::kOffRaw + (t % kNR) * C::kRawBytes;
    uint8_t *xs = smem + C::kOffX + buf * C::kXBytes;
    const uint32_t wide = convert_rows<D>(L, t, raw, xs, ms, buf);
    if (wide) wide_rows<D>(L, t, wide, raw, xs, ms, buf);   // warp-uniform
    // X' to the tensor cores; the raw slots just read to the copy engine
    fence_proxy_async_smem();
    mbar_arrive_warp(&ms->x_full[buf]);
    if (L.lw == 0 && L.lane == 0 && t < 2) CSLA_TL_MARK_ANY(t == 0 ? 1 : 5);
    if (t + kNR < L.n_tiles) {
        issue_rows<D>(a, L, t + kNR, smem, ms);
        *issued = t + kNR;
    }
    return true;
}

// q_in_raw: q is staged into the raw buffers too (copies wait for Qhat);
// q_in_two: q fits in X'[0] and X'[1], so tile 0 (X'[kNX-1]) may be
// converted before Qhat is built.
template <int D>
__device__ void loader_role(const AttendArgs &a, int b, const Req &rq, Span sp, uint8_t *smem, Misc *ms,
                            bool q_in_raw, bool q_in_two) {
    LoadCtx L;
    L.b = b;
    L.lw = (threadIdx.x >> 5) - kSoftWarps;
    L.lane = threadIdx.x & 31;
    L.r_begin = sp.c0 * rq.chunk;
    L.r_end = min(rq.n_rows, sp.c1 * rq.chunk);
    L.n_tiles = (L.r_end - L.r_begin + kTile - 1) / kTile;
    if (L.n_tiles <= 0) return;
    // Prologue: tiles 0..kAhead-1 fully resolved (lane l: row l % 4 of tile
    // l / 4, one independent chain each), and in the same round tile kAhead
    // through stage 2 (lanes 0-3) and tile kAhead+1 through stage 1 (lanes 4-7).
    {
        const int i = kRowsPerWarp * L.lw + L.lane % kRowsPerWarp, j = L.lane / kRowsPerWarp;
        const int r = L.r_begin + j * kTile + i;
        int e = 0;
        uint32_t loc = 0;
        uint8_t kind = kLocNone;
        if (j < L.n_tiles && r < L.r_end) {
            e = resolve_s1(a, b, rq, r);
            kind = resolve_s2(a, rq, r, e, &loc);
        }
        const float s = resolve_s3(a, kind, loc);
        const int tp = kAhead + j, rp = L.r_begin + tp * kTile + i;
        int ep = 0;
        uint32_t locp = 0;
        uint8_t kindp = kLocNone;
        if (j < 2 && tp < L.n_tiles && rp < L.r_end) {
            ep = resolve_s1(a, b, rq, rp);
            if (j == 0) kindp = resolve_s2(a, rq, rp, ep, &locp);
        }
        if (j < L.n_tiles) {
            ms->kind[j % kRing][i] = kind;
            ms->loc[j % kRing][i] = loc;
            ms->scl[j % kRing][i] = s;
        }
        if (j < 2 && tp < L.n_tiles) {
            ms->ent[tp % kRing][i] = ep;
            if (j == 0) {
                ms->kind[tp % kRing][i] = kindp;
                ms->loc[tp % kRing][i] = locp;
            }
        }
        __syncwarp();
    }
    // q may be staged in the raw buffers (f32 q): copy rows only once Qhat is built
    if (q_in_raw && !warp_all(mbar_wait(&ms->q_ready, 0, &ms->abort))) return;
    int landed = -1, issued = -1;
    for (int t = 0; t < kNR && t < L.n_tiles; ++t) {
        issue_rows<D>(a, L, t, smem, ms);
        issued = t;
    }
    // q is staged in the X' buffers: convert into them only once Qhat is built
    ResolveRegs rr;
    int t = 0;
    bool ok = true;
    // (with few tiles the conversion would only slow the Qhat build, which
    // is then on the critical path)
    if (q_in_two && !q_in_raw && L.n_tiles >= 4) ok = loader_step<D>(a, rq, L, t++, smem, ms, rr, &landed, &issued);
    if (ok && warp_all(mbar_wait(&ms->q_ready, 0, &ms->abort))) {
        for (; t < L.n_tiles; ++t)
            if (!loader_step<D>(a, rq, L, t, smem, ms, rr, &landed, &issued)) break;
    }
    // copies this warp started but has not seen land (only after an abort)
    // must land before the CTA exits (each tile's phase has had its arrival)
    for (int t = landed + 1; t <= issued; ++t) mbar_wait(&ms->raw_full[L.lw][t % kNR], (t / kNR) & 1, nullptr);
}

// ---------------------------------------------------------------- MMA role
template <int D>
__device__ void mma_role(const Req &rq, Span sp, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    constexpr uint32_t kIdescS = idesc_f16(64, kTile, false, false);
    constexpr uint32_t kIdescO = idesc_f16(128, 64, true, false);
    const uint32_t tmem = ms->tmem;
    const uint32_t q0 = smem_u32(smem + C::kOffQ);
    const uint32_t p0 = smem_u32(smem + C::kOffP);
    const int r_begin = sp.c0 * rq.chunk;
    const int r_end = min(rq.n_rows, sp.c1 * rq.chunk);
    const int n_tiles = (r_end - r_begin + kTile - 1) / kTile;
    const int tpc = rq.chunk / kTile;   // tiles per chunk (chunks are whole tiles)
    if (!mbar_wait(&ms->q_ready, 0, &ms->abort)) return;
    CSLA_TL_MARK_ANY(0);
    for (int g = 0; g <= n_tiles; ++g) {
        if (g < n_tiles) {
            // S[g & 1] = Qhat . X'[g & 1]^T
            const int sb = g & 1, xg = xbuf(g);
            if (!mbar_wait(&ms->x_full[xg], (g / kNX) & 1, &ms->abort)) return;
            if (g >= 2 && !mbar_wait(&ms->s_free[sb], ((g - 2) >> 1) & 1, &ms->abort)) return;
            tc_fence_after();
            const uint32_t x0 = smem_u32(smem + C::kOffX + xg * C::kXBytes);
#pragma unroll 1
            for (int kb = 0; kb < C::kKB; ++kb)
#pragma unroll
                for (int ks = 0; ks < 4; ++ks)
                    umma_kind_f16(tmem + C::kColS + kTile * sb, sdesc(q0 + kb * C::kQKB + ks * 32, 16, 1024),
                                  sdesc(x0 + kb * C::kKBBytes + ks * 32, 16, 1024), kIdescS, (kb | ks) ? 1u : 0u);
            umma_commit(&ms->s_full[sb]);
            if (g == 0) CSLA_TL_MARK_ANY(4);
        }
        if (g >= 1) {
            // O^T += X'[h & 1]^T . P^T for tile h = g - 1
            const int h = g - 1, xb = xbuf(h);
            const int ti = h % tpc, c = h / tpc;
            if (!mbar_wait(&ms->p_full, h & 1, &ms->abort)) return;
            if (ti == 0 && c > 0 && !mbar_wait(&ms->o_free, (c - 1) & 1, &ms->abort)) return;
            tc_fence_after();
            const uint32_t x0 = smem_u32(smem + C::kOffX + xb * C::kXBytes);
#pragma unroll
            for (int mb = 0; mb < C::kMB; ++mb)
#pragma unroll
                for (int ks = 0; ks < kTile / 16; ++ks)
                    umma_kind_f16(tmem + C::kColO + 64 * mb,
                                  sdesc(x0 + 2 * mb * C::kKBBytes + 2 * ks * 1024, C::kKBBytes, 1024),
                                  sdesc(p0 + ks * 32, 16, 1024), kIdescO, (ti > 0 || ks > 0) ? 1u : 0u);
            umma_commit(&ms->x_empty[xb]);
            umma_commit(&ms->pv_done);
            if (g == n_tiles) CSLA_TL_MARK_ANY(7);
        }
    }
}

// ---------------------------------------------------------------- softmax role
template <int D>
__device__ void softmax_role(const AttendArgs &a, int b, const Req &rq, Span sp, uint8_t *smem, Misc *ms) {
    using C = Cfg<D>;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lane_base = (uint32_t)(32 * warp) << 16;
    // The M = 64 TMEM layout puts head 16w + l in lane l < 16 of warp w; lane
    // l + 16 takes the second half of that head's columns of each tile
    // (handed over by shuffles), so all 32 lanes share the exponentials.
    const int h = 16 * warp + (lane & 15);
    const int half = lane >> 4;
    const bool head_thread = lane < 16;
    const float cscale = kLog2e / sqrtf((float)D);
    const uint32_t tmem = ms->tmem;
    uint8_t *pp = smem + C::kOffP;

    int g = 0, nfac = 0;
    for (int c = sp.c0; c < sp.c1; ++c) {
        const int lo = c * rq.chunk;
        const int hi = min(rq.n_rows, lo + rq.chunk);
        float m_run = -INFINITY, l_run = 0.f;
        for (int r0 = lo, ti = 0; r0 < hi; r0 += kTile, ++ti, ++g) {
            const int sb = g & 1, xg = xbuf(g);
            if (!warp_all(mbar_wait(&ms->x_full[xg], (g / kNX) & 1, &ms->abort))) return;
            if (!warp_all(mbar_wait(&ms->s_full[sb], (g >> 1) & 1, &ms->abort))) return;
            tc_fence_after();
            const float4 *ts4 = reinterpret_cast<const float4 *>(ms->tscale[xg]);
            float s[kTile];
            float mt = -INFINITY;
            {
                static_assert(kTile == 32, "one 32-column TMEM load per tile");
                uint32_t rv[32];
                tmem_ld32x32(tmem + lane_base + C::kColS + kTile * sb, rv);
                tmem_wait_ld();
#pragma unroll
                for (int j4 = 0; j4 < kTile / 4; ++j4) {
                    const float4 t4 = ts4[j4];
                    const float tv[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int j = 4 * j4 + e;
                        const float v = __uint_as_float(rv[j]);
                        s[j] = tv[e] > 0.f ? __fmul_rn(__fmul_rn(v, tv[e]), cscale) : -INFINITY;
                        mt = fmaxf(mt, s[j]);
                    }
                }
            }
            // lanes 16..31: columns 16..31 of head h (and its tile maximum) from lane l - 16
#pragma unroll
            for (int j = 0; j < kTile / 2; ++j) {
                const float t = __shfl_up_sync(0xffffffffu, s[kTile / 2 + j], 16);
                if (half) s[j] = t;
            }
            mt = __shfl_sync(0xffffffffu, mt, lane & 15);
            tc_fence_before();
            mbar_arrive_warp(&ms->s_free[sb]);   // S[sb] may be overwritten by tile g + 2
            // PV of the previous tile must be done before P and O^T are touched.
            if (g > 0 && !warp_all(mbar_wait(&ms->pv_done, (g - 1) & 1, &ms->abort))) return;
            tc_fence_after();
            float f = 1.f;
            {
                // both lanes of head h take the same decisions (same mt, m_run, l_run)
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
                for (int c8l = 0; c8l < kTile / 16; ++c8l) {
                    const int c8 = 2 * half + c8l;   // this lane's 8-column groups
                    const float4 ta = ts4[2 * c8], tb = ts4[2 * c8 + 1];
                    const float tv[8] = {ta.x, ta.y, ta.z, ta.w, tb.x, tb.y, tb.z, tb.w};
                    float p[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        p[e] = exp2f(__fsub_rn(s[c8l * 8 + e], muse));
                        lsum = __fadd_rn(lsum, p[e]);
                    }
                    uint4 u;
                    u.x = pack_f16x2(__fmul_rn(p[0], tv[0]), __fmul_rn(p[1], tv[1]));
                    u.y = pack_f16x2(__fmul_rn(p[2], tv[2]), __fmul_rn(p[3], tv[3]));
                    u.z = pack_f16x2(__fmul_rn(p[4], tv[4]), __fmul_rn(p[5], tv[5]));
                    u.w = pack_f16x2(__fmul_rn(p[6], tv[6]), __fmul_rn(p[7], tv[7]));
                    const uint32_t off = (uint32_t)((h >> 3) * 1024 + (h & 7) * 128 + ((c8 ^ (h & 7)) << 4));
                    *reinterpret_cast<uint4 *>(pp + off) = u;
                }
                // the tile's sum: columns 0..15 plus columns 16..31 (the same on both lanes)
                lsum = __fadd_rn(lsum, __shfl_xor_sync(0xffffffffu, lsum, 16));
                l_run = (ti == 0) ? lsum : __fadd_rn(__fmul_rn(l_run, f), lsum);
                m_run = mnew;
                if (head_thread) ms->fac[g & 1][h] = f;
            }
            // every head's factor is needed by every thread (each owns one O^T
            // row); a chunk's first tile has none (every factor is 1)
            bool any_rescale = false;
            if (ti > 0) {
                mbar_arrive_warp(&ms->fac_ready);
                if (!warp_all(mbar_wait(&ms->fac_ready, nfac & 1, &ms->abort))) return;
                ++nfac;
                const float4 *f4 = reinterpret_cast<const float4 *>(ms->fac[g & 1]);
#pragma unroll
                for (int j = 0; j < kHP / 4; ++j) {
                    const float4 v = f4[j];
                    any_rescale |= (v.x != 1.f) | (v.y != 1.f) | (v.z != 1.f) | (v.w != 1.f);
                }
            }
            if (any_rescale) {
                // O^T columns are heads: every thread scales its own dim lane,
                // 16 columns (heads) at a time
#pragma unroll 1
                for (int it = 0; it < 4 * C::kMB; ++it) {
                    const int blk = it >> 2, q4 = it & 3;
                    uint32_t v[16];
                    const uint32_t addr = tmem + lane_base + C::kColO + 64 * blk + 16 * q4;
                    tmem_ld32x16(addr, v);
                    tmem_wait_ld();
                    const float4 *f4 = reinterpret_cast<const float4 *>(&ms->fac[g & 1][16 * q4]);
#pragma unroll
                    for (int j4 = 0; j4 < 4; ++j4) {
                        const float4 fv = f4[j4];
                        v[4 * j4] = __float_as_uint(__fmul_rn(__uint_as_float(v[4 * j4]), fv.x));
                        v[4 * j4 + 1] = __float_as_uint(__fmul_rn(__uint_as_float(v[4 * j4 + 1]), fv.y));
                        v[4 * j4 + 2] = __float_as_uint(__fmul_rn(__uint_as_float(v[4 * j4 + 2]), fv.z));
                        v[4 * j4 + 3] = __float_as_uint(__fmul_rn(__uint_as_float(v[4 * j4 + 3]), fv.w));
                    }
                    tmem_st32x16(addr, v);
                }
                tmem_wait_st();
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive_warp(&ms->p_full);
            if (threadIdx.x == 0 && g < 2) CSLA_TL_MARK_ANY(g == 0 ? 2 : 6);
        }
        // chunk done: drain its last PV and read O^T out as the partial
        if (!warp_all(mbar_wait(&ms->pv_done, (g - 1) & 1, &ms->abort))) return;
        tc_fence_after();
        float *part = partial_ptr(a, b, c, D);
        float *ml = part + (size_t)a.H * D;
#pragma unroll 1
        for (int blk = 0; blk < C::kMB; ++blk) {
            const int dim = 128 * blk + 32 * warp + lane;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t v[32];
                tmem_ld32x32(tmem + lane_base + C::kColO + 64 * blk + 32 * half, v);
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < 32; ++j) {
                    const int hh = 32 * half + j;
                    if (hh < a.H) part[(size_t)hh * D + dim] = __uint_as_float(v[j]);
                }
            }
        }
        if (head_thread && h < a.H) {
            ml[h] = m_run;
            ml[a.H + h] = l_run;
        }
        tc_fence_before();
        mbar_arrive_warp(&ms->o_free);
        if (threadIdx.x == 0 && c == sp.c0) CSLA_TL_MARK_ANY(3);
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
    // q of request b is staged from X'[0] on: in the X' buffers (bf16 q of
    // up to 64 heads fills two of them), reaching into the raw buffers for
    // f32 q
    const uint32_t q_bytes = (uint32_t)(a.H * D * (q_bf16 ? 2 : 4));
    uint8_t *stage = smem + C::kOffX;
    const bool q_in_raw = q_bytes > (uint32_t)(kNX * C::kXBytes);

    // ---- before the wait: barriers, TMEM, the q copy
    if (threadIdx.x == 0) {
        mbar_init(&ms->q_staged, 1);
        mbar_init(&ms->q_ready, kSoftWarps);
        for (int i = 0; i < kNX; ++i) {
            mbar_init(&ms->x_full[i], kLoadWarps);
            mbar_init(&ms->x_empty[i], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ms->s_full[i], 1);
            mbar_init(&ms->s_free[i], kSoftWarps);
        }
        mbar_init(&ms->p_full, kSoftWarps);
        mbar_init(&ms->pv_done, 1);
        mbar_init(&ms->o_free, kSoftWarps);
        mbar_init(&ms->fac_ready, kSoftWarps);
        mbar_init(&ms->drain, 1);
        for (int w = 0; w < kLoadWarps; ++w)
            for (int i = 0; i < kNR; ++i) mbar_init(&ms->raw_full[w][i], 1);
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
    if (threadIdx.x == 32 * kMmaWarp) {
        const uint8_t *src = reinterpret_cast<const uint8_t *>(a.q) + (size_t)b * q_bytes;
        mbar_arrive_expect_tx(&ms->q_staged, q_bytes);
        bulk_load(stage, src, q_bytes, &ms->q_staged);
    }
    bool q_ok = true;
    if (warp < kSoftWarps) {
        q_ok = build_q_normed<D>(a, smem, stage, q_bf16, ms);
    }
    pdl_wait();
    CSLA_TL_WAITED();

    const Req rq = request(a, b);
    if (!rq.ok && threadIdx.x == 0 && (kSaturated || blockIdx.x == 0)) set_dev_err(CSLA_DEVERR_LEN);
    const bool run = rq.ok && (kSaturated || (int)blockIdx.x < rq.n_chunks);
    const Span sp = kSaturated ? Span{0, rq.n_chunks} : Span{(int)blockIdx.x, (int)blockIdx.x + 1};
    if (!run) {
        // nothing to do: fall through to the teardown
    } else if (warp < kSoftWarps) {
        if (q_ok) {
            build_q_rope<D>(a, (long long)rq.L - 1, smem, stage, q_bf16, ms);
            softmax_role<D>(a, b, rq, sp, smem, ms);
        }
    } else if (warp < kSoftWarps + kLoadWarps) {
        loader_role<D>(a, b, rq, sp, smem, ms, q_in_raw, q_bytes <= (uint32_t)(2 * C::kXBytes));
    } else if ((threadIdx.x & 31) == 0) {
        mma_role<D>(rq, sp, smem, ms);
    }
    if (threadIdx.x == 32 * kMmaWarp) {
        // the q copy has landed (it is waited for even when nothing ran), and
        // every MMA this thread issued has completed, before the CTA tears down
        mbar_wait(&ms->q_staged, 0, nullptr);
        umma_commit(&ms->drain);
        mbar_wait(&ms->drain, 0, nullptr);
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
        // into the X' area the loader no longer uses.
        float *wall = reinterpret_cast<float *>(smem + C::kOffX);   // [H][33]: w_0..w_31, l
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
