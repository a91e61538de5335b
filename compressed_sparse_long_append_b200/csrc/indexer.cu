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
//  2. indexer: persistent, warp-specialised tcgen05 kernel.  A tile is 128
//     compressed entries of one request (4 pages of 32 entries).  Warp 0
//     streams key tiles and the request's query operand with TMA into a
//     4-stage ring; warp 1 issues UMMA (M=128 entries, N=NQ query rows,
//     K=dI) into one of two TMEM accumulators; warps 2-5 read the
//     accumulator (one entry per thread) and reduce
//       score = sum_j w_j * relu((acc[j] + acc[HI + j]) + acc[2HI + j])
//     in head order.  Every score depends only on its own entry and request.
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

template <typename TC, typename TW>
__global__ void __launch_bounds__(kProjThreads) iq_project_kernel(IndexerArgs a) {
    const int r = blockIdx.x * (kProjThreads / 32) + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (r >= a.HI * a.dI) return;
    const int j = r / a.dI, e = r % a.dI;
    const TW *w = reinterpret_cast<const TW *>(a.W) + (size_t)r * a.dc;
    const int nch = a.dc / 8;
    for (int b = 0; b < a.B; ++b) {
        const TC *c = reinterpret_cast<const TC *>(a.cq) + (size_t)b * a.dc;
        float acc = 0.f;
        for (int ch = lane; ch < nch; ch += 32) {
            float wv[8], cv[8];
            load8<TW>(w + ch * 8, wv);
            load8<TC>(c + ch * 8, cv);
#pragma unroll
            for (int i = 0; i < 8; ++i) acc = fmaf(wv[i], cv[i], acc);
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

constexpr int kStages = 4;
constexpr int kTileE = 128;          // entries per tile
constexpr int kPageE = 32;           // CSA entries per 128-token page
constexpr int kIdxThreads = 192;     // warp 0: TMA, warp 1: MMA, warps 2..5: epilogue

template <int DI, int NQ>
struct IdxSmem {
    static constexpr int kKeyBytes = kTileE * DI * 2;
    static constexpr int kQBytes = NQ * DI * 2;
    static constexpr int kStageBytes = kKeyBytes + kQBytes;
    static constexpr int kBytes = kStages * kStageBytes + 1024 /*align*/ + 256 /*barriers*/;
};

// Two accumulators of NQ columns, rounded up to a power of two >= 32.
template <int NQ>
constexpr uint32_t kTmemCols() {
    return 2 * NQ <= 32 ? 32 : (2 * NQ <= 64 ? 64 : 128);
}

// Tile bookkeeping shared by the three roles (all must skip the same tiles).
struct TileInfo {
    int b, tt, slot, nv;
    bool live;
};
__device__ __forceinline__ TileInfo tile_info(const IndexerArgs &a, int tile) {
    TileInfo t;
    t.b = tile / a.tiles_per_req;
    t.tt = tile % a.tiles_per_req;
    t.slot = __ldg(a.slots + t.b);
    const bool slot_ok = t.slot >= 0 && t.slot < a.n_slots;
    const int L = slot_ok ? __ldg(a.len + t.slot) : 0;
    t.nv = (slot_ok && L <= a.max_len) ? L / a.m : 0;
    t.live = t.tt * kTileE < t.nv;
    return t;
}

template <int DI, int NQ, int HI>
__global__ void __launch_bounds__(kIdxThreads, 1)
    indexer_kernel(IndexerArgs a, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap qmap) {
    using S = IdxSmem<DI, NQ>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t *bars = reinterpret_cast<uint64_t *>(base + kStages * S::kStageBytes);
    uint64_t *full = bars, *empty = bars + kStages, *tfull = bars + 2 * kStages, *tempty = tfull + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(tempty + 2);
    __shared__ volatile int abort_flag;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = a.B * a.tiles_per_req;

    if (threadIdx.x == 0) {
        abort_flag = 0;
        for (int s = 0; s < kStages; ++s) {
            mbar_init(full + s, 1);
            mbar_init(empty + s, 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(tfull + i, 1);
            mbar_init(tempty + i, 128);
        }
        fence_mbar_init();
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&qmap);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, kTmemCols<NQ>());
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            int n = 0;
            for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
                const TileInfo t = tile_info(a, tile);
                if (!t.live) continue;
                const int s = n % kStages;
                if (n >= kStages && !mbar_wait(empty + s, ((n / kStages) - 1) & 1, &abort_flag)) break;
                uint8_t *kb = base + s * S::kStageBytes;
                uint8_t *qb = kb + S::kKeyBytes;
                int pages[4];
                int np = 0;
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    const int e0 = t.tt * kTileE + p * kPageE;
                    pages[p] = -1;
                    if (e0 < t.nv) {
                        const int col = e0 / kPageE;
                        const int pg = col < a.bt_stride ? __ldg(a.block_table + (size_t)t.slot * a.bt_stride + col) : -1;
                        if (pg >= 0 && pg < a.n_pages) {
                            pages[p] = pg;
                            ++np;
                        } else {
                            set_dev_err(CSLA_DEVERR_PAGE);
                        }
                    }
                }
                mbar_arrive_expect_tx(full + s, (uint32_t)(S::kQBytes + np * kPageE * DI * 2));
#pragma unroll
                for (int h = 0; h < DI / 64; ++h)
                    tma_load_2d(qb + h * NQ * 128, &qmap, h * 64, t.b * NQ, full + s);
#pragma unroll
                for (int p = 0; p < 4; ++p) {
                    if (pages[p] < 0) continue;
#pragma unroll
                    for (int h = 0; h < DI / 64; ++h)
                        tma_load_2d(kb + h * (kTileE * 128) + p * (kPageE * 128), &kmap, h * 64,
                                    pages[p] * kPageE, full + s);
                }
                ++n;
            }
            // every issued copy must land before the CTA may exit
            for (int i = (n > kStages ? n - kStages : 0); i < n; ++i)
                mbar_wait(full + (i % kStages), (i / kStages) & 1, nullptr);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(128, NQ, false, false);
            int n = 0;
            for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
                const TileInfo t = tile_info(a, tile);
                if (!t.live) continue;
                const int s = n % kStages;
                const int acc = n & 1;
                if (!mbar_wait(full + s, (n / kStages) & 1, &abort_flag)) break;
                if (n >= 2 && !mbar_wait(tempty + acc, ((n / 2) - 1) & 1, &abort_flag)) break;
                tc_fence_after();
                const uint32_t kb = smem_u32(base + s * S::kStageBytes);
                const uint32_t qb = kb + S::kKeyBytes;
#pragma unroll
                for (int k = 0; k < DI / 16; ++k) {
                    const uint32_t half = k / 4, ko = (k % 4) * 32;
                    const uint64_t ad = sdesc(kb + half * (kTileE * 128) + ko, 16, 1024);
                    const uint64_t bd = sdesc(qb + half * (NQ * 128) + ko, 16, 1024);
                    umma_bf16(tmem + acc * NQ, ad, bd, idesc, k > 0 ? 1u : 0u);
                }
                umma_commit(empty + s);
                umma_commit(tfull + acc);
                ++n;
            }
            if (n > 0) mbar_wait(tfull + ((n - 1) & 1), ((n - 1) / 2) & 1, nullptr);
        }
    } else {
        const int lane_base = 32 * (warp & 3);
        const int row = lane_base + lane;
        int n = 0;
        for (int tile = blockIdx.x; tile < total && !abort_flag; tile += gridDim.x) {
            const TileInfo t = tile_info(a, tile);
            if (!t.live) continue;
            const int acc = n & 1;
            if (!mbar_wait(tfull + acc, (n / 2) & 1, &abort_flag)) break;
            tc_fence_after();
            uint32_t r[NQ];
            const uint32_t ta = tmem + ((uint32_t)lane_base << 16) + acc * NQ;
            if constexpr (NQ == 16) {
                tmem_ld32x16(ta, r);
            } else if constexpr (NQ == 32) {
                tmem_ld32x32(ta, r);
            } else {
                static_assert(NQ == 48, "query operand rows");
                uint32_t (&r0)[32] = *reinterpret_cast<uint32_t (*)[32]>(r);
                uint32_t (&r1)[16] = *reinterpret_cast<uint32_t (*)[16]>(r + 32);
                tmem_ld32x32(ta, r0);
                tmem_ld32x16(ta + 32, r1);
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(tempty + acc);
            const int e = t.tt * kTileE + row;
            if (e < t.nv) {
                const float *w = a.head_w + (size_t)t.b * HI;
                float sc = 0.f;
#pragma unroll
                for (int j = 0; j < HI; ++j) {
                    const float dot = __fadd_rn(__fadd_rn(__uint_as_float(r[j]), __uint_as_float(r[HI + j])),
                                                __uint_as_float(r[2 * HI + j]));
                    sc = __fmaf_rn(__ldg(w + j), fmaxf(dot, 0.f), sc);
                }
                a.scores[(size_t)t.b * a.scores_stride + e] = sc;
            }
            ++n;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols<NQ>());
    }
}

template <int DI, int NQ, int HI>
cudaError_t launch_indexer_t(const IndexerArgs &a, const CUtensorMap &kmap, const CUtensorMap &qmap,
                             int num_sms, cudaStream_t stream) {
    using S = IdxSmem<DI, NQ>;
    static int configured_dev = -1;
    int dev = 0;
    cudaGetDevice(&dev);
    if (configured_dev != dev) {
        cudaError_t e = cudaFuncSetAttribute(indexer_kernel<DI, NQ, HI>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::kBytes);
        if (e != cudaSuccess) return e;
        configured_dev = dev;
    }
    const int total = a.B * a.tiles_per_req;
    int grid = total < num_sms ? total : num_sms;
    if (grid < 1) grid = 1;
    indexer_kernel<DI, NQ, HI><<<grid, kIdxThreads, S::kBytes, stream>>>(a, kmap, qmap);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_indexer(const IndexerArgs &a, bool cq_bf16, bool w_bf16, const CUtensorMap &kmap,
                           const CUtensorMap &qmap, int num_sms, cudaStream_t stream) {
    if (a.NQ > 3 * a.HI) {
        cudaError_t e = cudaMemsetAsync(a.q_ws, 0, (size_t)a.B * a.NQ * a.dI * 2, stream);
        if (e != cudaSuccess) return e;
    }
    const int pblocks = (a.HI * a.dI + kProjThreads / 32 - 1) / (kProjThreads / 32);
    if (cq_bf16 && w_bf16) iq_project_kernel<__nv_bfloat16, __nv_bfloat16><<<pblocks, kProjThreads, 0, stream>>>(a);
    else if (cq_bf16) iq_project_kernel<__nv_bfloat16, float><<<pblocks, kProjThreads, 0, stream>>>(a);
    else if (w_bf16) iq_project_kernel<float, __nv_bfloat16><<<pblocks, kProjThreads, 0, stream>>>(a);
    else iq_project_kernel<float, float><<<pblocks, kProjThreads, 0, stream>>>(a);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // HI is a template parameter so the epilogue's head loop is unrolled.
    if (a.dI == 128) {
        switch (a.HI) {
            case 16: return launch_indexer_t<128, 48, 16>(a, kmap, qmap, num_sms, stream);
            case 8: return launch_indexer_t<128, 32, 8>(a, kmap, qmap, num_sms, stream);
            case 4: return launch_indexer_t<128, 16, 4>(a, kmap, qmap, num_sms, stream);
            default: break;
        }
    } else if (a.dI == 64) {
        switch (a.HI) {
            case 16: return launch_indexer_t<64, 48, 16>(a, kmap, qmap, num_sms, stream);
            case 8: return launch_indexer_t<64, 32, 8>(a, kmap, qmap, num_sms, stream);
            case 4: return launch_indexer_t<64, 16, 4>(a, kmap, qmap, num_sms, stream);
            default: break;
        }
    }
    return cudaErrorInvalidValue;
}

}  // namespace csla
