// Context-parallel prefill: the two data-movement steps around the
// all-gather of compressed entries (haiqwa "DeepSeek-V4" blog, §百万 token
// 怎么切分到多张卡, global gather and reassembly).  Each rank compresses the
// blocks that close inside its token range into its own copy of the
// request's paged cache; csla_cp_select packs those entries, in block order,
// into a fixed-length run of entry records (zero records pad the run to the
// same length on every rank, so one all-gather of equal-sized buffers moves
// them); csla_cp_place writes every rank's valid records back into the
// paged cache at their global block index, dropping the padding.
//
// One warp moves one record: the entry's row (row_bytes), its index key
// (CSA), its row scale and key scale, as 16-byte vectors.  The record is
//   [row | key | scale f32 | key scale f32 | zero pad to 16 bytes].
#include "common.cuh"
#include "kernels.h"

namespace csla {
namespace {

constexpr int kCpWarps = 8;

__device__ __forceinline__ void copy16(uint8_t *dst, const uint8_t *src, int bytes, int lane) {
    for (int o = 16 * lane; o < bytes; o += 16 * 32)
        *reinterpret_cast<uint4 *>(dst + o) = *reinterpret_cast<const uint4 *>(src + o);
}

__global__ void __launch_bounds__(32 * kCpWarps) cp_move_kernel(CpArgs a) {
    pdl_trigger();
    const int lane = threadIdx.x & 31;
    const long long rec = (long long)blockIdx.x * kCpWarps + (threadIdx.x >> 5);
    if (rec >= (long long)a.R * a.E_max) return;
    const int r = (int)(rec / a.E_max), j = (int)(rec % a.E_max);
    uint8_t *R8 = a.recs + rec * a.rec_bytes;
    pdl_wait();
    if (j >= a.n[r]) {
        // select: padding record; place: nothing to write
        if (!a.place)
            for (int o = 16 * lane; o < a.rec_bytes; o += 16 * 32)
                *reinterpret_cast<uint4 *>(R8 + o) = make_uint4(0u, 0u, 0u, 0u);
        return;
    }
    const long long bk = (long long)a.b_lo[r] + j;
    const long long col = bk / a.epp;
    const int page = col < a.bt_stride ? __ldg(a.block_table + (size_t)a.slot * a.bt_stride + (size_t)col) : -1;
    if (page < 0 || page >= a.n_pages) {
        if (lane == 0) set_dev_err(CSLA_DEVERR_PAGE);
        return;
    }
    const size_t ent = (size_t)page * a.epp + (size_t)(bk % a.epp);
    uint8_t *row = a.rows + ent * a.row_bytes;
    uint8_t *key = a.key_bytes ? a.kidx + ent * a.key_bytes : nullptr;
    float *tail = reinterpret_cast<float *>(R8 + a.row_bytes + a.key_bytes);
    if (a.place) {
        copy16(row, R8, a.row_bytes, lane);
        if (key) copy16(key, R8 + a.row_bytes, a.key_bytes, lane);
        if (lane == 0) {
            a.scales[ent] = tail[0];
            if (a.kscale) a.kscale[ent] = tail[1];
        }
    } else {
        copy16(R8, row, a.row_bytes, lane);
        if (key) copy16(R8 + a.row_bytes, key, a.key_bytes, lane);
        const int used = a.row_bytes + a.key_bytes;
        for (int o = used + 16 * lane; o < a.rec_bytes; o += 16 * 32)
            *reinterpret_cast<uint4 *>(R8 + o) = make_uint4(0u, 0u, 0u, 0u);
        __syncwarp();
        if (lane == 0) {
            tail[0] = a.scales[ent];
            tail[1] = a.kscale ? a.kscale[ent] : 0.f;
        }
    }
}

}  // namespace

cudaError_t launch_cp_move(const CpArgs &a, cudaStream_t stream) {
    const long long recs = (long long)a.R * a.E_max;
    if (recs == 0) return cudaSuccess;
    const unsigned blocks = (unsigned)((recs + kCpWarps - 1) / kCpWarps);
    return launch_pdl(cp_move_kernel, dim3(blocks), dim3(32 * kCpWarps), 0, stream, a);
}

}  // namespace csla
