// indexer_noalloc.cu -- csla_indexer_scores_noalloc: the lightning indexer
// for callers that cannot allocate device memory.
//
// Who needs it: code that runs where cudaMalloc is off limits -- inside a
// host callback or a custom allocator hook, in a process whose memory pool
// is owned and fully reserved by a framework, or in an embedding that may
// only touch memory it was handed.  Such a caller can still pass its inputs
// and outputs, but has nowhere to put the indexer's scratch (the bf16
// query operand, 3*HI rows x dI per request).
//
// Here that scratch lives in one fixed array inside the library image.  Every
// GPU that loads libcsla holds these bytes until the process exits.  All
// calls share the array, so two calls that overlap on the GPU (different
// streams without ordering between them) race on it; calls on one stream, or
// otherwise ordered, are safe.  The array keeps whatever the last call wrote;
// the padding rows of the operand, which must read as zero, are cleared on
// every call.
#include <atomic>

#include "../../include/csla.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// 64 requests x 48 operand rows x 128 dims x 2 bytes.
constexpr size_t kScratchBytes = (size_t)CSLA_NOALLOC_INDEXER_SCRATCH_BYTES;
static __device__ __align__(256) uint8_t g_indexer_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
// Per-device cache of the array's address.  Host threads may make their first
// call on a device at the same time: each looks the address up and stores the
// same value, so relaxed atomics suffice.  The cache is never refreshed, so it
// would be stale after a cudaDeviceReset of that device.
std::atomic<void *> g_scratch_ptr[kMaxDevices];

// Device address of the array on the current device, looked up once per
// device.  Returns null if the lookup fails.
void *scratch_address(int *status) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        *status = CSLA_ERR_CUDA;
        return nullptr;
    }
    void *p = g_scratch_ptr[dev].load(std::memory_order_relaxed);
    if (!p) {
        if (cudaGetSymbolAddress(&p, g_indexer_scratch) != cudaSuccess || p == nullptr) {
            *status = CSLA_ERR_CUDA;
            return nullptr;
        }
        g_scratch_ptr[dev].store(p, std::memory_order_relaxed);
    }
    *status = CSLA_OK;
    return p;
}

}  // namespace

extern "C" int csla_indexer_scores_noalloc(const csla_cfg *cfg, const csla_state *st, const csla_cache *cache,
                                           const int32_t *slots, int32_t B, const csla_queries *qs,
                                           int32_t max_len, const void *cq,
                                           int32_t cq_dtype, const void *W_iq, int32_t w_dtype,
                                           const float *head_w, float *scores, int32_t scores_stride,
                                           csla_stream_t stream) {
    if (!cfg || B < 1) return CSLA_ERR_ARG;
    const size_t need = csla_workspace_size(cfg, CSLA_OP_INDEXER, B, max_len > 0 ? max_len : 0);
    if (need == 0) return cfg->m != 4 ? CSLA_ERR_UNSUPPORTED : CSLA_ERR_ARG;
    if (need > kScratchBytes) return CSLA_ERR_ARG;   // batch too large for the fixed scratch
    int status = CSLA_OK;
    void *ws = scratch_address(&status);
    if (!ws) return status;
    return csla_indexer_scores(cfg, st, cache, slots, B, qs, max_len, cq, cq_dtype, W_iq, w_dtype, head_w, scores,
                               scores_stride, ws, kScratchBytes, stream);
}
