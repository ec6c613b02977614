// hif4_noalloc.cu — a calibration entry point for callers that cannot
// allocate device memory.
//
// hif4_calib_percentile_mask needs a scratch workspace (per-channel
// histograms) that the caller normally allocates.  Some callers cannot do
// that: a serving runtime that hands all device memory to its own pool at
// start-up and forbids cudaMalloc afterwards, a plugin host that does not
// allow allocation inside its enqueue callback, or code that must not call
// the allocator while other work is being recorded.  For them this file keeps
// the scratch in a fixed, file-scope device array and forwards to the normal
// entry point with that array as the workspace.
#include <mutex>

#include "hif4_internal.cuh"

namespace {

// 16 MiB per device, resident in every GPU that loads the library until the
// process exits.
constexpr size_t kScratchBytes = 16u << 20;
static __device__ __align__(256) uint8_t g_calib_scratch[kScratchBytes];

std::mutex g_mu;
void *g_scratch_ptr[64] = {nullptr};

// Device address of g_calib_scratch on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up
// once per device (with that device current) and cached for the life of the
// process; a device reset (a new primary context) would leave the cached
// address stale, which the header tells callers.
hif4_status scratch_for_current_device(void **out)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HIF4_ERR_CUDA;
    if (dev < 0 || dev >= 64) return HIF4_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_calib_scratch) != cudaSuccess || !p) return HIF4_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return HIF4_OK;
}

} // namespace

extern "C" size_t hif4_calib_noalloc_scratch_bytes(void) { return kScratchBytes; }

extern "C" hif4_status hif4_calib_percentile_mask_noalloc(const void *acts, int64_t tokens, int64_t channels,
                                                          int64_t lda, uint32_t q_num, uint32_t q_den,
                                                          uint32_t mask_num, uint32_t mask_den, void *pct,
                                                          float *ratio, uint8_t *mask, int32_t *mask_idx_out,
                                                          hif4_stream_t stream)
{
    if (tokens <= 0 || channels <= 0) return HIF4_ERR_INVALID_ARG;
    if (hif4_calib_workspace(tokens, channels) > kScratchBytes) return HIF4_ERR_WORKSPACE;
    void *scratch = nullptr;
    hif4_status st = scratch_for_current_device(&scratch);
    if (st != HIF4_OK) return st;
    return hif4_calib_percentile_mask(acts, tokens, channels, lda, q_num, q_den, mask_num, mask_den, pct, ratio,
                                      mask, mask_idx_out, scratch, kScratchBytes, stream);
}
