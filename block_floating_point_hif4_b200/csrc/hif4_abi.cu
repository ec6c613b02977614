// hif4_abi.cu — status handling and per-device caches of libhif4.
#include <atomic>
#include <mutex>

#include <cuda.h>

#include "hif4_internal.cuh"

namespace hif4 {

namespace {
std::mutex g_mu;
constexpr int kMaxDev = 64;
int g_sms[kMaxDev] = {0};
struct OccEntry {
    const void *kernel;
    int dev, threads;
    size_t smem;
    int blocks;
};
OccEntry g_occ[256];
int g_nocc = 0;
} // namespace

namespace {
std::atomic<uint32_t> g_withhold{0};
std::atomic<uint64_t> g_wait_limit{0};
} // namespace

uint32_t wait_test_withhold() { return g_withhold.load(std::memory_order_relaxed); }

uint64_t wait_limit_ns(uint64_t dflt)
{
    const uint64_t v = g_wait_limit.load(std::memory_order_relaxed);
    return v ? v : dflt;
}

int sm_count()
{
    int dev = 0;
    cudaGetDevice(&dev);
    std::lock_guard<std::mutex> lk(g_mu);
    int &v = g_sms[dev & (kMaxDev - 1)];
    if (v == 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1) n = 148;
        v = n;
    }
    return v;
}

namespace {
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
} // namespace

bool make_tensor_map_bf16_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128)
{
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void *p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                g_encode = reinterpret_cast<EncodeTiledFn>(p);
        }
    }
    if (!g_encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 8-bit 2-D tensor map with 128-byte swizzle (the FP8 GEMM's operands).
bool make_tensor_map_u8_2d_sw128(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer)
{
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void *p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                g_encode = reinterpret_cast<EncodeTiledFn>(p);
        }
    }
    if (!g_encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// FP32 2-D tensor map with 128-byte swizzle (the HiGPTQ update's operands).
bool make_tensor_map_f32_2d_sw128(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer)
{
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (!g_encode) {
            void *p = nullptr;
            cudaDriverEntryPointQueryResult q;
            if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
                q == cudaDriverEntryPointSuccess)
                g_encode = reinterpret_cast<EncodeTiledFn>(p);
        }
    }
    if (!g_encode) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
    cuuint64_t strides[1] = {(cuuint64_t)row_stride_bytes};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    return g_encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int blocks_per_sm(const void *kernel, int threads, size_t dyn_smem)
{
    int dev = 0;
    cudaGetDevice(&dev);
    {
        std::lock_guard<std::mutex> lk(g_mu);
        for (int i = 0; i < g_nocc; ++i)
            if (g_occ[i].kernel == kernel && g_occ[i].dev == dev && g_occ[i].threads == threads &&
                g_occ[i].smem == dyn_smem)
                return g_occ[i].blocks;
    }
    int b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, kernel, threads, dyn_smem) != cudaSuccess || b < 1)
        b = 1;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_nocc < 256) g_occ[g_nocc++] = OccEntry{kernel, dev, threads, dyn_smem, b};
    return b;
}

} // namespace hif4

extern "C" hif4_status hif4_get_status(const uint32_t *status_word, hif4_stream_t stream)
{
    if (!status_word) return HIF4_ERR_INVALID_ARG;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint32_t w = 0;
    if (cudaMemcpyAsync(&w, status_word, sizeof w, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return HIF4_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return HIF4_ERR_CUDA;
    if (w & HIF4_FLAG_TIMEOUT) return HIF4_ERR_TIMEOUT;
    if (w & (HIF4_FLAG_BAD_INDEX | HIF4_FLAG_NOT_SPD)) return HIF4_ERR_INVALID_ARG;
    if (w & HIF4_FLAG_NONFINITE) return HIF4_ERR_NONFINITE;
    return HIF4_OK;
}

extern "C" hif4_status hif4_reset_status(uint32_t *status_word, hif4_stream_t stream)
{
    if (!status_word) return HIF4_ERR_INVALID_ARG;
    if (cudaMemsetAsync(status_word, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return HIF4_ERR_CUDA;
    return HIF4_OK;
}

namespace hif4 {
namespace {
thread_local cudaError_t t_last_cuda_error = cudaSuccess;
} // namespace

hif4_status cuda_failed(cudaError_t e)
{
    t_last_cuda_error = e;
    return HIF4_ERR_CUDA;
}
} // namespace hif4

extern "C" const char *hif4_last_cuda_error(void)
{
    return hif4::t_last_cuda_error == cudaSuccess ? "" : cudaGetErrorName(hif4::t_last_cuda_error);
}

extern "C" const char *hif4_status_string(hif4_status s)
{
    switch (s) {
    case HIF4_OK: return "ok";
    case HIF4_ERR_INVALID_ARG: return "invalid argument";
    case HIF4_ERR_ALIGNMENT: return "pointer or leading dimension not 16-byte aligned";
    case HIF4_ERR_SHAPE: return "shape error (cols/K must be a multiple of 64, ld >= cols)";
    case HIF4_ERR_WORKSPACE: return "workspace missing or too small";
    case HIF4_ERR_CUDA: return "CUDA runtime error";
    case HIF4_ERR_NONFINITE: return "non-finite input mapped (NaN -> 0, Inf -> +-FLT_MAX)";
    case HIF4_ERR_TIMEOUT: return "bounded device wait timed out";
    case HIF4_ERR_UNSUPPORTED: return "unsupported device or size";
    case HIF4_ERR_FORMAT: return "serialized state malformed, truncated or corrupted";
    }
    return "unknown status";
}

extern "C" int hif4_version(void) { return 100; }

extern "C" void hif4_debug_wait_test(uint32_t withhold, uint64_t limit_ns)
{
    hif4::g_withhold.store(withhold ? 1u : 0u);
    hif4::g_wait_limit.store(limit_ns);
}
