// hif4_internal.cuh — shared device/host helpers of libhif4 (sm_100a).
//
// The HiF4 unit [Huawei HiF4 calibration article, section 1 "HiFloat4 (HiF4)
// format"]: 64 elements, one E6M2 level-1 scale, 8 level-2 and 16 level-3 E1
// exponents, S1P2 element codes.  The scale is unsigned with bias 31,
// v(c) = 2^(E-31) (1 + f/4); every quantity the encoder compares against
// (6.5 v, 1.75 v, 3.5 v and the rounding half-way points) is exact in FP32,
// so every rounding decision below is taken by exact FP32 comparison.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hif4.h"

#define HIF4_UNIT 64

namespace hif4 {

// ------------------------------------------------------------------ host

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline bool aligned_to(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Records the CUDA runtime error behind an HIF4_ERR_CUDA return (per host
// thread; hif4_last_cuda_error reports it) and returns HIF4_ERR_CUDA.
hif4_status cuda_failed(cudaError_t e);

inline hif4_status launch_status()
{
    cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? HIF4_OK : cuda_failed(e);
}

// Number of SMs of the current device (cached per device ordinal).
int sm_count();
// Failure-handling diagnostics (hif4_debug_wait_test): whether TMA-fed
// launches withhold the first copy of their block 0, and the limit of their
// bounded waits (dflt unless a test set one).
uint32_t wait_test_withhold();
uint64_t wait_limit_ns(uint64_t dflt);
// Resident blocks per SM for `kernel` at this block size (cached per kernel
// and device).
int blocks_per_sm(const void *kernel, int threads, size_t dyn_smem);
// 2-D BF16 tensor map (inner x outer elements, rows row_stride_bytes apart)
// with box_inner x box_outer boxes, optionally 128-byte swizzled; the driver's
// encoder is resolved once through the runtime.  False if unavailable.
bool make_tensor_map_bf16_2d(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                             uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128);

// Exact unsigned 32-bit division by a fixed divisor d >= 1 via a multiply:
// q = (umulhi(n, m) + n) >> s with s = ceil(log2 d),
// m = floor(2^32 (2^s - d) / d) + 1 (exact for every n < 2^32).
struct FastDiv {
    uint32_t m;
    uint32_t s;
    FastDiv() = default;
    explicit FastDiv(uint32_t d)
    {
        uint32_t sh = 0;
        while (sh < 32 && (1ull << sh) < d) ++sh;
        s = sh;
        m = (uint32_t)(((1ull << 32) * ((1ull << sh) - d)) / d + 1ull);
    }
    __device__ __forceinline__ uint32_t div(uint32_t n) const
    {
        return (uint32_t)(((uint64_t)__umulhi(n, m) + n) >> s);
    }
};

// ---------------------------------------------------------------- device

__device__ __forceinline__ float bits_f(uint32_t u) { return __uint_as_float(u); }
__device__ __forceinline__ uint32_t f_bits(float f) { return __float_as_uint(f); }

// FP32 value of the E6M2 code c: exponent field E + 96 (= E - 31 + 127),
// top two mantissa bits f.
__device__ __forceinline__ float e6m2_value(uint32_t c)
{
    return bits_f(((c >> 2) + 96u) << 23 | (c & 3u) << 21);
}

// Largest code c with 6.5 * v(c) < a (0 if none; 255 above the top).
// The candidate comes from truncating a / 6.5 onto the E6M2 grid; the FP32
// quotient is within a few ulp of the true one, and consecutive grid values
// differ by at least 8/7, so one exact correction step in each direction
// suffices.  6.5 * v(c) has at most 7 significant bits: the products below
// are exact.
__device__ __forceinline__ uint32_t select_scale_code(float a)
{
    float r = a * (1.0f / 6.5f);
    int32_t ef = (int32_t)(f_bits(r) >> 23);          // a >= 0: no sign bit
    int32_t c = ((ef - 96) << 2) | (int32_t)((f_bits(r) >> 21) & 3u);
    c = ef < 96 ? 0 : c;
    c = c > 255 ? 255 : c;
    if (c > 0 && 6.5f * e6m2_value((uint32_t)c) >= a) c -= 1;
    if (c < 255 && 6.5f * e6m2_value((uint32_t)c + 1u) < a) c += 1;
    return (uint32_t)c;
}

// 2^k * v for a normal FP32 v and small k (exact exponent shift).
__device__ __forceinline__ float ldexp_small(float v, int k)
{
    return bits_f(f_bits(v) + ((uint32_t)k << 23));
}

// Map NaN -> 0 and +-Inf -> +-FLT_MAX; *bad |= 1 when it did.
__device__ __forceinline__ float sanitize(float v, uint32_t &bad)
{
    uint32_t u = f_bits(v);
    if ((u & 0x7F800000u) == 0x7F800000u) {
        bad = 1u;
        if (u & 0x007FFFFFu) return 0.0f;
        return bits_f((u & 0x80000000u) | 0x7F7FFFFFu);
    }
    return v;
}

// BF16 pair in a 32-bit word -> two FP32 values (exact widening).
__device__ __forceinline__ float bf16_lo(uint32_t w) { return bits_f(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return bits_f(w & 0xFFFF0000u); }
// Two FP32 values whose low 16 bits are zero -> packed BF16 pair (exact).
__device__ __forceinline__ uint32_t pack_bf16_exact(float lo, float hi)
{
    return __byte_perm(f_bits(lo), f_bits(hi), 0x7632);
}

__device__ __forceinline__ void status_or(uint32_t *status, uint32_t bits)
{
    if (status && bits) atomicOr(status, bits);
}

} // namespace hif4
