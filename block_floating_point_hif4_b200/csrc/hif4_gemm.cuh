// hif4_gemm.cuh — the persistent tcgen05 GEMM kernel behind hif4_gemm_bf16,
// hif4_gemm_bf16_fq, hif4_linear_w4a4 and the FFN calls (included by
// hif4_linear.cu, where its host entry points live).  Structure, epilogue
// options and time-out behaviour are described at the top of hif4_linear.cu.
#pragma once

#include <cuda_bf16.h>

#include "hif4_encode.cuh"
#include "hif4_internal.cuh"
#include "hif4_sm100.cuh"

namespace hif4 {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int THREADS = 192;
constexpr int GROUP_M = 16;
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint64_t TIMEOUT_NS = 4000000000ull;   // 4 s: far above any launch

struct Args {
    int M, N, K;
    int num_m, num_n, num_k, num_tiles;
    const uint16_t *bias;   // BF16 [N] or null
    void *y;                // BF16 (or F32 with HIF4_LINEAR_OUT_F32) M x N, leading dimension ldy
    int64_t ldy;
    uint32_t flags;
    const uint8_t *out_mask;  // HIF4_LINEAR_FAKE_QUANT_OUT: u8 [N] protected output columns, or null
    uint32_t *status;
    uint64_t timeout_ns;
    uint32_t withhold;      // block 0 withholds its first copy (failure-handling test)
    int group_m;            // m-tiles per rasterization group
};

__device__ __forceinline__ void tile_coords(int t, const Args &g, int &mb, int &nb)
{
    const int per_group = g.group_m * g.num_n;
    const int gi = t / per_group;
    const int first_m = gi * g.group_m;
    const int gm = min(g.num_m - first_m, g.group_m);
    const int r = t - gi * per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

// tanh-form GELU, 0.5 x (1 + tanh(u)) with u = sqrt(2/pi) (x + 0.044715 x^3),
// evaluated as the identical x / (1 + exp(-2u)) with the fast exponential
// and division intrinsics: relative error a few 1e-6 for |x| up to ~10
// (three orders below BF16's half-ulp), no per-element branches, so the
// epilogue stays hidden behind the mainloop.  x -> -inf: exp overflows and
// the result is -0 (below about -10 the exact value is already < 1e-37);
// x -> +inf: the result is x.
__device__ __forceinline__ float gelu_tanh(float x)
{
    const float u = 0.7978845608028654f * fmaf(0.044715f * x, x * x, x);
    return __fdividef(x, 1.0f + __expf(-2.0f * u));
}

// 32 accumulator columns of one row -> + bias (BF16, 16-byte aligned, or
// null) -> optional tanh-GELU -> 16 packed BF16 pairs (round to nearest
// even; column 2j in the low half of w[j]).
__device__ __forceinline__ void epi_pack32(const uint32_t (&r)[32], const uint16_t *bias, bool gelu,
                                           uint32_t *w)
{
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
    if (bias) {
        const uint4 *bp = reinterpret_cast<const uint4 *>(bias);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 b = __ldg(bp + i);
            const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                v[8 * i + 2 * h] += __uint_as_float(bw[h] << 16);
                v[8 * i + 2 * h + 1] += __uint_as_float(bw[h] & 0xFFFF0000u);
            }
        }
    }
    if (gelu) {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
    }
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
        w[j] = *reinterpret_cast<uint32_t *>(&h2);
    }
}

// One accumulator's rows of this warp's TMEM lane quarter (tacc: lane
// quarter and accumulator column base) -> output row `row` (stored only if
// row < M), columns nb * BN ... + BN - 1: + bias, optional tanh-GELU, FP32,
// or BF16 (round to nearest even) with optional HiF4 fake quantization of
// the row's 64-column units (compiled in only with FQ).
template <bool FQ>
__device__ __forceinline__ void store_tile_rows(const Args &g, uint32_t tacc, int row, int nb, uint32_t &nonfinite)
{
    using namespace sm100;
    const bool gelu = (g.flags & HIF4_LINEAR_GELU_TANH) != 0;
    const bool out_f32 = (g.flags & HIF4_LINEAR_OUT_F32) != 0;
    const bool fq_out = FQ && (g.flags & HIF4_LINEAR_FAKE_QUANT_OUT) != 0;
    uint16_t *yrow = static_cast<uint16_t *>(g.y) + (int64_t)row * g.ldy;
    float *yrow32 = static_cast<float *>(g.y) + (int64_t)row * g.ldy;
    // HiF4 fake-quant of the output along N: a thread holds whole
    // 64-column units of its row (N % 64 == 0), so every unit
    // decision is thread-local.
#pragma unroll 1
    for (int u = 0; fq_out && u < BN / 64; ++u) {
        const int n0 = nb * BN + u * 64;
        if (n0 >= g.N) break;                          // warp-uniform
        uint32_t w[32];
        {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tacc + u * 64, r);
            tmem_ld_wait();
            epi_pack32(r, g.bias ? g.bias + n0 : nullptr, gelu, w);
            tmem_ld_32x32b_x32(tacc + u * 64 + 32, r);
            tmem_ld_wait();
            epi_pack32(r, g.bias ? g.bias + n0 + 32 : nullptr, gelu, w + 16);
        }
        uint32_t out[32];
        uint32_t mraw[16];
        uint32_t any = 0;
        if (g.out_mask) {
            const uint4 *mp = reinterpret_cast<const uint4 *>(g.out_mask + n0);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint4 m = __ldg(mp + i);
                mraw[4 * i] = m.x;
                mraw[4 * i + 1] = m.y;
                mraw[4 * i + 2] = m.z;
                mraw[4 * i + 3] = m.w;
                any |= m.x | m.y | m.z | m.w;
            }
        }
        if (any) {                                     // warp-uniform: same columns
            uint32_t mw[32];
#pragma unroll
            for (int i = 0; i < 4; ++i) enc::mask_words16(mraw + 4 * i, mw + 8 * i);
            enc::fq_unit64<true>(w, mw, out, nonfinite);
        } else {
            enc::fq_unit64<false>(w, w, out, nonfinite);
        }
        if (row < g.M) {
            uint4 *dst = reinterpret_cast<uint4 *>(yrow + n0);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                dst[i] = make_uint4(out[4 * i], out[4 * i + 1], out[4 * i + 2], out[4 * i + 3]);
        }
    }
#pragma unroll 1
    for (int c = 0; !fq_out && c < BN / 32; ++c) {
        const int n0 = nb * BN + c * 32;
        if (n0 >= g.N) break;                          // warp-uniform
        uint32_t r[32];
        tmem_ld_32x32b_x32(tacc + c * 32, r);
        tmem_ld_wait();
        float v[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(r[j]);
        if (g.bias) {
            if (n0 + 32 <= g.N) {
                const uint4 *bp = reinterpret_cast<const uint4 *>(g.bias + n0);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint4 b = __ldg(bp + i);
                    const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int h = 0; h < 4; ++h) {
                        v[8 * i + 2 * h] += __uint_as_float(bw[h] << 16);
                        v[8 * i + 2 * h + 1] += __uint_as_float(bw[h] & 0xFFFF0000u);
                    }
                }
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (n0 + j < g.N) v[j] += __uint_as_float((uint32_t)g.bias[n0 + j] << 16);
            }
        }
        if (gelu) {
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] = gelu_tanh(v[j]);
        }
        if (out_f32) {
            if (row < g.M) {
                if (n0 + 32 <= g.N) {
                    float4 *dst = reinterpret_cast<float4 *>(yrow32 + n0);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                } else {
#pragma unroll
                    for (int j = 0; j < 32; ++j)
                        if (n0 + j < g.N) yrow32[n0 + j] = v[j];
                }
            }
            continue;
        }
        uint32_t packed[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            __nv_bfloat162 h2 = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
            packed[j] = *reinterpret_cast<uint32_t *>(&h2);
        }
        if (row < g.M) {
            if (n0 + 32 <= g.N) {
                uint4 *dst = reinterpret_cast<uint4 *>(yrow + n0);
#pragma unroll
                for (int i = 0; i < 4; ++i)
                    dst[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
            } else {
#pragma unroll
                for (int j = 0; j < 32; ++j)
                    if (n0 + j < g.N) yrow[n0 + j] = (uint16_t)(packed[j >> 1] >> (16 * (j & 1)));
            }
        }
    }
}

__global__ void __launch_bounds__(THREADS, 1)
k_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Args g)
{
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = smem + STAGES * A_BYTES;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + STAGES * STAGE_BYTES);
    uint64_t *full = bars;
    uint64_t *empty = bars + STAGES;
    uint64_t *tfull = bars + 2 * STAGES;
    uint64_t *tempty = tfull + 2;
    uint64_t *drain = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], 4);
        }
        mbar_init(drain, 1);
        *abort_flag = 0u;
        fence_barrier_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmA);
        prefetch_tensormap(&tmB);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_holder;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer
            uint32_t stage = 0, phase = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < g.num_tiles; t += gridDim.x) {
                int mb, nb;
                tile_coords(t, g, mb, nb);
                for (int kb = 0; kb < g.num_k; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, g.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    if (!(g.withhold && t == 0 && kb == 0)) {      // else its wait can only run out
                        mbar_arrive_expect_tx(&full[stage], STAGE_BYTES);
                        tma_load_2d(sA + stage * A_BYTES, &tmA, kb * BK, mb * BM, &full[stage]);
                        tma_load_2d(sB + stage * B_BYTES, &tmB, kb * BK, nb * BN, &full[stage]);
                        ++issued;
                    }
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // Let our own copies land before the block leaves: wait (with
                // a short limit, ignoring the abort flag) on the most recent
                // phase of every stage we loaded.
                for (uint32_t i = 0; i < STAGES && i < issued; ++i) {
                    uint32_t s = (stage + STAGES - 1 - i) % STAGES;
                    uint32_t ph = (s < stage) ? phase : (phase ^ 1u);
                    mbar_wait_bounded(&full[s], ph, nullptr, 100000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------- MMA issuer
            const uint32_t idesc = idesc_bf16_f32(BM, BN);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < g.num_tiles; t += gridDim.x) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, g.timeout_ns)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = 0; kb < g.num_k; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, g.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_addr(sA + stage * A_BYTES);
                    const uint32_t b0 = smem_addr(sB + stage * B_BYTES);
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k)
                        mma_bf16(d, smem_desc_sw128(a0 + k * 32), smem_desc_sw128(b0 + k * 32), idesc,
                                 (kb | k) != 0);
                    mma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            }
            // No MMA may still be running when TMEM is released.
            mma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, 100000000ull);
        }
    } else {
        // -------------------------------------------------------- epilogue
        const int q = warp & 3;                 // TMEM lane quarter of this warp
        uint32_t nonfinite = 0;
        uint32_t acc = 0, acc_phase = 0;
        for (int t = blockIdx.x; t < g.num_tiles; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, g, mb, nb);
            if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, g.timeout_ns)) break;
            tc_fence_after();
            store_tile_rows<true>(g, tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN, mb * BM + q * 32 + lane, nb,
                                  nonfinite);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (nonfinite) status_or(g.status, HIF4_FLAG_NONFINITE);
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
    if (threadIdx.x == 0 && *abort_flag) status_or(g.status, HIF4_FLAG_TIMEOUT);
}



// ----------------------------------------------------------- host helpers

// BF16 rows x cols (K-major, leading dimension ld elements), boxes of
// box_rows x 64 with 128-byte swizzle.
bool make_map(CUtensorMap *map, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_rows)
{
    return make_tensor_map_bf16_2d(map, base, cols, rows, ld * 2, BK, box_rows, true);
}

} // namespace gemm
} // namespace hif4
