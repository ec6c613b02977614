// hif4_gemm_f8.cu — the W4A4 HiF4 product on the FP8 tensor cores, with the
// HiF4 unit scales applied in FP32 per 64-element unit.
//
// Every HiF4 element is (-1)^s (m/4) 2^E S with m <= 7, E = e2 + e3 <= 2 and
// S the unit's E6M2 scale [Huawei HiF4 calibration article, section 1
// "HiFloat4 (HiF4) format"].  Its scale-free part m 2^(E-2) has at most three
// significant bits, so it is exact in FP8 E4M3 (hif4_to_e4m3).  The products
// of two such values are multiples of 1/16 up to 49, and a 64-element unit's
// sum of them is below 2^12 with granularity 2^-4: 16 significant bits.  S is
// not a power of two (1 + f/4 has two fraction bits) and differs per unit of
// each row of A and of B, so it cannot enter the FP8 operands or a
// power-of-two block scale; it is applied after the tensor core: each unit's
// 64-deep product goes to its own TMEM accumulator, and the epilogue warps
// read it back and add S_a[m] S_b[n] P[m, n] into FP32 totals held in
// registers.
//
// Structure (one CTA per SM, 320 threads; 128 x 256 output tiles):
//   warp 0      TMA producer: 128 x 128-byte A and 256 x 128-byte B tiles
//               (two units of K) with 128-byte swizzle, and the two units'
//               row and column scales (bulk copies of the K-unit-major scale
//               arrays), into a 4-stage ring;
//   warp 1      allocates 512 TMEM columns (two 128 x 256 FP32 unit
//               accumulators) and issues tcgen05.mma kind::f8f6f4 (E4M3,
//               M = 128, N = 256, K = 32; two per unit), alternating the
//               accumulators unit by unit;
//   warps 2-9   promotion: warp w reads TMEM lane quarter w % 4, columns
//               0-127 (warps 2-5) or 128-255 (warps 6-9), releases the
//               accumulator, and adds S_a S_b P into its 128 FP32 totals;
//               after the last unit of a tile it stores the totals (FP32 or
//               BF16, round to nearest even).
// A smem stage is released when its MMAs have completed and every promotion
// warp has read its scales.  Every mbarrier wait is bounded (4 s); a role that
// gives up sets the block's abort flag, the producer lets its copies land,
// the MMA thread drains its MMAs before TMEM is freed, and HIF4_FLAG_TIMEOUT
// is raised.
#include <cuda_bf16.h>

#include "hif4_internal.cuh"
#include "hif4_sm100.cuh"

namespace hif4 {

bool make_tensor_map_u8_2d_sw128(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                                 uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);

namespace gemm8 {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int KS = 128;                         // K elements (bytes) per stage: two units
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * KS;                // 16 KB
constexpr int B_BYTES = BN * KS;                // 32 KB
constexpr int SA_BYTES = 2 * BM * 4;            // two units' row scales
constexpr int SB_BYTES = 2 * BN * 4;            // two units' column scales
constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SA_BYTES + SB_BYTES;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;
constexpr int TMEM_COLS = 2 * BN;
constexpr int GROUP_M = 16;
constexpr size_t SMEM_BYTES = (size_t)STAGES * STAGE_BYTES + 1024 + 256;
constexpr uint64_t TIMEOUT_NS = 4000000000ull;

struct Args {
    int M, N, K;
    int num_m, num_n, num_u, num_s, num_tiles;
    const float *sa;        // [K/64][lds_a] row scales (rows past M read, never stored)
    int64_t lds_a;
    const float *sb;        // [K/64][lds_b] column scales
    int64_t lds_b;
    void *y;
    int64_t ldy;
    uint32_t out_f32;
    uint32_t *status;
    uint64_t timeout_ns;
};

// Two FP32 lanes at once (sm_100 packed FP32): d = a * b + d and d = a * b.
__device__ __forceinline__ void fma2(float &d0, float &d1, float a0, float a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\tmov.b64 pd, {%0, %1};\n\t"
        "fma.rn.f32x2 pd, pa, pb, pd;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void mul2(float &d0, float &d1, float a0, float a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
        "mov.b64 pa, {%2, %3};\n\tmov.b64 pb, {%4, %5};\n\t"
        "mul.rn.f32x2 pd, pa, pb;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// acc[0..7] += (sx * sw[0..7]) * p[0..7], in packed pairs.
__device__ __forceinline__ void promote8(float *acc, const uint32_t (&p)[8], float sx, const float4 *sw)
{
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const float4 w = sw[j];
        float c0, c1, c2, c3;
        mul2(c0, c1, w.x, w.y, sx, sx);
        mul2(c2, c3, w.z, w.w, sx, sx);
        fma2(acc[4 * j], acc[4 * j + 1], __uint_as_float(p[4 * j]), __uint_as_float(p[4 * j + 1]), c0, c1);
        fma2(acc[4 * j + 2], acc[4 * j + 3], __uint_as_float(p[4 * j + 2]), __uint_as_float(p[4 * j + 3]), c2, c3);
    }
}

__device__ __forceinline__ void tile_coords(int t, const Args &g, int &mb, int &nb)
{
    const int per_group = GROUP_M * g.num_n;
    const int gi = t / per_group;
    const int first_m = gi * GROUP_M;
    const int gm = min(g.num_m - first_m, GROUP_M);
    const int r = t - gi * per_group;
    mb = first_m + r % gm;
    nb = r / gm;
}

__global__ void __launch_bounds__(THREADS, 1)
k_gemm_f8(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Args g)
{
    using namespace sm100;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem;
    uint8_t *sB = sA + STAGES * A_BYTES;
    float *sSa = reinterpret_cast<float *>(sB + STAGES * B_BYTES);       // [stage][2][BM]
    float *sSb = sSa + STAGES * 2 * BM;                                   // [stage][2][BN]
    uint64_t *bars = reinterpret_cast<uint64_t *>(sSb + STAGES * 2 * BN);
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
            mbar_init(&empty[s], 1 + EPI_WARPS);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&tfull[a], 1);
            mbar_init(&tempty[a], EPI_WARPS);
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
                for (int s = 0; s < g.num_s; ++s) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, g.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const int nu = min(2, g.num_u - 2 * s);
                    mbar_arrive_expect_tx(&full[stage], A_BYTES + B_BYTES + nu * (BM + BN) * 4);
                    tma_load_2d(sA + stage * A_BYTES, &tmA, s * KS, mb * BM, &full[stage]);
                    tma_load_2d(sB + stage * B_BYTES, &tmB, s * KS, nb * BN, &full[stage]);
                    for (int v = 0; v < nu; ++v) {
                        const int64_t u = 2 * s + v;
                        bulk_load(sSa + (stage * 2 + v) * BM, g.sa + u * g.lds_a + (int64_t)mb * BM, BM * 4,
                                  &full[stage]);
                        bulk_load(sSb + (stage * 2 + v) * BN, g.sb + u * g.lds_b + (int64_t)nb * BN, BN * 4,
                                  &full[stage]);
                    }
                    ++issued;
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let our own copies land before the block leaves
                for (uint32_t i = 0; i < STAGES && i < issued; ++i) {
                    const uint32_t s = (stage + STAGES - 1 - i) % STAGES;
                    const uint32_t ph = (s < stage) ? phase : (phase ^ 1u);
                    mbar_wait_bounded(&full[s], ph, nullptr, 100000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------------------------------------------- MMA issuer
            const uint32_t idesc = idesc_e4m3_f32(BM, BN);
            uint32_t stage = 0, phase = 0, ug = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < g.num_tiles; t += gridDim.x) {
                for (int s = 0; ok && s < g.num_s; ++s) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, g.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    const int nu = min(2, g.num_u - 2 * s);
                    const uint32_t a0 = smem_addr(sA + stage * A_BYTES);
                    const uint32_t b0 = smem_addr(sB + stage * B_BYTES);
                    for (int v = 0; v < nu; ++v, ++ug) {
                        const uint32_t b = ug & 1u;
                        if (!mbar_wait_bounded(&tempty[b], ((ug >> 1) & 1u) ^ 1u, abort_flag, g.timeout_ns)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t d = tmem_base + b * BN;
#pragma unroll
                        for (int k = 0; k < 2; ++k)
                            mma_f8f6f4(d, smem_desc_sw128(a0 + v * 64 + k * 32), smem_desc_sw128(b0 + v * 64 + k * 32),
                                       idesc, (uint32_t)k);
                        mma_commit(&tfull[b]);
                    }
                    if (!ok) break;
                    mma_commit(&empty[stage]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            // no MMA may still be running when TMEM is released
            mma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, 100000000ull);
        }
    } else {
        // ------------------------------------------------------- promotion
        const int q = warp & 3;                         // TMEM lane quarter
        const int half = (warp - 2) >> 2;               // column half of the tile
        uint32_t stage = 0, phase = 0, ug = 0;
        bool ok = true;
        for (int t = blockIdx.x; ok && t < g.num_tiles; t += gridDim.x) {
            int mb, nb;
            tile_coords(t, g, mb, nb);
            float acc[128];
#pragma unroll
            for (int j = 0; j < 128; ++j) acc[j] = 0.0f;
            for (int s = 0; ok && s < g.num_s; ++s) {
                if (!mbar_wait_bounded(&full[stage], phase, abort_flag, g.timeout_ns)) {
                    ok = false;
                    break;
                }
                const int nu = min(2, g.num_u - 2 * s);
                for (int v = 0; v < nu; ++v, ++ug) {
                    const float sx = sSa[(stage * 2 + v) * BM + q * 32 + lane];
                    const float4 *sw = reinterpret_cast<const float4 *>(sSb + (stage * 2 + v) * BN + half * 128);
                    const uint32_t b = ug & 1u;
                    if (!mbar_wait_bounded(&tfull[b], (ug >> 1) & 1u, abort_flag, g.timeout_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + b * BN + half * 128;
                    // double-buffered 8-column reads: the load of chunk c + 1 is
                    // in flight while chunk c is promoted
                    uint32_t p0[8], p1[8];
                    tmem_ld_32x32b_x8(taddr, p0);
                    tmem_ld_wait_regs(p0);
#pragma unroll
                    for (int c = 0; c < 16; c += 2) {
                        tmem_ld_32x32b_x8(taddr + (c + 1) * 8, p1);
                        promote8(acc + c * 8, p0, sx, sw + c * 2);
                        tmem_ld_wait_regs(p1);
                        if (c + 2 < 16) {
                            tmem_ld_32x32b_x8(taddr + (c + 2) * 8, p0);
                        } else {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&tempty[b]);
                        }
                        promote8(acc + (c + 1) * 8, p1, sx, sw + (c + 1) * 2);
                        if (c + 2 < 16) tmem_ld_wait_regs(p0);
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[stage]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
            if (!ok) break;
            const int row = mb * BM + q * 32 + lane;
            const int n0 = nb * BN + half * 128;
            if (row < g.M) {
                if (g.out_f32) {
                    float *yr = static_cast<float *>(g.y) + (int64_t)row * g.ldy + n0;
                    if (n0 + 128 <= g.N) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            reinterpret_cast<float4 *>(yr)[j] =
                                make_float4(acc[4 * j], acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
                    } else {
#pragma unroll
                        for (int j = 0; j < 128; ++j)
                            if (n0 + j < g.N) yr[j] = acc[j];
                    }
                } else {
                    uint16_t *yr = static_cast<uint16_t *>(g.y) + (int64_t)row * g.ldy + n0;
                    if (n0 + 128 <= g.N) {
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            uint32_t w[4];
#pragma unroll
                            for (int i = 0; i < 4; ++i) {
                                __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[8 * j + 2 * i], acc[8 * j + 2 * i + 1]);
                                w[i] = *reinterpret_cast<uint32_t *>(&h2);
                            }
                            reinterpret_cast<uint4 *>(yr)[j] = make_uint4(w[0], w[1], w[2], w[3]);
                        }
                    } else {
#pragma unroll
                        for (int j = 0; j < 128; ++j)
                            if (n0 + j < g.N) {
                                __nv_bfloat16 h = __float2bfloat16_rn(acc[j]);
                                yr[j] = *reinterpret_cast<uint16_t *>(&h);
                            }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, TMEM_COLS);
    if (threadIdx.x == 0 && *abort_flag) status_or(g.status, HIF4_FLAG_TIMEOUT);
}

// E4M3 byte of the scale-free HiF4 magnitude m 2^(E-2), E = 0: exponent field
// (bias 7) and mantissa of m/4 for m = 0..7; E adds to the exponent field.
__constant__ uint8_t c_e4m3_m[8] = {0x00, 0x28, 0x30, 0x34, 0x38, 0x3A, 0x3C, 0x3E};

// One thread per 8 elements (a 32-bit code word): their E4M3 bytes, and the
// unit's E6M2 scale value into the K-unit-major scale array.
__global__ void k_to_e4m3(const uint32_t *codes, const uint32_t *meta, int64_t rows, int64_t cols, uint8_t *q8,
                          int64_t ldq, float *scale, int64_t lds)
{
    const int64_t words = rows * (cols / 8);
    const int64_t wpr = cols / 8;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < words;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = i / wpr;
        const int64_t wc = i - r * wpr;                 // word within the row
        const int64_t unit = r * (cols / 64) + wc / 8;
        const uint32_t mw = __ldg(meta + unit);
        const uint32_t j = (uint32_t)(wc & 7);          // 8-element group within the unit
        const uint32_t e2 = (mw >> (8 + j)) & 1u;
        const uint32_t cw = __ldg(codes + i);
        uint32_t out[2] = {0, 0};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t nib = (cw >> (4 * e)) & 15u;
            const uint32_t m = nib & 7u;
            const uint32_t E = e2 + ((mw >> (16 + 2 * j + (e >> 2))) & 1u);
            const uint32_t byte = m ? (((uint32_t)c_e4m3_m[m] + (E << 3)) | ((nib >> 3) << 7)) : 0u;
            out[e >> 2] |= byte << (8 * (e & 3));
        }
        *reinterpret_cast<uint2 *>(q8 + r * ldq + wc * 8) = make_uint2(out[0], out[1]);
        if (j == 0) scale[(wc / 8) * lds + r] = e6m2_value(mw & 0xFFu);
    }
}

} // namespace gemm8
} // namespace hif4

using namespace hif4;

extern "C" hif4_status hif4_to_e4m3(const uint8_t *codes, const uint32_t *meta, int64_t rows, int64_t cols,
                                    uint8_t *q8, int64_t ldq, float *scale, int64_t lds, hif4_stream_t stream)
{
    if (rows < 0 || cols < 0) return HIF4_ERR_INVALID_ARG;
    if (cols % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (rows == 0 || cols == 0) return HIF4_OK;
    if (!codes || !meta || !q8 || !scale) return HIF4_ERR_INVALID_ARG;
    if (ldq < cols || lds < rows) return HIF4_ERR_SHAPE;
    if (!aligned_to(codes, 4) || !aligned_to(meta, 4) || !aligned_to(q8, 8) || ldq % 8 != 0 || !aligned_to(scale, 4))
        return HIF4_ERR_ALIGNMENT;
    const int64_t words = rows * (cols / 8);
    int64_t blocks = (words + 255) / 256;
    if (blocks > 16 * (int64_t)sm_count()) blocks = 16 * (int64_t)sm_count();
    gemm8::k_to_e4m3<<<(unsigned)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        reinterpret_cast<const uint32_t *>(codes), meta, rows, cols, q8, ldq, scale, lds);
    return launch_status();
}

extern "C" hif4_status hif4_gemm_f8(const uint8_t *a, int64_t M, int64_t K, int64_t lda, const float *sa,
                                    int64_t lds_a, const uint8_t *b, int64_t N, int64_t ldb, const float *sb,
                                    int64_t lds_b, void *y, int64_t ldy, uint32_t flags, uint32_t *status,
                                    hif4_stream_t stream)
{
    using namespace gemm8;
    if (M < 0 || N < 0 || K < 0) return HIF4_ERR_INVALID_ARG;
    if (K % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (M == 0 || N == 0) return HIF4_OK;
    if (K < KS) return HIF4_ERR_SHAPE;              // the 128-byte operand box must fit inside a row
    if (!a || !b || !sa || !sb || !y) return HIF4_ERR_INVALID_ARG;
    if (flags & ~(uint32_t)HIF4_LINEAR_OUT_F32) return HIF4_ERR_INVALID_ARG;
    const int64_t mp = (M + BM - 1) / BM * BM, np = (N + BN - 1) / BN * BN;
    if (lda < K || ldb < K || ldy < N || lds_a < mp || lds_b < np) return HIF4_ERR_SHAPE;
    if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return HIF4_ERR_UNSUPPORTED;
    const int64_t ysz = (flags & HIF4_LINEAR_OUT_F32) ? 4 : 2;
    if (!aligned16(a) || !aligned16(b) || !aligned16(y) || !aligned16(sa) || !aligned16(sb) || lda % 16 ||
        ldb % 16 || lds_a % 4 || lds_b % 4 || (ldy * ysz) % 16)
        return HIF4_ERR_ALIGNMENT;
    CUtensorMap tmA, tmB;
    if (!make_tensor_map_u8_2d_sw128(&tmA, a, (uint64_t)K, (uint64_t)M, (uint64_t)lda, KS, BM) ||
        !make_tensor_map_u8_2d_sw128(&tmB, b, (uint64_t)K, (uint64_t)N, (uint64_t)ldb, KS, BN))
        return HIF4_ERR_UNSUPPORTED;                // the driver's encoder refused the layout
    Args g{};
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.num_m = (int)(mp / BM);
    g.num_n = (int)(np / BN);
    g.num_u = (int)(K / HIF4_UNIT);
    g.num_s = (g.num_u + 1) / 2;
    g.num_tiles = g.num_m * g.num_n;
    g.sa = sa;
    g.lds_a = lds_a;
    g.sb = sb;
    g.lds_b = lds_b;
    g.y = y;
    g.ldy = ldy;
    g.out_f32 = (flags & HIF4_LINEAR_OUT_F32) ? 1u : 0u;
    g.status = status;
    g.timeout_ns = wait_limit_ns(TIMEOUT_NS);
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr_set[dev & 63]) {
        const cudaError_t e =
            cudaFuncSetAttribute(k_gemm_f8, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return cuda_failed(e);
        attr_set[dev & 63] = true;
    }
    int grid = sm_count();
    if (grid > g.num_tiles) grid = g.num_tiles;
    k_gemm_f8<<<grid, THREADS, SMEM_BYTES, reinterpret_cast<cudaStream_t>(stream)>>>(tmA, tmB, g);
    return launch_status();
}
