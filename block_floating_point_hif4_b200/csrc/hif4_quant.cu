// hif4_quant.cu — HiF4 quantize / dequantize / activation fake-quant kernels.
//
// HBM-bound streaming kernels.  One lane owns one 16-byte input vector: the
// 8 elements of one level-2 group (two level-3 groups) of a 64-element unit;
// the 8 lanes of a unit combine their maxima with three xor-shuffles, so a
// warp covers 4 consecutive units (512 contiguous BF16 bytes per load
// instruction).  Each lane keeps UNR vectors in flight before it computes.
//
// Encode rule [Huawei HiF4 calibration article, section 1; the rule itself is
// the library's reading of a step the page leaves open]:
//   S   = largest E6M2 value with 6.5 S < max|x| over the unit,
//   t   = 0/1/2 for each 4-group by max4 <= 1.75 S / <= 3.5 S / more,
//   e2  = [max t of the 8-group == 2],  e3 = max(0, t - e2),
//   m   = RNE(|x| / (S 2^(e2+e3) / 4)), ties to even, min 7.
// Rounding: r = |x| * fl(4 / (S 2^E)) is within 2^-20 of the true quotient
// (two FP32 roundings, quotient <= 7.5), so RNE(r) is exact unless r lies
// within 2^-19 of a half-integer; such lanes redo their 8 elements with exact
// comparisons against the half-way points (k + 1/2) S 2^E / 4 (exact in FP32).
#include <cuda_bf16.h>

#include "hif4_encode.cuh"
#include "hif4_internal.cuh"
#include "hif4_sm100.cuh"

namespace hif4 {

namespace {

using namespace enc;

constexpr int kThreads = 256;
constexpr int kUnroll = 4;
#ifndef HIF4_DQ_UNROLL
#define HIF4_DQ_UNROLL 4
#endif
constexpr int kDqUnroll = HIF4_DQ_UNROLL;            // units in flight per dequantize lane

struct QuantArgs {
    const void *x;
    int64_t ldx;
    const uint8_t *chan_mask;  // nullable
    uint8_t *codes;            // MODE 0
    uint32_t *meta;            // MODE 0
    void *out;                 // MODE 1 (BF16 xhat)
    int64_t ldo;
    uint32_t upr;              // units per row
    FastDiv upr_div;
    uint32_t total_units;
    uint32_t *status;
    uint32_t withhold;         // TMA kernels: block 0 withholds its first copy (failure-handling test)
    uint64_t wait_ns;          // TMA kernels: limit of every bounded wait
};

// Loads the 8 elements of lane vector `e` (element offset) as FP32.
template <bool BF16>
__device__ __forceinline__ void load_vec(const void *x, int64_t e, uint4 (&raw)[2])
{
    if (BF16) {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const uint16_t *>(x) + e);
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(raw[0].x), "=r"(raw[0].y), "=r"(raw[0].z), "=r"(raw[0].w)
                     : "l"(p));
    } else {
        const uint4 *p = reinterpret_cast<const uint4 *>(static_cast<const float *>(x) + e);
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(raw[0].x), "=r"(raw[0].y), "=r"(raw[0].z), "=r"(raw[0].w)
                     : "l"(p));
        asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                     : "=r"(raw[1].x), "=r"(raw[1].y), "=r"(raw[1].z), "=r"(raw[1].w)
                     : "l"(p + 1));
    }
}

template <bool BF16>
__device__ __forceinline__ void widen(const uint4 (&raw)[2], float (&v)[8], uint32_t &nonfinite)
{
    uint32_t acc = 0;
    if (BF16) {
        const uint32_t w[4] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = bf16_lo(w[i]);
            v[2 * i + 1] = bf16_hi(w[i]);
            acc |= (w[i] & 0x7F807F80u) + 0x00800080u;   // bit 15/31 set <=> exponent all ones
        }
        nonfinite = acc & 0x80008000u;
    } else {
        const uint32_t w[8] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w,
                               raw[1].x, raw[1].y, raw[1].z, raw[1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[i] = bits_f(w[i]);
            acc |= (w[i] & 0x7F800000u) + 0x00800000u;
        }
        nonfinite = acc & 0x80000000u;
    }
}

// Quantize (MODE 0) or fake-quantize (MODE 1) one lane vector.  All 8 lanes
// of a unit must call this together (shuffles over xor 1, 2, 4).
template <int MODE>
__device__ __forceinline__ void encode_lane(float (&v)[8], const float (&orig)[8], uint32_t mbits,
                                            uint32_t lane8, uint32_t &codes_out,
                                            uint32_t &meta_out, uint32_t (&y)[4])
{
    float alo = 0.0f, ahi = 0.0f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        alo = fmaxf(alo, fabsf(v[i]));
        ahi = fmaxf(ahi, fabsf(v[i + 4]));
    }
    float a8 = fmaxf(alo, ahi);
    float a = a8;
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));

    const uint32_t c = select_scale_code(a);
    const float S = e6m2_value(c);
    const float T1 = 1.75f * S, T2 = 3.5f * S;
    const uint32_t e2 = a8 > T2;
    const uint32_t e3lo = e2 ? (alo > T2) : (alo > T1);
    const uint32_t e3hi = e2 ? (ahi > T2) : (ahi > T1);
    // step = S 2^E / 4; inv = 4 / (S 2^E) (reciprocal of S rounded once)
    const float rS = __frcp_rn(S);
    const float step_lo = ldexp_small(S, (int)(e2 + e3lo) - 2);
    const float step_hi = ldexp_small(S, (int)(e2 + e3hi) - 2);
    const float inv_lo = ldexp_small(rS, 2 - (int)(e2 + e3lo));
    const float inv_hi = ldexp_small(rS, 2 - (int)(e2 + e3hi));

    uint32_t m[8];
    float near = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const float inv = i < 4 ? inv_lo : inv_hi;
        const float r = fminf(fabsf(v[i]) * inv, 7.0f);
        const float t = r + 12582912.0f;                 // 1.5 * 2^23: RNE in the low bits
        const float mf = t - 12582912.0f;
        near = fmaxf(near, fabsf(r - mf));
        m[i] = f_bits(t) & 7u;
    }
    if (near >= 0.49999809f) {                           // 0.5 - 2^-19: exact re-decision
#pragma unroll
        for (int i = 0; i < 8; ++i)
            m[i] = round_exact(fabsf(v[i]), i < 4 ? inv_lo : inv_hi, i < 4 ? step_lo : step_hi);
    }

    uint32_t codes = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint32_t s = (m[i] != 0u) ? (f_bits(v[i]) >> 31) : 0u;
        codes |= (m[i] | (s << 3)) << (4 * i);
    }
    codes_out = codes;

    if (MODE == 0) {
        uint32_t part = (e2 << (8 + lane8)) | (e3lo << (16 + 2 * lane8)) | (e3hi << (17 + 2 * lane8));
        part |= __shfl_xor_sync(0xffffffffu, part, 1);
        part |= __shfl_xor_sync(0xffffffffu, part, 2);
        part |= __shfl_xor_sync(0xffffffffu, part, 4);
        meta_out = part | c;
    } else {
        float o[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float step = i < 4 ? step_lo : step_hi;
            float q = (float)m[i] * step;                          // exact (<= 6 bits)
            q = bits_f(f_bits(q) | (((codes >> (4 * i + 3)) & 1u) << 31));
            o[i] = ((mbits >> i) & 1u) ? orig[i] : q;
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) y[i] = pack_bf16_exact(o[2 * i], o[2 * i + 1]);
        meta_out = 0;
    }
}

template <bool BF16, bool MASK, bool CONTIG, int MODE>
__global__ void __launch_bounds__(kThreads) k_quant(QuantArgs a)
{
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t lane8 = lane & 7u;
    const uint32_t nquads = (a.total_units + 3u) >> 2;
    const uint32_t gwarp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    uint32_t bad = 0;

    for (uint32_t q0 = gwarp; q0 < nquads; q0 += nwarps * kUnroll) {
        uint4 raw[kUnroll][2];
        uint32_t unit[kUnroll], row[kUnroll], cu[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t q = q0 + (uint32_t)u * nwarps;
            unit[u] = q * 4u + (lane >> 3);
            const bool active = q < nquads && unit[u] < a.total_units;
            row[u] = (!CONTIG || MASK) ? a.upr_div.div(unit[u]) : 0u;
            cu[u] = unit[u] - row[u] * a.upr;
            const int64_t e = CONTIG ? (int64_t)unit[u] * HIF4_UNIT + lane8 * 8
                                     : (int64_t)row[u] * a.ldx + (int64_t)cu[u] * HIF4_UNIT + lane8 * 8;
            if (active) load_vec<BF16>(a.x, e, raw[u]);
            else raw[u][0] = raw[u][1] = make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t q = q0 + (uint32_t)u * nwarps;
            if (q >= nquads) break;                     // warp-uniform
            const bool active = unit[u] < a.total_units;
            float v[8], orig[8];
            uint32_t nf;
            widen<BF16>(raw[u], v, nf);
#pragma unroll
            for (int i = 0; i < 8; ++i) orig[i] = v[i];  // pass-through keeps the raw value
            if (nf) {
#pragma unroll
                for (int i = 0; i < 8; ++i) v[i] = sanitize(v[i], bad);
            }
            uint32_t mbits = 0;
            if (MASK && active) {
                const uint2 mb = *reinterpret_cast<const uint2 *>(a.chan_mask + (size_t)cu[u] * HIF4_UNIT + lane8 * 8);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    mbits |= (((mb.x >> (8 * i)) & 0xFFu) ? 1u : 0u) << i;
                    mbits |= (((mb.y >> (8 * i)) & 0xFFu) ? 1u : 0u) << (i + 4);
                }
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if ((mbits >> i) & 1u) v[i] = 0.0f;
            }
            uint32_t codes, meta, y[4];
            encode_lane<MODE>(v, orig, mbits, lane8, codes, meta, y);
            if (!active) continue;
            if (MODE == 0) {
                reinterpret_cast<uint32_t *>(a.codes)[(size_t)unit[u] * 8 + lane8] = codes;
                if (lane8 == 0) a.meta[unit[u]] = meta;
            } else {
                const int64_t o = CONTIG ? (int64_t)unit[u] * HIF4_UNIT + lane8 * 8
                                         : (int64_t)row[u] * a.ldo + (int64_t)cu[u] * HIF4_UNIT + lane8 * 8;
                *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.out) + o) =
                    make_uint4(y[0], y[1], y[2], y[3]);
            }
        }
    }
    if (bad) status_or(a.status, HIF4_FLAG_NONFINITE);
}

// ------------------------------------------------- BF16 input, fast kernel
//
// One lane owns 16 consecutive elements of a unit (one 256-bit load; two
// level-2 groups, four level-3 groups); 4 lanes share a unit, a warp covers 8
// units (1 KB of BF16).
//   * Maxima are taken on 16-bit magnitude keys (bits & 0x7FFF, whose order is
//     the |x| order) with max.u16x2; a unit key >= 0x7F80 means a NaN/Inf.
//   * The scale code comes from the bits of the unit maximum a: within a's
//     binade the four thresholds 6.5 v(c) sit at mantissa offsets
//     2^17 {1, 14, 27, 40}, so c = 4 (e - 99) + #{thresholds below the mantissa}.
//   * 1.75 S and 3.5 S are exact BF16 values, so the group exponents are
//     integer comparisons of keys.
//   * |x| / step = |x| (H + L) with H + L a two-term expansion of
//     16 / (4 + f) (times a power of two): for BF16 inputs the FP32 result of
//     fma(|x|, H, |x| L) is exact at every rounding tie and at least 1/448 away
//     from a tie otherwise, so round-to-nearest-even by the 1.5 * 2^23 magic
//     addition is exact.  Products run as packed f32x2 operations.
//   * Units with a non-finite input or a scale clamped at the top code (255)
//     take the generic FP32 path (sanitize, exact half-way comparisons).

__device__ __forceinline__ void ld256(const void *p, uint32_t (&w)[8])
{
    asm volatile("ld.global.nc.L1::no_allocate.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]), "=r"(w[4]), "=r"(w[5]), "=r"(w[6]), "=r"(w[7])
                 : "l"(p));
}
__device__ __forceinline__ void st256(void *p, const uint32_t (&w)[8])
{
    asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
                 "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

// Generic FP32 path for one lane's 16 elements (all 4 lanes of the unit call
// it together; `mask` = the lanes taking this path).
template <int MODE>
__device__ __forceinline__ void slow_lane16(const uint32_t (&w)[8], const uint32_t (&mw)[8], uint32_t q4,
                                         uint32_t mask, uint32_t &bad, uint32_t (&out)[8], uint32_t &meta)
{
    float v[16];
    for (int i = 0; i < 8; ++i) {
        v[2 * i] = sanitize(bf16_lo(w[i] & ~mw[i]), bad);
        v[2 * i + 1] = sanitize(bf16_hi(w[i] & ~mw[i]), bad);
    }
    float a4[4];
    for (int k = 0; k < 4; ++k) {
        a4[k] = 0.0f;
        for (int i = 0; i < 4; ++i) a4[k] = fmaxf(a4[k], fabsf(v[4 * k + i]));
    }
    float a = fmaxf(fmaxf(a4[0], a4[1]), fmaxf(a4[2], a4[3]));
    a = fmaxf(a, __shfl_xor_sync(mask, a, 1));
    a = fmaxf(a, __shfl_xor_sync(mask, a, 2));
    const uint32_t c = select_scale_code(a);
    const float S = e6m2_value(c);
    const float T1 = 1.75f * S, T2 = 3.5f * S;
    const float rS = __frcp_rn(S);
    uint32_t part = 0;
    for (int j = 0; j < 2; ++j) {
        const uint32_t e2 = fmaxf(a4[2 * j], a4[2 * j + 1]) > T2;
        part |= e2 << (8 + 2 * q4 + j);
        for (int h = 0; h < 2; ++h) {
            const int k = 2 * j + h;
            const uint32_t e3 = e2 ? (a4[k] > T2) : (a4[k] > T1);
            part |= e3 << (16 + 4 * q4 + k);
            const int E = (int)(e2 + e3);
            const float step = ldexp_small(S, E - 2), inv = ldexp_small(rS, 2 - E);
            for (int i = 4 * k; i < 4 * k + 4; ++i) {
                const uint32_t m = round_exact(fabsf(v[i]), inv, step);
                const uint32_t sgn = (m != 0u) ? (f_bits(v[i]) >> 31) : 0u;
                if (MODE == 0) {
                    if ((i & 7) == 0) out[i >> 3] = 0;
                    out[i >> 3] |= (m | (sgn << 3)) << (4 * (i & 7));
                } else {
                    v[i] = bits_f(f_bits((float)m * step) | (sgn << 31));
                }
            }
        }
    }
    if (MODE == 0) {
        part |= __shfl_xor_sync(mask, part, 1);
        part |= __shfl_xor_sync(mask, part, 2);
        meta = part | c;
    } else {
        for (int i = 0; i < 8; ++i) {
            const uint32_t y = pack_bf16_exact(v[2 * i], v[2 * i + 1]);
            out[i] = (y & ~mw[i]) | (w[i] & mw[i]);
        }
    }
}

// mw: the protected halves of the 8 input words as 16-bit lane masks (all
// ones where the channel is protected; read only with MASK).
template <bool MASK, int MODE>
__device__ __forceinline__ void encode16(const uint32_t (&w)[8], const uint32_t (&mw)[8], uint32_t q4,
                                         uint32_t &bad, uint32_t (&out)[8], uint32_t &meta)
{
    const u64 MAGIC2 = pk(12582912.0f, 12582912.0f);
    uint32_t mk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) mk[i] = (MASK ? (w[i] & ~mw[i]) : w[i]) & 0x7FFF7FFFu;
    uint32_t A01, A23, A8;
    quarter_max(mk, A01, A23, A8);
    uint32_t ak = max(A8 & 0xFFFFu, A8 >> 16);
    ak = max(ak, __shfl_xor_sync(0xffffffffu, ak, 1));
    ak = max(ak, __shfl_xor_sync(0xffffffffu, ak, 2));
    const uint32_t c = scale_code_from_bits(ak << 16);
    meta = 0;
    const bool slow = ak >= 0x7F80u || c == 255u;                 // unit-uniform
    if (slow) {
        slow_lane16<MODE>(w, mw, q4, __activemask(), bad, out, meta);
    } else {
        const float S = e6m2_value(c);
        Quarter pq;
        plan_quarter(A01, A23, A8, c, S, pq);
        const uint32_t e2_0 = pq.e2_0, e2_1 = pq.e2_1;
        const uint32_t *e3 = pq.e3;
        if (MODE == 0) {
            uint32_t tb[16];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const u64 ax = pk(bits_f(imad(mk[p], 65536u, 0u)), bits_f(mk[p] & 0xFFFF0000u));
                const u64 r = ffma2(ax, pq.HH[p >> 1], fmul2(ax, pq.LL[p >> 1]));
                const u64 t = fadd2(r, MAGIC2);                    // low byte = RNE(r) <= 8
                float tl, th;
                upk(t, tl, th);
                tb[2 * p] = f_bits(tl);
                tb[2 * p + 1] = f_bits(th);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t *t8 = tb + 8 * h;
                const uint32_t *w4 = w + 4 * h;
                // nibble i = t_i - 0x4B400000 = m_i (0..8): a digit sum, no carries
                const uint32_t c01 = imad(t8[1], 16u, t8[0]), c23 = imad(t8[3], 16u, t8[2]);
                const uint32_t c45 = imad(t8[5], 16u, t8[4]), c67 = imad(t8[7], 16u, t8[6]);
                const uint32_t c03 = imad(c23, 256u, c01), c47 = imad(c67, 256u, c45);
                uint32_t C = imad(c47, 65536u, c03 - 0x4B400000u * 0x11111111u);
                const uint32_t nz = (C + 0x77777777u) & 0x88888888u;   // bit 3 of nibble <=> m >= 1
                C -= (C >> 3) & 0x11111111u;                           // m = 8 -> 7 (saturation)
                const uint32_t SE = prmt(prmt(w4[0], w4[1], 0x00D9), prmt(w4[2], w4[3], 0x00D9), 0x5410);
                const uint32_t SO = prmt(prmt(w4[0], w4[1], 0x00FB), prmt(w4[2], w4[3], 0x00FB), 0x5410);
                const uint32_t sg = (SE & 0x0F0F0F0Fu) | (SO & 0xF0F0F0F0u);
                out[h] = C | (sg & nz);                                // sign only where m != 0
            }
            uint32_t part = (e2_0 << (8 + 2 * q4)) | (e2_1 << (9 + 2 * q4)) |
                            ((e3[0] | e3[1] << 1 | e3[2] << 2 | e3[3] << 3) << (16 + 4 * q4));
            part |= __shfl_xor_sync(0xffffffffu, part, 1);
            part |= __shfl_xor_sync(0xffffffffu, part, 2);
            meta = part | c;
        } else {
            fq_quarter<MASK>(w, mw, pq, S, out);
        }
    }
}

constexpr int kUnroll16 = 2;

template <bool MASK, bool CONTIG, int MODE>
__global__ void __launch_bounds__(kThreads, 3) k_quant_bf16(QuantArgs a)
{
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t q4 = lane & 3u;
    const uint32_t nocts = (a.total_units + 7u) >> 3;                 // 8 units per warp step
    const uint32_t gwarp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;
    uint32_t bad = 0;

    for (uint32_t o0 = gwarp; o0 < nocts; o0 += nwarps * kUnroll16) {
        uint32_t raw[kUnroll16][8], mraw[kUnroll16][4] = {}, unit[kUnroll16], row[kUnroll16], cu[kUnroll16];
#pragma unroll
        for (int u = 0; u < kUnroll16; ++u) {
            const uint32_t o = o0 + (uint32_t)u * nwarps;
            unit[u] = o * 8u + (lane >> 2);
            const bool active = o < nocts && unit[u] < a.total_units;
            row[u] = (!CONTIG || MASK) ? a.upr_div.div(unit[u]) : 0u;
            cu[u] = unit[u] - row[u] * a.upr;
            const int64_t e = CONTIG ? (int64_t)unit[u] * HIF4_UNIT + q4 * 16
                                     : (int64_t)row[u] * a.ldx + (int64_t)cu[u] * HIF4_UNIT + q4 * 16;
            if (active) {
                ld256(static_cast<const uint16_t *>(a.x) + e, raw[u]);
            } else {
#pragma unroll
                for (int i = 0; i < 8; ++i) raw[u][i] = 0;
            }
            if (MASK) {
                if (active) {
                    const uint4 m4 = __ldg(reinterpret_cast<const uint4 *>(a.chan_mask + (size_t)cu[u] * HIF4_UNIT + q4 * 16));
                    mraw[u][0] = m4.x; mraw[u][1] = m4.y; mraw[u][2] = m4.z; mraw[u][3] = m4.w;
                } else {
                    mraw[u][0] = mraw[u][1] = mraw[u][2] = mraw[u][3] = 0;
                }
            }
        }
#pragma unroll
        for (int u = 0; u < kUnroll16; ++u) {
            const uint32_t o = o0 + (uint32_t)u * nwarps;
            if (o >= nocts) break;                                      // warp-uniform
            const bool active = unit[u] < a.total_units;
            const uint32_t (&w)[8] = raw[u];
            uint32_t mw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (MASK) mask_words16(mraw[u], mw);
            uint32_t out[8], meta;
            encode16<MASK, MODE>(w, mw, q4, bad, out, meta);
            if (!active) continue;
            if (MODE == 0) {
                asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(a.codes + (size_t)unit[u] * 32 + q4 * 8),
                             "r"(out[0]), "r"(out[1])
                             : "memory");
                if (q4 == 0) a.meta[unit[u]] = meta;
            } else {
                const int64_t e = CONTIG ? (int64_t)unit[u] * HIF4_UNIT + q4 * 16
                                         : (int64_t)row[u] * a.ldo + (int64_t)cu[u] * HIF4_UNIT + q4 * 16;
                st256(static_cast<uint16_t *>(a.out) + e, out);
            }
        }
    }
    if (bad) status_or(a.status, HIF4_FLAG_NONFINITE);
}

// ------------------------------------------- BF16 input, TMA-staged kernel
//
// Contiguous rows only.  A block streams chunks of 64 units (8 KB of BF16)
// through a 6-stage shared-memory ring filled by cp.async.bulk copies that
// complete on per-stage mbarriers, so each SM keeps ~100-150 KB of reads in
// flight without holding them in registers.  Chunks are dealt to blocks
// round-robin; thread t of the block encodes elements [16 (t % 4), +16) of
// unit (chunk * 64 + t / 4) with encode16 above.

#ifndef HIF4_QT_STAGES
#define HIF4_QT_STAGES 6
#endif
#ifndef HIF4_QT_MINB
#define HIF4_QT_MINB 3
#endif
constexpr int kStages = HIF4_QT_STAGES;
constexpr int kChunkUnits = kThreads / 4;                 // 64 units
constexpr uint32_t kChunkBytes = kChunkUnits * HIF4_UNIT * 2;   // 8 KB
constexpr size_t kTmaSmem = (size_t)kStages * kChunkBytes + 128;
constexpr uint64_t kWaitNs = 2000000000ull;               // 2 s: far above any chunk

// FIXED (with MASK): the grid is a multiple of upr / gcd(upr, 64), so the
// chunk stride gridDim.x * 64 units is a whole number of rows and a thread's
// channels are the same in every chunk: its protected-lane masks are built
// once, before the loop.
template <bool MASK, int MODE, bool FIXED>
__global__ void __launch_bounds__(kThreads, HIF4_QT_MINB) k_quant_tma(QuantArgs a)
{
    using namespace sm100;
    extern __shared__ __align__(128) uint8_t sm[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + (size_t)kStages * kChunkBytes);
    __shared__ uint32_t abort_flag;
    const uint32_t tid = threadIdx.x, lane = tid & 31u, q4 = lane & 3u;
    const uint32_t nchunks = (a.total_units + kChunkUnits - 1) / kChunkUnits;
    const uint32_t my_n = nchunks > blockIdx.x ? (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;
    const uint16_t *x = static_cast<const uint16_t *>(a.x);

    if (tid == 0) {
        for (int st = 0; st < kStages; ++st) mbar_init(&full[st], 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    auto issue = [&](uint32_t i) {
        if (a.withhold && blockIdx.x == 0 && i == 0) return;   // its wait can only run out
        const uint32_t chunk = blockIdx.x + i * gridDim.x;
        const uint32_t u0 = chunk * kChunkUnits;
        const uint32_t nu = min((uint32_t)kChunkUnits, a.total_units - u0);
        const uint32_t st = i % kStages;
        mbar_arrive_expect_tx(&full[st], nu * HIF4_UNIT * 2);
        bulk_load(sm + (size_t)st * kChunkBytes, x + (size_t)u0 * HIF4_UNIT, nu * HIF4_UNIT * 2, &full[st]);
    };
    if (tid == 0)
        for (uint32_t i = 0; i < my_n && i < (uint32_t)kStages; ++i) issue(i);

    uint32_t mw_fixed[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (MASK && FIXED) {
        const uint32_t unit0 = blockIdx.x * kChunkUnits + (tid >> 2);
        const uint32_t cu0 = unit0 - a.upr_div.div(unit0) * a.upr;
        const uint4 m4 = __ldg(reinterpret_cast<const uint4 *>(a.chan_mask + (size_t)cu0 * HIF4_UNIT + q4 * 16));
        const uint32_t mraw[4] = {m4.x, m4.y, m4.z, m4.w};
        mask_words16(mraw, mw_fixed);
    }

    uint32_t bad = 0, i = 0;
    for (; i < my_n; ++i) {
        const uint32_t st = i % kStages;
        const uint32_t unit = (blockIdx.x + i * gridDim.x) * kChunkUnits + (tid >> 2);
        const bool active = unit < a.total_units;
        // the mask bytes do not depend on the stage: their load overlaps the wait
        uint32_t mraw[4] = {0, 0, 0, 0};
        if (MASK && !FIXED && active) {
            const uint32_t cu = unit - a.upr_div.div(unit) * a.upr;
            const uint4 m4 = __ldg(reinterpret_cast<const uint4 *>(a.chan_mask + (size_t)cu * HIF4_UNIT + q4 * 16));
            mraw[0] = m4.x; mraw[1] = m4.y; mraw[2] = m4.z; mraw[3] = m4.w;
        }
        const bool ok = mbar_wait_bounded(&full[st], (i / kStages) & 1u, &abort_flag, a.wait_ns);
        uint32_t w[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (ok && active) {
            const uint4 *src = reinterpret_cast<const uint4 *>(sm + (size_t)st * kChunkBytes + tid * 32u);
            const uint4 lo = src[0], hi = src[1];
            w[0] = lo.x; w[1] = lo.y; w[2] = lo.z; w[3] = lo.w;
            w[4] = hi.x; w[5] = hi.y; w[6] = hi.z; w[7] = hi.w;
        }
        // stage st consumed by every thread; leave together if any wait gave up
        if (__syncthreads_or(!ok)) break;
        if (tid == 0 && i + kStages < my_n) issue(i + kStages);
        uint32_t mw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (MASK && FIXED) {
#pragma unroll
            for (int j = 0; j < 8; ++j) mw[j] = mw_fixed[j];
        } else if (MASK) {
            mask_words16(mraw, mw);
        }
        uint32_t out[8], meta;
        encode16<MASK, MODE>(w, mw, q4, bad, out, meta);
        if (!active) continue;
        if (MODE == 0) {
            asm volatile("st.global.v2.u32 [%0], {%1, %2};" ::"l"(a.codes + (size_t)unit * 32 + q4 * 8), "r"(out[0]),
                         "r"(out[1])
                         : "memory");
            if (q4 == 0) a.meta[unit] = meta;
        } else {
            st256(static_cast<uint16_t *>(a.out) + (size_t)unit * HIF4_UNIT + q4 * 16, out);
        }
    }
    if (bad) status_or(a.status, HIF4_FLAG_NONFINITE);
    if (tid == 0 && i < my_n) {
        // gave up: let the copies this block still has in flight land first
        for (uint32_t j = i; j < my_n && j < i + kStages; ++j)
            mbar_wait_bounded(&full[j % kStages], (j / kStages) & 1u, nullptr, 100000000ull);
        status_or(a.status, HIF4_FLAG_TIMEOUT);
    }
}

// ------------------------------- BF16 quantize, 32 elements per lane, TMA 2-D
//
// Halves the per-unit work of encode16 per element: two lanes share a unit,
// each encodes 32 elements (four level-2 groups).  A block stages chunks of
// 128 units (16 KB) with 2-D TMA tile loads whose 128-byte swizzle makes the
// per-lane 64-byte shared-memory reads bank-conflict free: 16-byte piece p of
// unit row r sits at piece p ^ (r % 8).  The per-group scaling 4/(S 2^E) is
// derived from the E = 0 value by subtracting E from the FP32 exponent field.

#ifndef HIF4_Q32_STAGES
#define HIF4_Q32_STAGES 3
#endif
#ifndef HIF4_Q32_MINB
#define HIF4_Q32_MINB 4
#endif
constexpr int kQ32Stages = HIF4_Q32_STAGES;
constexpr int kQ32Units = kThreads / 2;                       // 128 units per chunk
constexpr uint32_t kQ32Bytes = kQ32Units * HIF4_UNIT * 2;     // 16 KB
constexpr size_t kQ32Smem = (size_t)kQ32Stages * kQ32Bytes + 1024 + 128;

// Generic FP32 path for a lane holding NW words (2 NW elements) of a unit
// split over 64 / (2 NW) lanes; `part` = this lane's index within the unit.
template <int NW>
__device__ __forceinline__ void slow_codes(const uint32_t (&w)[NW], const uint32_t (&mw)[NW], uint32_t part_idx,
                                           uint32_t mask, uint32_t &bad, uint32_t (&out)[NW / 4], uint32_t &meta)
{
    constexpr int NE = 2 * NW, NG = NE / 4;
    float v[NE];
    for (int i = 0; i < NW; ++i) {
        v[2 * i] = sanitize(bf16_lo(w[i] & ~mw[i]), bad);
        v[2 * i + 1] = sanitize(bf16_hi(w[i] & ~mw[i]), bad);
    }
    float a4[NG];
    float a = 0.0f;
    for (int k = 0; k < NG; ++k) {
        a4[k] = 0.0f;
        for (int i = 0; i < 4; ++i) a4[k] = fmaxf(a4[k], fabsf(v[4 * k + i]));
        a = fmaxf(a, a4[k]);
    }
    for (int o = 1; o < 64 / NE; o <<= 1) a = fmaxf(a, __shfl_xor_sync(mask, a, o));
    const uint32_t c = select_scale_code(a);
    const float S = e6m2_value(c);
    const float T1 = 1.75f * S, T2 = 3.5f * S;
    const float rS = __frcp_rn(S);
    uint32_t part = 0;
    for (int i = 0; i < NW / 4; ++i) out[i] = 0;
    for (int j = 0; j < NG / 2; ++j) {
        const uint32_t e2 = fmaxf(a4[2 * j], a4[2 * j + 1]) > T2;
        part |= e2 << (8 + (NG / 2) * part_idx + j);
        for (int h = 0; h < 2; ++h) {
            const int k = 2 * j + h;
            const uint32_t e3 = e2 ? (a4[k] > T2) : (a4[k] > T1);
            part |= e3 << (16 + NG * part_idx + k);
            const int E = (int)(e2 + e3);
            const float step = ldexp_small(S, E - 2), inv = ldexp_small(rS, 2 - E);
            for (int i = 4 * k; i < 4 * k + 4; ++i) {
                const uint32_t m = round_exact(fabsf(v[i]), inv, step);
                const uint32_t sgn = (m != 0u) ? (f_bits(v[i]) >> 31) : 0u;
                out[i >> 3] |= (m | (sgn << 3)) << (4 * (i & 7));
            }
        }
    }
    for (int o = 1; o < 64 / NE; o <<= 1) part |= __shfl_xor_sync(mask, part, o);
    meta = part | c;
}

// Codes of 8 elements from their rounded values t (low bits m <= 8) and the
// 4 BF16 words holding them (for the signs).
__device__ __forceinline__ uint32_t pack8(const uint32_t *t8, const uint32_t *w4)
{
    const uint32_t c01 = imad(t8[1], 16u, t8[0]), c23 = imad(t8[3], 16u, t8[2]);
    const uint32_t c45 = imad(t8[5], 16u, t8[4]), c67 = imad(t8[7], 16u, t8[6]);
    const uint32_t c03 = imad(c23, 256u, c01), c47 = imad(c67, 256u, c45);
    uint32_t C = imad(c47, 65536u, c03 - 0x4B400000u * 0x11111111u);    // nibble i = m_i
    const uint32_t nz = (C + 0x77777777u) & 0x88888888u;                // bit 3 <=> m >= 1
    C -= (C >> 3) & 0x11111111u;                                        // m = 8 -> 7
    const uint32_t SE = prmt(prmt(w4[0], w4[1], 0x00D9), prmt(w4[2], w4[3], 0x00D9), 0x5410);
    const uint32_t SO = prmt(prmt(w4[0], w4[1], 0x00FB), prmt(w4[2], w4[3], 0x00FB), 0x5410);
    return C | (((SE & 0x0F0F0F0Fu) | (SO & 0xF0F0F0F0u)) & nz);
}

template <bool MASK>
__device__ __forceinline__ void encode32(const uint32_t (&w)[16], const uint32_t (&mraw)[8], uint32_t p2,
                                         uint32_t &bad, uint32_t (&out)[4], uint32_t &meta)
{
    const u64 MAGIC2 = pk(12582912.0f, 12582912.0f);
    uint32_t mw[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) mw[i] = 0;
    if (MASK) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const uint32_t x = mraw[i];
            const uint32_t nz = (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x);
            mw[2 * i] = prmt(nz, 0, 0x9988);
            mw[2 * i + 1] = prmt(nz, 0, 0xBBAA);
        }
    }
    uint32_t mk[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) mk[i] = w[i] & ~mw[i] & 0x7FFF7FFFu;
    uint32_t A[4];                                           // [a4_2j, a4_2j+1]
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t G0 = max_u16x2(mk[4 * j], mk[4 * j + 1]), G1 = max_u16x2(mk[4 * j + 2], mk[4 * j + 3]);
        A[j] = max_u16x2(prmt(G0, G1, 0x5410), prmt(G0, G1, 0x7632));
    }
    const uint32_t A8a = max_u16x2(prmt(A[0], A[1], 0x5410), prmt(A[0], A[1], 0x7632));   // [a8_0, a8_1]
    const uint32_t A8b = max_u16x2(prmt(A[2], A[3], 0x5410), prmt(A[2], A[3], 0x7632));   // [a8_2, a8_3]
    const uint32_t m2 = max_u16x2(A8a, A8b);
    uint32_t ak = max(m2 & 0xFFFFu, m2 >> 16);
    ak = max(ak, __shfl_xor_sync(0xffffffffu, ak, 1));
    const uint32_t c = scale_code_from_bits(ak << 16);
    if (ak >= 0x7F80u || c == 255u) {                        // unit-uniform
        slow_codes<16>(w, mw, p2, __activemask(), bad, out, meta);
        return;
    }
    const float S = e6m2_value(c);
    const uint32_t T1 = f_bits(1.75f * S) >> 16, T2 = f_bits(3.5f * S) >> 16;
    // Level decisions on pairs of 16-bit keys (all below 0x8000): key > T
    // exactly when bit 15 of key + 0x7FFF - T is set, with no carry into the
    // other half.  e2 of the 8-groups from their maxima; the 4-groups' e3
    // against T2 where e2 is set, else T1 (selected by a byte-permute mask).
    const uint32_t K1 = (0x7FFFu - T1) * 0x10001u, K2 = (0x7FFFu - T2) * 0x10001u;
    const uint32_t G2a = (A8a + K2) & 0x80008000u, G2b = (A8b + K2) & 0x80008000u;
    float ih, il;
    recip_pair(c & 3u, ih, il);
    if ((c & 3u) == 0) il = bits_f(0x21800000u);             // 2^-60: keeps the exponent arithmetic valid
    const float pw0 = bits_f((160u - (c >> 2)) << 23);       // 2^(33 - E6)
    const uint32_t H0 = f_bits(ih * pw0), L0 = f_bits(il * pw0);
    uint32_t Hk[8], Lk[8], Z = 0;                            // per 4-group: H0, L0 scaled by 2^-E
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t G = j < 2 ? G2a : G2b;
        const uint32_t Mj = prmt(G, 0, (j & 1) ? 0xBBBBu : 0x9999u);        // all ones where e2_j
        const uint32_t P1 = (A[j] + K1) & 0x80008000u, P2 = (A[j] + K2) & 0x80008000u;
        const uint32_t y = ((P1 & ~Mj) | (P2 & Mj)) >> 15;                  // e3 of 4-groups 2j (bit 0), 2j+1 (bit 16)
        const uint32_t Ep = y + (Mj & 0x10001u);                             // [E_2j, E_2j+1] in 16-bit halves
        Hk[2 * j] = imad(Ep, 0xFF800000u, H0);                               // (the high half vanishes mod 2^32)
        Lk[2 * j] = imad(Ep, 0xFF800000u, L0);
        Hk[2 * j + 1] = imad(Ep & 0xFFFF0000u, 0xFFFFFF80u, H0);
        Lk[2 * j + 1] = imad(Ep & 0xFFFF0000u, 0xFFFFFF80u, L0);
        Z = imad(y, 1u << (2 * j), Z);
    }
    const uint32_t u2 = (G2a >> 15) | (G2b >> 13);           // e2 of 8-groups 0, 2 at bits 0, 2; 1, 3 at 16, 18
    const uint32_t e2bits = (u2 & 5u) | ((u2 >> 15) & 0xAu);
    const uint32_t e3bits = (Z & 0x55u) | ((Z >> 15) & 0xAAu);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        uint32_t tb[16];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
            const int k = 4 * hh + (p >> 1);
            const float H = bits_f(Hk[k]), L = bits_f(Lk[k]);   // exponent - E
            const uint32_t m = mk[8 * hh + p];
            const u64 ax = pk(bits_f(imad(m, 65536u, 0u)), bits_f(m & 0xFFFF0000u));
            const u64 r = ffma2(ax, pk(H, H), fmul2(ax, pk(L, L)));
            float tl, th;
            upk(fadd2(r, MAGIC2), tl, th);
            tb[2 * p] = f_bits(tl);
            tb[2 * p + 1] = f_bits(th);
        }
        out[2 * hh] = pack8(tb, w + 8 * hh);
        out[2 * hh + 1] = pack8(tb + 8, w + 8 * hh + 4);
    }
    uint32_t part = (e2bits << (8 + 4 * p2)) | (e3bits << (16 + 8 * p2));
    part |= __shfl_xor_sync(0xffffffffu, part, 1);
    meta = part | c;
}

template <bool MASK>
__global__ void __launch_bounds__(kThreads, HIF4_Q32_MINB) k_quant32(const __grid_constant__ CUtensorMap tm, QuantArgs a)
{
    using namespace sm100;
    extern __shared__ uint8_t sm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(sm_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + (size_t)kQ32Stages * kQ32Bytes);
    __shared__ uint32_t abort_flag;
    const uint32_t tid = threadIdx.x, p2 = tid & 1u, r = tid >> 1;
    const uint32_t nchunks = (a.total_units + kQ32Units - 1) / kQ32Units;
    const uint32_t my_n = nchunks > blockIdx.x ? (nchunks - blockIdx.x + gridDim.x - 1) / gridDim.x : 0u;

    if (tid == 0) {
        for (int st = 0; st < kQ32Stages; ++st) mbar_init(&full[st], 1);
        abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm);
    }
    __syncthreads();
    auto issue = [&](uint32_t i) {
        if (a.withhold && blockIdx.x == 0 && i == 0) return;   // its wait can only run out
        const uint32_t st = i % kQ32Stages;
        mbar_arrive_expect_tx(&full[st], kQ32Bytes);
        tma_load_2d(sm + (size_t)st * kQ32Bytes, &tm, 0, (int32_t)((blockIdx.x + i * gridDim.x) * kQ32Units),
                    &full[st]);
    };
    if (tid == 0)
        for (uint32_t i = 0; i < my_n && i < (uint32_t)kQ32Stages; ++i) issue(i);

    uint32_t bad = 0, i = 0;
    for (; i < my_n; ++i) {
        const uint32_t st = i % kQ32Stages;
        const bool ok = mbar_wait_bounded(&full[st], (i / kQ32Stages) & 1u, &abort_flag, a.wait_ns);
        const uint32_t unit = (blockIdx.x + i * gridDim.x) * kQ32Units + r;
        const bool active = unit < a.total_units;
        uint32_t w[16];
        if (ok) {
            const uint8_t *row = sm + (size_t)st * kQ32Bytes + r * 128u;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint4 v = *reinterpret_cast<const uint4 *>(row + (((4u * p2 + kk) ^ (r & 7u)) << 4));
                w[4 * kk] = v.x; w[4 * kk + 1] = v.y; w[4 * kk + 2] = v.z; w[4 * kk + 3] = v.w;
            }
        } else {
#pragma unroll
            for (int k = 0; k < 16; ++k) w[k] = 0;
        }
        if (__syncthreads_or(!ok)) break;                    // stage consumed; leave together on a time-out
        if (tid == 0 && i + kQ32Stages < my_n) issue(i + kQ32Stages);
        uint32_t mraw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (MASK && active) {
            const uint32_t cu = unit - a.upr_div.div(unit) * a.upr;
            const uint4 *mp = reinterpret_cast<const uint4 *>(a.chan_mask + (size_t)cu * HIF4_UNIT + p2 * 32);
            const uint4 m0 = __ldg(mp), m1 = __ldg(mp + 1);
            mraw[0] = m0.x; mraw[1] = m0.y; mraw[2] = m0.z; mraw[3] = m0.w;
            mraw[4] = m1.x; mraw[5] = m1.y; mraw[6] = m1.z; mraw[7] = m1.w;
        }
        uint32_t out[4], meta;
        encode32<MASK>(w, mraw, p2, bad, out, meta);
        if (!active) continue;
        asm volatile("st.global.v4.u32 [%0], {%1, %2, %3, %4};" ::"l"(a.codes + (size_t)unit * 32 + p2 * 16),
                     "r"(out[0]), "r"(out[1]), "r"(out[2]), "r"(out[3])
                     : "memory");
        if (p2 == 0) a.meta[unit] = meta;
    }
    if (bad) status_or(a.status, HIF4_FLAG_NONFINITE);
    if (tid == 0 && i < my_n) {
        for (uint32_t j = i; j < my_n && j < i + kQ32Stages; ++j)
            mbar_wait_bounded(&full[j % kQ32Stages], (j / kQ32Stages) & 1u, nullptr, 100000000ull);
        status_or(a.status, HIF4_FLAG_TIMEOUT);
    }
}

template <bool MASK>
hif4_status launch_quant32(const QuantArgs &qa, cudaStream_t s, bool &done)
{
    done = false;
    CUtensorMap tm;
    if (!make_tensor_map_bf16_2d(&tm, qa.x, HIF4_UNIT, qa.total_units, HIF4_UNIT * 2, HIF4_UNIT, kQ32Units, true))
        return HIF4_OK;                                      // no encoder: caller uses another kernel
    auto k = k_quant32<MASK>;
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr[dev & 63]) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kQ32Smem) != cudaSuccess)
            return HIF4_ERR_CUDA;
        attr[dev & 63] = true;
    }
    const uint32_t nchunks = (qa.total_units + kQ32Units - 1) / kQ32Units;
    int grid = blocks_per_sm(reinterpret_cast<const void *>(k), kThreads, kQ32Smem) * sm_count();
    if ((uint32_t)grid > nchunks) grid = (int)nchunks;
    k<<<grid, kThreads, kQ32Smem, s>>>(tm, qa);
    done = true;
    return launch_status();
}

// ------------------------------------------------------------- dequantize

struct DequantArgs {
    const uint8_t *codes;
    const uint32_t *meta;
    void *y;
    int64_t ldy;
    uint32_t upr;
    FastDiv upr_div;
    uint32_t total_units;
};


template <bool F32OUT, bool CONTIG>
__global__ void __launch_bounds__(kThreads) k_dequant(DequantArgs a)
{
    __shared__ __align__(16) uint32_t tab[4][4];       // [f] = {low bytes m 0-3, 4-7, high bytes m 0-3, 4-7}
    if (!F32OUT) {
        if (threadIdx.x < 16)
            tab[threadIdx.x >> 2][threadIdx.x & 3u] = dequant_table_word(threadIdx.x >> 2, threadIdx.x & 3u);
        __syncthreads();
    }
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t lane8 = lane & 7u;
    const uint32_t nquads = (a.total_units + 3u) >> 2;
    const uint32_t gwarp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;

    for (uint32_t q0 = gwarp; q0 < nquads; q0 += nwarps * kDqUnroll) {
        uint32_t cw[kDqUnroll], mw[kDqUnroll], unit[kDqUnroll];
#pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const uint32_t q = q0 + (uint32_t)u * nwarps;
            unit[u] = q * 4u + (lane >> 3);
            if (q < nquads && unit[u] < a.total_units) {
                asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];"
                             : "=r"(cw[u]) : "l"(a.codes + (size_t)unit[u] * 32 + lane8 * 4));
                mw[u] = __ldg(a.meta + unit[u]);
            } else {
                cw[u] = 0;
                mw[u] = 0;
            }
        }
#pragma unroll
        for (int u = 0; u < kDqUnroll; ++u) {
            const uint32_t q = q0 + (uint32_t)u * nwarps;
            if (q >= nquads) break;
            if (unit[u] >= a.total_units) continue;
            const uint32_t w = mw[u];
            const uint32_t e2 = (w >> (8 + lane8)) & 1u;
            const uint32_t e3lo = (w >> (16 + 2 * lane8)) & 1u;
            const uint32_t e3hi = (w >> (17 + 2 * lane8)) & 1u;
            float o[8];
            uint32_t ob[4];
            if (F32OUT) {
                const float S = e6m2_value(w & 0xFFu);
                const float step_lo = ldexp_small(S, (int)(e2 + e3lo) - 2);
                const float step_hi = ldexp_small(S, (int)(e2 + e3hi) - 2);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const uint32_t nib = (cw[u] >> (4 * i)) & 15u;
                    const float mf = bits_f(0x4B000000u | (nib & 7u)) - 8388608.0f;   // exact m
                    const float q = mf * (i < 4 ? step_lo : step_hi);
                    o[i] = bits_f(f_bits(q) | ((nib >> 3) << 31));
                }
            } else {
                const uint4 T = *reinterpret_cast<const uint4 *>(tab[w & 3u]);
                dequant8_bf16(cw[u], (w & 0xFFu) >> 2, e2 + e3lo, e2 + e3hi, T, ob);
            }
            int64_t off;
            if (CONTIG) {
                off = (int64_t)unit[u] * HIF4_UNIT + lane8 * 8;
            } else {
                const uint32_t r = a.upr_div.div(unit[u]);
                const uint32_t cu = unit[u] - r * a.upr;
                off = (int64_t)r * a.ldy + (int64_t)cu * HIF4_UNIT + lane8 * 8;
            }
            if (F32OUT) {
                float4 *p = reinterpret_cast<float4 *>(static_cast<float *>(a.y) + off);
                p[0] = make_float4(o[0], o[1], o[2], o[3]);
                p[1] = make_float4(o[4], o[5], o[6], o[7]);
            } else {
                *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.y) + off) = make_uint4(ob[0], ob[1], ob[2], ob[3]);
            }
        }
    }
}

template <typename K>
int grid_for(K kernel, uint32_t total_units, int unroll = kUnroll)
{
    const int per_sm = blocks_per_sm(reinterpret_cast<const void *>(kernel), kThreads, 0);
    const uint64_t quads = (total_units + 3ull) / 4ull;
    const uint64_t warps_needed = (quads + unroll - 1) / unroll;
    const uint64_t blocks_needed = (warps_needed + kThreads / 32 - 1) / (kThreads / 32);
    uint64_t g = (uint64_t)per_sm * (uint64_t)sm_count();
    if (blocks_needed < g) g = blocks_needed;
    return (int)(g < 1 ? 1 : g);
}

template <typename K>
int grid_for16(K kernel, uint32_t total_units)
{
    const int per_sm = blocks_per_sm(reinterpret_cast<const void *>(kernel), kThreads, 0);
    const uint64_t octs = (total_units + 7ull) / 8ull;
    const uint64_t warps_needed = (octs + kUnroll16 - 1) / kUnroll16;
    const uint64_t blocks_needed = (warps_needed + kThreads / 32 - 1) / (kThreads / 32);
    uint64_t g = (uint64_t)per_sm * (uint64_t)sm_count();
    if (blocks_needed < g) g = blocks_needed;
    return (int)(g < 1 ? 1 : g);
}

// Opts the kernel into kTmaSmem of dynamic shared memory (once per device).
template <bool MASK, int MODE, bool FIXED>
bool quant_tma_attr()
{
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr[dev & 63]) {
        if (cudaFuncSetAttribute(k_quant_tma<MASK, MODE, FIXED>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kTmaSmem) != cudaSuccess)
            return false;
        attr[dev & 63] = true;
    }
    return true;
}

template <bool MASK, int MODE, bool FIXED>
hif4_status launch_quant_tma_grid(const QuantArgs &qa, int grid, cudaStream_t s)
{
    if (!quant_tma_attr<MASK, MODE, FIXED>()) return HIF4_ERR_CUDA;
    k_quant_tma<MASK, MODE, FIXED><<<grid, kThreads, kTmaSmem, s>>>(qa);
    return launch_status();
}

template <bool MASK, int MODE>
hif4_status launch_quant_tma(const QuantArgs &qa, cudaStream_t s)
{
    if (!quant_tma_attr<MASK, MODE, false>()) return HIF4_ERR_CUDA;
    const uint32_t nchunks = (qa.total_units + kChunkUnits - 1) / kChunkUnits;
    int grid = blocks_per_sm(reinterpret_cast<const void *>(k_quant_tma<MASK, MODE, false>), kThreads, kTmaSmem) *
               sm_count();
    if ((uint32_t)grid > nchunks) grid = (int)nchunks;
    if (MASK) {
        // the largest grid whose chunk stride is a whole number of rows, if
        // it keeps at least 7/8 of the blocks
        uint32_t g = qa.upr, b = (uint32_t)kChunkUnits;
        while (b) {
            const uint32_t r = g % b;
            g = b;
            b = r;
        }
        const uint32_t step = qa.upr / g;
        const uint32_t gf = ((uint32_t)grid / step) * step;
        if (gf >= 1 && gf * 8 >= (uint32_t)grid * 7) return launch_quant_tma_grid<MASK, MODE, MASK>(qa, (int)gf, s);
    }
    return launch_quant_tma_grid<MASK, MODE, false>(qa, grid, s);
}

template <bool BF16, bool MASK, int MODE>
hif4_status launch_quant(const QuantArgs &qa0, bool contig, bool fast, cudaStream_t s)
{
    QuantArgs qa = qa0;
    qa.withhold = wait_test_withhold();
    qa.wait_ns = wait_limit_ns(kWaitNs);
    if (BF16 && MODE == 0 && fast && contig) {
        bool done = false;
        const hif4_status st = launch_quant32<MASK>(qa, s, done);
        if (done || st != HIF4_OK) return st;
    }
    if (BF16 && fast && contig) return launch_quant_tma<MASK, MODE>(qa, s);
    if (BF16 && fast) {
        if (contig) {
            auto k = k_quant_bf16<MASK, true, MODE>;
            k<<<grid_for16(k, qa.total_units), kThreads, 0, s>>>(qa);
        } else {
            auto k = k_quant_bf16<MASK, false, MODE>;
            k<<<grid_for16(k, qa.total_units), kThreads, 0, s>>>(qa);
        }
        return launch_status();
    }
    if (contig) {
        auto k = k_quant<BF16, MASK, true, MODE>;
        k<<<grid_for(k, qa.total_units), kThreads, 0, s>>>(qa);
    } else {
        auto k = k_quant<BF16, MASK, false, MODE>;
        k<<<grid_for(k, qa.total_units), kThreads, 0, s>>>(qa);
    }
    return launch_status();
}

hif4_status check_units(int64_t rows, int64_t cols)
{
    if (rows < 0 || cols < 0) return HIF4_ERR_INVALID_ARG;
    if (cols % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (rows > 0 && cols > 0 && (uint64_t)rows * (uint64_t)(cols / HIF4_UNIT) >= (1ull << 32) - 64)
        return HIF4_ERR_UNSUPPORTED;
    return HIF4_OK;
}

} // namespace

// Internal entry used by the linear layer (BF16 in, BF16 out).
hif4_status fake_quantize_bf16(const void *x, int64_t rows, int64_t cols, int64_t ldx,
                               const uint8_t *chan_mask, void *xhat, int64_t ldxh,
                               uint32_t *status, cudaStream_t s)
{
    if (rows == 0 || cols == 0) return HIF4_OK;
    QuantArgs qa{};
    qa.x = x;
    qa.ldx = ldx;
    qa.chan_mask = chan_mask;
    qa.out = xhat;
    qa.ldo = ldxh;
    qa.upr = (uint32_t)(cols / HIF4_UNIT);
    qa.upr_div = FastDiv(qa.upr);
    qa.total_units = (uint32_t)(rows * (cols / HIF4_UNIT));
    qa.status = status;
    const bool contig = (ldx == cols) && (ldxh == cols);
    // 256-bit accesses need 32-byte aligned rows; otherwise the 16-byte kernel
    const bool fast = aligned_to(x, 32) && aligned_to(xhat, 32) && (ldx * 2) % 32 == 0 && (ldxh * 2) % 32 == 0 &&
                      (!chan_mask || aligned_to(chan_mask, 16));
    return chan_mask ? launch_quant<true, true, 1>(qa, contig, fast, s)
                     : launch_quant<true, false, 1>(qa, contig, fast, s);
}

} // namespace hif4

using namespace hif4;

extern "C" hif4_status hif4_quantize(const void *x, hif4_dtype dtype, int64_t rows, int64_t cols,
                                     int64_t ldx, const uint8_t *chan_mask, uint8_t *codes,
                                     uint32_t *meta, uint32_t *status, hif4_stream_t stream)
{
    hif4_status st = check_units(rows, cols);
    if (st != HIF4_OK) return st;
    if (dtype != HIF4_F32 && dtype != HIF4_BF16) return HIF4_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return HIF4_OK;
    if (!x || !codes || !meta) return HIF4_ERR_INVALID_ARG;
    if (ldx < cols) return HIF4_ERR_SHAPE;
    const int64_t esz = dtype == HIF4_BF16 ? 2 : 4;
    if (!aligned16(x) || (ldx * esz) % 16 != 0) return HIF4_ERR_ALIGNMENT;
    if (!aligned_to(codes, 4) || !aligned_to(meta, 4) || (chan_mask && !aligned_to(chan_mask, 8)))
        return HIF4_ERR_ALIGNMENT;
    QuantArgs qa{};
    qa.x = x;
    qa.ldx = ldx;
    qa.chan_mask = chan_mask;
    qa.codes = codes;
    qa.meta = meta;
    qa.upr = (uint32_t)(cols / HIF4_UNIT);
    qa.upr_div = FastDiv(qa.upr);
    qa.total_units = (uint32_t)(rows * (cols / HIF4_UNIT));
    qa.status = status;
    const bool contig = ldx == cols;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // 256-bit loads need 32-byte aligned rows; otherwise the 16-byte kernel
    const bool fast = aligned_to(x, 32) && (ldx * 2) % 32 == 0 && aligned_to(codes, 8) &&
                      (!chan_mask || aligned_to(chan_mask, 16));
    if (dtype == HIF4_BF16)
        return chan_mask ? launch_quant<true, true, 0>(qa, contig, fast, s)
                         : launch_quant<true, false, 0>(qa, contig, fast, s);
    return chan_mask ? launch_quant<false, true, 0>(qa, contig, false, s)
                     : launch_quant<false, false, 0>(qa, contig, false, s);
}

extern "C" hif4_status hif4_dequantize(const uint8_t *codes, const uint32_t *meta, int64_t rows,
                                       int64_t cols, hif4_dtype out_dtype, void *y, int64_t ldy,
                                       hif4_stream_t stream)
{
    hif4_status st = check_units(rows, cols);
    if (st != HIF4_OK) return st;
    if (out_dtype != HIF4_F32 && out_dtype != HIF4_BF16) return HIF4_ERR_INVALID_ARG;
    if (rows == 0 || cols == 0) return HIF4_OK;
    if (!codes || !meta || !y) return HIF4_ERR_INVALID_ARG;
    if (ldy < cols) return HIF4_ERR_SHAPE;
    const int64_t esz = out_dtype == HIF4_BF16 ? 2 : 4;
    if (!aligned16(y) || (ldy * esz) % 16 != 0) return HIF4_ERR_ALIGNMENT;
    if (!aligned_to(codes, 4) || !aligned_to(meta, 4)) return HIF4_ERR_ALIGNMENT;
    DequantArgs da{codes, meta, y, ldy, (uint32_t)(cols / HIF4_UNIT), FastDiv((uint32_t)(cols / HIF4_UNIT)),
                   (uint32_t)(rows * (cols / HIF4_UNIT))};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const bool contig = ldy == cols;
    if (out_dtype == HIF4_F32) {
        if (contig) { auto k = k_dequant<true, true>; k<<<grid_for(k, da.total_units, kDqUnroll), kThreads, 0, s>>>(da); }
        else { auto k = k_dequant<true, false>; k<<<grid_for(k, da.total_units, kDqUnroll), kThreads, 0, s>>>(da); }
    } else {
        if (contig) { auto k = k_dequant<false, true>; k<<<grid_for(k, da.total_units, kDqUnroll), kThreads, 0, s>>>(da); }
        else { auto k = k_dequant<false, false>; k<<<grid_for(k, da.total_units, kDqUnroll), kThreads, 0, s>>>(da); }
    }
    return launch_status();
}

extern "C" hif4_status hif4_fake_quantize(const void *x, int64_t rows, int64_t cols, int64_t ldx,
                                          const uint8_t *chan_mask, void *xhat, int64_t ldxh,
                                          uint32_t *status, hif4_stream_t stream)
{
    hif4_status st = check_units(rows, cols);
    if (st != HIF4_OK) return st;
    if (rows == 0 || cols == 0) return HIF4_OK;
    if (!x || !xhat) return HIF4_ERR_INVALID_ARG;
    if (ldx < cols || ldxh < cols) return HIF4_ERR_SHAPE;
    if (!aligned16(x) || !aligned16(xhat) || (ldx * 2) % 16 != 0 || (ldxh * 2) % 16 != 0)
        return HIF4_ERR_ALIGNMENT;
    if (chan_mask && !aligned_to(chan_mask, 8)) return HIF4_ERR_ALIGNMENT;
    return fake_quantize_bf16(x, rows, cols, ldx, chan_mask, xhat, ldxh, status,
                              reinterpret_cast<cudaStream_t>(stream));
}
