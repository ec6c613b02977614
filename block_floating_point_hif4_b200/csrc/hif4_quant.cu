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

#include "hif4_internal.cuh"

namespace hif4 {

namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

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
};

// Exact RNE of |x| / step onto 0..7 (slow path).
__device__ __forceinline__ uint32_t round_exact(float ax, float inv, float step)
{
    float k = floorf(fminf(ax * inv, 7.0f));
    float mid = fmaf(k, step, 0.5f * step);       // (k + 1/2) step, exact
    uint32_t ki = (uint32_t)k;
    uint32_t up = (ax > mid) || (ax == mid && (ki & 1u));
    uint32_t m = ki + up;
    return m > 7u ? 7u : m;
}

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
    const uint32_t lane = threadIdx.x & 31u;
    const uint32_t lane8 = lane & 7u;
    const uint32_t nquads = (a.total_units + 3u) >> 2;
    const uint32_t gwarp = (blockIdx.x * kThreads + threadIdx.x) >> 5;
    const uint32_t nwarps = (gridDim.x * kThreads) >> 5;

    for (uint32_t q0 = gwarp; q0 < nquads; q0 += nwarps * kUnroll) {
        uint32_t cw[kUnroll], mw[kUnroll], unit[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
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
        for (int u = 0; u < kUnroll; ++u) {
            const uint32_t q = q0 + (uint32_t)u * nwarps;
            if (q >= nquads) break;
            if (unit[u] >= a.total_units) continue;
            const uint32_t w = mw[u];
            const float S = e6m2_value(w & 0xFFu);
            const uint32_t e2 = (w >> (8 + lane8)) & 1u;
            const uint32_t e3lo = (w >> (16 + 2 * lane8)) & 1u;
            const uint32_t e3hi = (w >> (17 + 2 * lane8)) & 1u;
            const float step_lo = ldexp_small(S, (int)(e2 + e3lo) - 2);
            const float step_hi = ldexp_small(S, (int)(e2 + e3hi) - 2);
            float o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const uint32_t nib = (cw[u] >> (4 * i)) & 15u;
                const float mf = bits_f(0x4B000000u | (nib & 7u)) - 8388608.0f;   // exact m
                const float q = mf * (i < 4 ? step_lo : step_hi);
                o[i] = bits_f(f_bits(q) | ((nib >> 3) << 31));
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
                *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(a.y) + off) =
                    make_uint4(pack_bf16_exact(o[0], o[1]), pack_bf16_exact(o[2], o[3]),
                               pack_bf16_exact(o[4], o[5]), pack_bf16_exact(o[6], o[7]));
            }
        }
    }
}

template <typename K>
int grid_for(K kernel, uint32_t total_units)
{
    const int per_sm = blocks_per_sm(reinterpret_cast<const void *>(kernel), kThreads, 0);
    const uint64_t quads = (total_units + 3ull) / 4ull;
    const uint64_t warps_needed = (quads + kUnroll - 1) / kUnroll;
    const uint64_t blocks_needed = (warps_needed + kThreads / 32 - 1) / (kThreads / 32);
    uint64_t g = (uint64_t)per_sm * (uint64_t)sm_count();
    if (blocks_needed < g) g = blocks_needed;
    return (int)(g < 1 ? 1 : g);
}

template <bool BF16, bool MASK, int MODE>
hif4_status launch_quant(const QuantArgs &qa, bool contig, cudaStream_t s)
{
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
    return chan_mask ? launch_quant<true, true, 1>(qa, contig, s)
                     : launch_quant<true, false, 1>(qa, contig, s);
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
    if (dtype == HIF4_BF16)
        return chan_mask ? launch_quant<true, true, 0>(qa, contig, s) : launch_quant<true, false, 0>(qa, contig, s);
    return chan_mask ? launch_quant<false, true, 0>(qa, contig, s) : launch_quant<false, false, 0>(qa, contig, s);
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
        if (contig) { auto k = k_dequant<true, true>; k<<<grid_for(k, da.total_units), kThreads, 0, s>>>(da); }
        else { auto k = k_dequant<true, false>; k<<<grid_for(k, da.total_units), kThreads, 0, s>>>(da); }
    } else {
        if (contig) { auto k = k_dequant<false, true>; k<<<grid_for(k, da.total_units), kThreads, 0, s>>>(da); }
        else { auto k = k_dequant<false, false>; k<<<grid_for(k, da.total_units), kThreads, 0, s>>>(da); }
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
