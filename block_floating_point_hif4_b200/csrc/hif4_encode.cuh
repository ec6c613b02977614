// hif4_encode.cuh — exact FP32 HiF4 element arithmetic shared by the
// streaming quantizers and the GEMM epilogue.
//
// Encode rule [Huawei HiF4 calibration article, section 1; the rule itself is
// the library's reading of a step the page leaves open]:
//   S   = largest E6M2 value with 6.5 S < max|x| over the 64-element unit,
//   t   = 0/1/2 for each 4-group by max4 <= 1.75 S / <= 3.5 S / more,
//   e2  = [max t of the 8-group == 2],  e3 = max(0, t - e2),
//   m   = RNE(|x| / (S 2^(e2+e3) / 4)), ties to even, min 7.
// The fast path works on 16-bit BF16 magnitude keys (bits & 0x7FFF, whose
// order is the |x| order):
//   * the scale code comes from the bits of the unit maximum a: within a's
//     binade the four thresholds 6.5 v(c) sit at mantissa offsets
//     2^17 {1, 14, 27, 40}, so c = 4 (e - 99) + #{thresholds below};
//   * 1.75 S and 3.5 S are exact BF16 values, so the group exponents are
//     integer comparisons of keys;
//   * |x| / step = |x| (H + L) with H + L a two-term expansion of
//     16 / (4 + f) (times a power of two): for BF16 inputs the FP32 result
//     of fma(|x|, H, |x| L) is exact at every rounding tie and at least 1/448
//     away from a tie otherwise, so round-to-nearest-even by the 1.5 * 2^23
//     magic addition is exact.  Products run as packed f32x2 operations.
// Units with a non-finite input or a scale clamped at the top code (255) take
// the generic FP32 path (sanitize, exact half-way comparisons).
#pragma once

#include "hif4_internal.cuh"

namespace hif4 {
namespace enc {

typedef unsigned long long u64;

__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
// PTX prmt (byte permute); a selector nibble with bit 3 set replicates the
// sign bit of the selected byte into the whole byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
// a * b + c on the integer multiply-add path (keeps byte/nibble packing off
// the ALU pipe).
__device__ __forceinline__ uint32_t imad(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("mad.lo.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ u64 pk(float lo, float hi)
{
    u64 r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void upk(u64 v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ u64 fmul2(u64 a, u64 b)
{
    u64 d;
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ u64 ffma2(u64 a, u64 b, u64 c)
{
    u64 d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ u64 fadd2(u64 a, u64 b)
{
    u64 d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}

// Scale code from the FP32 bits of the unit maximum (exact; see above).
__device__ __forceinline__ uint32_t scale_code_from_bits(uint32_t bits)
{
    const int32_t ea = (int32_t)(bits >> 23);
    const int32_t qm = ((int32_t)(bits & 0x7FFFFFu) - 1) >> 17;       // -1 .. 63
    int32_t f = ((qm + 12) * 79) >> 10;                                 // floor((qm + 12) / 13)
    f = f > 4 ? 4 : f;
    int32_t c = ((ea - 99) << 2) + f;
    c = c < 0 ? 0 : c;
    return (uint32_t)(c > 255 ? 255 : c);
}

// 4 / (4 + f) as an unevaluated sum hi + lo of two FP32 values.
__device__ __forceinline__ void recip_pair(uint32_t f, float &hi, float &lo)
{
    const uint32_t h = f == 0 ? 0x3F800000u : f == 1 ? 0x3F4CCCCDu : f == 2 ? 0x3F2AAAABu : 0x3F124925u;
    const uint32_t l = f == 0 ? 0u : f == 1 ? 0xB24CCCCDu : f == 2 ? 0xB2AAAAABu : 0xB2DB6DB7u;
    hi = bits_f(h);
    lo = bits_f(l);
}

// Exact RNE of |x| / step onto 0..7 (generic path).
__device__ __forceinline__ uint32_t round_exact(float ax, float inv, float step)
{
    float k = floorf(fminf(ax * inv, 7.0f));
    float mid = fmaf(k, step, 0.5f * step);       // (k + 1/2) step, exact
    uint32_t ki = (uint32_t)k;
    uint32_t up = (ax > mid) || (ax == mid && (ki & 1u));
    uint32_t m = ki + up;
    return m > 7u ? 7u : m;
}

// Protected-column masks of 16 elements: 16 mask bytes (4 words) -> 8 words
// of 16-bit lanes, all ones where the mask byte is nonzero.
__device__ __forceinline__ void mask_words16(const uint32_t *mraw, uint32_t *mw)
{
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t x = mraw[i];
        const uint32_t nz = (((x & 0x7F7F7F7Fu) + 0x7F7F7F7Fu) | x);   // bit 7 set <=> byte != 0
        mw[2 * i] = prmt(nz, 0, 0x9988);                            // bytes 0,0,1,1 (sign-replicated)
        mw[2 * i + 1] = prmt(nz, 0, 0xBBAA);                        // bytes 2,2,3,3
    }
}

// Maxima keys of a 16-element quarter from its 8 masked key words
// (mk[i] = BF16 pair with protected halves zeroed and signs cleared):
// A01 / A23 = the four level-3 (4-element) maxima as 16-bit pairs,
// A8 = the two level-2 (8-element) maxima.
__device__ __forceinline__ void quarter_max(const uint32_t *mk, uint32_t &A01, uint32_t &A23, uint32_t &A8)
{
    const uint32_t G0 = max_u16x2(mk[0], mk[1]), G1 = max_u16x2(mk[2], mk[3]);
    const uint32_t G2 = max_u16x2(mk[4], mk[5]), G3 = max_u16x2(mk[6], mk[7]);
    A01 = max_u16x2(prmt(G0, G1, 0x5410), prmt(G0, G1, 0x7632));
    A23 = max_u16x2(prmt(G2, G3, 0x5410), prmt(G2, G3, 0x7632));
    A8 = max_u16x2(prmt(A01, A23, 0x5410), prmt(A01, A23, 0x7632));
}

// Level decisions and per-4-group reciprocal factors of one quarter, given
// the unit's scale code c (< 255) and S = v(c).
struct Quarter {
    uint32_t e2_0, e2_1, e3[4];
    u64 HH[4], LL[4];
};

__device__ __forceinline__ void plan_quarter(uint32_t A01, uint32_t A23, uint32_t A8, uint32_t c, float S,
                                             Quarter &p)
{
    const uint32_t T1 = f_bits(1.75f * S) >> 16, T2 = f_bits(3.5f * S) >> 16;
    const uint32_t a4[4] = {A01 & 0xFFFFu, A01 >> 16, A23 & 0xFFFFu, A23 >> 16};
    p.e2_0 = (A8 & 0xFFFFu) > T2;
    p.e2_1 = (A8 >> 16) > T2;
    const uint32_t th0 = p.e2_0 ? T2 : T1, th1 = p.e2_1 ? T2 : T1;
    p.e3[0] = a4[0] > th0;
    p.e3[1] = a4[1] > th0;
    p.e3[2] = a4[2] > th1;
    p.e3[3] = a4[3] > th1;
    float ih, il;
    recip_pair(c & 3u, ih, il);
    const uint32_t E6 = c >> 2;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t E = (k < 2 ? p.e2_0 : p.e2_1) + p.e3[k];
        const float pw = bits_f((160u - E6 - E) << 23);                 // 2^(33 - E6 - E)
        p.HH[k] = pk(ih * pw, ih * pw);
        p.LL[k] = pk(il * pw, il * pw);
    }
}

// Fake-quantized BF16 pairs of one quarter (fast path): w = the 8 input
// words, mw = protected halves (MASK only; passed through unchanged).  The
// two halves of a pair are computed independently and a protected half's
// result is replaced by its input, so the products run on w unmasked.
template <bool MASK>
__device__ __forceinline__ void fq_quarter(const uint32_t *w, const uint32_t *mw, const Quarter &p, float S,
                                           uint32_t *out)
{
    const u64 MAGIC2 = pk(12582912.0f, 12582912.0f);
    const u64 NMAGIC2 = pk(-12582912.0f, -12582912.0f);
    u64 ST[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const uint32_t E = (k < 2 ? p.e2_0 : p.e2_1) + p.e3[k];
        const float st = ldexp_small(S, (int)E - 2);
        ST[k] = pk(st, st);
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        const u64 x = pk(bits_f(w[q] << 16), bits_f(w[q] & 0xFFFF0000u));
        const u64 r = ffma2(x, p.HH[q >> 1], fmul2(x, p.LL[q >> 1]));
        const u64 mf = fadd2(fadd2(r, MAGIC2), NMAGIC2);   // signed RNE(r), +0 when 0
        float ml, mh;
        upk(mf, ml, mh);
        ml = fminf(fmaxf(ml, -7.0f), 7.0f);
        mh = fminf(fmaxf(mh, -7.0f), 7.0f);
        float yl, yh;
        upk(fmul2(pk(ml, mh), ST[q >> 1]), yl, yh);
        const uint32_t y = pack_bf16_exact(yl, yh);
        out[q] = MASK ? ((y & ~mw[q]) | (w[q] & mw[q])) : y;
    }
}

// Generic FP32 fake-quant of one whole unit held by one thread (non-finite
// inputs, or the scale clamped at code 255).  w: 32 words of BF16 pairs
// (element 2i in the low half of w[i]); mw as in fq_quarter.  Fully unrolled
// so that the caller's arrays stay in registers.
template <bool MASK>
__device__ __forceinline__ void fq_unit64_generic(const uint32_t *w, const uint32_t *mw, uint32_t *out,
                                                  uint32_t &bad)
{
    float a4[16];
#pragma unroll
    for (int k = 0; k < 16; ++k) {
        a4[k] = 0.0f;
#pragma unroll
        for (int i = 2 * k; i < 2 * k + 2; ++i) {
            const uint32_t wz = MASK ? (w[i] & ~mw[i]) : w[i];
            a4[k] = fmaxf(a4[k], fmaxf(fabsf(sanitize(bf16_lo(wz), bad)), fabsf(sanitize(bf16_hi(wz), bad))));
        }
    }
    float a = 0.0f;
#pragma unroll
    for (int k = 0; k < 16; ++k) a = fmaxf(a, a4[k]);
    const uint32_t c = select_scale_code(a);
    const float S = e6m2_value(c);
    const float T1 = 1.75f * S, T2 = 3.5f * S;
    const float rS = __frcp_rn(S);
    uint32_t seen = 0;                                  // already reported above
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t e2 = fmaxf(a4[2 * j], a4[2 * j + 1]) > T2;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int k = 2 * j + h;
            const uint32_t e3 = e2 ? (a4[k] > T2) : (a4[k] > T1);
            const int E = (int)(e2 + e3);
            const float step = ldexp_small(S, E - 2), inv = ldexp_small(rS, 2 - E);
#pragma unroll
            for (int i = 2 * k; i < 2 * k + 2; ++i) {
                const uint32_t wz = MASK ? (w[i] & ~mw[i]) : w[i];
                const float v0 = sanitize(bf16_lo(wz), seen), v1 = sanitize(bf16_hi(wz), seen);
                const uint32_t m0 = round_exact(fabsf(v0), inv, step), m1 = round_exact(fabsf(v1), inv, step);
                const uint32_t s0 = m0 ? (f_bits(v0) >> 31) : 0u, s1 = m1 ? (f_bits(v1) >> 31) : 0u;
                const float y0 = bits_f(f_bits((float)m0 * step) | (s0 << 31));
                const float y1 = bits_f(f_bits((float)m1 * step) | (s1 << 31));
                const uint32_t y = pack_bf16_exact(y0, y1);
                out[i] = MASK ? ((y & ~mw[i]) | (w[i] & mw[i])) : y;
            }
        }
    }
}

// Fake-quantizes one 64-element unit held entirely by one thread:
// out = deq(q(w with protected halves -> 0)), protected halves passed
// through.  w, mw, out: 32 words each (mw read only with MASK).
template <bool MASK>
__device__ __forceinline__ void fq_unit64(const uint32_t *w, const uint32_t *mw, uint32_t *out, uint32_t &bad)
{
    uint32_t A01[4], A23[4], A8[4];
    uint32_t ak = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t mk[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) mk[i] = (MASK ? (w[8 * q + i] & ~mw[8 * q + i]) : w[8 * q + i]) & 0x7FFF7FFFu;
        quarter_max(mk, A01[q], A23[q], A8[q]);
        ak = max(ak, max(A8[q] & 0xFFFFu, A8[q] >> 16));
    }
    const uint32_t c = scale_code_from_bits(ak << 16);
    if (ak >= 0x7F80u || c == 255u) {
        fq_unit64_generic<MASK>(w, mw, out, bad);
        return;
    }
    const float S = e6m2_value(c);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        Quarter p;
        plan_quarter(A01[q], A23[q], A8[q], c, S, p);
        fq_quarter<MASK>(w + 8 * q, mw + 8 * q, p, S, out + 8 * q);
    }
}

// BF16 decode of 8 elements by byte permutes (the dequantizer's and the
// weight-decoding GEMM's).  Table word [f][which] for the scale fraction f:
// the low (which < 2) or high bytes of the BF16 pattern of m (4 + f) 2^-35
// for m = 0-3 (which even) or 4-7 (which odd), four per word.
__device__ __forceinline__ uint32_t dequant_table_word(uint32_t f, uint32_t which)
{
    uint32_t v = 0;
    for (uint32_t k = 0; k < 4; ++k) {
        const uint32_t m = (which & 1u) * 4u + k;
        const uint32_t t = m ? f_bits((float)(m * (4u + f)) * 0x1p-35f) >> 16 : 0u;
        v |= ((which >> 1) ? (t >> 8) : (t & 0xFFu)) << (8 * k);
    }
    return v;
}

// BF16 output by byte-permute lookups.  Element value m S 2^(E-2) with
// S = 2^(e6-31) (1 + f/4) equals [m (4 + f)] 2^-35 2^(e6 + E): the BF16 bits
// of the first factor (small integers scaled by 2^-35, exact) form one
// 8-entry table per f, split into low and high bytes; one prmt looks up 4
// elements' bytes at once, and adding (e6 + E) << 7 to a BF16 pair word
// scales both halves (every result is a normal number, no carry crosses the
// halves).  m = 0 entries are masked to zero; the sign bit is the code's.
__device__ __forceinline__ void dequant8_bf16(uint32_t cw, uint32_t e6, uint32_t Elo, uint32_t Ehi, uint4 T,
                                              uint32_t (&out)[4])
{
    const uint32_t n8 = ((cw & 0x77777777u) + 0x77777777u) & 0x88888888u;   // bit 3 of nibble: m != 0
    const uint32_t nA = n8 << 4, sA = cw << 4;                              // byte MSBs: even nibbles
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const uint32_t sel = (cw >> (16 * half)) & 0x7777u;
        const uint32_t lo4 = prmt(T.x, T.y, sel), hi4 = prmt(T.z, T.w, sel);
        const uint32_t add = imad((e6 + (half ? Ehi : Elo)) << 7, 0x10001u, 0u);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int k = 2 * half + j;
            const uint32_t v = prmt(lo4, hi4, j ? 0x7362u : 0x5140u);
            const uint32_t msk = prmt(nA, n8, 0xCC88u + 0x1111u * k);      // 0xFFFF halves where m != 0
            const uint32_t sg = prmt(sA, cw, 0xC888u + 0x1111u * k) & 0x80008000u;
            out[k] = ((v + add) & msk) | sg;
        }
    }
}

} // namespace enc
} // namespace hif4
