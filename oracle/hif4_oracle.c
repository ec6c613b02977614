/*
 * hif4_oracle.c — plain, slow CPU reference for the HiF4 W4A4 hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This file defines what "correct" means for the
 * CUDA library; it shares no code, header, table or constant generator with
 * it.  Only the tests, the package smoke check and the benchmark's CPU
 * baseline / reference arm may load it.  The product path never does.
 *
 * Arithmetic is IEEE double throughout (every HiF4 quantity is exact in
 * double); loops are written in the order the method states its steps, with
 * no blocking or fusion.
 *
 * Sources, cited by page title and section:
 *   [HiF4 format]  Huawei HiF4 calibration article (hwcomputing.csdn.net),
 *                  section 1 "HiFloat4 (HiF4) format" and its Fig. 1.
 *   [HiGPTQ]       same article, section 3.1 (groups of 64 along the
 *                  input-channel columns of W).
 *   [HiAutoRound]  same article, section 3.2 (E' = E + RZ(K) on the level-3
 *                  exponent: a larger exponent means a larger value).
 *   [TA abstract]  "Tail-Aware HiFloat4: W4A4 Post-Training Quantization for
 *                  Wan2.2", arXiv 2605.26628 record, abstract.
 *   [TA summary]   agents-report.net summary of the same report, "Method
 *                  overview" and "Why tail percentiles".
 * Where those pages leave a step open, the reading taken is stated beside the
 * step and marked "[reading]".
 *
 * Parity pins: every function below is pinned by the CPU tests in
 * tests/test_oracle_*.py (invariants, brute force, textbook routines).
 */
#include <float.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_UNIT 64

/* ---------------------------------------------------------------- scalars */

/* BF16 bit pattern -> double (exact widening). */
static double orc_bf16_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* E6M2 level-1 scale value [HiF4 format; reading: unsigned, bias 31, no
 * specials]:  v(code) = 2^(E-31) * (1 + f/4),  code = E<<2 | f. */
double orc_e6m2_value(int code)
{
    int E = (code >> 2) & 63;
    int f = code & 3;
    return ldexp(1.0 + f / 4.0, E - 31);
}

/* Level-1 scale choice [reading]: the largest code whose value v satisfies
 * 6.5 * v < a; code 0 when none does (a <= 6.5 * 2^-31, a = 0 included). */
int orc_select_scale_code(double a)
{
    int best = 0;
    for (int c = 0; c < 256; ++c)
        if (6.5 * orc_e6m2_value(c) < a)
            best = c;
    return best;
}

/* Round |x| onto the element grid {0, step, 2 step, ..., 7 step} to the
 * nearest point, ties to the even multiple, saturating at 7 [reading].
 * step = S * 2^E / 4 is the spacing of the S1P2 magnitudes m/4 [HiF4 format].
 * The half-way points (m + 1/2) * step are exact in double, so each
 * comparison is exact. */
int orc_round_magnitude(double ax, double step)
{
    for (int m = 0; m < 7; ++m) {
        double mid = (m + 0.5) * step;
        if (ax < mid)
            return m;
        if (ax == mid)
            return (m % 2 == 0) ? m : m + 1;
    }
    return 7;
}

/* ------------------------------------------------------------ one unit */

/* Quantize one 64-element unit [HiF4 format; encode rule: reading].
 *   x      64 finite values (already mapped from NaN/Inf by the caller)
 *   masked 64 flags or NULL; a masked element counts as 0 and gets code 0
 *   nib    out: 64 codes, bit 3 = sign, bits 2..0 = m
 *   meta   out: c | e2 << 8 | e3 << 16 */
void orc_quantize_unit(const double *x, const unsigned char *masked,
                       unsigned char *nib, uint32_t *meta)
{
    double v[ORC_UNIT];
    for (int i = 0; i < ORC_UNIT; ++i)
        v[i] = (masked && masked[i]) ? 0.0 : x[i];

    /* step 2: unit maximum -> level-1 scale */
    double a = 0.0;
    for (int i = 0; i < ORC_UNIT; ++i)
        if (fabs(v[i]) > a)
            a = fabs(v[i]);
    int c = orc_select_scale_code(a);
    double S = orc_e6m2_value(c);

    /* step 3: exponent need of each 4-element group */
    int t[16];
    for (int k = 0; k < 16; ++k) {
        double a4 = 0.0;
        for (int i = 4 * k; i < 4 * k + 4; ++i)
            if (fabs(v[i]) > a4)
                a4 = fabs(v[i]);
        if (a4 <= 1.75 * S)
            t[k] = 0;
        else if (a4 <= 3.5 * S)
            t[k] = 1;
        else
            t[k] = 2;
    }

    /* steps 4-5: level-2 bit per 8 elements, level-3 bit per 4 elements */
    int e2[8], e3[16];
    for (int j = 0; j < 8; ++j) {
        int tm = t[2 * j] > t[2 * j + 1] ? t[2 * j] : t[2 * j + 1];
        e2[j] = (tm == 2) ? 1 : 0;
    }
    for (int k = 0; k < 16; ++k) {
        int r = t[k] - e2[k / 2];
        e3[k] = r > 0 ? r : 0;
    }

    /* step 6: element codes */
    for (int i = 0; i < ORC_UNIT; ++i) {
        int E = e2[i / 8] + e3[i / 4];
        double step = S * ldexp(1.0, E) / 4.0;
        int m = orc_round_magnitude(fabs(v[i]), step);
        int s = (v[i] < 0.0 && m > 0) ? 1 : 0;
        nib[i] = (unsigned char)((s << 3) | m);
    }

    uint32_t w = (uint32_t)c;
    for (int j = 0; j < 8; ++j)
        w |= (uint32_t)e2[j] << (8 + j);
    for (int k = 0; k < 16; ++k)
        w |= (uint32_t)e3[k] << (16 + k);
    *meta = w;
}

/* Decode element i of a unit [HiF4 format; decode sign convention: reading,
 * supported by HiAutoRound]:  y = (-1)^s * (m/4) * 2^(e2 + e3) * v(c). */
double orc_decode_element(unsigned nib, uint32_t meta, int i)
{
    int c = (int)(meta & 0xFFu);
    int e2 = (int)((meta >> (8 + i / 8)) & 1u);
    int e3 = (int)((meta >> (16 + i / 4)) & 1u);
    int m = (int)(nib & 7u);
    int s = (int)((nib >> 3) & 1u);
    double y = (m / 4.0) * ldexp(1.0, e2 + e3) * orc_e6m2_value(c);
    return s ? -y : y;
}

/* --------------------------------------------------------------- tensors */

/* Map a non-finite input as the encode rule states [reading]: NaN -> 0,
 * +-Inf -> +-FLT_MAX.  Counts what it mapped. */
static double orc_sanitize(double v, long *n_nonfinite)
{
    if (isnan(v)) {
        ++*n_nonfinite;
        return 0.0;
    }
    if (isinf(v)) {
        ++*n_nonfinite;
        return v > 0 ? (double)FLT_MAX : -(double)FLT_MAX;
    }
    return v;
}

/* Quantize a row-major rows x cols matrix along its rows in units of 64
 * [HiGPTQ: groups run along the input-channel dimension].
 *   dtype 0: x is float; dtype 1: x is BF16 bit patterns (uint16).
 *   chan_mask: NULL or cols flags (nonzero = masked column).
 *   codes: rows x cols/2 bytes, element 2b in the low nibble of byte b.
 *   meta:  rows x cols/64 words.
 * Returns the number of non-finite inputs, or -1 on a bad shape. */
long orc_quantize(const void *x, int dtype, long rows, long cols, long ldx,
                  const unsigned char *chan_mask, unsigned char *codes,
                  uint32_t *meta)
{
    if (cols % ORC_UNIT != 0 || ldx < cols || rows < 0)
        return -1;
    long n_nonfinite = 0;
    long upr = cols / ORC_UNIT;
    for (long r = 0; r < rows; ++r) {
        for (long u = 0; u < upr; ++u) {
            double xv[ORC_UNIT];
            unsigned char nib[ORC_UNIT];
            for (int i = 0; i < ORC_UNIT; ++i) {
                long col = u * ORC_UNIT + i;
                double v;
                if (dtype == 0)
                    v = (double)((const float *)x)[r * ldx + col];
                else
                    v = orc_bf16_to_double(((const uint16_t *)x)[r * ldx + col]);
                xv[i] = orc_sanitize(v, &n_nonfinite);
            }
            uint32_t w;
            orc_quantize_unit(xv, chan_mask ? chan_mask + u * ORC_UNIT : NULL,
                              nib, &w);
            meta[r * upr + u] = w;
            for (int i = 0; i < ORC_UNIT; i += 2)
                codes[r * (cols / 2) + (u * ORC_UNIT + i) / 2] =
                    (unsigned char)(nib[i] | (nib[i + 1] << 4));
        }
    }
    return n_nonfinite;
}

/* Dequantize a rows x cols HiF4 matrix into doubles (y has stride ldy). */
void orc_dequantize(const unsigned char *codes, const uint32_t *meta,
                    long rows, long cols, double *y, long ldy)
{
    long upr = cols / ORC_UNIT;
    for (long r = 0; r < rows; ++r)
        for (long col = 0; col < cols; ++col) {
            unsigned byte = codes[r * (cols / 2) + col / 2];
            unsigned nib = (col % 2 == 0) ? (byte & 15u) : (byte >> 4);
            uint32_t w = meta[r * upr + col / ORC_UNIT];
            y[r * ldy + col] = orc_decode_element(nib, w, (int)(col % ORC_UNIT));
        }
}

/* Activation fake quantization [TA abstract: W4A4 fake quantization of the
 * main linears; mask semantics: reading]:  xhat = deq(q(x with masked -> 0)),
 * and xhat = x on the masked channels.  x: BF16 rows x cols, stride ldx.
 * mask_idx: n_masked column indices (any order).  Output rows x cols
 * doubles (dense).  Returns the number of non-finite inputs, -1 on bad args. */
long orc_fake_quantize(const uint16_t *x, long rows, long cols, long ldx,
                       const int32_t *mask_idx, int n_masked, double *xhat)
{
    unsigned char *mask = calloc((size_t)(cols > 0 ? cols : 1), 1);
    unsigned char *codes = malloc((size_t)(cols / 2 > 0 ? cols / 2 : 1));
    uint32_t *meta = malloc(sizeof(uint32_t) * (size_t)(cols / 64 > 0 ? cols / 64 : 1));
    long n_nonfinite = 0;
    if (!mask || !codes || !meta || cols % ORC_UNIT != 0) {
        free(mask); free(codes); free(meta);
        return -1;
    }
    for (int j = 0; j < n_masked; ++j) {
        if (mask_idx[j] < 0 || mask_idx[j] >= cols) {
            free(mask); free(codes); free(meta);
            return -1;
        }
        mask[mask_idx[j]] = 1;
    }
    for (long r = 0; r < rows; ++r) {
        long nf = orc_quantize(x + r * ldx, 1, 1, cols, cols, mask, codes, meta);
        n_nonfinite += nf;
        orc_dequantize(codes, meta, 1, cols, xhat + r * cols, cols);
        for (long col = 0; col < cols; ++col)
            if (mask[col])
                xhat[r * cols + col] = orc_bf16_to_double(x[r * ldx + col]);
    }
    free(mask); free(codes); free(meta);
    return n_nonfinite;
}

/* Dequantized weight with the protected columns restored from BF16
 * [TA abstract; mask semantics: reading].  codes/meta: N x K HiF4;
 * w_masked: N x n_masked BF16 (row n holds W[n, mask_idx[0..]]).
 * Output N x K doubles. */
void orc_weight_hat(const unsigned char *codes, const uint32_t *meta,
                    long N, long K, const int32_t *mask_idx, int n_masked,
                    const uint16_t *w_masked, double *what)
{
    orc_dequantize(codes, meta, N, K, what, K);
    for (long n = 0; n < N; ++n)
        for (int j = 0; j < n_masked; ++j)
            what[n * K + mask_idx[j]] = orc_bf16_to_double(w_masked[n * n_masked + j]);
}

/* tanh-form GELU (the FFN activation; standard definition, not on the
 * pages):  0.5 x (1 + tanh(sqrt(2/pi) (x + 0.044715 x^3))). */
double orc_gelu_tanh(double x)
{
    const double k = sqrt(2.0 / 3.14159265358979323846);
    return 0.5 * x * (1.0 + tanh(k * (x + 0.044715 * x * x * x)));
}

/* double -> BF16 bit pattern in one rounding: to nearest, ties to even (no
 * intermediate FP32 rounding) [reading: the FFN's hidden activation is held
 * in BF16 between the two linears].  BF16 keeps 8 significant bits, so the
 * quantum is 2^(e-8) for |x| = m 2^e (m in [0.5, 1)), and 2^-133 below the
 * normal range.  Magnitudes at or above the midpoint past the largest finite
 * BF16 value go to Inf; NaN gives the quiet NaN with the input's sign. */
uint16_t orc_round_bf16(double x)
{
    if (isnan(x)) return signbit(x) ? 0xFFC0u : 0x7FC0u;
    const uint16_t sign = signbit(x) ? 0x8000u : 0u;
    const double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80u;
    int e;
    frexp(a, &e);
    int qe = e - 8;
    if (qe < -133) qe = -133;
    const double q = ldexp(1.0, qe);
    const double r = nearbyint(a / q) * q;          /* a / q exact; default mode = ties to even */
    if (r > ldexp(255.0, 120)) return sign | 0x7F80u;
    const float f = (float)r;                        /* exact: r is a BF16 value */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return sign | (uint16_t)(u >> 16);
}

void orc_round_bf16_array(const double *x, long n, uint16_t *out)
{
    for (long i = 0; i < n; ++i) out[i] = orc_round_bf16(x[i]);
}

/* Fake-quantized linear layer [TA abstract]:  y = xhat * what^T + bias,
 * summed in double;  with gelu != 0 the GELU above is applied to each output.
 *   xhat M x K, what N x K, bias N or NULL, y M x N (all dense, row-major). */
void orc_linear(const double *xhat, const double *what, const double *bias,
                long M, long N, long K, int gelu, double *y)
{
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k)
                acc += xhat[m * K + k] * what[n * K + k];
            if (bias)
                acc += bias[n];
            y[m * N + n] = gelu ? orc_gelu_tanh(acc) : acc;
        }
}

/* ------------------------------------------------- calibration statistics */

static int orc_cmp_u16(const void *a, const void *b)
{
    uint16_t x = *(const uint16_t *)a, y = *(const uint16_t *)b;
    return (x > y) - (x < y);
}

/* Per-channel tail percentile [TA summary "Why tail percentiles"; rank rule:
 * reading]: for each of the C channels (columns) of the T x C BF16 matrix,
 * sort the 15-bit magnitude keys (bits & 0x7FFF) ascending and take the one at
 * 0-based rank k = floor(q_num * (T-1) / q_den).  pct[c] is that key, i.e. the
 * non-negative BF16 value.  Returns 0, or -1 on bad arguments. */
int orc_percentile(const uint16_t *acts, long T, long C, long lda,
                   unsigned q_num, unsigned q_den, uint16_t *pct)
{
    if (T <= 0 || C <= 0 || lda < C || q_den == 0 || q_num > q_den)
        return -1;
    uint16_t *col = malloc(sizeof(uint16_t) * (size_t)T);
    if (!col)
        return -1;
    long k = (long)(((unsigned long long)q_num * (unsigned long long)(T - 1)) / q_den);
    for (long c = 0; c < C; ++c) {
        for (long t = 0; t < T; ++t)
            col[t] = (uint16_t)(acts[t * lda + c] & 0x7FFFu);
        qsort(col, (size_t)T, sizeof(uint16_t), orc_cmp_u16);
        pct[c] = col[k];
    }
    free(col);
    return 0;
}

typedef struct {
    uint16_t key;
    long idx;
} orc_rank_item;

/* Order: key descending, channel index ascending. */
static int orc_cmp_rank(const void *a, const void *b)
{
    const orc_rank_item *x = a, *y = b;
    if (x->key != y->key)
        return x->key > y->key ? -1 : 1;
    return (x->idx > y->idx) - (x->idx < y->idx);
}

/* Channel mask from the percentiles [TA summary; median over channels and
 * tie rule: reading].  med = lower median over channels of pct;
 * ratio[c] = float(pct[c]) / float(med) in IEEE single precision (+Inf / 0
 * when med = 0); mask marks the floor(C * mask_num / mask_den) channels with
 * the largest pct, ties broken by lower channel index.  Returns the number of
 * masked channels, or -1 on bad arguments. */
long orc_channel_mask(const uint16_t *pct, long C, unsigned mask_num,
                      unsigned mask_den, float *ratio, unsigned char *mask)
{
    if (C <= 0 || mask_den == 0 || mask_num > mask_den)
        return -1;
    uint16_t *sorted = malloc(sizeof(uint16_t) * (size_t)C);
    orc_rank_item *items = malloc(sizeof(orc_rank_item) * (size_t)C);
    if (!sorted || !items) {
        free(sorted); free(items);
        return -1;
    }
    memcpy(sorted, pct, sizeof(uint16_t) * (size_t)C);
    qsort(sorted, (size_t)C, sizeof(uint16_t), orc_cmp_u16);
    uint16_t med_key = sorted[(C - 1) / 2];
    float med = (float)orc_bf16_to_double(med_key);
    for (long c = 0; c < C; ++c) {
        float p = (float)orc_bf16_to_double(pct[c]);
        if (med_key == 0)
            ratio[c] = (pct[c] & 0x7FFFu) ? INFINITY : 0.0f;
        else
            ratio[c] = p / med;
        items[c].key = (uint16_t)(pct[c] & 0x7FFFu);
        items[c].idx = c;
        mask[c] = 0;
    }
    long n_top = (long)(((unsigned long long)C * mask_num) / mask_den);
    qsort(items, (size_t)C, sizeof(orc_rank_item), orc_cmp_rank);
    for (long j = 0; j < n_top; ++j)
        mask[items[j].idx] = 1;
    free(sorted);
    free(items);
    return n_top;
}

/* ----------------------------------------------------------------- HiGPTQ */

/* Upper-triangular error-feedback factor of GPTQ, as HiGPTQ uses it [HiF4
 * article, section 3.1 (HiGPTQ is GPTQ adapted to the HiF4 unit); GPTQ's
 * Hessian factor]:
 *   Hd = H + damp * mean(diag H) * I, after a zero diagonal entry (an input
 *        channel that never fires) is set to 1 and flagged dead;
 *   Hd^{-1} = U^T U with U upper triangular.
 * Steps as stated: Cholesky factor of Hd, the inverse from it, the Cholesky
 * factor of that inverse.  H and U are K x K, row-major.  dead: K flags or
 * NULL.  Returns 0, or -1 when Hd is not positive definite. */
int orc_gptq_factor(const double *H, long K, double damp, double *U, unsigned char *dead)
{
    double *A = malloc(sizeof(double) * K * K);
    double *Li = calloc((size_t)K * K, sizeof(double));
    if (!A || !Li) {
        free(A);
        free(Li);
        return -1;
    }
    memcpy(A, H, sizeof(double) * K * K);
    double mean = 0.0;
    for (long i = 0; i < K; ++i) {
        int d = A[i * K + i] == 0.0;
        if (d) A[i * K + i] = 1.0;
        if (dead) dead[i] = (unsigned char)d;
        mean += A[i * K + i];
    }
    mean /= (double)K;
    for (long i = 0; i < K; ++i) A[i * K + i] += damp * mean;
    int rc = 0;
    /* 1. Hd = L L^T (lower L, in the lower triangle of A) */
    for (long j = 0; j < K && rc == 0; ++j) {
        double s = A[j * K + j];
        for (long k = 0; k < j; ++k) s -= A[j * K + k] * A[j * K + k];
        if (!(s > 0.0)) {
            rc = -1;
            break;
        }
        A[j * K + j] = sqrt(s);
        for (long i = j + 1; i < K; ++i) {
            double t = A[i * K + j];
            for (long k = 0; k < j; ++k) t -= A[i * K + k] * A[j * K + k];
            A[i * K + j] = t / A[j * K + j];
        }
    }
    if (rc == 0) {
        /* 2. L^{-1} (lower), then Hd^{-1} = L^{-T} L^{-1} into U's storage */
        for (long j = 0; j < K; ++j) {
            Li[j * K + j] = 1.0 / A[j * K + j];
            for (long i = j + 1; i < K; ++i) {
                double t = 0.0;
                for (long k = j; k < i; ++k) t += A[i * K + k] * Li[k * K + j];
                Li[i * K + j] = -t / A[i * K + i];
            }
        }
        for (long i = 0; i < K; ++i)
            for (long j = 0; j < K; ++j) {
                double t = 0.0;
                for (long k = i > j ? i : j; k < K; ++k) t += Li[k * K + i] * Li[k * K + j];
                U[i * K + j] = t;
            }
        /* 3. Hd^{-1} = C C^T (lower C), U = C^T */
        memcpy(A, U, sizeof(double) * K * K);
        for (long j = 0; j < K && rc == 0; ++j) {
            double s = A[j * K + j];
            for (long k = 0; k < j; ++k) s -= A[j * K + k] * A[j * K + k];
            if (!(s > 0.0)) {
                rc = -1;
                break;
            }
            A[j * K + j] = sqrt(s);
            for (long i = j + 1; i < K; ++i) {
                double t = A[i * K + j];
                for (long k = 0; k < j; ++k) t -= A[i * K + k] * A[j * K + k];
                A[i * K + j] = t / A[j * K + j];
            }
        }
        for (long i = 0; i < K && rc == 0; ++i)
            for (long j = 0; j < K; ++j) U[i * K + j] = j >= i ? A[j * K + i] : 0.0;
    }
    free(A);
    free(Li);
    return rc;
}

/* HiGPTQ, scheme one [HiF4 article, section 3.1, first scheme: 64 columns are
 * quantized at a time; the level-1, level-2 and level-3 exponents of the
 * group are fixed together, then the remaining weights of the block are
 * updated].  W: N x K BF16 bits (row-major; a group of 64 columns is one HiF4
 * unit per row).  U, dead: from orc_gptq_factor.  Per group g of the block
 * [b0, b1) (blocksize a multiple of 64), for each row:
 *   Q_g = the unit quantized from the row's current values (encode rule of
 *         orc_quantize_unit, protected columns excluded from the scale);
 *         a protected column's value is the BF16 rounding of its current
 *         weight (what the product uses), since it is not HiF4-coded;
 *   D   = W_g - Q_g,   E = D U_gg^{-1}   (E U_gg = D, U_gg upper),
 *   W_c -= E U_{g,c} for the later columns c of the block;
 * then, once per block, W_c -= E_block U_{block,c} for the columns after it
 * [GPTQ's error feedback and its lazy blocked update, here per group].
 * Dead input channels are zeroed first.  Outputs: codes (N x K/2), meta
 * (N x K/64), wq (N x K quantized values, protected columns included) and
 * w_masked (N x n_masked BF16 bits of the protected columns in ascending
 * order; may be NULL).  Returns 0, or -1 on bad arguments. */
long orc_higptq1(const uint16_t *w, long N, long K, const double *U, const unsigned char *dead,
                 const unsigned char *chan_mask, long blocksize, unsigned char *codes, uint32_t *meta,
                 double *wq, uint16_t *w_masked)
{
    if (N <= 0 || K <= 0 || K % ORC_UNIT || blocksize <= 0 || blocksize % ORC_UNIT) return -1;
    double *W = malloc(sizeof(double) * K);
    double *E = malloc(sizeof(double) * blocksize);
    if (!W || !E) {
        free(W);
        free(E);
        return -1;
    }
    for (long n = 0; n < N; ++n) {
        for (long k = 0; k < K; ++k) W[k] = (dead && dead[k]) ? 0.0 : orc_bf16_to_double(w[n * K + k]);
        for (long b0 = 0; b0 < K; b0 += blocksize) {
            const long b1 = b0 + blocksize < K ? b0 + blocksize : K;
            for (long g0 = b0; g0 < b1; g0 += ORC_UNIT) {
                unsigned char nib[ORC_UNIT];
                uint32_t m;
                orc_quantize_unit(W + g0, chan_mask ? chan_mask + g0 : NULL, nib, &m);
                double D[ORC_UNIT];
                for (int i = 0; i < ORC_UNIT; ++i) {
                    const long col = g0 + i;
                    double q;
                    if (chan_mask && chan_mask[col])
                        q = orc_bf16_to_double(orc_round_bf16(W[col]));
                    else
                        q = orc_decode_element(nib[i], m, i);
                    wq[n * K + col] = q;
                    D[i] = W[col] - q;
                    if (i % 2 == 0) codes[n * (K / 2) + col / 2] = 0;
                    codes[n * (K / 2) + col / 2] |= (unsigned char)(nib[i] << (4 * (i % 2)));
                }
                meta[n * (K / ORC_UNIT) + g0 / ORC_UNIT] = m;
                /* E U_gg = D, U_gg upper triangular: forward over the columns */
                for (int j = 0; j < ORC_UNIT; ++j) {
                    double t = D[j];
                    for (int i = 0; i < j; ++i) t -= E[g0 - b0 + i] * U[(g0 + i) * K + g0 + j];
                    E[g0 - b0 + j] = t / U[(g0 + j) * K + g0 + j];
                }
                /* the later columns of this block */
                for (long c = g0 + ORC_UNIT; c < b1; ++c) {
                    double t = 0.0;
                    for (int j = 0; j < ORC_UNIT; ++j) t += E[g0 - b0 + j] * U[(g0 + j) * K + c];
                    W[c] -= t;
                }
            }
            /* the columns after the block, once */
            for (long c = b1; c < K; ++c) {
                double t = 0.0;
                for (long j = b0; j < b1; ++j) t += E[j - b0] * U[j * K + c];
                W[c] -= t;
            }
        }
    }
    free(W);
    free(E);
    if (w_masked && chan_mask) {
        long nm = 0;
        for (long k = 0; k < K; ++k) nm += chan_mask[k] != 0;
        for (long n = 0; n < N; ++n) {
            long j = 0;
            for (long k = 0; k < K; ++k)
                if (chan_mask[k]) w_masked[n * nm + j++] = orc_round_bf16(wq[n * K + k]);
        }
    }
    return 0;
}
