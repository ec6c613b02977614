/*
 * hif4.h — C ABI of libhif4: the data-parallel hot path of Tail-Aware
 * HiFloat4 W4A4 post-training quantization on NVIDIA B200 (sm_100a).
 *
 * Sources, cited by page title and section:
 *   [HiF4 format]  Huawei HiF4 calibration article (hwcomputing.csdn.net),
 *                  section 1 "HiFloat4 (HiF4) format" (64-element unit, E6M2
 *                  level-1 scale, 8 + 16 E1 micro-exponents, S1P2 elements).
 *   [HiGPTQ]       same article, section 3.1 (units run along the input
 *                  channels, i.e. along the reduction dimension K).
 *   [TA abstract]  "Tail-Aware HiFloat4: W4A4 Post-Training Quantization for
 *                  Wan2.2", arXiv 2605.26628 record, abstract (W4A4 fake
 *                  quantization of the main linears, tail-aware percentile
 *                  calibration for channel-mask construction).
 *   [TA summary]   agents-report.net summary of that report, "Method
 *                  overview" and "Why tail percentiles".
 *
 * Numerics (decode sign convention, encode rule, percentile rank and mask
 * rule — the parts the pages leave open) are fixed in the repository's
 * specification and restated in each call's comment below.
 *
 * Conventions for every call:
 *   - Ownership: the caller allocates every buffer; the library allocates
 *     nothing and keeps no state between calls except, per device, one
 *     resolved driver entry point (tensor-map encoder) and cached occupancy.
 *   - Pointers named x, y, codes, meta, acts, pct, ratio, mask, workspace,
 *     status are DEVICE pointers unless stated otherwise.
 *   - Execution: asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  Arguments are checked on the host before any launch;
 *     a failed check launches nothing and returns its error.  After each
 *     launch the library checks cudaGetLastError and returns HIF4_ERR_CUDA.
 *   - Layout: row-major; "ld" arguments are leading dimensions in ELEMENTS.
 *     Units are 64 consecutive elements of a row, so cols (K) % 64 == 0.
 *   - Alignment: x / y / acts base pointers and ld * element size must be
 *     multiples of 16 bytes (HIF4_ERR_ALIGNMENT otherwise).
 *   - Device-side errors are sticky bits in an optional caller-provided
 *     device word `status` (HIF4_FLAG_*); read it with hif4_get_status.
 */
#ifndef HIF4_H
#define HIF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *hif4_stream_t; /* == cudaStream_t */

typedef enum {
    HIF4_OK = 0,
    HIF4_ERR_INVALID_ARG = 1, /* null pointer, negative size, bad ratio */
    HIF4_ERR_ALIGNMENT = 2,   /* pointer or leading dimension not 16-byte aligned */
    HIF4_ERR_SHAPE = 3,       /* cols / K not a multiple of 64, ld < cols */
    HIF4_ERR_WORKSPACE = 4,   /* workspace null or smaller than *_workspace() */
    HIF4_ERR_CUDA = 5,        /* a CUDA runtime call or launch failed */
    HIF4_ERR_NONFINITE = 6,   /* device flag: a NaN/Inf input was mapped */
    HIF4_ERR_TIMEOUT = 7,     /* device flag: a bounded wait gave up */
    HIF4_ERR_UNSUPPORTED = 8, /* no sm_100 device, or size beyond a limit */
    HIF4_ERR_FORMAT = 9       /* serialized state malformed, truncated or corrupted */
} hif4_status;

typedef enum { HIF4_F32 = 0, HIF4_BF16 = 1 } hif4_dtype;

/* Bits of the device status word. */
#define HIF4_FLAG_NONFINITE 0x1u /* NaN -> 0, +-Inf -> +-FLT_MAX was applied */
#define HIF4_FLAG_TIMEOUT 0x2u   /* a pipeline wait hit its iteration limit */
#define HIF4_FLAG_BAD_INDEX 0x4u /* a mask index was out of range or unsorted */
#define HIF4_FLAG_NOT_SPD 0x8u   /* a damped Hessian was not positive definite (HiGPTQ) */

/* Flags of hif4_linear_w4a4 / hif4_gemm_bf16. */
#define HIF4_LINEAR_GELU_TANH 0x1u /* y = gelu_tanh(acc + bias) */
#define HIF4_LINEAR_OUT_F32 0x2u   /* y is FP32 (the accumulator, unrounded) instead of BF16 */
/* y (BF16) is replaced by its HiF4 fake quantization along N in 64-column
 * units: deq(q(y with protected columns -> 0)), protected columns kept
 * (hif4_gemm_bf16_fq; hif4_ffn_w4a4 uses it for the hidden activation). */
#define HIF4_LINEAR_FAKE_QUANT_OUT 0x4u

/*
 * hif4_quantize — HiF4 "direct conversion" (round to nearest) of a
 * rows x cols matrix along its rows [HiF4 format; HiGPTQ].
 *
 * For each 64-element unit (masked columns counted as 0):
 *   c  = largest E6M2 code with 6.5 * v(c) < max|x|  (0 if none),
 *        v(c) = 2^(E-31) (1 + f/4), c = E<<2 | f;
 *   t_k = 0 / 1 / 2 as max|x| of 4-group k is <= 1.75 S / <= 3.5 S / more;
 *   e2[j] = [max(t_2j, t_2j+1) == 2],  e3[k] = max(0, t_k - e2[k/2]);
 *   m_i = RNE(|x_i| / (S 2^(e2+e3) / 4)), ties to even, min 7; sign dropped at 0.
 *   NaN -> 0 and +-Inf -> +-FLT_MAX (sets HIF4_FLAG_NONFINITE).
 *
 * x         rows x cols, F32 or BF16, leading dimension ldx (elements).
 * chan_mask NULL or `cols` bytes (device); nonzero = protected column: it is
 *           excluded from the scale choice and gets code 0.
 * codes     out, rows x cols/2 bytes, dense; element 2b in the low nibble of
 *           byte b, code = sign << 3 | m.
 * meta      out, rows x cols/64 uint32, dense; c | e2 << 8 | e3 << 16.
 * status    NULL or a device word that receives HIF4_FLAG_* bits (OR-ed).
 * Errors: INVALID_ARG (null x/codes/meta with rows > 0, rows < 0, dtype),
 *         SHAPE (cols % 64, ldx < cols), ALIGNMENT (x, ldx; codes/meta 4 B).
 */
hif4_status hif4_quantize(const void *x, hif4_dtype dtype, int64_t rows, int64_t cols,
                          int64_t ldx, const uint8_t *chan_mask, uint8_t *codes,
                          uint32_t *meta, uint32_t *status, hif4_stream_t stream);

/*
 * hif4_dequantize — y = (-1)^s (m/4) 2^(e2+e3) v(c) [HiF4 format; the
 * decode formula is an image on that page — this sign convention, an E1 bit
 * of 1 doubling the value, is the library's reading].  Exact in BF16/F32.
 * codes/meta as produced by hif4_quantize (dense); y rows x cols with ldy.
 * Code 8 (sign with m = 0) decodes to -0.
 */
hif4_status hif4_dequantize(const uint8_t *codes, const uint32_t *meta, int64_t rows,
                            int64_t cols, hif4_dtype out_dtype, void *y, int64_t ldy,
                            hif4_stream_t stream);

/*
 * hif4_fake_quantize — activation fake quantization of the W4A4 linear
 * [TA abstract]: xhat = deq(q(x with masked -> 0)) and xhat = x on masked
 * columns.  x, xhat: BF16 rows x cols (ldx, ldxh).  chan_mask as in
 * hif4_quantize.  Bit-identical to hif4_quantize followed by hif4_dequantize
 * with the masked columns copied.
 */
hif4_status hif4_fake_quantize(const void *x, int64_t rows, int64_t cols, int64_t ldx,
                               const uint8_t *chan_mask, void *xhat, int64_t ldxh,
                               uint32_t *status, hif4_stream_t stream);

/*
 * hif4_linear_w4a4 — the fake-quantized W4A4 linear layer [TA abstract]:
 *   y = xhat * what^T + bias   (FP32 accumulation, BF16 output),
 * xhat = hif4_fake_quantize(x) with the columns in mask_idx kept in BF16;
 * what = deq(w_codes, w_meta) with column mask_idx[j] replaced by
 * w_masked[:, j].  The dequantized operands are exact in BF16, so the
 * product runs on the tcgen05 BF16 tensor cores.
 *
 * x        BF16 M x K, ldx.            w_codes/w_meta  HiF4 N x K (dense),
 *          quantized with hif4_quantize using the same protected columns.
 * mask_idx NULL or n_masked sorted distinct column indices (device int32).
 * w_masked NULL or BF16 N x n_masked, dense (row n = W[n, mask_idx[:]]).
 * bias     NULL or BF16 [N].           y  BF16 (FP32 with OUT_F32) M x N, ldy.
 * flags    HIF4_LINEAR_GELU_TANH: tanh-form GELU applied to acc + bias;
 *          HIF4_LINEAR_OUT_F32: store the FP32 result instead of its BF16
 *          round-to-nearest-even (the BF16 output is exactly that rounding).
 * workspace >= hif4_linear_w4a4_workspace(M, N, K) bytes, 256-byte aligned.
 * The weight is decoded once per call into the workspace (a streaming pass
 * at full occupancy), then read by the GEMM.  For repeated calls on a static
 * weight, decode it once with hif4_weight_decode and call hif4_fake_quantize
 * + hif4_gemm_bf16 per input: the same products, bit for bit.
 * Errors: SHAPE (K % 64, M/N/K <= 0), ALIGNMENT, WORKSPACE, INVALID_ARG.
 * Bad mask indices are reported through status (HIF4_FLAG_BAD_INDEX).
 */
size_t hif4_linear_w4a4_workspace(int64_t M, int64_t N, int64_t K);
hif4_status hif4_linear_w4a4(const void *x, int64_t M, int64_t K, int64_t ldx,
                             const uint8_t *w_codes, const uint32_t *w_meta, int64_t N,
                             const int32_t *mask_idx, int32_t n_masked, const void *w_masked,
                             const void *bias, void *y, int64_t ldy, uint32_t flags,
                             void *workspace, size_t ws_bytes, uint32_t *status,
                             hif4_stream_t stream);

/*
 * hif4_weight_decode — the weight half of the fake-quantized linear:
 * what = deq(w_codes, w_meta) as BF16 (N x K, leading dimension ldw) with
 * column mask_idx[j] replaced by w_masked[:, j] (BF16 N x n_masked, dense).
 * Stage 3 of hif4_linear_w4a4; callers with static weights may run it once.
 * Errors as hif4_linear_w4a4.
 */
hif4_status hif4_weight_decode(const uint8_t *w_codes, const uint32_t *w_meta, int64_t N, int64_t K,
                               const int32_t *mask_idx, int32_t n_masked, const void *w_masked,
                               void *what, int64_t ldw, uint32_t *status, hif4_stream_t stream);

/*
 * hif4_gemm_bf16 — the product stage of hif4_linear_w4a4 on operands that are
 * already BF16: y = a * b^T + bias (FP32 accumulation in tensor memory,
 * BF16 round-to-nearest-even output), optional tanh-GELU (flags as for the
 * linear).  a: M x K (lda), b: N x K (ldb), both K-major; K % 64 == 0.
 * Persistent tcgen05 kernel, 128 x 256 output tiles, TMA-fed.
 */
hif4_status hif4_gemm_bf16(const void *a, int64_t M, int64_t K, int64_t lda, const void *b, int64_t N,
                           int64_t ldb, const void *bias, void *y, int64_t ldy, uint32_t flags,
                           uint32_t *status, hif4_stream_t stream);

/*
 * hif4_gemm_bf16_fq — hif4_gemm_bf16 whose BF16 output is fake-quantized in
 * the epilogue [TA abstract: W4A4 HiF4 fake quantization of the activations
 * that enter the main linears; fusion of the second FFN activation]:
 *   h    = bf16_rne(acc + bias), or of gelu_tanh(acc + bias) with GELU,
 *   y    = deq(q(h with the out_chan_mask columns -> 0)) along N in 64-column
 *          units, the out_chan_mask columns keeping h.
 * Identical, bit for bit, to hif4_gemm_bf16 followed by hif4_fake_quantize
 * with that mask.  HIF4_LINEAR_FAKE_QUANT_OUT is implied; OUT_F32 is refused.
 * out_chan_mask  NULL (no protected column) or u8 [N], nonzero = protected,
 *                16-byte aligned.
 * Errors: SHAPE (N % 64 != 0, others as hif4_gemm_bf16), ALIGNMENT,
 * INVALID_ARG.  Non-finite h values raise HIF4_FLAG_NONFINITE (mapped as the
 * quantizer maps them).
 */
hif4_status hif4_gemm_bf16_fq(const void *a, int64_t M, int64_t K, int64_t lda, const void *b, int64_t N,
                              int64_t ldb, const void *bias, const uint8_t *out_chan_mask, void *y,
                              int64_t ldy, uint32_t flags, uint32_t *status, hif4_stream_t stream);

/*
 * hif4_to_e4m3 — exact remap of HiF4 codes onto FP8 E4M3 plus one FP32 scale
 * per 64-element unit [HiF4 format: an element is (-1)^s (m/4) 2^(e2+e3) S;
 * m/4 2^E with m <= 7, E <= 2 has at most three significant bits]:
 *   q8[r][c]          = E4M3 byte of (-1)^s (m/4) 2^E (0x00 for m = 0),
 *   scale[u * lds + r] = S, the E6M2 value of unit u of row r (FP32, exact),
 * so that q8 * scale is hif4_dequantize's value, bit for bit.  codes / meta
 * as hif4_quantize writes them (rows x cols/2, rows x cols/64, dense).
 * q8 rows x cols bytes (ldq, a multiple of 8; 8-byte aligned); scale is
 * K-unit-major, (cols/64) x lds FP32, lds >= rows, 4-byte aligned; entries
 * of rows >= `rows` are left untouched.
 * Errors: SHAPE (cols % 64, ldq < cols, lds < rows), ALIGNMENT, INVALID_ARG.
 */
hif4_status hif4_to_e4m3(const uint8_t *codes, const uint32_t *meta, int64_t rows, int64_t cols, uint8_t *q8,
                         int64_t ldq, float *scale, int64_t lds, hif4_stream_t stream);

/*
 * hif4_gemm_f8 — the W4A4 HiF4 product on the FP8 tensor cores [HiF4 format;
 * TA abstract: W4A4 fake-quantized linears]:
 *   y[m][n] = sum over units u of  sa[u][m] sb[u][n] sum_{k in u} a[m][k] b[n][k]
 * with a, b E4M3 operands (hif4_to_e4m3 of HiF4 codes) and the unit scales
 * applied in FP32 after each unit's 64-deep FP8 product (tcgen05 kind::f8f6f4,
 * FP32 accumulation; exact for HiF4 operands, see the source), FP32 or BF16
 * (round to nearest even) out.  Protected channels are not covered: they are
 * the BF16 linear's job (hif4_gemm_bf16).
 * a  M x K E4M3 bytes (lda >= K, a multiple of 16), sa (K/64) x lds_a FP32,
 *    lds_a >= M rounded up to 128 (rows past M are read, never affect y);
 * b  N x K E4M3 bytes (ldb), sb (K/64) x lds_b FP32, lds_b >= N rounded up to
 *    256; all 16-byte aligned, lds_a and lds_b multiples of 4.
 * flags  0 (BF16 y) or HIF4_LINEAR_OUT_F32.
 * Errors: SHAPE (K % 64, K < 128, leading dimensions), ALIGNMENT,
 * INVALID_ARG, UNSUPPORTED (sizes, or a layout the driver's tensor-map
 * encoder refuses).  Bounded waits raise HIF4_FLAG_TIMEOUT as
 * hif4_gemm_bf16.
 */
hif4_status hif4_gemm_f8(const uint8_t *a, int64_t M, int64_t K, int64_t lda, const float *sa, int64_t lds_a,
                         const uint8_t *b, int64_t N, int64_t ldb, const float *sb, int64_t lds_b, void *y,
                         int64_t ldy, uint32_t flags, uint32_t *status, hif4_stream_t stream);

/*
 * hif4_ffn_w4a4 — the W4A4 HiF4 feed-forward block of a DiT layer [TA
 * abstract: fake-quantized main linears, protected channels in BF16; the
 * tanh-form GELU between them is the library's reading]:
 *   xhat1 = fake_quantize(x, mask1)                       M x D
 *   Hhat  = fake_quantize(bf16(gelu_tanh(xhat1 what1^T + b1)), mask2)   M x F
 *   y     = Hhat what2^T + b2                             M x D
 * what1 = deq(w1) with columns mask1 restored from w1_masked (F x n_mask1);
 * what2 = deq(w2) with columns mask2 restored from w2_masked (D x n_mask2).
 * Hhat is produced inside the first GEMM's epilogue (hif4_gemm_bf16_fq).
 * x      BF16 M x D, ldx.   w1_codes/w1_meta HiF4 F x D, quantized with
 *        hif4_quantize and mask1; w2_codes/w2_meta HiF4 D x F with mask2.
 * mask1_idx / mask2_idx  NULL or sorted distinct column indices (device
 *        int32) of D / F.   b1 BF16 [F] or NULL; b2 BF16 [D] or NULL.
 * y      BF16 M x D (FP32 with HIF4_LINEAR_OUT_F32, the only flag), ldy.
 * workspace >= hif4_ffn_w4a4_workspace(M, D, F) bytes, 256-byte aligned.
 * Errors: SHAPE (D or F not a multiple of 64), ALIGNMENT, WORKSPACE,
 * INVALID_ARG; bad mask indices through status (HIF4_FLAG_BAD_INDEX).
 */
size_t hif4_ffn_w4a4_workspace(int64_t M, int64_t D, int64_t F);
hif4_status hif4_ffn_w4a4(const void *x, int64_t M, int64_t D, int64_t ldx,
                          const uint8_t *w1_codes, const uint32_t *w1_meta, int64_t F,
                          const int32_t *mask1_idx, int32_t n_mask1, const void *w1_masked,
                          const void *b1, const uint8_t *w2_codes, const uint32_t *w2_meta,
                          const int32_t *mask2_idx, int32_t n_mask2, const void *w2_masked,
                          const void *b2, void *y, int64_t ldy, uint32_t flags, void *workspace,
                          size_t ws_bytes, uint32_t *status, hif4_stream_t stream);

/*
 * hif4_ffn_w4a4_host — hif4_ffn_w4a4 on HOST activations: x_host (BF16
 * M x D, ldx) and y_host (BF16, or FP32 with HIF4_LINEAR_OUT_F32, M x D,
 * ldy) are host buffers.  The rows stream through the GPU in chunks of
 * chunk_rows (0 = automatic: at most 4096 rows in whole 128-row tiles,
 * ramping 1024 / 2048 rows up at the start and down at the end), the
 * copies of neighbouring chunks overlapping the compute of chunk i.  Chunks
 * alternate between `stream` and one internal compute stream, so a chunk's
 * kernels can start on the SMs the previous chunk's last GEMM wave leaves
 * idle; two internal copy streams; staging and scratch double-buffered in
 * the workspace.  The results equal hif4_ffn_w4a4 on the same rows.
 * Page-locked host buffers (cudaHostAlloc / cudaHostRegister) are needed for
 * the overlap; pageable ones give the same results with serialized copies.
 * Asynchronous on `stream`: when `stream` completes, y_host holds the
 * result; x_host and y_host must stay valid until then.
 * workspace >= hif4_ffn_w4a4_host_workspace(M, D, F, chunk_rows, flags)
 * bytes, 256-byte aligned.  Other arguments and errors as hif4_ffn_w4a4.
 */
size_t hif4_ffn_w4a4_host_workspace(int64_t M, int64_t D, int64_t F, int64_t chunk_rows, uint32_t flags);
hif4_status hif4_ffn_w4a4_host(const void *x_host, int64_t M, int64_t D, int64_t ldx,
                               const uint8_t *w1_codes, const uint32_t *w1_meta, int64_t F,
                               const int32_t *mask1_idx, int32_t n_mask1, const void *w1_masked,
                               const void *b1, const uint8_t *w2_codes, const uint32_t *w2_meta,
                               const int32_t *mask2_idx, int32_t n_mask2, const void *w2_masked,
                               const void *b2, void *y_host, int64_t ldy, int64_t chunk_rows,
                               uint32_t flags, void *workspace, size_t ws_bytes, uint32_t *status,
                               hif4_stream_t stream);

/*
 * hif4_calib_percentile_mask — tail-aware percentile calibration and the
 * channel mask [TA summary "Why tail percentiles"; TA abstract].
 *   pct[c]   = the |x| value (as non-negative BF16) at 0-based ascending rank
 *              k = floor(q_num (T-1) / q_den) among the T tokens of channel c,
 *              keys compared as 15-bit BF16 magnitudes (+-0 equal);
 *   med      = lower median over channels of pct (rank floor((C-1)/2));
 *   ratio[c] = fp32(pct[c]) / fp32(med)  (+Inf / 0 when med == 0);
 *   mask[c]  = 1 for the floor(C mask_num / mask_den) channels with the
 *              largest pct, ties to the lower channel index.
 * acts  BF16 T x C (lda; 2-byte alignment suffices).  pct BF16 [C], ratio
 *       F32 [C], mask u8 [C] (device).
 * mask_idx_out  NULL or int32 [floor(C mask_num / mask_den)]: the masked
 *               channels in ascending order (ready for hif4_linear_w4a4).
 * workspace >= hif4_calib_workspace(T, C) bytes.
 * Every wait on a tile copy inside the passes is bounded (2 s); if one runs
 * out, the passes stop and the outputs are poisoned instead of computed:
 * every ratio NaN, mask all zero, every mask_idx_out entry -1.
 */
size_t hif4_calib_workspace(int64_t tokens, int64_t channels);
hif4_status hif4_calib_percentile_mask(const void *acts, int64_t tokens, int64_t channels,
                                       int64_t lda, uint32_t q_num, uint32_t q_den,
                                       uint32_t mask_num, uint32_t mask_den, void *pct,
                                       float *ratio, uint8_t *mask, int32_t *mask_idx_out,
                                       void *workspace, size_t ws_bytes,
                                       hif4_stream_t stream);

/*
 * hif4_calib_percentile_mask_noalloc — the same computation as
 * hif4_calib_percentile_mask, for callers that cannot allocate device memory
 * (a runtime that gives all device memory to its own pool at start-up, a
 * plugin host that forbids allocation inside its enqueue callback).  The
 * source pages have no counterpart of this call; it exists only for such
 * callers.
 *
 * Its scratch is one fixed array of hif4_calib_noalloc_scratch_bytes()
 * bytes (16 MiB) in device memory, which every GPU that loads the library
 * holds until the process exits.  The call allocates nothing: it forwards to
 * hif4_calib_percentile_mask with that array as the workspace, which clears
 * what must start at zero on every call.
 *   - Sizes whose hif4_calib_workspace(tokens, channels) exceeds the array
 *     are rejected with HIF4_ERR_WORKSPACE before any launch (with the
 *     current histogram layout: channels <= 5445).
 *   - The first call on a device looks up the array's device address once
 *     (that device must be current); make that first call before any stream
 *     capture begins.  The address stays cached for the life of the
 *     process: after cudaDeviceReset, or anything else that tears down and
 *     re-creates the device's primary context, it is stale, so do not use
 *     this call on that device again in the same process.
 *   - All calls on a device share the one array, which keeps the last call's
 *     contents: calls whose execution overlaps on the GPU (different streams
 *     without ordering) race and give wrong results.  Order them.
 * Arguments and outputs are those of hif4_calib_percentile_mask.
 */
size_t hif4_calib_noalloc_scratch_bytes(void);
hif4_status hif4_calib_percentile_mask_noalloc(const void *acts, int64_t tokens, int64_t channels,
                                               int64_t lda, uint32_t q_num, uint32_t q_den,
                                               uint32_t mask_num, uint32_t mask_den, void *pct,
                                               float *ratio, uint8_t *mask, int32_t *mask_idx_out,
                                               hif4_stream_t stream);

/*
 * hif4_hessian — H = X^T X (FP32, K x K) of a layer's input activations X
 * (BF16 T x K, ldx), the second-moment matrix HiGPTQ weighs the weight
 * error with.  Tensor-core product with FP32 accumulation (the BF16 products
 * are exact).  workspace >= hif4_hessian_workspace(T, K) bytes (X^T, rows
 * padded to a multiple of 64), 256-byte aligned; H 16-byte aligned.
 * Errors: SHAPE (K % 64, ldx < K), ALIGNMENT, WORKSPACE, INVALID_ARG.
 */
size_t hif4_hessian_workspace(int64_t T, int64_t K);
hif4_status hif4_hessian(const void *x, int64_t T, int64_t K, int64_t ldx, float *H, void *workspace,
                         size_t ws_bytes, uint32_t *status, hif4_stream_t stream);

/*
 * hif4_higptq1 — HiGPTQ, scheme one [HiF4 article, section 3.1: 64 columns
 * (one HiF4 unit per row) are quantized at a time with the level-1, level-2
 * and level-3 exponents fixed together; the remaining weights of the block
 * are then updated; GPTQ's Hessian error feedback]:
 *   Hd = H + damp * mean(diag H) * I (a zero diagonal entry -- a dead input
 *        channel -- is set to 1 and its weights to 0); Hd^{-1} = U^T U;
 *   for each block of `blocksize` columns and each 64-column group g in it,
 *   per row:  Q_g = HiF4 quantization of the row's current values (encode
 *   rule of hif4_quantize; protected columns are excluded from the scale and
 *   take the BF16 rounding of their current value),  E = (W_g - Q_g) U_gg^-1,
 *   W_c -= E U_{g,c} for the later columns of the block, and after the block
 *   W_c -= E_block U_{block,c} for every later column.
 * w       BF16 N x K (ldw), the layer weight.   H  FP32 K x K (symmetric).
 * mask_idx  NULL or n_masked sorted distinct columns kept in BF16.
 * damp    relative damping (>= 0; 0.01 is customary).
 * blocksize  64, 128 (0 = 128), 192 or 256.
 * codes / meta  out: HiF4 N x K/2 and N x K/64 (as hif4_quantize writes
 *         them, protected columns coded 0), ready for hif4_linear_w4a4;
 * w_masked  out: BF16 N x n_masked, the protected columns' final values.
 * workspace >= hif4_higptq1_workspace(N, K, blocksize), 256-byte aligned.
 * The factor runs in FP64, the group loop in FP32 (its lazy update on the
 * TF32 tensor cores with each operand split in two TF32 parts: three
 * products per FP32 product, FP32 accumulation).  Device flags: NOT_SPD
 * (Hd not positive definite), BAD_INDEX, NONFINITE (non-finite weights,
 * mapped as hif4_quantize maps them).  Errors: SHAPE (K % 64, ldw < K),
 * UNSUPPORTED (K > 32768), ALIGNMENT, WORKSPACE, INVALID_ARG.
 */
size_t hif4_higptq1_workspace(int64_t N, int64_t K, int64_t blocksize);
hif4_status hif4_higptq1(const void *w, int64_t N, int64_t K, int64_t ldw, const float *H,
                         const int32_t *mask_idx, int32_t n_masked, double damp, int64_t blocksize,
                         uint8_t *codes, uint32_t *meta, void *w_masked, void *workspace, size_t ws_bytes,
                         uint32_t *status, hif4_stream_t stream);
/*
 * hif4_higptq1_group_inputs_offset — byte offset, inside a hif4_higptq1
 * workspace of the same N, K and blocksize, of an FP32 N x K array (row
 * stride K) that, once the call has completed on its stream, holds for every
 * 64-column group the weights that group was quantized from: the layer
 * weight after the error feedback of every earlier group (dead input
 * channels zeroed) [HiF4 article, section 3.1: each group is quantized from
 * its current, updated values].  Lets a caller inspect the feedback, or check
 * each group's codes against a plain quantization of those values.  The array
 * stays valid until the workspace is reused.  Returns (size_t)-1 for shapes
 * hif4_higptq1_workspace refuses.
 */
size_t hif4_higptq1_group_inputs_offset(int64_t N, int64_t K, int64_t blocksize);

/*
 * Compact PTQ state of one linear layer [TA summary, "Method overview":
 * compact deltas that restore the quantized behaviour are stored instead of
 * the full BF16 weights]: its HiF4 codes and metadata (as hif4_quantize
 * writes them, N x K), the protected-column indices and those columns' BF16
 * weights (as hif4_linear_w4a4 takes them) in one self-describing record.
 * Version 1 layout (little-endian; sections at 64-byte offsets):
 *   0 "HIF4PTQS" | 8 u32 version 1 | 12 u32 64 | 16 i64 N | 24 i64 K |
 *   32 i32 n_masked | 36 u32 0 | 40 u64 total bytes | 48 16 zero bytes |
 *   64 mask_idx i32[n_masked] | codes u8[N][K/2] | meta u32[N][K/64] |
 *   w_masked u16[N][n_masked] | u32 CRC-32 (IEEE, reflected 0xEDB88320) of
 *   every byte before it.
 * All pointers are HOST pointers; no device is needed.  mask_idx must be
 * sorted and distinct in [0, K).
 * hif4_ptq_state_bytes   record size (0 for invalid sizes).
 * hif4_ptq_state_pack    writes the record into out (>= that size; else
 *                        WORKSPACE); SHAPE if K % 64, INVALID_ARG otherwise.
 * hif4_ptq_state_info    checks a record (magic, version, sizes, checksum,
 *                        indices; FORMAT when any fails) and reports N, K,
 *                        n_masked (each output pointer may be NULL).
 * hif4_ptq_state_unpack  checks the record as info does and copies its
 *                        sections into caller buffers of those sizes.
 */
size_t hif4_ptq_state_bytes(int64_t N, int64_t K, int32_t n_masked);
hif4_status hif4_ptq_state_pack(int64_t N, int64_t K, const uint8_t *codes, const uint32_t *meta,
                                const int32_t *mask_idx, int32_t n_masked, const void *w_masked,
                                void *out, size_t out_bytes);
hif4_status hif4_ptq_state_info(const void *buf, size_t bytes, int64_t *N, int64_t *K,
                                int32_t *n_masked);
hif4_status hif4_ptq_state_unpack(const void *buf, size_t bytes, uint8_t *codes, uint32_t *meta,
                                  int32_t *mask_idx, void *w_masked);

/*
 * hif4_debug_wait_test — failure-handling diagnostic; off by default and not
 * meant for production runs.  Every wait of the TMA-fed kernels on an
 * asynchronous copy is bounded by wall time (4 s in the tcgen05 GEMM, 2 s in
 * the quantizers and the calibration passes): a block whose wait runs out
 * stops, lets the copies it issued land (and, in the GEMM, its MMAs
 * complete before the tensor memory is freed), and reports
 * HIF4_FLAG_TIMEOUT in the status word; the calibration then poisons its
 * outputs (ratios NaN, mask 0, indices -1).  While `withhold` is nonzero,
 * block 0 of every later launch of those kernels from this process leaves
 * its first copy un-issued, so the wait on it can only end at its limit;
 * `limit_ns` (0 = the defaults) replaces every such limit.  Call
 * hif4_debug_wait_test(0, 0) to return to normal operation.  Process-wide,
 * not thread-safe against concurrent launches; no device work.
 */
void hif4_debug_wait_test(uint32_t withhold, uint64_t limit_ns);

/* Synchronizes `stream`, reads the device status word and maps its bits:
 * TIMEOUT -> HIF4_ERR_TIMEOUT, BAD_INDEX or NOT_SPD -> HIF4_ERR_INVALID_ARG,
 * NONFINITE -> HIF4_ERR_NONFINITE, none -> HIF4_OK.  The word is not cleared. */
hif4_status hif4_get_status(const uint32_t *status_word, hif4_stream_t stream);
/* Clears the device status word (asynchronously, on `stream`). */
hif4_status hif4_reset_status(uint32_t *status_word, hif4_stream_t stream);

const char *hif4_status_string(hif4_status s);
/* Name of the last CUDA runtime error that made a call of this host thread
 * return HIF4_ERR_CUDA where the call records it (every kernel launch; ""
 * when none was recorded): a diagnostic beside the status code. */
const char *hif4_last_cuda_error(void);
/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
int hif4_version(void);

#ifdef __cplusplus
}
#endif

#endif /* HIF4_H */
