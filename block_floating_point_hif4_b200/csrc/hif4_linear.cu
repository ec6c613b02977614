// hif4_linear.cu — the W4A4 HiF4 fake-quantized linear layer on sm_100a.
//
//   y = xhat * what^T + bias        [Tail-Aware HiFloat4 arXiv abstract:
//                                    W4A4 fake quantization of the main linears]
// xhat: activations fake-quantized along K in 64-element units (protected
//       channels kept in BF16), written once to the workspace;
// what: HiF4 weights decoded to BF16 (protected columns restored from the
//       caller's BF16 copy), written once to the workspace;
// GEMM: persistent, warp-specialized tcgen05 kernel.  Every dequantized
//       operand is exact in BF16 (at most 6 significant bits), so the BF16
//       tensor-core product with FP32 accumulation is the fake-quant linear.
//
// GEMM structure (one CTA per SM, 192 threads):
//   warp 0      TMA producer: 128x64 A and 256x64 B BF16 tiles, 128-byte
//               swizzle, 4-stage smem ring (48 KB per stage);
//   warp 1      allocates 512 TMEM columns (two 128x256 FP32 accumulators)
//               and issues tcgen05.mma (M=128, N=256, K=16) from one thread;
//   warps 2-5   epilogue: tcgen05.ld of its 32-lane quarter, + bias,
//               optional tanh-GELU, BF16 round-to-nearest-even, optional
//               HiF4 fake quantization of the row's 64-column units, global
//               store; it drains one accumulator while the next tile
//               accumulates.
// Every mbarrier wait is bounded; a wait that gives up sets the block's abort
// flag, the others leave their loops, TMEM is freed and HIF4_FLAG_TIMEOUT is
// raised in the status word.
#include <cuda_bf16.h>

#include <vector>

#include "hif4_encode.cuh"
#include "hif4_gemm.cuh"
#include "hif4_internal.cuh"
#include "hif4_sm100.cuh"

namespace hif4 {

hif4_status fake_quantize_bf16(const void *x, int64_t rows, int64_t cols, int64_t ldx,
                               const uint8_t *chan_mask, void *xhat, int64_t ldxh,
                               uint32_t *status, cudaStream_t s);

namespace {

// mask[k] = 1 for k in mask_idx, else 0; flags out-of-range or unsorted
// indices in the status word (they are then ignored).
__global__ void k_mask_prep(uint8_t *mask, int K, const int32_t *idx, int n, uint32_t *status)
{
    uint32_t bad = 0;
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < K || i < n; i += gridDim.x * blockDim.x) {
        if (i < n) {
            const int v = idx[i];
            if (v < 0 || v >= K || (i > 0 && idx[i - 1] >= v)) bad = 1;
        }
        if (i < K) {
            int lo = 0, hi = n;                    // first index with idx >= i
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (idx[mid] < i) lo = mid + 1;
                else hi = mid;
            }
            mask[i] = (lo < n && idx[lo] == i) ? 1 : 0;
        }
    }
    if (bad) status_or(status, HIF4_FLAG_BAD_INDEX);
}

// what[n, idx[j]] = w_masked[n, j] (protected weight columns kept in BF16).
__global__ void k_scatter_cols(uint16_t *what, int64_t K, const uint16_t *wm, const int32_t *idx, int n_m,
                               int64_t N)
{
    const int64_t total = N * (int64_t)n_m;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = e / n_m;
        const int j = (int)(e - n * n_m);
        const int k = idx[j];
        if (k >= 0 && k < K) what[n * K + k] = wm[e];
    }
}

size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

} // namespace
} // namespace hif4

using namespace hif4;

namespace hif4 {
namespace {

hif4_status launch_gemm(const void *a, int64_t M, int64_t K, int64_t lda, const void *b, int64_t N, int64_t ldb,
                        const void *bias, const uint8_t *out_mask, void *y, int64_t ldy, uint32_t flags,
                        uint32_t *status, cudaStream_t s)
{
    using namespace gemm;
    Args g{};
    g.M = (int)M;
    g.N = (int)N;
    g.K = (int)K;
    g.num_n = (int)((N + BN - 1) / BN);
    g.num_k = (int)(K / BK);
    g.bias = static_cast<const uint16_t *>(bias);
    g.y = y;
    g.ldy = ldy;
    g.flags = flags;
    g.out_mask = out_mask;
    g.status = status;
    g.timeout_ns = wait_limit_ns(TIMEOUT_NS);
    g.withhold = wait_test_withhold();
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_set[64] = {false};
    CUtensorMap tmA, tmB;
    if (!make_map(&tmA, a, M, K, lda, BM) || !make_map(&tmB, b, N, K, ldb, BN)) return HIF4_ERR_CUDA;
    g.num_m = (int)((M + BM - 1) / BM);
    g.num_tiles = g.num_m * g.num_n;
    g.group_m = GROUP_M;
    if (!attr_set[dev & 63]) {
        const cudaError_t e = cudaFuncSetAttribute(k_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
        if (e != cudaSuccess) return cuda_failed(e);
        attr_set[dev & 63] = true;
    }
    int grid = sm_count();
    if (grid > g.num_tiles) grid = g.num_tiles;
    k_gemm<<<grid, THREADS, SMEM_BYTES, s>>>(tmA, tmB, g);
    return launch_status();
}

hif4_status check_gemm_args(const void *a, int64_t M, int64_t K, int64_t lda, const void *b, int64_t N,
                            int64_t ldb, const void *bias, const void *y, int64_t ldy, uint32_t flags)
{
    if (M < 0 || N < 0 || K < 0) return HIF4_ERR_INVALID_ARG;
    if (K % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (M == 0 || N == 0) return HIF4_OK;
    if (K == 0) return HIF4_ERR_SHAPE;
    if (!a || !b || !y) return HIF4_ERR_INVALID_ARG;
    if (flags & ~(HIF4_LINEAR_GELU_TANH | HIF4_LINEAR_OUT_F32 | HIF4_LINEAR_FAKE_QUANT_OUT))
        return HIF4_ERR_INVALID_ARG;
    if (flags & HIF4_LINEAR_FAKE_QUANT_OUT) {
        if (flags & HIF4_LINEAR_OUT_F32) return HIF4_ERR_INVALID_ARG;   // fake quant writes BF16
        if (N % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    }
    if (lda < K || ldb < K || ldy < N) return HIF4_ERR_SHAPE;
    if (M > INT32_MAX / 2 || N > INT32_MAX / 2 || K > INT32_MAX / 2) return HIF4_ERR_UNSUPPORTED;
    const int64_t ysz = (flags & HIF4_LINEAR_OUT_F32) ? 4 : 2;
    if (!aligned16(a) || !aligned16(b) || !aligned16(y) || (lda * 2) % 16 || (ldb * 2) % 16 || (ldy * ysz) % 16)
        return HIF4_ERR_ALIGNMENT;
    if (bias && !aligned16(bias)) return HIF4_ERR_ALIGNMENT;
    return HIF4_OK;
}

} // namespace
} // namespace hif4

extern "C" hif4_status hif4_gemm_bf16(const void *a, int64_t M, int64_t K, int64_t lda, const void *b, int64_t N,
                                      int64_t ldb, const void *bias, void *y, int64_t ldy, uint32_t flags,
                                      uint32_t *status, hif4_stream_t stream)
{
    hif4_status st = check_gemm_args(a, M, K, lda, b, N, ldb, bias, y, ldy, flags);
    if (st != HIF4_OK || M == 0 || N == 0) return st;
    return launch_gemm(a, M, K, lda, b, N, ldb, bias, nullptr, y, ldy, flags, status,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" hif4_status hif4_gemm_bf16_fq(const void *a, int64_t M, int64_t K, int64_t lda, const void *b,
                                         int64_t N, int64_t ldb, const void *bias, const uint8_t *out_chan_mask,
                                         void *y, int64_t ldy, uint32_t flags, uint32_t *status,
                                         hif4_stream_t stream)
{
    flags |= HIF4_LINEAR_FAKE_QUANT_OUT;
    hif4_status st = check_gemm_args(a, M, K, lda, b, N, ldb, bias, y, ldy, flags);
    if (st != HIF4_OK || M == 0 || N == 0) return st;
    if (out_chan_mask && !aligned16(out_chan_mask)) return HIF4_ERR_ALIGNMENT;
    return launch_gemm(a, M, K, lda, b, N, ldb, bias, out_chan_mask, y, ldy, flags, status,
                       reinterpret_cast<cudaStream_t>(stream));
}

extern "C" hif4_status hif4_weight_decode(const uint8_t *w_codes, const uint32_t *w_meta, int64_t N, int64_t K,
                                          const int32_t *mask_idx, int32_t n_masked, const void *w_masked,
                                          void *what, int64_t ldw, uint32_t *status, hif4_stream_t stream)
{
    (void)status;
    if (N < 0 || K < 0 || n_masked < 0) return HIF4_ERR_INVALID_ARG;
    if (K % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (N == 0 || K == 0) return HIF4_OK;
    if (!w_codes || !w_meta || !what) return HIF4_ERR_INVALID_ARG;
    if (n_masked > 0 && (!mask_idx || !w_masked)) return HIF4_ERR_INVALID_ARG;
    if (n_masked > K) return HIF4_ERR_INVALID_ARG;
    if (n_masked > 0 && (!aligned_to(mask_idx, 4) || !aligned_to(w_masked, 2))) return HIF4_ERR_ALIGNMENT;
    hif4_status st = hif4_dequantize(w_codes, w_meta, N, K, HIF4_BF16, what, ldw, stream);
    if (st != HIF4_OK || n_masked == 0) return st;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t total = N * (int64_t)n_masked;
    int blocks = (int)((total + 255) / 256);
    if (blocks > 4 * sm_count()) blocks = 4 * sm_count();
    k_scatter_cols<<<blocks, 256, 0, s>>>(static_cast<uint16_t *>(what), ldw, static_cast<const uint16_t *>(w_masked),
                                          mask_idx, n_masked, N);
    return launch_status();
}

extern "C" size_t hif4_linear_w4a4_workspace(int64_t M, int64_t N, int64_t K)
{
    if (M <= 0 || N <= 0 || K <= 0) return 0;
    return align256((size_t)M * K * 2) + align256((size_t)N * K * 2) + align256((size_t)K);
}

extern "C" hif4_status hif4_linear_w4a4(const void *x, int64_t M, int64_t K, int64_t ldx,
                                        const uint8_t *w_codes, const uint32_t *w_meta, int64_t N,
                                        const int32_t *mask_idx, int32_t n_masked, const void *w_masked,
                                        const void *bias, void *y, int64_t ldy, uint32_t flags,
                                        void *workspace, size_t ws_bytes, uint32_t *status,
                                        hif4_stream_t stream)
{
    if (n_masked < 0) return HIF4_ERR_INVALID_ARG;
    if (flags & HIF4_LINEAR_FAKE_QUANT_OUT) return HIF4_ERR_INVALID_ARG;   // needs an output mask: hif4_ffn_w4a4
    hif4_status st = check_gemm_args(x, M, K, ldx, x, N, K, bias, y, ldy, flags);
    if (st != HIF4_OK || M == 0 || N == 0) return st;
    if (!w_codes || !w_meta) return HIF4_ERR_INVALID_ARG;
    if (n_masked > 0 && (!mask_idx || !w_masked)) return HIF4_ERR_INVALID_ARG;
    if (n_masked > K) return HIF4_ERR_INVALID_ARG;
    if (!aligned_to(w_codes, 4) || !aligned_to(w_meta, 4)) return HIF4_ERR_ALIGNMENT;
    if (n_masked > 0 && (!aligned_to(mask_idx, 4) || !aligned_to(w_masked, 2))) return HIF4_ERR_ALIGNMENT;
    const size_t need = hif4_linear_w4a4_workspace(M, N, K);
    if (!workspace || ws_bytes < need) return HIF4_ERR_WORKSPACE;
    if (!aligned_to(workspace, 256)) return HIF4_ERR_ALIGNMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *xhat = reinterpret_cast<uint16_t *>(ws);
    uint16_t *what = reinterpret_cast<uint16_t *>(ws + align256((size_t)M * K * 2));
    uint8_t *mask = ws + align256((size_t)M * K * 2) + align256((size_t)N * K * 2);

    // 1. protected-channel mask (u8 per input channel) from the sorted indices
    const uint8_t *chan_mask = nullptr;
    if (n_masked > 0) {
        const int64_t work = K > n_masked ? K : n_masked;
        k_mask_prep<<<(int)((work + 255) / 256), 256, 0, s>>>(mask, (int)K, mask_idx, n_masked, status);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
        chan_mask = mask;
    }
    // 2. activation fake quantization along K
    st = fake_quantize_bf16(x, M, K, ldx, chan_mask, xhat, K, status, s);
    if (st != HIF4_OK) return st;
    // 3. weight decode to BF16, protected columns restored
    st = hif4_weight_decode(w_codes, w_meta, N, K, mask_idx, n_masked, w_masked, what, K, status, stream);
    if (st != HIF4_OK) return st;
    // 4. tcgen05 GEMM + bias (+ GELU)
    return launch_gemm(xhat, M, K, K, what, N, K, bias, nullptr, y, ldy, flags, status, s);
}

// ----------------------------------------------------------------- FFN block
//
//   H    = gelu_tanh(xhat1 * what1^T + b1)   rounded to BF16,
//   Hhat = HiF4 fake quantization of H along F (mask2 columns kept),
//   y    = Hhat * what2^T + b2,
// with xhat1 the fake quantization of x along D (mask1 columns kept) and
// what1 / what2 the decoded weights (protected columns restored).  The
// second activation's fake quantization runs inside the first GEMM's
// epilogue, so H never goes through HBM unquantized.
// Workspace: xhat1 M x D | what1 F x D | Hhat M x F | what2 D x F (BF16) |
// mask1 D | mask2 F (u8), each 256-byte aligned.

namespace hif4 {
namespace {

// The FFN on `rows` device rows once the masks are built and the weights
// decoded: fake quantization of x along D into xhat1 (rows x D), the first
// GEMM with bias, GELU and the fake quantization of H into hhat (rows x F),
// the second GEMM with bias into y.
hif4_status ffn_rows(const void *x, int64_t rows, int64_t D, int64_t ldx, const uint16_t *what1,
                     const uint16_t *what2, int64_t F, const uint8_t *mask1, const uint8_t *mask2, const void *b1,
                     const void *b2, uint16_t *xhat1, uint16_t *hhat, void *y, int64_t ldy, uint32_t flags,
                     uint32_t *status, cudaStream_t s)
{
    hif4_status st = fake_quantize_bf16(x, rows, D, ldx, mask1, xhat1, D, status, s);
    if (st != HIF4_OK) return st;
    st = launch_gemm(xhat1, rows, D, D, what1, F, D, b1, mask2, hhat, F,
                     HIF4_LINEAR_GELU_TANH | HIF4_LINEAR_FAKE_QUANT_OUT, status, s);
    if (st != HIF4_OK) return st;
    return launch_gemm(hhat, rows, F, F, what2, D, F, b2, nullptr, y, ldy, flags, status, s);
}

// Host-side checks shared by both FFN entry points (device x / y pointers
// are checked by the caller where they exist).
hif4_status check_ffn_weights(int64_t D, int64_t F, const uint8_t *w1_codes, const uint32_t *w1_meta,
                              const int32_t *mask1_idx, int32_t n_mask1, const void *w1_masked, const void *b1,
                              const uint8_t *w2_codes, const uint32_t *w2_meta, const int32_t *mask2_idx,
                              int32_t n_mask2, const void *w2_masked, const void *b2)
{
    if (n_mask1 < 0 || n_mask2 < 0 || D < 0 || F < 0) return HIF4_ERR_INVALID_ARG;
    if (D % HIF4_UNIT != 0 || F % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (D == 0 || F == 0) return HIF4_ERR_SHAPE;
    if (D > INT32_MAX / 2 || F > INT32_MAX / 2) return HIF4_ERR_UNSUPPORTED;
    if (!w1_codes || !w1_meta || !w2_codes || !w2_meta) return HIF4_ERR_INVALID_ARG;
    if (n_mask1 > D || n_mask2 > F) return HIF4_ERR_INVALID_ARG;
    if ((n_mask1 > 0 && (!mask1_idx || !w1_masked)) || (n_mask2 > 0 && (!mask2_idx || !w2_masked)))
        return HIF4_ERR_INVALID_ARG;
    if (!aligned_to(w1_codes, 4) || !aligned_to(w1_meta, 4) || !aligned_to(w2_codes, 4) || !aligned_to(w2_meta, 4))
        return HIF4_ERR_ALIGNMENT;
    if ((n_mask1 > 0 && (!aligned_to(mask1_idx, 4) || !aligned_to(w1_masked, 2))) ||
        (n_mask2 > 0 && (!aligned_to(mask2_idx, 4) || !aligned_to(w2_masked, 2))))
        return HIF4_ERR_ALIGNMENT;
    if ((b1 && !aligned16(b1)) || (b2 && !aligned16(b2))) return HIF4_ERR_ALIGNMENT;
    return HIF4_OK;
}

// Masks from the sorted index lists and both weight decodes (once per call).
hif4_status ffn_prepare(int64_t D, int64_t F, const uint8_t *w1_codes, const uint32_t *w1_meta,
                        const int32_t *mask1_idx, int32_t n_mask1, const void *w1_masked, const uint8_t *w2_codes,
                        const uint32_t *w2_meta, const int32_t *mask2_idx, int32_t n_mask2, const void *w2_masked,
                        uint16_t *what1, uint16_t *what2, uint8_t *mask1, uint8_t *mask2, uint32_t *status,
                        cudaStream_t s)
{
    if (n_mask1 > 0) {
        const int64_t work = D > n_mask1 ? D : n_mask1;
        k_mask_prep<<<(int)((work + 255) / 256), 256, 0, s>>>(mask1, (int)D, mask1_idx, n_mask1, status);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    }
    if (n_mask2 > 0) {
        const int64_t work = F > n_mask2 ? F : n_mask2;
        k_mask_prep<<<(int)((work + 255) / 256), 256, 0, s>>>(mask2, (int)F, mask2_idx, n_mask2, status);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    }
    hif4_stream_t hs = reinterpret_cast<hif4_stream_t>(s);
    hif4_status st = hif4_weight_decode(w1_codes, w1_meta, F, D, mask1_idx, n_mask1, w1_masked, what1, D, status, hs);
    if (st != HIF4_OK) return st;
    return hif4_weight_decode(w2_codes, w2_meta, D, F, mask2_idx, n_mask2, w2_masked, what2, F, status, hs);
}

} // namespace
} // namespace hif4

extern "C" size_t hif4_ffn_w4a4_workspace(int64_t M, int64_t D, int64_t F)
{
    if (M <= 0 || D <= 0 || F <= 0) return 0;
    return align256((size_t)M * D * 2) + align256((size_t)F * D * 2) + align256((size_t)M * F * 2) +
           align256((size_t)D * F * 2) + align256((size_t)D) + align256((size_t)F);
}

extern "C" hif4_status hif4_ffn_w4a4(const void *x, int64_t M, int64_t D, int64_t ldx,
                                     const uint8_t *w1_codes, const uint32_t *w1_meta, int64_t F,
                                     const int32_t *mask1_idx, int32_t n_mask1, const void *w1_masked,
                                     const void *b1, const uint8_t *w2_codes, const uint32_t *w2_meta,
                                     const int32_t *mask2_idx, int32_t n_mask2, const void *w2_masked,
                                     const void *b2, void *y, int64_t ldy, uint32_t flags, void *workspace,
                                     size_t ws_bytes, uint32_t *status, hif4_stream_t stream)
{
    if (flags & ~HIF4_LINEAR_OUT_F32) return HIF4_ERR_INVALID_ARG;
    if (M < 0) return HIF4_ERR_INVALID_ARG;
    hif4_status st = check_ffn_weights(D, F, w1_codes, w1_meta, mask1_idx, n_mask1, w1_masked, b1, w2_codes,
                                       w2_meta, mask2_idx, n_mask2, w2_masked, b2);
    if (st != HIF4_OK || M == 0) return st;
    // first GEMM (x -> Hhat) and second GEMM (Hhat -> y) shapes and pointers
    st = check_gemm_args(x, M, D, ldx, x, F, D, b1, x, F, HIF4_LINEAR_GELU_TANH | HIF4_LINEAR_FAKE_QUANT_OUT);
    if (st != HIF4_OK) return st;
    st = check_gemm_args(x, M, F, F, x, D, F, b2, y, ldy, flags);
    if (st != HIF4_OK) return st;
    const size_t need = hif4_ffn_w4a4_workspace(M, D, F);
    if (!workspace || ws_bytes < need) return HIF4_ERR_WORKSPACE;
    if (!aligned_to(workspace, 256)) return HIF4_ERR_ALIGNMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *p = static_cast<uint8_t *>(workspace);
    uint16_t *xhat1 = reinterpret_cast<uint16_t *>(p);
    p += align256((size_t)M * D * 2);
    uint16_t *what1 = reinterpret_cast<uint16_t *>(p);
    p += align256((size_t)F * D * 2);
    uint16_t *hhat = reinterpret_cast<uint16_t *>(p);
    p += align256((size_t)M * F * 2);
    uint16_t *what2 = reinterpret_cast<uint16_t *>(p);
    p += align256((size_t)D * F * 2);
    uint8_t *mask1 = p;
    p += align256((size_t)D);
    uint8_t *mask2 = p;

    st = ffn_prepare(D, F, w1_codes, w1_meta, mask1_idx, n_mask1, w1_masked, w2_codes, w2_meta, mask2_idx,
                     n_mask2, w2_masked, what1, what2, mask1, mask2, status, s);
    if (st != HIF4_OK) return st;
    return ffn_rows(x, M, D, ldx, what1, what2, F, n_mask1 > 0 ? mask1 : nullptr, n_mask2 > 0 ? mask2 : nullptr,
                    b1, b2, xhat1, hhat, y, ldy, flags, status, s);
}

// ---------------------------------------------- FFN block on host activations
//
// The tokens stream through the GPU in chunks of at most C rows.  Two copy
// streams run beside two compute streams (the caller's and one more): chunk
// i is copied in, computed on compute stream i % 2 and copied out, so the
// copies of neighbouring chunks overlap its compute and the next chunk's
// kernels fill the SMs that the tail of chunk i's GEMMs leaves idle.
// Staging (xs, ys) and scratch (xhat1, hhat) are double-buffered by slot
// s = i % 2 and ordered by events:
//   h2d:       wait x_free[s]  -> copy x rows into xs[s]  -> record x_ready[s]
//   compute s: wait x_ready[s] -> fake-quant xs[s]        -> record x_free[s]
//              GEMM 1 (+ fake quant of H) -> wait y_free[s] -> GEMM 2 into
//              ys[s] -> record y_ready[s]
//   d2h:       wait y_ready[s] -> copy ys[s] out          -> record y_free[s]
// The weights are decoded once per call.  The streams and events are created
// per call and released once their work completes.
// Workspace: what1 F x D | what2 D x F | mask1 D | mask2 F | xhat1 2 x C x D |
// hhat 2 x C x F | xs 2 x C x D | ys 2 x C x D (x 2 for FP32 output).

namespace hif4 {
namespace {

size_t ffn_host_layout(int64_t C, int64_t D, int64_t F, uint32_t flags, size_t *off)
{
    const size_t ysz = (flags & HIF4_LINEAR_OUT_F32) ? 4 : 2;
    size_t o = 0;
    const size_t sizes[8] = {(size_t)F * D * 2, (size_t)D * F * 2, (size_t)D, (size_t)F,
                             2 * align256((size_t)C * D * 2), 2 * align256((size_t)C * F * 2),
                             2 * align256((size_t)C * D * 2), 2 * align256((size_t)C * D * ysz)};
    for (int i = 0; i < 8; ++i) {
        if (off) off[i] = o;
        o += align256(sizes[i]);
    }
    return o;
}

// Largest chunk: the caller's chunk_rows, or (0) at most 4096 rows in whole
// 128-row GEMM tiles.  Host copies and compute run at about the same rate
// here (PCIe both ways vs the power-capped GEMMs), so the pipeline gains
// nothing from longer chunks and loses their longer fill and drain.
int64_t ffn_host_chunk(int64_t M, int64_t chunk_rows)
{
    if (chunk_rows > 0) return chunk_rows < M ? chunk_rows : M;
    const int64_t n = (M + 4095) / 4096;
    int64_t c = (M + n - 1) / n;
    c = (c + 127) / 128 * 128;
    return c < M ? c : M;
}

// Row ranges of the chunks.  An explicit chunk_rows gives equal chunks.  The
// automatic schedule ramps up (1024, 2048 rows) and back down at the end, so
// that the copy in of the first chunk and the copy out of the last one,
// which nothing overlaps, stay short; the middle runs in chunks of at most C
// rows.
void ffn_host_schedule(int64_t M, int64_t chunk_rows, int64_t C, int64_t *starts, int64_t *counts, int &n)
{
    n = 0;
    const int64_t ramp[2] = {1024, 2048};
    const int64_t ends = 2 * (ramp[0] + ramp[1]);
    if (chunk_rows > 0 || M < ends + 2 * C) {
        for (int64_t r = 0; r < M; r += C) {
            starts[n] = r;
            counts[n++] = M - r < C ? M - r : C;
        }
        return;
    }
    int64_t r = 0;
    for (int i = 0; i < 2; ++i) {
        starts[n] = r;
        counts[n++] = ramp[i];
        r += ramp[i];
    }
    const int64_t mid = M - ends;
    const int64_t pieces = (mid + C - 1) / C;
    int64_t per = (mid + pieces - 1) / pieces;
    per = (per + 127) / 128 * 128;
    for (int64_t left = mid; left > 0;) {
        const int64_t c = left < per ? left : per;
        starts[n] = r;
        counts[n++] = c;
        r += c;
        left -= c;
    }
    for (int i = 1; i >= 0; --i) {
        starts[n] = r;
        counts[n++] = ramp[i];
        r += ramp[i];
    }
}

struct HostPipe {
    cudaStream_t h2d = nullptr, d2h = nullptr, cs1 = nullptr;
    cudaEvent_t start = nullptr, done = nullptr, prepared = nullptr;
    cudaEvent_t x_ready[2] = {}, x_free[2] = {}, y_ready[2] = {}, y_free[2] = {};
    bool make()
    {
        if (cudaStreamCreateWithFlags(&h2d, cudaStreamNonBlocking) != cudaSuccess) return false;
        if (cudaStreamCreateWithFlags(&d2h, cudaStreamNonBlocking) != cudaSuccess) return false;
        if (cudaStreamCreateWithFlags(&cs1, cudaStreamNonBlocking) != cudaSuccess) return false;
        cudaEvent_t *all[11] = {&start, &done, &prepared, &x_ready[0], &x_ready[1], &x_free[0],
                                &x_free[1], &y_ready[0], &y_ready[1], &y_free[0], &y_free[1]};
        for (cudaEvent_t *e : all)
            if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return false;
        return true;
    }
    ~HostPipe()
    {
        // Destroying a stream or an event with work pending is allowed: its
        // resources are released once that work completes.
        cudaEvent_t all[11] = {start, done, prepared, x_ready[0], x_ready[1], x_free[0],
                               x_free[1], y_ready[0], y_ready[1], y_free[0], y_free[1]};
        for (cudaEvent_t e : all)
            if (e) cudaEventDestroy(e);
        if (h2d) cudaStreamDestroy(h2d);
        if (d2h) cudaStreamDestroy(d2h);
        if (cs1) cudaStreamDestroy(cs1);
    }
};

} // namespace
} // namespace hif4

extern "C" size_t hif4_ffn_w4a4_host_workspace(int64_t M, int64_t D, int64_t F, int64_t chunk_rows, uint32_t flags)
{
    if (M <= 0 || D <= 0 || F <= 0) return 0;
    return ffn_host_layout(ffn_host_chunk(M, chunk_rows), D, F, flags, nullptr);
}

extern "C" hif4_status hif4_ffn_w4a4_host(const void *x_host, int64_t M, int64_t D, int64_t ldx,
                                          const uint8_t *w1_codes, const uint32_t *w1_meta, int64_t F,
                                          const int32_t *mask1_idx, int32_t n_mask1, const void *w1_masked,
                                          const void *b1, const uint8_t *w2_codes, const uint32_t *w2_meta,
                                          const int32_t *mask2_idx, int32_t n_mask2, const void *w2_masked,
                                          const void *b2, void *y_host, int64_t ldy, int64_t chunk_rows,
                                          uint32_t flags, void *workspace, size_t ws_bytes, uint32_t *status,
                                          hif4_stream_t stream)
{
    if (flags & ~HIF4_LINEAR_OUT_F32) return HIF4_ERR_INVALID_ARG;
    if (M < 0 || chunk_rows < 0) return HIF4_ERR_INVALID_ARG;
    hif4_status st = check_ffn_weights(D, F, w1_codes, w1_meta, mask1_idx, n_mask1, w1_masked, b1, w2_codes,
                                       w2_meta, mask2_idx, n_mask2, w2_masked, b2);
    if (st != HIF4_OK || M == 0) return st;
    if (!x_host || !y_host) return HIF4_ERR_INVALID_ARG;
    if (ldx < D || ldy < D) return HIF4_ERR_SHAPE;
    if (M > INT32_MAX / 2) return HIF4_ERR_UNSUPPORTED;
    const size_t ysz = (flags & HIF4_LINEAR_OUT_F32) ? 4 : 2;
    const int64_t C = ffn_host_chunk(M, chunk_rows);
    size_t off[8];
    const size_t need = ffn_host_layout(C, D, F, flags, off);
    if (!workspace || ws_bytes < need) return HIF4_ERR_WORKSPACE;
    if (!aligned_to(workspace, 256)) return HIF4_ERR_ALIGNMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint16_t *what1 = reinterpret_cast<uint16_t *>(ws + off[0]);
    uint16_t *what2 = reinterpret_cast<uint16_t *>(ws + off[1]);
    uint8_t *mask1 = ws + off[2];
    uint8_t *mask2 = ws + off[3];
    uint16_t *xhat1[2] = {reinterpret_cast<uint16_t *>(ws + off[4]),
                          reinterpret_cast<uint16_t *>(ws + off[4] + align256((size_t)C * D * 2))};
    uint16_t *hhat[2] = {reinterpret_cast<uint16_t *>(ws + off[5]),
                         reinterpret_cast<uint16_t *>(ws + off[5] + align256((size_t)C * F * 2))};
    uint8_t *xs[2] = {ws + off[6], ws + off[6] + align256((size_t)C * D * 2)};
    uint8_t *ys[2] = {ws + off[7], ws + off[7] + align256((size_t)C * D * ysz)};

    HostPipe P;
    if (!P.make()) return HIF4_ERR_CUDA;
    // the copy streams start after everything already queued on the caller's stream
    if (cudaEventRecord(P.start, s) != cudaSuccess || cudaStreamWaitEvent(P.h2d, P.start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(P.d2h, P.start, 0) != cudaSuccess)
        return HIF4_ERR_CUDA;
    // On any failure below, the caller's stream still waits for the work
    // already queued on the other streams, so no buffer is released under it.
    auto join = [&](hif4_status result) {
        if (cudaEventRecord(P.done, P.h2d) == cudaSuccess) cudaStreamWaitEvent(s, P.done, 0);
        if (cudaEventRecord(P.done, P.cs1) == cudaSuccess) cudaStreamWaitEvent(s, P.done, 0);
        if (cudaEventRecord(P.done, P.d2h) == cudaSuccess) cudaStreamWaitEvent(s, P.done, 0);
        return result;
    };
    st = ffn_prepare(D, F, w1_codes, w1_meta, mask1_idx, n_mask1, w1_masked, w2_codes, w2_meta, mask2_idx,
                     n_mask2, w2_masked, what1, what2, mask1, mask2, status, s);
    if (st != HIF4_OK) return join(st);
    // the second compute stream starts after the masks and decoded weights
    if (cudaEventRecord(P.prepared, s) != cudaSuccess || cudaStreamWaitEvent(P.cs1, P.prepared, 0) != cudaSuccess)
        return join(HIF4_ERR_CUDA);
    cudaStream_t cs[2] = {s, P.cs1};
    const uint8_t *xh = static_cast<const uint8_t *>(x_host);
    uint8_t *yh = static_cast<uint8_t *>(y_host);
    // at most ceil(M / C) + 5 chunks: equal chunks, or the ramped schedule
    const int64_t max_chunks = (M + C - 1) / C + 5;
    std::vector<int64_t> starts((size_t)max_chunks), counts((size_t)max_chunks);
    int nchunks = 0;
    ffn_host_schedule(M, chunk_rows, C, starts.data(), counts.data(), nchunks);
    for (int i = 0; i < nchunks; ++i) {
        const int sl = i & 1;
        const int64_t r0 = starts[i];
        const int64_t rows = counts[i];
        // copy in (waits for the compute that last read this staging slot)
        if (i >= 2 && cudaStreamWaitEvent(P.h2d, P.x_free[sl], 0) != cudaSuccess) return join(HIF4_ERR_CUDA);
        if (cudaMemcpy2DAsync(xs[sl], (size_t)D * 2, xh + (size_t)r0 * ldx * 2, (size_t)ldx * 2, (size_t)D * 2,
                              (size_t)rows, cudaMemcpyHostToDevice, P.h2d) != cudaSuccess ||
            cudaEventRecord(P.x_ready[sl], P.h2d) != cudaSuccess)
            return join(HIF4_ERR_CUDA);
        // compute on stream sl
        cudaStream_t c = cs[sl];
        if (cudaStreamWaitEvent(c, P.x_ready[sl], 0) != cudaSuccess) return join(HIF4_ERR_CUDA);
        st = fake_quantize_bf16(xs[sl], rows, D, D, n_mask1 > 0 ? mask1 : nullptr, xhat1[sl], D, status, c);
        if (st != HIF4_OK) return join(st);
        if (cudaEventRecord(P.x_free[sl], c) != cudaSuccess) return join(HIF4_ERR_CUDA);
        st = launch_gemm(xhat1[sl], rows, D, D, what1, F, D, b1, n_mask2 > 0 ? mask2 : nullptr, hhat[sl], F,
                         HIF4_LINEAR_GELU_TANH | HIF4_LINEAR_FAKE_QUANT_OUT, status, c);
        if (st != HIF4_OK) return join(st);
        if (i >= 2 && cudaStreamWaitEvent(c, P.y_free[sl], 0) != cudaSuccess) return join(HIF4_ERR_CUDA);
        st = launch_gemm(hhat[sl], rows, F, F, what2, D, F, b2, nullptr, ys[sl], D, flags, status, c);
        if (st != HIF4_OK) return join(st);
        if (cudaEventRecord(P.y_ready[sl], c) != cudaSuccess) return join(HIF4_ERR_CUDA);
        // copy out
        if (cudaStreamWaitEvent(P.d2h, P.y_ready[sl], 0) != cudaSuccess ||
            cudaMemcpy2DAsync(yh + (size_t)r0 * ldy * ysz, (size_t)ldy * ysz, ys[sl], (size_t)D * ysz,
                              (size_t)D * ysz, (size_t)rows, cudaMemcpyDeviceToHost, P.d2h) != cudaSuccess ||
            cudaEventRecord(P.y_free[sl], P.d2h) != cudaSuccess)
            return join(HIF4_ERR_CUDA);
    }
    // the caller's stream completes only after the second compute stream and
    // the last row has landed on the host
    if (cudaEventRecord(P.done, P.cs1) != cudaSuccess || cudaStreamWaitEvent(s, P.done, 0) != cudaSuccess ||
        cudaEventRecord(P.done, P.d2h) != cudaSuccess || cudaStreamWaitEvent(s, P.done, 0) != cudaSuccess)
        return join(HIF4_ERR_CUDA);
    return HIF4_OK;
}
