// hif4_gptq.cu — HiGPTQ, scheme one, on the GPU [HiF4 calibration article,
// section 3.1: 64 columns (one HiF4 unit per row) are quantized at a time
// with their level-1, level-2 and level-3 exponents fixed together, and the
// rest of the block's weights are then updated (GPTQ's Hessian error
// feedback)].
//
//   Hd  = H + damp mean(diag H) I     (a dead input channel: H_ii = 0 -> 1,
//                                       its weights zeroed)
//   Hd^{-1} = U^T U,  U upper triangular
//   per 64-column group g of a block, per row:
//       Q_g = HiF4 unit quantization of the row's current values (protected
//             columns: their BF16 rounding),
//       E   = (W_g - Q_g) U_gg^{-1},   W_c -= E U_{g,c} for the later columns
//             of the block; then once per block W_c -= E_block U_{block,c}
//             for the columns after it.
//
// Factor: with P the index reversal, P Hd P = L' L'^T (Cholesky, lower) gives
// U = P L'^{-1} P (upper, positive diagonal: the Cholesky factor of Hd^{-1}),
// so one Cholesky factorization and one triangular inverse suffice, and the
// inverse of U's 64 x 64 diagonal block g is the reversed diagonal block of
// L' itself.  Both run in FP64 as 64 x 64 tile kernels (a single-block tile
// factorization, then tile products for the panel, the trailing update and
// the inverse's block rows).  The group loop runs in FP32: one warp per row
// quantizes with the exact FP32 encode rule of the streaming quantizer, and
// the lazy update after each block is an FP32 tile GEMM.
#include <cuda_bf16.h>

#include "hif4_encode.cuh"
#include "hif4_internal.cuh"

namespace hif4 {
namespace {

constexpr int TB = 64;            // factorization tile

// ---------------------------------------------------------------- factor

// dead[i] = (H_ii == 0); mean of the fixed diagonal -> *mean (one block).
__global__ void k_diag_mean(const float *H, int64_t K, uint8_t *dead, double *mean)
{
    __shared__ double part[32];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < K; i += blockDim.x) {
        const float d = H[i * K + i];
        dead[i] = d == 0.0f;
        s += d == 0.0f ? 1.0 : (double)d;
    }
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x < 32) {
        s = threadIdx.x < (blockDim.x >> 5) ? part[threadIdx.x] : 0.0;
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (threadIdx.x == 0) *mean = s / (double)K;
    }
}

// A = lower triangle of P Hd P in FP64 (A[i][j] = Hd[K-1-i][K-1-j], i >= j).
__global__ void k_fill_reversed(const float *H, int64_t K, const uint8_t *dead, const double *mean, double damp,
                                double *A)
{
    const int64_t i = blockIdx.y * (int64_t)blockDim.y + threadIdx.y;
    const int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= K || j > i) return;
    const int64_t hi = K - 1 - i, hj = K - 1 - j;
    double v = (double)H[hi * K + hj];
    if (i == j) v = (dead[hi] ? 1.0 : v) + damp * *mean;
    A[i * K + j] = v;
}

// Cholesky factorization of diagonal tile kb of A (lower, in place) and the
// inverse of the factor into Linv (64 x 64).  One block of 256 threads.
// One row of a padded 64 x 64 FP64 tile: 66 doubles (528 bytes) keep rows
// 16-byte aligned for paired loads and offset consecutive rows by 4 banks.
typedef double Tile[TB + 2];
constexpr size_t kTileBytes = sizeof(double) * TB * (TB + 2);

__global__ void __launch_bounds__(256) k_potrf_tile(double *A, int64_t K, int kb, double *Linv, uint32_t *status)
{
    extern __shared__ __align__(16) double smd[];
    Tile *T = reinterpret_cast<Tile *>(smd);
    Tile *I = T + TB;
    __shared__ int bad;
    const int tid = threadIdx.x;
    double *a0 = A + (int64_t)kb * TB * K + (int64_t)kb * TB;
    for (int e = tid; e < TB * TB; e += 256) {
        const int r = e / TB, c = e % TB;
        T[r][c] = c <= r ? a0[(int64_t)r * K + c] : 0.0;
        I[r][c] = 0.0;
    }
    if (tid == 0) bad = 0;
    __syncthreads();
    // left-looking by columns: T[r][j] -= sum_{k<j} T[r][k] T[j][k] for r >= j
    // (four threads per row share the dot product), then the pivot and the
    // scaling of the column below it
    __shared__ double rpiv;
    for (int j = 0; j < TB; ++j) {
        const int r = tid >> 2, part = tid & 3;
        double t = 0.0;
        if (r >= j)
            for (int k = part; k < j; k += 4) t += T[r][k] * T[j][k];
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        if (r >= j && part == 0) T[r][j] -= t;
        __syncthreads();
        if (tid == 0) {
            double d = T[j][j];
            if (!(d > 0.0)) {
                bad = 1;
                d = 1.0;
            }
            d = sqrt(d);
            T[j][j] = d;
            rpiv = 1.0 / d;
        }
        __syncthreads();
        if (r > j && part == 0) T[r][j] *= rpiv;
        __syncthreads();
    }
    // inverse of the lower factor, row by row: I[i][j] = -(sum_{k=j}^{i-1}
    // T[i][k] I[k][j]) / T[i][i] for j < i; four threads share each column's
    // dot product (lanes 4j..4j+3 of the block, combined by shuffles)
    if (tid < TB) I[tid][tid] = 1.0 / T[tid][tid];
    __syncthreads();
    for (int i = 1; i < TB; ++i) {
        const int j = tid >> 2, part = tid & 3;
        double t = 0.0;
        if (j < i)
            for (int k = j + part; k < i; k += 4) t += T[i][k] * I[k][j];
        t += __shfl_xor_sync(0xffffffffu, t, 1);
        t += __shfl_xor_sync(0xffffffffu, t, 2);
        if (j < i && part == 0) I[i][j] = -t * I[i][i];
        __syncthreads();
    }
    for (int e = tid; e < TB * TB; e += 256) {
        const int r = e / TB, c = e % TB;
        if (c <= r) a0[(int64_t)r * K + c] = T[r][c];
        Linv[e] = I[r][c];
    }
    if (tid == 0 && bad && status) atomicOr(status, HIF4_FLAG_NOT_SPD);
}

// 64 x 64 FP64 tile product helpers: 256 threads, each a 4 x 4 sub-block
// (rows 4 (tid / 16) + i, cols 4 (tid % 16) + j).
__device__ __forceinline__ void tile_load(Tile *S, const double *src, int64_t ld)
{
    for (int e = threadIdx.x; e < TB * TB; e += 256) S[e / TB][e % TB] = src[(int64_t)(e / TB) * ld + e % TB];
}

// S = src^T (S[k][c] = src[c][k]): the right operand of an X Y^T product
// stored k-major, so that the product reads it like an X Y operand.
__device__ __forceinline__ void tile_load_t(Tile *S, const double *src, int64_t ld)
{
    for (int e = threadIdx.x; e < TB * TB; e += 256) S[e % TB][e / TB] = src[(int64_t)(e / TB) * ld + e % TB];
}

// acc += X Y (X, Y: 64 x 64 in shared memory; Y read as pairs along a row)
__device__ __forceinline__ void tile_mma_nn(double (&acc)[4][4], const Tile *X, const Tile *Y)
{
    const int r0 = 4 * (threadIdx.x / 16), c0 = 4 * (threadIdx.x % 16);
#pragma unroll 4
    for (int k = 0; k < TB; ++k) {
        double x[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = X[r0 + i][k];
        const double2 ya = *reinterpret_cast<const double2 *>(&Y[k][c0]);
        const double2 yb = *reinterpret_cast<const double2 *>(&Y[k][c0 + 2]);
        const double y[4] = {ya.x, ya.y, yb.x, yb.y};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fma(x[i], y[j], acc[i][j]);
    }
}

// Panel below diagonal tile kb: L[r, kb] = A[r, kb] Linv^T for the row
// tiles r > kb.  One block per row tile (in place: the tile is read whole
// before it is written).
__global__ void __launch_bounds__(256) k_panel(double *A, int64_t K, int kb, const double *Linv)
{
    extern __shared__ __align__(16) double smd[];
    Tile *X = reinterpret_cast<Tile *>(smd);
    Tile *Y = X + TB;
    const int rt = kb + 1 + blockIdx.x;
    double *a = A + (int64_t)rt * TB * K + (int64_t)kb * TB;
    tile_load(X, a, K);
    tile_load_t(Y, Linv, TB);
    __syncthreads();
    double acc[4][4] = {};
    tile_mma_nn(acc, X, Y);
    const int r0 = 4 * (threadIdx.x / 16), c0 = 4 * (threadIdx.x % 16);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) a[(int64_t)(r0 + i) * K + c0 + j] = acc[i][j];
}

// Trailing update after tile kb: A[ti][tj] -= L[ti][kb] L[tj][kb]^T for
// kb < tj <= ti.  Grid (n, n) with n the trailing tile count; blocks above
// the diagonal exit at once, and so does tile (kb + 1, kb + 1) when
// skip_next_diag is set (it is updated first, by a one-block launch, so that
// its factorization can overlap the rest of this update).
__global__ void __launch_bounds__(256) k_syrk(double *A, int64_t K, int kb, int skip_next_diag)
{
    const int ti = kb + 1 + blockIdx.y, tj = kb + 1 + blockIdx.x;
    if (tj > ti || (skip_next_diag && blockIdx.x == 0 && blockIdx.y == 0)) return;
    extern __shared__ __align__(16) double smd[];
    Tile *X = reinterpret_cast<Tile *>(smd);
    Tile *Y = X + TB;
    tile_load(X, A + (int64_t)ti * TB * K + (int64_t)kb * TB, K);
    tile_load_t(Y, A + (int64_t)tj * TB * K + (int64_t)kb * TB, K);
    __syncthreads();
    double acc[4][4] = {};
    tile_mma_nn(acc, X, Y);
    double *c = A + (int64_t)ti * TB * K + (int64_t)tj * TB;
    const int r0 = 4 * (threadIdx.x / 16), c0 = 4 * (threadIdx.x % 16);
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) c[(int64_t)(r0 + i) * K + c0 + j] -= acc[i][j];
}

// Y = L^{-1} (lower, tile rows), right-looking.  Y starts at zero and
// accumulates S[i][j] = sum_{k<i} L[i][k] Y[k][j] in place; at step k block
// row k is finalized (k_trtri_finalize: Y[k][k] = Linv_k, Y[k][j] =
// -Linv_k S[k][j]) and its contribution is added to every later block row
// (k_trtri_update: S[i][j] += L[i][k] Y[k][j], i > k >= j).
__global__ void __launch_bounds__(256) k_trtri_finalize(int64_t K, int k, const double *LinvAll, double *Y)
{
    extern __shared__ __align__(16) double smd[];
    Tile *X = reinterpret_cast<Tile *>(smd);
    Tile *Z = X + TB;
    const int j = blockIdx.x;
    const double *lk = LinvAll + (int64_t)k * TB * TB;
    double *y = Y + (int64_t)k * TB * K + (int64_t)j * TB;
    if (j == k) {
        for (int e = threadIdx.x; e < TB * TB; e += 256) y[(int64_t)(e / TB) * K + e % TB] = lk[e];
        return;
    }
    tile_load(X, lk, TB);
    tile_load(Z, y, K);
    __syncthreads();
    double out[4][4] = {};
    tile_mma_nn(out, X, Z);
    const int r0 = 4 * (threadIdx.x / 16), c0 = 4 * (threadIdx.x % 16);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) y[(int64_t)(r0 + a) * K + c0 + b] = -out[a][b];
}

// grid (k + 1, nb - 1 - k): block (j, ii) updates S[k + 1 + ii][j]
__global__ void __launch_bounds__(256) k_trtri_update(const double *A, int64_t K, int k, double *Y)
{
    extern __shared__ __align__(16) double smd[];
    Tile *X = reinterpret_cast<Tile *>(smd);
    Tile *Z = X + TB;
    const int j = blockIdx.x, i = k + 1 + blockIdx.y;
    tile_load(X, A + (int64_t)i * TB * K + (int64_t)k * TB, K);            // L[i][k]
    tile_load(Z, Y + (int64_t)k * TB * K + (int64_t)j * TB, K);            // Y[k][j]
    __syncthreads();
    double acc[4][4] = {};
    tile_mma_nn(acc, X, Z);
    double *s = Y + (int64_t)i * TB * K + (int64_t)j * TB;
    const int r0 = 4 * (threadIdx.x / 16), c0 = 4 * (threadIdx.x % 16);
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int b = 0; b < 4; ++b) s[(int64_t)(r0 + a) * K + c0 + b] += acc[a][b];
}

// U[i][j] = Y[K-1-i][K-1-j] for j >= i (FP32, upper), 0 below; and the
// inverse of U's diagonal block g, Uinv_g[a][b] = L'[K-1-64g-a][K-1-64g-b]
// for b >= a (the reversed diagonal block of the Cholesky factor).
__global__ void k_build_u(const double *Y, const double *A, int64_t K, float *U, float *UinvG)
{
    const int64_t i = blockIdx.y * (int64_t)blockDim.y + threadIdx.y;
    const int64_t j = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (i >= K || j >= K) return;
    U[i * K + j] = j >= i ? (float)Y[(K - 1 - i) * K + (K - 1 - j)] : 0.0f;
    if (i / TB == j / TB) {
        const int64_t g = i / TB, a = i % TB, b = j % TB;
        UinvG[g * TB * TB + a * TB + b] = b >= a ? (float)A[(K - 1 - i) * K + (K - 1 - j)] : 0.0f;
    }
}

// ------------------------------------------------------------ group loop

constexpr int kRowsPerBlock = 8;            // one warp per weight row

// u8 mask and column -> protected rank (-1 when not protected) from the
// sorted indices; flags bad indices.
__global__ void k_mask_rank(const int32_t *idx, int n, int64_t K, uint8_t *mask, int32_t *rank, uint32_t *status)
{
    uint32_t bad = 0;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < K || i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        if (i < n) {
            const int v = idx[i];
            if (v < 0 || v >= K || (i > 0 && idx[i - 1] >= v)) bad = 1;
        }
        if (i < K) {
            int lo = 0, hi = n;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if (idx[mid] < i) lo = mid + 1;
                else hi = mid;
            }
            const bool hit = lo < n && idx[lo] == i;
            mask[i] = hit ? 1 : 0;
            rank[i] = hit ? lo : -1;
        }
    }
    if (bad && status) atomicOr(status, HIF4_FLAG_BAD_INDEX);
}

// W32 = BF16 w widened (dead input channels zeroed; NaN -> 0, +-Inf ->
// +-FLT_MAX as the quantizer maps them, flagged).
__global__ void k_w_to_f32(const uint16_t *w, int64_t ldw, int64_t N, int64_t K, const uint8_t *dead, float *W,
                           uint32_t *status)
{
    uint32_t bad = 0;
    const int64_t total = N * K;
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = e / K, k = e - n * K;
        const float v = sanitize(bf16_lo(w[n * ldw + k]), bad);
        W[e] = dead[k] ? 0.0f : v;
    }
    if (bad && status) atomicOr(status, HIF4_FLAG_NONFINITE);
}

struct GptqArgs {
    const float *W;          // N x K current weights (FP32)
    int64_t N, K;
    int64_t b0;              // first column of the block
    const float *U;          // K x K upper factor
    const float *UinvG;      // (K / 64) x 64 x 64: inverse of U's diagonal blocks
    const uint8_t *mask;     // u8 [K] or null
    const int32_t *rank;     // [K] protected rank or -1
    int n_masked;
    uint8_t *codes;          // N x K/2
    uint32_t *meta;          // N x K/64
    uint16_t *w_masked;      // N x n_masked
    float *Err;              // N x 64 NG
};

// One block of NG groups (64 NG columns) for kRowsPerBlock rows, a warp per
// row; lane l holds elements 2l, 2l+1 of each group.  Per group: the exact
// FP32 unit quantization (encode rule of the streaming quantizer), D = W - Q,
// E = D Uinv_g (Uinv_g upper), feedback into the block's later groups.
template <int NG>
__global__ void __launch_bounds__(32 * kRowsPerBlock) k_gptq_block(GptqArgs a)
{
    constexpr int NP = NG * (NG - 1) / 2;     // U tiles (g, h), g < h
    extern __shared__ float smf[];
    float *Ui = smf;                          // NG x 64 x 64
    float *Uo = Ui + NG * 4096;               // NP x 64 x 64
    float *Dsh = Uo + NP * 4096;              // kRowsPerBlock x 64
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g0 = a.b0 / 64;
    for (int e = threadIdx.x; e < NG * 4096; e += blockDim.x) Ui[e] = a.UinvG[(g0 + e / 4096) * 4096 + e % 4096];
    for (int p = 0, g = 0; g < NG; ++g)
        for (int h = g + 1; h < NG; ++h, ++p)
            for (int e = threadIdx.x; e < 4096; e += blockDim.x)
                Uo[p * 4096 + e] = a.U[(a.b0 + 64 * g + e / 64) * a.K + a.b0 + 64 * h + e % 64];
    __syncthreads();
    const int64_t n = blockIdx.x * (int64_t)kRowsPerBlock + warp;
    if (n >= a.N) return;                     // no block-wide barrier below
    float *dsh = Dsh + warp * 64;
    float x[NG][2];
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const float2 v = *reinterpret_cast<const float2 *>(a.W + n * a.K + a.b0 + 64 * g + 2 * lane);
        x[g][0] = v.x;
        x[g][1] = v.y;
    }
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const int64_t col = a.b0 + 64 * g + 2 * lane;
        const bool m0 = a.mask && a.mask[col], m1 = a.mask && a.mask[col + 1];
        const float v0 = m0 ? 0.0f : x[g][0], v1 = m1 ? 0.0f : x[g][1];
        // level 1: unit maximum -> scale code
        float am = fmaxf(fabsf(v0), fabsf(v1));
        float a4 = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));       // 4-element group: lanes 2k, 2k+1
        am = a4;
#pragma unroll
        for (int o = 2; o < 32; o <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
        const uint32_t c = select_scale_code(am);
        const float S = e6m2_value(c);
        const uint32_t t = a4 <= 1.75f * S ? 0u : a4 <= 3.5f * S ? 1u : 2u;
        const uint32_t tm = max(t, __shfl_xor_sync(0xffffffffu, t, 2));  // 8-element group: lanes 4j..4j+3
        const uint32_t e2 = tm == 2u, e3 = t > e2 ? t - e2 : 0u;
        const int E = (int)(e2 + e3);
        const float step = ldexp_small(S, E - 2), inv = ldexp_small(__frcp_rn(S), 2 - E);
        const uint32_t q0m = enc::round_exact(fabsf(v0), inv, step), q1m = enc::round_exact(fabsf(v1), inv, step);
        const uint32_t s0 = q0m ? f_bits(v0) >> 31 : 0u, s1 = q1m ? f_bits(v1) >> 31 : 0u;
        const float b0v = __bfloat162float(__float2bfloat16_rn(x[g][0]));
        const float b1v = __bfloat162float(__float2bfloat16_rn(x[g][1]));
        const float q0 = m0 ? b0v : bits_f(f_bits((float)q0m * step) | (s0 << 31));
        const float q1 = m1 ? b1v : bits_f(f_bits((float)q1m * step) | (s1 << 31));
        const uint32_t nib0 = m0 ? 0u : (q0m | (s0 << 3)), nib1 = m1 ? 0u : (q1m | (s1 << 3));
        a.codes[n * (a.K / 2) + col / 2] = (uint8_t)(nib0 | (nib1 << 4));
        const uint32_t b2 = __ballot_sync(0xffffffffu, e2 && (lane & 3) == 0);
        const uint32_t b3 = __ballot_sync(0xffffffffu, e3 && (lane & 1) == 0);
        if (lane == 0) {
            uint32_t mw = c;
#pragma unroll
            for (int j = 0; j < 8; ++j) mw |= ((b2 >> (4 * j)) & 1u) << (8 + j);
#pragma unroll
            for (int k = 0; k < 16; ++k) mw |= ((b3 >> (2 * k)) & 1u) << (16 + k);
            a.meta[n * (a.K / 64) + col / 64] = mw;
        }
        if (m0) a.w_masked[n * a.n_masked + a.rank[col]] = (uint16_t)(f_bits(b0v) >> 16);
        if (m1) a.w_masked[n * a.n_masked + a.rank[col + 1]] = (uint16_t)(f_bits(b1v) >> 16);
        // E = D Uinv_g
        __syncwarp();
        dsh[2 * lane] = x[g][0] - q0;
        dsh[2 * lane + 1] = x[g][1] - q1;
        __syncwarp();
        const float *ui = Ui + g * 4096 + 2 * lane;
        float e0 = 0.0f, e1 = 0.0f;
        for (int i = 0; i < 64; ++i) {
            const float d = dsh[i];
            const float2 u = *reinterpret_cast<const float2 *>(ui + i * 64);
            e0 = fmaf(d, u.x, e0);
            e1 = fmaf(d, u.y, e1);
        }
        *reinterpret_cast<float2 *>(a.Err + n * (64 * NG) + 64 * g + 2 * lane) = make_float2(e0, e1);
        // feedback into the later groups of the block
        if (g + 1 < NG) {
            __syncwarp();
            dsh[2 * lane] = e0;
            dsh[2 * lane + 1] = e1;
            __syncwarp();
#pragma unroll
            for (int h = g + 1; h < NG; ++h) {
                int p = 0;
                for (int gg = 0; gg < g; ++gg) p += NG - 1 - gg;
                p += h - g - 1;
                const float *uo = Uo + p * 4096 + 2 * lane;
                float d0 = 0.0f, d1 = 0.0f;
                for (int i = 0; i < 64; ++i) {
                    const float ei = dsh[i];
                    const float2 u = *reinterpret_cast<const float2 *>(uo + i * 64);
                    d0 = fmaf(ei, u.x, d0);
                    d1 = fmaf(ei, u.y, d1);
                }
                x[h][0] -= d0;
                x[h][1] -= d1;
            }
        }
    }
}

// C (M x Nc, ldc) -= A (M x Kd, lda) B (Kd x Nc, ldb) in FP32: 128 x 128
// tiles, 256 threads with 8 x 8 outputs each, k in steps of 8 through two
// shared-memory buffers (the next step's tiles are loaded into registers
// while the current one is multiplied, one barrier per step).  Kd, lda and
// ldb are multiples of 4 and A, B 16-byte aligned (float4 loads); M and Nc
// are ragged (guarded).
__global__ void __launch_bounds__(256, 2) k_sgemm_sub(float *C, int64_t ldc, const float *A, int64_t lda,
                                                   const float *B, int64_t ldb, int64_t M, int64_t Nc, int Kd)
{
    __shared__ __align__(16) float As[2][8][128 + 4];
    __shared__ __align__(16) float Bs[2][8][128 + 4];
    const int tid = threadIdx.x;
    const int64_t m0 = blockIdx.y * 128ll, n0 = blockIdx.x * 128ll;
    const int tr = tid / 16, tc = tid % 16;           // 16 x 16 threads, 8 x 8 outputs each
    const int ar = tid / 2, ak = 4 * (tid % 2);       // A: row ar, k columns ak..ak+3
    const int bk = tid / 32, bc = 4 * (tid % 32);     // B: k row bk, columns bc..bc+3
    const int64_t gm = m0 + ar, gn = n0 + bc;
    float4 ra, rb;
    auto gload = [&](int k0) {
        ra = gm < M ? *reinterpret_cast<const float4 *>(A + gm * lda + k0 + ak) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float *brow = B + (int64_t)(k0 + bk) * ldb;
        if (gn + 3 < Nc) {
            rb = *reinterpret_cast<const float4 *>(brow + gn);
        } else {
            rb.x = gn < Nc ? brow[gn] : 0.f;
            rb.y = gn + 1 < Nc ? brow[gn + 1] : 0.f;
            rb.z = gn + 2 < Nc ? brow[gn + 2] : 0.f;
            rb.w = 0.f;
        }
    };
    auto sstore = [&](int b) {
        As[b][ak][ar] = ra.x;
        As[b][ak + 1][ar] = ra.y;
        As[b][ak + 2][ar] = ra.z;
        As[b][ak + 3][ar] = ra.w;
        *reinterpret_cast<float4 *>(&Bs[b][bk][bc]) = rb;
    };
    float acc[8][8] = {};
    gload(0);
    sstore(0);
    __syncthreads();
    for (int k0 = 0, b = 0; k0 < Kd; k0 += 8, b ^= 1) {
        const bool more = k0 + 8 < Kd;
        if (more) gload(k0 + 8);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4 *>(&As[b][kk][tr * 8]);
            const float4 a1 = *reinterpret_cast<const float4 *>(&As[b][kk][tr * 8 + 4]);
            const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[b][kk][tc * 8]);
            const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[b][kk][tc * 8 + 4]);
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int jj = 0; jj < 8; ++jj) acc[i][jj] = fmaf(av[i], bv[jj], acc[i][jj]);
        }
        if (more) sstore(b ^ 1);
        __syncthreads();
    }
    // C -= acc, two float4 per row where the 8 columns are inside (C, ldc
    // and the column offset are multiples of 4 floats)
    const int64_t cn0 = n0 + tc * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t cm = m0 + tr * 8 + i;
        if (cm >= M) continue;
        float *crow = C + cm * ldc + cn0;
        if (cn0 + 7 < Nc) {
            float4 *c4 = reinterpret_cast<float4 *>(crow);
            float4 u = c4[0], v = c4[1];
            u.x -= acc[i][0]; u.y -= acc[i][1]; u.z -= acc[i][2]; u.w -= acc[i][3];
            v.x -= acc[i][4]; v.y -= acc[i][5]; v.z -= acc[i][6]; v.w -= acc[i][7];
            c4[0] = u;
            c4[1] = v;
        } else {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                if (cn0 + jj < Nc) crow[jj] -= acc[i][jj];
        }
    }
}

// Xt (K x Tp, BF16) = X^T with the rows past T zero-filled.  32 x 32 tiles.
__global__ void k_transpose_pad(const uint16_t *x, int64_t T, int64_t K, int64_t ldx, int64_t Tp, uint16_t *xt)
{
    __shared__ uint16_t t[32][33];
    const int64_t t0 = blockIdx.x * 32ll, k0 = blockIdx.y * 32ll;
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t tt = t0 + i, kk = k0 + threadIdx.x;
        t[i][threadIdx.x] = (tt < T && kk < K) ? x[tt * ldx + kk] : (uint16_t)0;
    }
    __syncthreads();
    for (int i = threadIdx.y; i < 32; i += blockDim.y) {
        const int64_t kk = k0 + i, tt = t0 + threadIdx.x;
        if (kk < K && tt < Tp) xt[kk * Tp + tt] = t[threadIdx.x][i];
    }
}

} // namespace
} // namespace hif4

using namespace hif4;

namespace hif4 {
namespace {

size_t al256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace sections of hif4_higptq1.
struct GptqLayout {
    size_t A, Y, Linv, U, UinvG, W, Err, mask, rank, dead, mean, total;
};

GptqLayout gptq_layout(int64_t N, int64_t K, int64_t B)
{
    GptqLayout L{};
    const size_t k = (size_t)K, nb = k / TB;
    size_t o = 0;
    auto take = [&](size_t &field, size_t bytes) {
        field = o;
        o += al256(bytes);
    };
    take(L.A, k * k * 8);
    take(L.Y, k * k * 8);
    take(L.Linv, nb * TB * TB * 8);
    take(L.U, k * k * 4);
    take(L.UinvG, nb * TB * TB * 4);
    take(L.W, (size_t)N * k * 4);
    take(L.Err, (size_t)N * (size_t)B * 4);
    take(L.mask, k);
    take(L.rank, k * 4);
    take(L.dead, k);
    take(L.mean, 8);
    L.total = o;
    return L;
}

template <typename F>
bool set_smem_once(F *kernel, size_t bytes, bool &done)
{
    if (done) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes) != cudaSuccess)
        return false;
    done = true;
    return true;
}

// Second stream and events of the factorization look-ahead (created per call,
// released once their work completes).
struct Aux {
    cudaStream_t s2 = nullptr;
    cudaEvent_t ev_diag = nullptr, ev_factored = nullptr;
    bool make()
    {
        return cudaStreamCreateWithFlags(&s2, cudaStreamNonBlocking) == cudaSuccess &&
               cudaEventCreateWithFlags(&ev_diag, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&ev_factored, cudaEventDisableTiming) == cudaSuccess;
    }
    ~Aux()
    {
        if (ev_diag) cudaEventDestroy(ev_diag);
        if (ev_factored) cudaEventDestroy(ev_factored);
        if (s2) cudaStreamDestroy(s2);
    }
};

template <int NG>
hif4_status launch_gptq_block(const GptqArgs &a, cudaStream_t s)
{
    constexpr int NP = NG * (NG - 1) / 2;
    const size_t smem = sizeof(float) * ((NG + NP) * 4096 + kRowsPerBlock * 64);
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!set_smem_once(k_gptq_block<NG>, smem, attr[dev & 63])) return HIF4_ERR_CUDA;
    k_gptq_block<NG><<<(unsigned)((a.N + kRowsPerBlock - 1) / kRowsPerBlock), 32 * kRowsPerBlock, smem, s>>>(a);
    return launch_status();
}

} // namespace
} // namespace hif4

extern "C" size_t hif4_hessian_workspace(int64_t T, int64_t K)
{
    if (T <= 0 || K <= 0) return 0;
    const int64_t Tp = (T + 63) / 64 * 64;
    return al256((size_t)K * (size_t)Tp * 2);
}

extern "C" hif4_status hif4_hessian(const void *x, int64_t T, int64_t K, int64_t ldx, float *H, void *workspace,
                                    size_t ws_bytes, uint32_t *status, hif4_stream_t stream)
{
    if (T <= 0 || K <= 0 || !x || !H) return HIF4_ERR_INVALID_ARG;
    if (K % HIF4_UNIT != 0 || ldx < K) return HIF4_ERR_SHAPE;
    if (K > 65536 || T > INT32_MAX / 2) return HIF4_ERR_UNSUPPORTED;
    if (!aligned_to(x, 2) || !aligned16(H)) return HIF4_ERR_ALIGNMENT;
    if (!workspace || ws_bytes < hif4_hessian_workspace(T, K)) return HIF4_ERR_WORKSPACE;
    if (!aligned_to(workspace, 256)) return HIF4_ERR_ALIGNMENT;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int64_t Tp = (T + 63) / 64 * 64;
    uint16_t *xt = static_cast<uint16_t *>(workspace);
    k_transpose_pad<<<dim3((unsigned)((Tp + 31) / 32), (unsigned)((K + 31) / 32)), dim3(32, 8), 0, s>>>(
        static_cast<const uint16_t *>(x), T, K, ldx, Tp, xt);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    // H = Xt Xt^T on the tensor cores, FP32 accumulation and output
    return hif4_gemm_bf16(xt, K, Tp, Tp, xt, K, Tp, nullptr, H, K, HIF4_LINEAR_OUT_F32, status, stream);
}

extern "C" size_t hif4_higptq1_workspace(int64_t N, int64_t K, int64_t blocksize)
{
    if (N <= 0 || K <= 0 || K % HIF4_UNIT != 0) return 0;
    const int64_t B = blocksize == 0 ? 128 : blocksize;
    if (B % HIF4_UNIT != 0 || B > 256 || B <= 0) return 0;
    return gptq_layout(N, K, B).total;
}

extern "C" hif4_status hif4_higptq1(const void *w, int64_t N, int64_t K, int64_t ldw, const float *H,
                                    const int32_t *mask_idx, int32_t n_masked, double damp, int64_t blocksize,
                                    uint8_t *codes, uint32_t *meta, void *w_masked, void *workspace,
                                    size_t ws_bytes, uint32_t *status, hif4_stream_t stream)
{
    if (N <= 0 || K <= 0 || n_masked < 0 || !(damp >= 0.0) || !(damp < 1e30)) return HIF4_ERR_INVALID_ARG;
    if (K % HIF4_UNIT != 0 || ldw < K) return HIF4_ERR_SHAPE;
    const int64_t B = blocksize == 0 ? 128 : blocksize;
    if (B <= 0 || B % HIF4_UNIT != 0 || B > 256) return HIF4_ERR_INVALID_ARG;
    if (K > 32768 || N > ((int64_t)1 << 31) || n_masked > K) return HIF4_ERR_UNSUPPORTED;
    if (!w || !H || !codes || !meta || (n_masked > 0 && (!mask_idx || !w_masked))) return HIF4_ERR_INVALID_ARG;
    if (!aligned_to(w, 2) || !aligned_to(H, 4) || !aligned_to(meta, 4) ||
        (n_masked > 0 && (!aligned_to(mask_idx, 4) || !aligned_to(w_masked, 2))))
        return HIF4_ERR_ALIGNMENT;
    const GptqLayout L = gptq_layout(N, K, B);
    if (!workspace || ws_bytes < L.total) return HIF4_ERR_WORKSPACE;
    if (!aligned_to(workspace, 256)) return HIF4_ERR_ALIGNMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    double *A = reinterpret_cast<double *>(ws + L.A);
    double *Y = reinterpret_cast<double *>(ws + L.Y);
    double *Linv = reinterpret_cast<double *>(ws + L.Linv);
    float *U = reinterpret_cast<float *>(ws + L.U);
    float *UinvG = reinterpret_cast<float *>(ws + L.UinvG);
    float *W = reinterpret_cast<float *>(ws + L.W);
    float *Err = reinterpret_cast<float *>(ws + L.Err);
    uint8_t *mask = ws + L.mask;
    int32_t *rank = reinterpret_cast<int32_t *>(ws + L.rank);
    uint8_t *dead = ws + L.dead;
    double *mean = reinterpret_cast<double *>(ws + L.mean);
    const int nb = (int)(K / TB);

    static bool attr2[64] = {false}, attr2b[64] = {false}, attr2c[64] = {false}, attr2d[64] = {false},
                attr2e[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!set_smem_once(k_potrf_tile, 2 * kTileBytes, attr2[dev & 63]) ||
        !set_smem_once(k_panel, 2 * kTileBytes, attr2b[dev & 63]) ||
        !set_smem_once(k_syrk, 2 * kTileBytes, attr2c[dev & 63]) ||
        !set_smem_once(k_trtri_finalize, 2 * kTileBytes, attr2d[dev & 63]) ||
        !set_smem_once(k_trtri_update, 2 * kTileBytes, attr2e[dev & 63]))
        return HIF4_ERR_CUDA;

    // 1. protected columns, Hessian diagonal statistics, FP32 working weights
    if (n_masked > 0) {
        const int64_t work = K > n_masked ? K : n_masked;
        k_mask_rank<<<(unsigned)((work + 255) / 256), 256, 0, s>>>(mask_idx, n_masked, K, mask, rank, status);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    }
    k_diag_mean<<<1, 1024, 0, s>>>(H, K, dead, mean);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    {
        const int64_t total = N * K;
        int64_t blocks = (total + 255) / 256;
        if (blocks > 8 * (int64_t)sm_count()) blocks = 8 * (int64_t)sm_count();
        k_w_to_f32<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint16_t *>(w), ldw, N, K, dead, W, status);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    }
    // 2. P Hd P = L' L'^T (FP64, 64 x 64 tiles, right-looking)
    k_fill_reversed<<<dim3((unsigned)((K + 31) / 32), (unsigned)((K + 7) / 8)), dim3(32, 8), 0, s>>>(
        H, K, dead, mean, damp, A);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    //    Look-ahead: after panel kb, diagonal tile kb + 1 is updated first and
    //    factored on a second stream while the rest of the trailing update
    //    runs (disjoint tiles); panel kb + 1 waits for it.
    Aux X;
    if (!X.make()) return HIF4_ERR_CUDA;
    auto join = [&](hif4_status r) {
        if (cudaEventRecord(X.ev_factored, X.s2) == cudaSuccess) cudaStreamWaitEvent(s, X.ev_factored, 0);
        return r;
    };
    k_potrf_tile<<<1, 256, 2 * kTileBytes, s>>>(A, K, 0, Linv, status);
    if (launch_status() != HIF4_OK) return join(HIF4_ERR_CUDA);
    for (int kb = 0; kb < nb; ++kb) {
        const int n = nb - 1 - kb;
        if (n == 0) break;
        if (kb > 0 && cudaStreamWaitEvent(s, X.ev_factored, 0) != cudaSuccess) return join(HIF4_ERR_CUDA);
        k_panel<<<n, 256, 2 * kTileBytes, s>>>(A, K, kb, Linv + (size_t)kb * TB * TB);
        k_syrk<<<1, 256, 2 * kTileBytes, s>>>(A, K, kb, 0);                   // tile (kb + 1, kb + 1)
        if (launch_status() != HIF4_OK || cudaEventRecord(X.ev_diag, s) != cudaSuccess ||
            cudaStreamWaitEvent(X.s2, X.ev_diag, 0) != cudaSuccess)
            return join(HIF4_ERR_CUDA);
        k_potrf_tile<<<1, 256, 2 * kTileBytes, X.s2>>>(A, K, kb + 1, Linv + (size_t)(kb + 1) * TB * TB, status);
        if (launch_status() != HIF4_OK || cudaEventRecord(X.ev_factored, X.s2) != cudaSuccess)
            return join(HIF4_ERR_CUDA);
        if (n > 1) k_syrk<<<dim3(n, n), 256, 2 * kTileBytes, s>>>(A, K, kb, 1);
        if (launch_status() != HIF4_OK) return join(HIF4_ERR_CUDA);
    }
    if (nb > 1 && cudaStreamWaitEvent(s, X.ev_factored, 0) != cudaSuccess) return join(HIF4_ERR_CUDA);
    // 3. Y = L'^{-1} (right-looking by block rows), then U = P Y P and the
    //    inverses of U's diagonal blocks
    if (cudaMemsetAsync(Y, 0, (size_t)K * K * 8, s) != cudaSuccess) return HIF4_ERR_CUDA;
    for (int k = 0; k < nb; ++k) {
        k_trtri_finalize<<<k + 1, 256, 2 * kTileBytes, s>>>(K, k, Linv, Y);
        if (k + 1 < nb) k_trtri_update<<<dim3(k + 1, nb - 1 - k), 256, 2 * kTileBytes, s>>>(A, K, k, Y);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    }
    k_build_u<<<dim3((unsigned)((K + 31) / 32), (unsigned)((K + 7) / 8)), dim3(32, 8), 0, s>>>(Y, A, K, U, UinvG);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    // 4. the group loop: per block, the groups with their in-block feedback,
    //    then the lazy update of every later column
    for (int64_t b0 = 0; b0 < K; b0 += B) {
        const int64_t b1 = b0 + B < K ? b0 + B : K;
        const int NG = (int)((b1 - b0) / HIF4_UNIT);
        GptqArgs a{};
        a.W = W;
        a.N = N;
        a.K = K;
        a.b0 = b0;
        a.U = U;
        a.UinvG = UinvG;
        a.mask = n_masked > 0 ? mask : nullptr;
        a.rank = rank;
        a.n_masked = n_masked;
        a.codes = codes;
        a.meta = meta;
        a.w_masked = static_cast<uint16_t *>(w_masked);
        a.Err = Err;
        hif4_status st = NG == 1 ? launch_gptq_block<1>(a, s)
                       : NG == 2 ? launch_gptq_block<2>(a, s)
                       : NG == 3 ? launch_gptq_block<3>(a, s)
                                 : launch_gptq_block<4>(a, s);
        if (st != HIF4_OK) return st;
        if (b1 < K) {
            k_sgemm_sub<<<dim3((unsigned)((K - b1 + 127) / 128), (unsigned)((N + 127) / 128)), 256, 0, s>>>(
                W + b1, K, Err, 64 * NG, U + b0 * K + b1, K, N, K - b1, 64 * NG);
            if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
        }
    }
    return HIF4_OK;
}
