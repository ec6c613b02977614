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
// L' itself.  Both run in FP64 by one recursion over halves whose products
// are FP64 tensor-core GEMMs (the factor section below).  The group loop
// runs in FP32: one warp per row quantizes with the exact FP32 encode rule
// of the streaming quantizer, and the lazy update after each block is a GEMM
// on the TF32 tensor cores with split operands (three TF32 products per
// FP32 product, FP32 accumulation).
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "hif4_encode.cuh"
#include "hif4_internal.cuh"
#include "hif4_pdl.cuh"
#include "hif4_sm100.cuh"

namespace hif4 {

bool make_tensor_map_f32_2d_sw128(CUtensorMap *map, const void *base, uint64_t inner, uint64_t outer,
                                  uint64_t row_stride_bytes, uint32_t box_inner, uint32_t box_outer);

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

// The factor and its inverse, recursively.  For a diagonal block of n rows
// at offset o (n a multiple of 64), split n = n1 + n2 and
//   (L11, L11^{-1}) of A11                    recursively
//   T   = A21 L11^{-T}                         (= L21)
//   A22 = A22 - T T^T                          (lower tiles)
//   T2  = T L11^{-1}
//   (L22, L22^{-1}) of A22                    recursively
//   Y21 = -L22^{-1} T2
// with Y holding L^{-1}: [[L11, 0], [L21, L22]]^{-1} has the off-diagonal
// block -L22^{-1} L21 L11^{-1}.  The split falls on a multiple of 128 rows
// where n allows it; a block of 128 (or 64) rows is a leaf: one thread block
// factors it and inverts its factor.  Only the leaves' blocks of L are kept
// (in A); every product is an FP64 GEMM that skips the tiles in which a
// triangular operand is zero, so the whole factor costs K^3/3 + K^3/3 FLOP.

constexpr int HB = TB / 2;               // panel of the leaf: one warp's Cholesky block
constexpr int HP = HB + 1;               // smem row of a diagonal (Cholesky) tile, doubles: lane = row
constexpr int LS = HB + 4;               // smem row of a product tile, doubles: conflict-free MMA fragments
constexpr int DT = HB * HP;              // doubles of a diagonal tile
constexpr int LT = HB * LS;              // doubles of a product tile

// d (8 x 8, two per lane: row lane / 4, columns 2 (lane % 4) + {0, 1}) +=
// a (8 x 4, row lane / 4, column lane % 4) b (4 x 8, row lane % 4, column lane / 4)
__device__ __forceinline__ void dmma884(double (&d)[2], double a, double b)
{
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(d[0]), "+d"(d[1])
                 : "d"(a), "d"(b));
}

// Cholesky of the 32 x 32 lower block S (shared memory) by one warp, lane r
// owning row r in registers.  Column j: every lane takes the pivot d (the
// diagonal entry as updated through column j - 1) from shared memory and
// forms l_r = a_rj / sqrt(d) (sqrt(d) on lane j); the column goes to shared
// memory once, lane j + 1 publishes the next pivot a_{j+1,j+1} - l^2, and
// after one __syncwarp each lane updates its later entries a_rw -= l_r l_w
// from 16-byte broadcast reads of the column.  The rank-one update of the
// later columns is off the critical path, which is one shared-memory round
// trip and one reciprocal square root per column.  On return S holds the
// factor, 0 above the diagonal.  Pivots that are not positive are replaced
// by 1 and counted in bad.
__device__ __forceinline__ void warp_chol32(double (*S)[HP], int &bad)
{
    __shared__ __align__(16) double colb[2][HB];
    __shared__ double piv[2];
    const int r = threadIdx.x & 31;
    double a[HB];
#pragma unroll
    for (int c = 0; c < HB; ++c) a[c] = c <= r ? S[r][c] : 0.0;
    if (r == 0) piv[0] = a[0];
    __syncwarp();
#pragma unroll
    for (int j = 0; j < HB; ++j) {
        double d = piv[j & 1];
        const bool ok = d > 0.0;
        if (!ok) d = 1.0;
        const double rs = rsqrt(d);
        const double l = r == j ? d * rs : (r > j ? a[j] * rs : 0.0);
        bad |= (int)(!ok && r == j);
        a[j] = l;
        if (j + 1 < HB) {
            colb[j & 1][r] = l;
            if (r == j + 1) piv[(j + 1) & 1] = fma(-l, l, a[j + 1]);
            __syncwarp();
            int w = j + 1;
            if (w & 1) {
                a[w] = fma(-l, colb[j & 1][w], a[w]);
                ++w;
            }
#pragma unroll
            for (; w < HB; w += 2) {
                const double2 c2 = *reinterpret_cast<const double2 *>(&colb[j & 1][w]);
                a[w] = fma(-l, c2.x, a[w]);
                a[w + 1] = fma(-l, c2.y, a[w + 1]);
            }
        }
    }
#pragma unroll
    for (int c = 0; c < HB; ++c) S[r][c] = c <= r ? a[c] : 0.0;
    __syncwarp();
}

// Inverse of the 32 x 32 lower factor L (shared memory) into X (row stride
// LS, 0 above the diagonal), one warp: lane c computes column c by forward
// substitution, L's rows read from shared memory as broadcasts.
__device__ __forceinline__ void warp_inv32(const double (*L)[HP], double *X)
{
    __shared__ double rdiag[HB];
    const int c = threadIdx.x & 31;
    rdiag[c] = 1.0 / L[c][c];
    __syncwarp();
    double x[HB];
#pragma unroll
    for (int r = 0; r < HB; ++r) {
        double s0 = 0.0, s1 = 0.0;
#pragma unroll
        for (int k = 0; k + 1 < r; k += 2) {
            s0 = fma(L[r][k], x[k], s0);
            s1 = fma(L[r][k + 1], x[k + 1], s1);
        }
        if (r & 1) s0 = fma(L[r][r - 1], x[r - 1], s0);
        x[r] = ((r == c ? 1.0 : 0.0) - (s0 + s1)) * rdiag[r];
    }
#pragma unroll
    for (int r = 0; r < HB; ++r) X[r * LS + c] = x[r];
    __syncwarp();
}

// One warp: the 32 x 32 lower block S -> its factor in S (0 above the
// diagonal) and the factor's inverse in X.  Not inlined: the leaf calls it
// once per panel, and one copy of the code keeps what the leaf fetches small.
__device__ __noinline__ void warp_factor_panel(double (*S)[HP], double *X, int &bad)
{
    warp_chol32(S, bad);
    warp_inv32(S, X);
}

// One warp, one 8-row strip s of a 32 x 32 product on the FP64 MMA:
// acc[n] += A[8 s .. 8 s + 8, :] B[:, 8 n .. 8 n + 8] over the 32-deep inner
// dimension.  A row-major (row stride LS); B row-major 32 x 32 (BT false) or
// given as B^T row-major (BT true), row stride LS.
template <bool BT>
__device__ __forceinline__ void strip_mma(double (&acc)[4][2], const double *A, const double *B, int s)
{
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    const double *ar = A + (8 * s + gid) * LS + tig;
#pragma unroll
    for (int k = 0; k < HB; k += 4) {
        const double a = ar[k];
        double b[4];
#pragma unroll
        for (int n = 0; n < 4; ++n) b[n] = BT ? B[(8 * n + gid) * LS + k + tig] : B[(k + tig) * LS + 8 * n + gid];
#pragma unroll
        for (int n = 0; n < 4; ++n) dmma884(acc[n], a, b[n]);
    }
}

// out strip (row stride ld) = alpha acc, or (SUB) out -= acc
template <bool SUB>
__device__ __forceinline__ void strip_store(double *out, int ld, int s, const double (&acc)[4][2], double alpha)
{
    const int lane = threadIdx.x & 31, gid = lane >> 2, tig = lane & 3;
    double *o = out + (8 * s + gid) * ld + 2 * tig;
#pragma unroll
    for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            if (SUB)
                o[8 * n + q] -= acc[n][q];
            else
                o[8 * n + q] = alpha * acc[n][q];
        }
}

// Shared memory of a leaf of P panels (32 P rows): the diagonal tiles of A
// (then L), the off-diagonal tiles of A (then L), the diagonal tiles of
// L^{-1}, its off-diagonal tiles, and P - 1 tiles for the products
// X_pp L_pk of the current panel.
template <int P>
constexpr size_t leaf_smem()
{
    return sizeof(double) * ((size_t)P * DT + (size_t)(P * (P - 1) + P + P - 1) * LT);
}
constexpr size_t kLeafSmem2 = leaf_smem<2>(), kLeafSmem4 = leaf_smem<4>();

// One diagonal block of 32 P rows (P = 2 or 4): its Cholesky factor (lower,
// in place in A) and the factor's inverse into Y (zeros above the diagonal),
// right-looking over 32-column panels p = 0 .. P - 1 with 32 x 32 tiles in
// shared memory.  Per panel:
//   warp 0:    L_pp = chol(A_pp), X_pp = L_pp^{-1}
//   all warps: L_ip = A_ip X_pp^T (i > p);  M_k = X_pp L_pk (k < p)
//   all warps: A_ij -= L_ip L_jp^T (p < j <= i);
//              Y_pj = -sum_{k = j}^{p - 1} M_k Y_kj (j < p, Y_jj = X_jj)
// (the last from L Y = I: L_pp Y_pj = -sum_{k < p} L_pk Y_kj).  The
// products run as 8 x 32 strips on the FP64 MMA, 8 warps taking strips in
// turn.  A pivot that is not positive is replaced by 1 and reported as
// HIF4_FLAG_NOT_SPD.  256 threads.
template <int P>
__global__ void __launch_bounds__(256, 1) k_leaf(double *A, int64_t lda, double *Y, int64_t ldy, uint32_t *status)
{
    constexpr int NO = P * (P - 1) / 2;                          // off-diagonal tiles
    pdl_enter();
    extern __shared__ __align__(16) double smd[];
    double *const Dg = smd;                                      // P diagonal tiles, row stride HP
    double *const Og = smd + P * DT;                             // NO off-diagonal tiles of A / L
    double *const Xg = Og + NO * LT;                             // P diagonal tiles of L^{-1}
    double *const Yg = Xg + P * LT;                              // NO off-diagonal tiles of L^{-1}
    double *const Mg = Yg + NO * LT;                             // P - 1 tiles X_pp L_pk
    auto D = [&](int p) { return reinterpret_cast<double(*)[HP]>(Dg + p * DT); };
    auto oi = [](int i, int j) { return i * (i - 1) / 2 + j; }; // i > j
    auto O = [&](int i, int j) { return Og + oi(i, j) * LT; };
    auto X = [&](int p) { return Xg + p * LT; };
    auto Yo = [&](int i, int j) { return Yg + oi(i, j) * LT; };
    auto M = [&](int k) { return Mg + k * LT; };
    __shared__ int bad_all;
    const int tid = threadIdx.x, warp = tid >> 5;

    // the lower tiles of A (zeros above the diagonal of the diagonal tiles),
    // as 16-byte pairs: a tile row is 16 pairs
    auto tile_of = [](int t, int &ti, int &tj) {                 // row-major over the lower tiles
        ti = 0;
        for (int u = t; u > ti; ++ti) u -= ti + 1;
        tj = t - ti * (ti + 1) / 2;
    };
    {
        double2 v[P + NO][2];
#pragma unroll
        for (int t = 0; t < P + NO; ++t) {
            int ti, tj;
            tile_of(t, ti, tj);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int e = tid + 256 * q, r = e >> 4, c = 2 * (e & 15);
                v[t][q] = *reinterpret_cast<const double2 *>(A + (int64_t)(HB * ti + r) * lda + HB * tj + c);
            }
        }
#pragma unroll
        for (int t = 0; t < P + NO; ++t) {
            int ti, tj;
            tile_of(t, ti, tj);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const int e = tid + 256 * q, r = e >> 4, c = 2 * (e & 15);
                if (ti == tj) {
                    D(ti)[r][c] = c <= r ? v[t][q].x : 0.0;
                    D(ti)[r][c + 1] = c + 1 <= r ? v[t][q].y : 0.0;
                } else {
                    *reinterpret_cast<double2 *>(O(ti, tj) + r * LS + c) = v[t][q];
                }
            }
        }
    }
    if (tid == 0) bad_all = 0;
    __syncthreads();

    int bad = 0;
#pragma unroll 1
    for (int p = 0; p < P; ++p) {
        if (warp == 0) warp_factor_panel(D(p), X(p), bad);
        __syncthreads();
        // L_ip = A_ip X_pp^T (in place: a strip reads only its own rows of A_ip), M_k = X_pp L_pk
        const int nL = 4 * (P - 1 - p), nM = 4 * p;
        for (int t = warp; t < nL + nM; t += 8) {
            double acc[4][2] = {};
            const int s = t & 3;
            if (t < nL) {
                double *o = O(p + 1 + (t >> 2), p);
                strip_mma<true>(acc, o, X(p), s);
                __syncwarp();
                strip_store<false>(o, LS, s, acc, 1.0);
            } else {
                const int k = (t - nL) >> 2;
                strip_mma<false>(acc, X(p), O(p, k), s);
                strip_store<false>(M(k), LS, s, acc, 1.0);
            }
        }
        __syncthreads();
        // trailing update of the lower tiles right of panel p; row p of L^{-1}
        const int nS = 2 * (P - 1 - p) * (P - p), nY = 4 * p;
        for (int t = warp; t < nS + nY; t += 8) {
            double acc[4][2] = {};
            const int s = t & 3;
            if (t < nS) {
                int i = p + 1, q = t >> 2;                       // q -> (i, j), p < j <= i
                while (q >= i - p) q -= i++ - p;
                const int j = p + 1 + q;
                strip_mma<true>(acc, O(i, p), O(j, p), s);
                if (i == j)
                    strip_store<true>(&D(j)[0][0], HP, s, acc, 0.0);
                else
                    strip_store<true>(O(i, j), LS, s, acc, 0.0);
            } else {
                const int j = (t - nS) >> 2;
                for (int k = j; k < p; ++k) strip_mma<false>(acc, M(k), k == j ? X(j) : Yo(k, j), s);
                strip_store<false>(Yo(p, j), LS, s, acc, -1.0);
            }
        }
        __syncthreads();
    }
    if (warp == 0 && bad) atomicOr(&bad_all, 1);

    // L (lower tiles, zeros above the diagonal) -> A; L^{-1} (the whole
    // block, zeros above the diagonal) -> Y; 16-byte pairs
#pragma unroll
    for (int t = 0; t < P * P; ++t) {
        const int ti = t / P, tj = t % P;
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int e = tid + 256 * q, r = e >> 4, c = 2 * (e & 15);
            const int64_t gr = HB * ti + r, gc = HB * tj + c;
            double2 y = make_double2(0.0, 0.0);
            if (ti == tj) {
                *reinterpret_cast<double2 *>(A + gr * lda + gc) = make_double2(D(ti)[r][c], D(ti)[r][c + 1]);
                y = *reinterpret_cast<const double2 *>(X(ti) + r * LS + c);
            } else if (ti > tj) {
                *reinterpret_cast<double2 *>(A + gr * lda + gc) =
                    *reinterpret_cast<const double2 *>(O(ti, tj) + r * LS + c);
                y = *reinterpret_cast<const double2 *>(Yo(ti, tj) + r * LS + c);
            }
            *reinterpret_cast<double2 *>(Y + gr * ldy + gc) = y;
        }
    }
    __syncthreads();
    if (tid == 0 && bad_all && status) atomicOr(status, HIF4_FLAG_NOT_SPD);
}

// FP64 GEMM on whole tiles: C = alpha op(A) op(B) (+ C if beta), on the FP64
// tensor-core MMA (m8n8k4).  One T x T tile of C per 128-thread block (T =
// 64, or 32 below), a T/2 x T/2 quarter per warp (T/16 x T/16 MMA tiles); the K loop
// runs in 32-deep stages that cp.async copies keep NS deep in shared memory
// (NS - 1 stages in flight ahead of the one in use: the small products'
// whole K range at once) in the operands' own layouts: A row-major, B k-major (B row-major)
// or n-major (BT, B^T row-major), whose fragments the MMA reads directly.  A
// is M x K row-major; B is K x N row-major, or (BT) N x K row-major holding
// B^T.  Triangular operands skip their zero tiles: tri_a (A lower) ends the
// K loop after tile ti; tri_b with B lower starts it at tile tj, with B^T
// lower (BT) ends it after tile tj.  lower_c computes only the tiles
// tj <= ti.  M, N, K are multiples of 64; pointers and leading dimensions
// keep 16-byte alignment.
constexpr int KC = 32;                    // K per stage
constexpr int AS = KC + 4;                // smem row of an n- or m-major stage (doubles; 16-byte multiple)
constexpr int kGemmThreads = 128;

// Tile T x T of C per block (T = 64, or 32 for products with few tiles, so
// that they still spread over the SMs): the A stage (T x 32) and the larger
// of the B stages (T x 32 n-major, 32 x (T + 4) k-major).
template <int T>
constexpr int stage_doubles()
{
    return T * AS + (T * AS > KC * (T + 4) ? T * AS : KC * (T + 4));
}
template <int T, int NS>
constexpr size_t gemm_smem()
{
    return sizeof(double) * NS * stage_doubles<T>();
}

struct Dgemm {
    const double *A;
    int64_t lda;
    const double *B;
    int64_t ldb;
    double *C;
    int64_t ldc;
    int M, N, K;
    double alpha;
    int beta, tri_a, tri_b, lower_c;
};

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(sm100::smem_addr(smem_dst)), "l"(gmem_src)
                 : "memory");
}

template <bool BT, int T, int NS>
__global__ void __launch_bounds__(kGemmThreads, 3) k_dgemm(Dgemm g)
{
    pdl_enter();
    constexpr int BS = T + 4;                 // smem row of a k-major B stage
    constexpr int SD = stage_doubles<T>();
    constexpr int F = T / 16;                 // MMA tiles per warp side (warp tile T/2 x T/2)
    constexpr int CH = T * KC / 2;            // 16-byte chunks of one operand stage
    const int tj = blockIdx.x, ti = blockIdx.y;
    if (g.lower_c && tj > ti) return;
    extern __shared__ __align__(16) double smd[];
    int k0 = 0, k1 = g.K;
    if (g.tri_a) k1 = min(k1, T * (ti + 1));
    if (g.tri_b) {
        if (BT)
            k1 = min(k1, T * (tj + 1));
        else
            k0 = max(k0, T * tj);
    }
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int wm = (T / 2) * (warp >> 1), wn = (T / 2) * (warp & 1), gid = lane >> 2, tig = lane & 3;
    const double *Ab = g.A + (int64_t)ti * T * g.lda;
    const double *Bb = BT ? g.B + (int64_t)tj * T * g.ldb : g.B + (int64_t)tj * T;
    // one stage: T x 32 of A and 32 x T of B as 16-byte chunks
    auto issue = [&](int k, int st) {
        double *As = smd + st * SD, *Bs = As + T * AS;
#pragma unroll
        for (int q = 0; q < CH / kGemmThreads; ++q) {
            const int idx = tid + kGemmThreads * q;                  // 0 .. CH - 1
            cp_async16(As + (idx >> 4) * AS + 2 * (idx & 15), Ab + (int64_t)(idx >> 4) * g.lda + k + 2 * (idx & 15));
            if (BT)
                cp_async16(Bs + (idx >> 4) * AS + 2 * (idx & 15),
                           Bb + (int64_t)(idx >> 4) * g.ldb + k + 2 * (idx & 15));
            else
                cp_async16(Bs + (idx / (T / 2)) * BS + 2 * (idx % (T / 2)),
                           Bb + (int64_t)(k + idx / (T / 2)) * g.ldb + 2 * (idx % (T / 2)));
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    double acc[F][F][2] = {};
    auto compute = [&](int st) {
        const double *As = smd + st * SD, *Bs = As + T * AS;
#pragma unroll
        for (int kk = 0; kk < KC; kk += 4) {
            double a[F], b[F];
#pragma unroll
            for (int i = 0; i < F; ++i) a[i] = As[(wm + 8 * i + gid) * AS + kk + tig];
#pragma unroll
            for (int j = 0; j < F; ++j)
                b[j] = BT ? Bs[(wn + 8 * j + gid) * AS + kk + tig] : Bs[(kk + tig) * BS + wn + 8 * j + gid];
#pragma unroll
            for (int i = 0; i < F; ++i)
#pragma unroll
                for (int j = 0; j < F; ++j) dmma884(acc[i][j], a[i], b[j]);
        }
    };
    if constexpr (NS == 2) {                  // double buffer: the next stage is issued before this one is awaited
        if (k0 < k1) {
            issue(k0, 0);
            int st = 0;
            for (int k = k0; k < k1; k += KC, st ^= 1) {
                if (k + KC < k1) {
                    issue(k + KC, st ^ 1);
                    asm volatile("cp.async.wait_group 1;" ::: "memory");
                } else {
                    asm volatile("cp.async.wait_group 0;" ::: "memory");
                }
                __syncthreads();
                compute(st);
                __syncthreads();              // stage st is refilled two steps on
            }
        }
    } else {
        const int nk = k0 < k1 ? (k1 - k0) / KC : 0;
#pragma unroll
        for (int q = 0; q < NS - 1; ++q) {    // one commit group per stage, empty past the end
            if (q < nk)
                issue(k0 + q * KC, q);
            else
                asm volatile("cp.async.commit_group;" ::: "memory");
        }
        for (int it = 0; it < nk; ++it) {
            asm volatile("cp.async.wait_group %0;" ::"n"(NS - 2) : "memory");
            __syncthreads();                  // stage it is in; stage it - 1 is consumed
            const int nx = it + NS - 1;       // refills the slot of stage it - 1
            if (nx < nk)
                issue(k0 + nx * KC, nx % NS);
            else
                asm volatile("cp.async.commit_group;" ::: "memory");
            compute(it % NS);
        }
    }
#pragma unroll
    for (int i = 0; i < F; ++i)
#pragma unroll
        for (int j = 0; j < F; ++j) {
            double2 *cp = reinterpret_cast<double2 *>(g.C + (int64_t)(ti * T + wm + 8 * i + gid) * g.ldc + tj * T +
                                                      wn + 8 * j + 2 * tig);
            double2 u = make_double2(g.alpha * acc[i][j][0], g.alpha * acc[i][j][1]);
            if (g.beta) {
                const double2 cu = *cp;
                u.x += cu.x;
                u.y += cu.y;
            }
            *cp = u;
        }
}

// ------------------------------------------------------------ group loop

constexpr int kWarpsPerBlock = 8;           // one warp per weight row at a time
constexpr int kRowsPerWarp = 4;             // rows a warp takes in turn (amortizes the U tiles' load)
constexpr int kRowsPerBlock = kWarpsPerBlock * kRowsPerWarp;

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
// W32 = BF16 w widened (dead input channels zeroed; NaN -> 0, +-Inf ->
// +-FLT_MAX as the quantizer maps them, flagged).  A thread converts 8
// consecutive elements of a row (one 16-byte load, two 16-byte stores; K and
// ldw are multiples of 8 and w 16-byte aligned on this path), rows and
// column octets in a grid-stride loop with one 32-bit division per octet.
__global__ void k_w_to_f32(const uint16_t *w, int64_t ldw, int64_t N, int64_t K, const uint8_t *dead, float *W,
                           uint32_t *status)
{
    uint32_t bad = 0;
    const uint32_t opr = (uint32_t)(K / 8);
    const int64_t total = N * (int64_t)opr;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / opr;
        const int64_t k = (i - n * opr) * 8;
        const uint4 v = *reinterpret_cast<const uint4 *>(w + n * ldw + k);
        const uint2 dk = *reinterpret_cast<const uint2 *>(dead + k);
        const uint32_t vw[4] = {v.x, v.y, v.z, v.w};
        float f[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            f[2 * j] = sanitize(bf16_lo(vw[j]), bad);
            f[2 * j + 1] = sanitize(bf16_hi(vw[j]), bad);
        }
        const uint32_t dw[2] = {dk.x, dk.y};
#pragma unroll
        for (int j = 0; j < 8; ++j)
            if ((dw[j >> 2] >> (8 * (j & 3))) & 0xFFu) f[j] = 0.0f;
        float4 *o = reinterpret_cast<float4 *>(W + n * K + k);
        o[0] = make_float4(f[0], f[1], f[2], f[3]);
        o[1] = make_float4(f[4], f[5], f[6], f[7]);
    }
    if (bad && status) atomicOr(status, HIF4_FLAG_NONFINITE);
}

// Any layout (2-byte aligned w, any ldw): one element per thread.
__global__ void k_w_to_f32_any(const uint16_t *w, int64_t ldw, int64_t N, int64_t K, const uint8_t *dead, float *W,
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

// FP32 -> TF32 (round to nearest, ties away): the low 13 mantissa bits cleared.
__device__ __forceinline__ uint32_t tf32_rna(float x)
{
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}

struct GptqArgs {
    float *W;                // N x K current weights (FP32); each group's columns get the values
                             // that group is quantized from
    int64_t N, K;
    int64_t b0;              // first column of the block
    const float *U;          // K x K upper factor (its blocks below the diagonal are not written)
    const float *UinvG;      // (K / 64) x 64 x 64: inverse of U's diagonal blocks
    const uint8_t *mask;     // u8 [K] or null
    const int32_t *rank;     // [K] protected rank or -1
    int n_masked;
    uint8_t *codes;          // N x K/2
    uint32_t *meta;          // N x K/64
    uint16_t *w_masked;      // N x n_masked
    float *Eh, *El;          // the block's error E = D U_gg^{-1} as TF32 parts (hi + lo): its 64 NG
                             // columns start at column e0 of N x ldE arrays (one per super-block)
    int64_t ldE, e0;
};

// One block of NG groups (64 NG columns) for kRowsPerBlock rows, a warp per
// kRowsPerWarp consecutive rows taken in lockstep (each U tile element read
// from shared memory serves all of them); lane l holds elements 2l, 2l+1 of
// each group of each row.  Per group: the exact FP32 unit quantization
// (encode rule of the streaming quantizer), D = W - Q, E = D Uinv_g (Uinv_g
// upper), feedback into the block's later groups.  The values a later group
// is quantized from (after the in-block feedback) are written back over its
// columns of W, so that on return W holds, for every group, exactly the
// weights that group was quantized from (later blocks never touch earlier
// columns).
template <int NG>
__global__ void __launch_bounds__(32 * kWarpsPerBlock) k_gptq_block(GptqArgs a)
{
    constexpr int NP = NG * (NG - 1) / 2;     // U tiles (g, h), g < h
    constexpr int R = kRowsPerWarp;
    extern __shared__ float smf[];
    float *Ui = smf;                          // NG x 64 x 64
    float *Uo = Ui + NG * 4096;               // NP x 64 x 64
    float *Dsh = Uo + NP * 4096;              // kWarpsPerBlock x R x 64
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t g0 = a.b0 / 64;
    for (int e = threadIdx.x; e < NG * 4096; e += blockDim.x) Ui[e] = a.UinvG[(g0 + e / 4096) * 4096 + e % 4096];
    for (int p = 0, g = 0; g < NG; ++g)
        for (int h = g + 1; h < NG; ++h, ++p)
            for (int e = threadIdx.x; e < 4096; e += blockDim.x)
                Uo[p * 4096 + e] = a.U[(a.b0 + 64 * g + e / 64) * a.K + a.b0 + 64 * h + e % 64];
    __syncthreads();
    // W is written by the previous launch of the chain (U is not): wait for it here
    pdl_enter();
    float *dsh = Dsh + warp * (R * 64);
    const int64_t nb = blockIdx.x * (int64_t)kRowsPerBlock + warp * R;
    if (nb >= a.N) return;                    // no block-wide barrier below
    bool valid[R];
    float x[R][NG][2];
#pragma unroll
    for (int r = 0; r < R; ++r) {
        valid[r] = nb + r < a.N;
#pragma unroll
        for (int g = 0; g < NG; ++g) {
            float2 v = make_float2(0.0f, 0.0f);
            if (valid[r]) v = *reinterpret_cast<const float2 *>(a.W + (nb + r) * a.K + a.b0 + 64 * g + 2 * lane);
            x[r][g][0] = v.x;
            x[r][g][1] = v.y;
        }
    }
    // y[r] = sum_i dsh[r][i] M[i][2l .. 2l+1] for a 64 x 64 tile M, all rows at once
    auto matvec = [&](const float *M, float (&y)[R][2]) {
#pragma unroll
        for (int r = 0; r < R; ++r) y[r][0] = y[r][1] = 0.0f;
        const float *mc = M + 2 * lane;
#pragma unroll 4
        for (int i = 0; i < 64; i += 4) {
            float2 u[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) u[k] = *reinterpret_cast<const float2 *>(mc + (i + k) * 64);
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const float4 d = *reinterpret_cast<const float4 *>(dsh + r * 64 + i);
                y[r][0] = fmaf(d.x, u[0].x, y[r][0]);
                y[r][1] = fmaf(d.x, u[0].y, y[r][1]);
                y[r][0] = fmaf(d.y, u[1].x, y[r][0]);
                y[r][1] = fmaf(d.y, u[1].y, y[r][1]);
                y[r][0] = fmaf(d.z, u[2].x, y[r][0]);
                y[r][1] = fmaf(d.z, u[2].y, y[r][1]);
                y[r][0] = fmaf(d.w, u[3].x, y[r][0]);
                y[r][1] = fmaf(d.w, u[3].y, y[r][1]);
            }
        }
    };
#pragma unroll
    for (int g = 0; g < NG; ++g) {
        const int64_t col = a.b0 + 64 * g + 2 * lane;
        const bool m0 = a.mask && a.mask[col], m1 = a.mask && a.mask[col + 1];
        __syncwarp();
#pragma unroll
        for (int r = 0; r < R; ++r) {
            const int64_t n = nb + r;
            if (g > 0 && valid[r]) *reinterpret_cast<float2 *>(a.W + n * a.K + col) = make_float2(x[r][g][0], x[r][g][1]);
            const float v0 = m0 ? 0.0f : x[r][g][0], v1 = m1 ? 0.0f : x[r][g][1];
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
            const float b0v = __bfloat162float(__float2bfloat16_rn(x[r][g][0]));
            const float b1v = __bfloat162float(__float2bfloat16_rn(x[r][g][1]));
            const float q0 = m0 ? b0v : bits_f(f_bits((float)q0m * step) | (s0 << 31));
            const float q1 = m1 ? b1v : bits_f(f_bits((float)q1m * step) | (s1 << 31));
            const uint32_t nib0 = m0 ? 0u : (q0m | (s0 << 3)), nib1 = m1 ? 0u : (q1m | (s1 << 3));
            const uint32_t b2 = __ballot_sync(0xffffffffu, e2 && (lane & 3) == 0);
            const uint32_t b3 = __ballot_sync(0xffffffffu, e3 && (lane & 1) == 0);
            if (valid[r]) {
                a.codes[n * (a.K / 2) + col / 2] = (uint8_t)(nib0 | (nib1 << 4));
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
            }
            dsh[r * 64 + 2 * lane] = x[r][g][0] - q0;
            dsh[r * 64 + 2 * lane + 1] = x[r][g][1] - q1;
        }
        __syncwarp();
        // E = D Uinv_g
        float e[R][2];
        matvec(Ui + g * 4096, e);
#pragma unroll
        for (int r = 0; r < R; ++r) {
            if (!valid[r]) continue;
            // E in two TF32 parts: the lazy update's split operand
            const uint32_t h0 = tf32_rna(e[r][0]), h1 = tf32_rna(e[r][1]);
            const int64_t o = (nb + r) * a.ldE + a.e0 + 64 * g + 2 * lane;
            *reinterpret_cast<float2 *>(a.Eh + o) = make_float2(__uint_as_float(h0), __uint_as_float(h1));
            *reinterpret_cast<float2 *>(a.El + o) = make_float2(__uint_as_float(tf32_rna(e[r][0] - __uint_as_float(h0))),
                                                              __uint_as_float(tf32_rna(e[r][1] - __uint_as_float(h1))));
        }
        // feedback into the later groups of the block
        if (g + 1 < NG) {
            __syncwarp();
#pragma unroll
            for (int r = 0; r < R; ++r) {
                dsh[r * 64 + 2 * lane] = e[r][0];
                dsh[r * 64 + 2 * lane + 1] = e[r][1];
            }
            __syncwarp();
#pragma unroll
            for (int h = g + 1; h < NG; ++h) {
                int p = 0;
                for (int gg = 0; gg < g; ++gg) p += NG - 1 - gg;
                p += h - g - 1;
                float dlt[R][2];
                matvec(Uo + p * 4096, dlt);
#pragma unroll
                for (int r = 0; r < R; ++r) {
                    x[r][h][0] -= dlt[r][0];
                    x[r][h][1] -= dlt[r][1];
                }
            }
        }
    }
}

// The lazy update C (M x Nc, ldc) -= E B after each block, on the tcgen05
// tensor cores, kind::tf32, as a persistent kernel: one CTA per SM walks
// 128 x 128 tiles of C, each accumulated in
// FP32 in one of two 128-column TMEM accumulators, so that the epilogue of a
// tile (C -= accumulator, read-modify-write in global memory) overlaps the
// loads and MMAs of the next.  Both operands come pre-split (x = hi + lo,
// hi = x rounded to TF32, lo = the rest rounded to TF32; A = the block's
// error E as E_hi, E_lo, N x Kd; B = U^T as U^T_hi, U^T_lo, K x K, so that a
// 128-column tile of C reads 128 K-major rows) and each 8-deep k-step issues
// lo hi + hi lo + hi hi (the dropped lo lo term and the TF32 rounding of lo
// leave an error of the order of FP32 rounding).  A 3-stage ring of four 128 x 32 FP32 tiles (64 KB
// each, 128-byte swizzle) is filled by TMA.  Warp 0: TMA producer; warp 1:
// TMEM allocation and the single MMA-issuing thread; warps 2-5: epilogue,
// thread = row.  Every wait is bounded; a time-out sets the abort flag, lets
// the copies in flight land, and reports HIF4_FLAG_TIMEOUT.
constexpr int UBM = 128, UBK = 32;
constexpr int kUThreads = 192;
constexpr uint64_t kUWaitNs = 2000000000ull;
// Tiles of 128 x BN (BN = 128: a 3-stage ring of 64 KB stages; BN = 256: a
// 2-stage ring of 96 KB stages and the whole 512-column TMEM for the two
// accumulators).
template <int BN>
struct UCfg {
    static constexpr int STG = BN == 128 ? 3 : 2;
    static constexpr uint32_t kA = UBM * UBK * 4;           // a 128 x 32 FP32 tile of E: 16 KB
    static constexpr uint32_t kB = BN * UBK * 4;            // a BN x 32 FP32 tile of U^T
    static constexpr uint32_t kStage = 2 * kA + 2 * kB;     // E_hi, E_lo, U^T_hi, U^T_lo
    static constexpr size_t kSmem = STG * kStage + 1024 + 256;
    static constexpr uint32_t kTmemCols = 2 * BN;
};

struct UpdArgs {
    float *W;                // C = W[:, b1 : b1 + Nc], row-major, ld ldw
    int64_t ldw, M, Nc;      // rows of W; columns updated (a multiple of 64)
    int b0, b1, nkb;         // the error's rows of U start at b0 (its columns of K); first column of C;
                             // 32-deep k-blocks
    int num_m, num_tiles;    // 128-row tiles of W; all tiles
    uint32_t *status;
    int a0;                  // first column of the error in the E arrays
};

// D[tmem] (+)= A[smem] * B[smem]^T, kind::tf32 (FP32 in smem read as TF32, FP32 accumulate).
__device__ __forceinline__ void mma_tf32_tc(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Instruction descriptor, kind::tf32: D = F32 (bits 4-5 = 1), A = B = TF32
// (2 in bits 7-9 and 10-12), both K-major, N >> 3 in bits 17-22, M >> 4 in
// bits 24-28.
constexpr uint32_t idesc_tf32_f32(uint32_t M, uint32_t N)
{
    return (1u << 4) | (2u << 7) | (2u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

template <int BN>
__global__ void __launch_bounds__(kUThreads, 1)
k_update_tf32(const __grid_constant__ CUtensorMap tmAh, const __grid_constant__ CUtensorMap tmAl,
              const __grid_constant__ CUtensorMap tmBh, const __grid_constant__ CUtensorMap tmBl, UpdArgs g)
{
    using namespace sm100;
    using C = UCfg<BN>;
    constexpr int USTG = C::STG;
    constexpr uint32_t kUStage = C::kStage;
    extern __shared__ uint8_t usm_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(usm_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + USTG * kUStage);
    uint64_t *full = bars, *empty = bars + USTG, *tfull = bars + 2 * USTG, *tempty = tfull + 2, *drain = tempty + 2;
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(drain + 1);
    volatile uint32_t *abort_flag = tmem_holder + 1;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int st = 0; st < USTG; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], 1);
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
        prefetch_tensormap(&tmAh);
        prefetch_tensormap(&tmAl);
        prefetch_tensormap(&tmBh);
        prefetch_tensormap(&tmBl);
    }
    if (warp == 1) {
        tmem_alloc(tmem_holder, C::kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;
    // the set-up above touches no data of the previous launch; E and W are its outputs
    pdl_enter();

    if (warp == 0) {
        if (lane == 0) {
            // ---------------------------------------------------- producer
            uint32_t stage = 0, phase = 0, issued = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < g.num_tiles; t += gridDim.x) {
                const int m0 = (t % g.num_m) * UBM, n0 = (t / g.num_m) * BN;
                for (int kb = 0; kb < g.nkb; ++kb) {
                    if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag, kUWaitNs)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = sm + stage * kUStage;
                    mbar_arrive_expect_tx(&full[stage], kUStage);
                    tma_load_2d(st, &tmAh, g.a0 + kb * UBK, m0, &full[stage]);
                    tma_load_2d(st + C::kA, &tmAl, g.a0 + kb * UBK, m0, &full[stage]);
                    tma_load_2d(st + 2 * C::kA, &tmBh, g.b0 + kb * UBK, g.b1 + n0, &full[stage]);
                    tma_load_2d(st + 2 * C::kA + C::kB, &tmBl, g.b0 + kb * UBK, g.b1 + n0, &full[stage]);
                    ++issued;
                    if (++stage == USTG) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                // let our own copies land: the most recent phase of every stage loaded
                for (uint32_t i = 0; i < USTG && i < issued; ++i) {
                    const uint32_t st = (stage + USTG - 1 - i) % USTG;
                    const uint32_t ph = (st < stage) ? phase : (phase ^ 1u);
                    mbar_wait_bounded(&full[st], ph, nullptr, 100000000ull);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ------------------------------------------------- MMA issuer
            const uint32_t idesc = idesc_tf32_f32(UBM, BN);
            uint32_t stage = 0, phase = 0, acc = 0, acc_phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; ok && t < g.num_tiles; t += gridDim.x) {
                if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, abort_flag, kUWaitNs)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * BN;
                for (int kb = 0; kb < g.nkb; ++kb) {
                    if (!mbar_wait_bounded(&full[stage], phase, abort_flag, kUWaitNs)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t ah = smem_addr(sm + stage * kUStage), al = ah + C::kA, bh = ah + 2 * C::kA,
                                   bl = bh + C::kB;
#pragma unroll
                    for (int k = 0; k < UBK / 8; ++k) {                // 8 TF32 = 32 bytes per step
                        mma_tf32_tc(d, smem_desc_sw128(al + 32 * k), smem_desc_sw128(bh + 32 * k), idesc,
                                    (kb | k) != 0);
                        mma_tf32_tc(d, smem_desc_sw128(ah + 32 * k), smem_desc_sw128(bl + 32 * k), idesc, 1u);
                        mma_tf32_tc(d, smem_desc_sw128(ah + 32 * k), smem_desc_sw128(bh + 32 * k), idesc, 1u);
                    }
                    mma_commit(&empty[stage]);
                    if (++stage == USTG) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (!ok) break;
                mma_commit(&tfull[acc]);
                acc ^= 1u;
                if (acc == 0) acc_phase ^= 1u;
            }
            // no MMA may still be running when TMEM is released
            mma_commit(drain);
            mbar_wait_bounded(drain, 0, nullptr, 100000000ull);
        }
    } else {
        // ---------------------------------------------------- epilogue
        // The TMEM read gives thread = row; each 32 x 32 chunk goes through
        // shared memory (row stride 33: no bank conflicts either way) so that
        // W is read and written a row at a time, lane = column (128 bytes
        // per row).  A chunk's W values are requested before its TMEM read.
        __shared__ float ebuf[4][32][33];
        const int q = warp & 3;                                        // TMEM lane quarter of this warp
        float(*buf)[33] = ebuf[q];
        uint32_t acc = 0, acc_phase = 0;
        for (int t = blockIdx.x; t < g.num_tiles; t += gridDim.x) {
            const int m0 = (t % g.num_m) * UBM, n0 = (t / g.num_m) * BN;
            const int64_t r0 = (int64_t)m0 + 32 * q;                   // this warp's 32 rows
            const int nrows = (int)(g.M - r0 < 32 ? g.M - r0 : 32);   // may be 0 or less
            if (!mbar_wait_bounded(&tfull[acc], acc_phase, abort_flag, kUWaitNs)) break;
            tc_fence_after();
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                const int64_t col = (int64_t)n0 + 32 * c;              // 32 columns: all inside Nc or all past it
                const bool live = col < g.Nc;
                float *wp = g.W + r0 * g.ldw + g.b1 + col + lane;
                float w[32];
                if (live) {
#pragma unroll
                    for (int rr = 0; rr < 32; ++rr) w[rr] = rr < nrows ? wp[rr * g.ldw] : 0.0f;
                }
                uint32_t r[32];
                tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + acc * BN + 32 * c, r);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 32; ++j) buf[lane][j] = __uint_as_float(r[j]);
                __syncwarp();
                if (live) {
#pragma unroll
                    for (int rr = 0; rr < 32; ++rr)
                        if (rr < nrows) wp[rr * g.ldw] = w[rr] - buf[rr][lane];
                }
                __syncwarp();
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            acc ^= 1u;
            if (acc == 0) acc_phase ^= 1u;
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kTmemCols);
    if (threadIdx.x == 0 && *abort_flag) status_or(g.status, HIF4_FLAG_TIMEOUT);
}

// U[i][j] = Y[K-1-i][K-1-j] for j >= i (FP32, upper), 0 below; the inverse
// of U's diagonal block g, Uinv_g[a][b] = L'[K-1-64g-a][K-1-64g-b] for b >= a
// (the reversed diagonal block of the Cholesky factor); and U^T in TF32
// parts, U^T = UTh + UTl (UTh = U rounded to TF32, UTl = the rest rounded to
// TF32), the K-major B operand of the lazy update.  One 32 x 32 tile per
// block of 32 x 8 threads, transposed through shared memory.  U's (and U^T's)
// 64 x 64 blocks below the diagonal are zero and never read (the group
// kernel reads U's blocks right of the diagonal, the updates E U[k0:k1, c0:c1]
// have k1 <= c0): they are left unwritten.
__global__ void k_build_u(const double *Y, const double *A, int64_t K, float *U, float *UinvG, float *UTh,
                          float *UTl)
{
    __shared__ float t[32][33];
    const int64_t i0 = blockIdx.y * 32ll, j0 = blockIdx.x * 32ll;
    if (i0 / TB > j0 / TB) return;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const int64_t i = i0 + threadIdx.y + 8 * q, j = j0 + threadIdx.x;
        const float u = j >= i ? (float)Y[(K - 1 - i) * K + (K - 1 - j)] : 0.0f;
        U[i * K + j] = u;
        t[threadIdx.y + 8 * q][threadIdx.x] = u;
        if (i / TB == j / TB) {
            const int64_t g = i / TB, a = i % TB, b = j % TB;
            UinvG[g * TB * TB + a * TB + b] = b >= a ? (float)A[(K - 1 - i) * K + (K - 1 - j)] : 0.0f;
        }
    }
    __syncthreads();
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const float v = t[threadIdx.x][threadIdx.y + 8 * q];
        const uint32_t h = tf32_rna(v);
        const int64_t o = (j0 + threadIdx.y + 8 * q) * K + i0 + threadIdx.x;
        UTh[o] = __uint_as_float(h);
        UTl[o] = __uint_as_float(tf32_rna(v - __uint_as_float(h)));
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
    size_t A, Y, T, U, UinvG, UTh, UTl, W, Eh, El, mask, rank, dead, mean, total;
};

// Columns of a super-block of the two-level lazy update: whole blocks, 512
// columns when the block divides it (64, 128, 256), 576 for 192.
int64_t super_cols(int64_t B) { return B * (512 / B > 1 ? 512 / B : 1); }

// The factor's split of a diagonal block of n > 128 rows: n1 = about half,
// a multiple of 128 rows when n is one (so that the leaves have 128 rows),
// else of 64.
int64_t factor_split(int64_t n)
{
    const int64_t u = n % (2 * TB) == 0 ? 2 * TB : TB;
    return n / u / 2 * u;
}

// Largest n1 x n2 split block (doubles) at each depth of the factor's
// recursion over n rows (the root is depth 0).
void factor_depth_sizes(int64_t n, size_t d, std::vector<int64_t> &mx)
{
    if (n <= 2 * TB) return;
    const int64_t n1 = factor_split(n), n2 = n - n1;
    if (mx.size() <= d) mx.resize(d + 1, 0);
    mx[d] = std::max(mx[d], n1 * n2);
    factor_depth_sizes(n1, d + 1, mx);
    factor_depth_sizes(n2, d + 1, mx);
}

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
    // the factor's scratch: two split blocks per depth of the recursion (a
    // level's blocks are read and written by its side product while deeper
    // levels run)
    {
        std::vector<int64_t> mx;
        factor_depth_sizes(K, 0, mx);
        size_t t = 0;
        for (int64_t v : mx) t += 2 * al256((size_t)v * 8);
        take(L.T, t > 0 ? t : 256);
    }
    take(L.U, k * k * 4);
    take(L.UinvG, nb * TB * TB * 4);
    take(L.UTh, k * k * 4);
    take(L.UTl, k * k * 4);
    take(L.W, (size_t)N * k * 4);
    take(L.Eh, (size_t)N * (size_t)super_cols(B) * 4);
    take(L.El, (size_t)N * (size_t)super_cols(B) * 4);
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

// Internal streams of hif4_higptq1, per device: the call's critical chain runs
// on `hi` (the device's greatest stream priority), forked from and joined back
// to the caller's stream; the factor's off-path products run on `side[d]`
// (least priority), one per depth of the recursion, so that the critical
// chain's small kernels take SMs first as they free up, except those of
// blocks of at most 384 rows, which run on `side_hi[d]` (greatest priority)
// so that they do not queue behind a large one; the FP32 working weights are
// formed on `prep` (least priority) while the factor runs.  Created on first
// use; `mu` serializes the calls that share them.
constexpr int kMaxDepth = 16;
struct GptqStreams {
    std::mutex mu;
    bool ready = false;
    cudaStream_t hi = nullptr, prep = nullptr, side[kMaxDepth] = {}, side_hi[kMaxDepth] = {};
    cudaEvent_t in = nullptr, out = nullptr, prep_fork = nullptr, prep_join = nullptr, fork[kMaxDepth] = {},
                join[kMaxDepth] = {};
};
GptqStreams g_streams[64];

hif4_status gptq_streams_ready(GptqStreams &g)
{
    if (g.ready) return HIF4_OK;
    int least = 0, greatest = 0;
    cudaError_t e = cudaDeviceGetStreamPriorityRange(&least, &greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&g.hi, cudaStreamNonBlocking, greatest);
    if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&g.prep, cudaStreamNonBlocking, least);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&g.prep_fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&g.prep_join, cudaEventDisableTiming);
    for (int d = 0; e == cudaSuccess && d < kMaxDepth; ++d) {
        e = cudaStreamCreateWithPriority(&g.side[d], cudaStreamNonBlocking, least);
        if (e == cudaSuccess) e = cudaStreamCreateWithPriority(&g.side_hi[d], cudaStreamNonBlocking, greatest);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&g.fork[d], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&g.join[d], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&g.in, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&g.out, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_failed(e);
    g.ready = true;
    return HIF4_OK;
}

// The factor of section "Factor": A (lower triangle of P Hd P on entry) and
// Y = L^{-1}, both K x K; T[d], T2[d] the split blocks of recursion depth d.
// At each split, T2 = T L11^{-1} does not depend on the lower-right block's
// factor, so it runs on the depth's side stream while that block is
// factored, and is joined before Y21 = -L22^{-1} T2 (the kernels and their
// operands are the same as in program order; only their overlap changes).
struct Factor {
    double *A, *Y;
    double *T[kMaxDepth], *T2[kMaxDepth];
    int64_t K;
    uint32_t *status;
    cudaStream_t s;
    GptqStreams *gs;

    hif4_status gemm(cudaStream_t st, bool bt, const double *a, int64_t lda, const double *b, int64_t ldb, double *c,
                     int64_t ldc, int64_t M, int64_t N, int64_t Kd, double alpha, int beta, int tri_a, int tri_b,
                     int lower_c)
    {
        Dgemm g{a, lda, b, ldb, c, ldc, (int)M, (int)N, (int)Kd, alpha, beta, tri_a, tri_b, lower_c};
        const int64_t mt = M / TB, nt = N / TB, tiles = lower_c ? mt * (mt + 1) / 2 : mt * nt;
        if (tiles < 3 * sm_count()) {             // few tiles: 32 x 32 ones, four times as many blocks
            const dim3 grid((unsigned)(N / 32), (unsigned)(M / 32));
            return bt ? launch_pdl(k_dgemm<true, 32, 4>, grid, dim3(kGemmThreads), gemm_smem<32, 4>(), st, g)
                      : launch_pdl(k_dgemm<false, 32, 4>, grid, dim3(kGemmThreads), gemm_smem<32, 4>(), st, g);
        }
        const dim3 grid((unsigned)nt, (unsigned)mt);
        return bt ? launch_pdl(k_dgemm<true, 64, 2>, grid, dim3(kGemmThreads), gemm_smem<64, 2>(), st, g)
                  : launch_pdl(k_dgemm<false, 64, 2>, grid, dim3(kGemmThreads), gemm_smem<64, 2>(), st, g);
    }

    // rows [o, o + n) of the factor and of its inverse, at recursion depth d
    hif4_status run(int64_t o, int64_t n, int d)
    {
        if (n == TB)
            return launch_pdl(k_leaf<2>, dim3(1), dim3(256), kLeafSmem2, s, A + o * K + o, K, Y + o * K + o, K,
                              status);
        if (n == 2 * TB)
            return launch_pdl(k_leaf<4>, dim3(1), dim3(256), kLeafSmem4, s, A + o * K + o, K, Y + o * K + o, K,
                              status);
        const int64_t n1 = factor_split(n), n2 = n - n1, a = o, b = o + n1;
        hif4_status st = run(a, n1, d + 1);
        if (st != HIF4_OK) return st;
        double *A21 = A + b * K + a, *A22 = A + b * K + b, *Y11 = Y + a * K + a, *Y21 = Y + b * K + a,
               *Y22 = Y + b * K + b, *Td = T[d], *T2d = T2[d];
        if ((st = gemm(s, true, A21, K, Y11, K, Td, n1, n2, n1, n1, 1.0, 0, 0, 1, 0)) != HIF4_OK) return st;
        if ((st = gemm(s, true, Td, n1, Td, n1, A22, K, n2, n2, n1, -1.0, 1, 0, 0, 1)) != HIF4_OK) return st;
        cudaStream_t sd = n <= 384 ? gs->side_hi[d] : gs->side[d];
        cudaError_t e = cudaEventRecord(gs->fork[d], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(sd, gs->fork[d], 0);
        if (e != cudaSuccess) return cuda_failed(e);
        if ((st = gemm(sd, false, Td, n1, Y11, K, T2d, n1, n2, n1, n1, 1.0, 0, 0, 1, 0)) != HIF4_OK) return st;
        if ((e = cudaEventRecord(gs->join[d], sd)) != cudaSuccess) return cuda_failed(e);
        st = run(b, n2, d + 1);
        if ((e = cudaStreamWaitEvent(s, gs->join[d], 0)) != cudaSuccess) return cuda_failed(e);
        if (st != HIF4_OK) return st;
        return gemm(s, false, Y22, K, T2d, n1, Y21, K, n2, n1, n2, -1.0, 0, 1, 0, 0);
    }
};

template <int NG>
hif4_status launch_gptq_block(const GptqArgs &a, cudaStream_t s)
{
    constexpr int NP = NG * (NG - 1) / 2;
    const size_t smem = sizeof(float) * ((NG + NP) * 4096 + kWarpsPerBlock * kRowsPerWarp * 64);
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!set_smem_once(k_gptq_block<NG>, smem, attr[dev & 63])) return HIF4_ERR_CUDA;
    return launch_pdl(k_gptq_block<NG>, dim3((unsigned)((a.N + kRowsPerBlock - 1) / kRowsPerBlock)),
                      dim3(32 * kWarpsPerBlock), smem, s, a);
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

extern "C" size_t hif4_higptq1_group_inputs_offset(int64_t N, int64_t K, int64_t blocksize)
{
    if (hif4_higptq1_workspace(N, K, blocksize) == 0) return (size_t)-1;
    return gptq_layout(N, K, blocksize == 0 ? 128 : blocksize).W;
}

namespace hif4 {
namespace {

// Everything hif4_higptq1 enqueues, on the internal critical-chain stream s.
hif4_status higptq1_enqueue(const void *w, int64_t N, int64_t K, int64_t ldw, const float *H,
                            const int32_t *mask_idx, int32_t n_masked, double damp, int64_t B, uint8_t *codes,
                            uint32_t *meta, void *w_masked, void *workspace, uint32_t *status, cudaStream_t s,
                            GptqStreams *gs)
{
    const GptqLayout L = gptq_layout(N, K, B);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    double *A = reinterpret_cast<double *>(ws + L.A);
    double *Y = reinterpret_cast<double *>(ws + L.Y);
    double *T = reinterpret_cast<double *>(ws + L.T);
    float *U = reinterpret_cast<float *>(ws + L.U);
    float *UinvG = reinterpret_cast<float *>(ws + L.UinvG);
    float *W = reinterpret_cast<float *>(ws + L.W);
    float *UTh = reinterpret_cast<float *>(ws + L.UTh);
    float *UTl = reinterpret_cast<float *>(ws + L.UTl);
    float *Eh = reinterpret_cast<float *>(ws + L.Eh);
    float *El = reinterpret_cast<float *>(ws + L.El);
    uint8_t *mask = ws + L.mask;
    int32_t *rank = reinterpret_cast<int32_t *>(ws + L.rank);
    uint8_t *dead = ws + L.dead;
    double *mean = reinterpret_cast<double *>(ws + L.mean);

    static bool attr_leaf[64] = {false}, attr_leaf4[64] = {false}, attr_g0[64] = {false}, attr_g1[64] = {false}, attr_g2[64] = {false},
                attr_g3[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    static bool attr_up[64] = {false}, attr_up2[64] = {false};
    if (!set_smem_once(k_update_tf32<128>, UCfg<128>::kSmem, attr_up[dev & 63]) ||
        !set_smem_once(k_update_tf32<256>, UCfg<256>::kSmem, attr_up2[dev & 63]) ||
        !set_smem_once(k_leaf<2>, kLeafSmem2, attr_leaf[dev & 63]) ||
        !set_smem_once(k_leaf<4>, kLeafSmem4, attr_leaf4[dev & 63]) ||
        !set_smem_once(k_dgemm<false, 64, 2>, gemm_smem<64, 2>(), attr_g0[dev & 63]) ||
        !set_smem_once(k_dgemm<true, 64, 2>, gemm_smem<64, 2>(), attr_g1[dev & 63]) ||
        !set_smem_once(k_dgemm<false, 32, 4>, gemm_smem<32, 4>(), attr_g2[dev & 63]) ||
        !set_smem_once(k_dgemm<true, 32, 4>, gemm_smem<32, 4>(), attr_g3[dev & 63]))
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
        cudaError_t e = cudaEventRecord(gs->prep_fork, s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(gs->prep, gs->prep_fork, 0);
        if (e != cudaSuccess) return cuda_failed(e);
        cudaStream_t ps = gs->prep;
        const bool vec = aligned16(w) && ldw % 8 == 0;          // K is a multiple of 64
        const int64_t work = vec ? N * K / 8 : N * K;
        int64_t blocks = (work + 255) / 256;
        if (blocks > 8 * (int64_t)sm_count()) blocks = 8 * (int64_t)sm_count();
        if (vec)
            k_w_to_f32<<<(unsigned)blocks, 256, 0, ps>>>(static_cast<const uint16_t *>(w), ldw, N, K, dead, W, status);
        else
            k_w_to_f32_any<<<(unsigned)blocks, 256, 0, ps>>>(static_cast<const uint16_t *>(w), ldw, N, K, dead, W,
                                                             status);
        if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
        if ((e = cudaEventRecord(gs->prep_join, ps)) != cudaSuccess) return cuda_failed(e);
    }
    // 2. P Hd P = L' L'^T and Y = L'^{-1} (FP64, recursive), then U = P Y P
    //    and the inverses of U's diagonal blocks
    k_fill_reversed<<<dim3((unsigned)((K + 31) / 32), (unsigned)((K + 7) / 8)), dim3(32, 8), 0, s>>>(
        H, K, dead, mean, damp, A);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    Factor F{};
    F.A = A;
    F.Y = Y;
    F.K = K;
    F.status = status;
    F.s = s;
    F.gs = gs;
    {
        std::vector<int64_t> mx;
        factor_depth_sizes(K, 0, mx);
        if ((int)mx.size() > kMaxDepth) return HIF4_ERR_UNSUPPORTED;
        uint8_t *t = reinterpret_cast<uint8_t *>(T);
        for (size_t d = 0; d < mx.size(); ++d) {
            F.T[d] = reinterpret_cast<double *>(t);
            t += al256((size_t)mx[d] * 8);
            F.T2[d] = reinterpret_cast<double *>(t);
            t += al256((size_t)mx[d] * 8);
        }
    }
    const hif4_status fst = F.run(0, K, 0);
    if (fst != HIF4_OK) return fst;
    k_build_u<<<dim3((unsigned)(K / 32), (unsigned)(K / 32)), dim3(32, 8), 0, s>>>(Y, A, K, U, UinvG, UTh, UTl);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    {
        const cudaError_t e = cudaStreamWaitEvent(s, gs->prep_join, 0);   // the FP32 working weights
        if (e != cudaSuccess) return cuda_failed(e);
    }
    CUtensorMap mBh, mBl, mBh2, mBl2;                  // boxes of 128 and 256 rows of U^T
    if (!make_tensor_map_f32_2d_sw128(&mBh, UTh, (uint64_t)K, (uint64_t)K, (uint64_t)K * 4, UBK, 128) ||
        !make_tensor_map_f32_2d_sw128(&mBl, UTl, (uint64_t)K, (uint64_t)K, (uint64_t)K * 4, UBK, 128) ||
        !make_tensor_map_f32_2d_sw128(&mBh2, UTh, (uint64_t)K, (uint64_t)K, (uint64_t)K * 4, UBK, 256) ||
        !make_tensor_map_f32_2d_sw128(&mBl2, UTl, (uint64_t)K, (uint64_t)K, (uint64_t)K * 4, UBK, 256))
        return HIF4_ERR_CUDA;
    // 3. the group loop, a two-level lazy update: within a super-block of
    //    S columns (whole blocks), each block's groups (with their in-block
    //    feedback), then the rest of the super-block updated by the block's
    //    error; after the super-block, every later column updated once by
    //    the super-block's whole error.  The same sum as GPTQ's per-block
    //    update, reordered; W's later columns are read and written once per
    //    super-block instead of once per block.
    const int64_t S = super_cols(B);
    CUtensorMap mAh, mAl;
    if (!make_tensor_map_f32_2d_sw128(&mAh, Eh, (uint64_t)S, (uint64_t)N, (uint64_t)S * 4, UBK, UBM) ||
        !make_tensor_map_f32_2d_sw128(&mAl, El, (uint64_t)S, (uint64_t)N, (uint64_t)S * 4, UBK, UBM))
        return HIF4_ERR_CUDA;
    auto update = [&](int64_t a0, int64_t k0, int64_t k1, int64_t c0, int64_t c1) -> hif4_status {
        // W[:, c0:c1] -= E[:, a0 : a0 + k1 - k0] U[k0:k1, c0:c1]
        // 128 x 256 tiles for the wide updates (half the E traffic per output), 128 x 128 otherwise
        const bool wide = (c1 - c0) % 256 == 0 && c1 - c0 >= 512;
        const int bn = wide ? 256 : 128;
        const int num_m = (int)((N + UBM - 1) / UBM), num_n = (int)((c1 - c0 + bn - 1) / bn);
        UpdArgs ua{W, K, N, c1 - c0, (int)k0, (int)c0, (int)((k1 - k0) / UBK), num_m, num_m * num_n, status,
                   (int)a0};
        const int grid = std::min(num_m * num_n, sm_count());
        return wide ? launch_pdl(k_update_tf32<256>, dim3(grid), dim3(kUThreads), UCfg<256>::kSmem, s, mAh, mAl, mBh2,
                                 mBl2, ua)
                    : launch_pdl(k_update_tf32<128>, dim3(grid), dim3(kUThreads), UCfg<128>::kSmem, s, mAh, mAl, mBh,
                                 mBl, ua);
    };
    for (int64_t s0 = 0; s0 < K; s0 += S) {
        const int64_t s1 = s0 + S < K ? s0 + S : K;
        for (int64_t b0 = s0; b0 < s1; b0 += B) {
            const int64_t b1 = b0 + B < s1 ? b0 + B : s1;
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
            a.Eh = Eh;
            a.El = El;
            a.ldE = S;
            a.e0 = b0 - s0;
            hif4_status st = NG == 1 ? launch_gptq_block<1>(a, s)
                           : NG == 2 ? launch_gptq_block<2>(a, s)
                           : NG == 3 ? launch_gptq_block<3>(a, s)
                                     : launch_gptq_block<4>(a, s);
            if (st != HIF4_OK) return st;
            if (b1 < s1 && (st = update(b0 - s0, b0, b1, b1, s1)) != HIF4_OK) return st;
        }
        if (s1 < K) {
            const hif4_status st = update(0, s0, s1, s1, K);
            if (st != HIF4_OK) return st;
        }
    }
    return HIF4_OK;
}

} // namespace
} // namespace hif4

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

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return HIF4_ERR_CUDA;
    GptqStreams &gs = g_streams[dev];
    std::lock_guard<std::mutex> lk(gs.mu);
    hif4_status st = gptq_streams_ready(gs);
    if (st != HIF4_OK) return st;
    // fork onto the critical-chain stream, join back whatever happens
    cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaEventRecord(gs.in, cs);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(gs.hi, gs.in, 0);
    if (e != cudaSuccess) return cuda_failed(e);
    st = higptq1_enqueue(w, N, K, ldw, H, mask_idx, n_masked, damp, B, codes, meta, w_masked, workspace, status,
                         gs.hi, &gs);
    e = cudaEventRecord(gs.out, gs.hi);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(cs, gs.out, 0);
    if (st == HIF4_OK && e != cudaSuccess) st = cuda_failed(e);
    return st;
}
