// hif4_calib.cu — tail-aware percentile calibration and channel mask.
//
// [Tail-Aware HiFloat4 summary on agents-report.net, "Why tail percentiles";
// arXiv abstract: "activation-tail-aware percentile calibration module for
// channel-mask construction".]  Rank rule and mask rule are the library's
// readings: per channel, the |x| key at ascending rank
// k = floor(q_num (T-1) / q_den); mask = top floor(C m_num / m_den) channels
// by (percentile desc, channel asc); ratio = percentile / lower median over
// channels.
//
// Exact order statistic by a two-pass radix select on the 15-bit BF16
// magnitude key (bits & 0x7FFF, whose order is the |x| order):
//   pass 1  per-channel histogram of key >> 7 (the exponent byte, 256 bins);
//   pass 2  per-channel histogram of key & 127 restricted to the bin that
//           holds rank k (128 bins);
//   final   bin + low bits -> the key; one warp per channel;
//   mask    one block: 32768-bin histogram of the C percentiles, block scans
//           for the median and the top-n threshold, index-order scan for
//           ties and for the sorted index list.
// Histogram blocks own a 64-channel slab and a token range; a warp reads one
// 128-byte row segment per load (lane = channel pair), so the slab's shared
// histogram (bin-major, channel-minor) is updated without bank conflicts.
#include <cuda_bf16.h>

#include "hif4_internal.cuh"

namespace hif4 {
namespace {

constexpr int kSlab = 64;          // channels per histogram block
constexpr int kHistThreads = 256;  // 8 warps
constexpr int kRowUnroll = 16;     // rows in flight per warp
constexpr int kBins1 = 256;
constexpr int kBins2 = 128;

struct HistArgs {
    const uint16_t *acts;
    int64_t T;
    int C;
    int64_t lda;
    int nslab;
    int64_t rows_per_split;
    uint32_t *hist1;   // [C][256]
    uint32_t *hist2;   // [C][128]
    uint32_t k;        // target ascending rank
    const uint32_t *needed;   // null, or per 64-channel slab: nonzero = process
};

__device__ __forceinline__ uint32_t ldg_nc_u32(const void *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

// Bin holding ascending rank k of a histogram of `nbins` counts, and the
// number of elements in lower bins.  Called by a full warp.
__device__ __forceinline__ void warp_select_bin(const uint32_t *h, int nbins, uint32_t k, uint32_t &bin,
                                                uint32_t &below, uint32_t *total = nullptr)
{
    const int lane = threadIdx.x & 31;
    const int per = nbins / 32;
    uint32_t c[8];
    uint32_t sum = 0;
    for (int i = 0; i < per; ++i) {
        c[i] = h[lane * per + i];
        sum += c[i];
    }
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
    }
    const uint32_t excl = incl - sum;
    const bool mine = excl <= k && k < incl;
    const uint32_t ballot = __ballot_sync(0xffffffffu, mine);
    const int owner = ballot ? __ffs(ballot) - 1 : 31;
    uint32_t b = 0, bl = 0;
    if (lane == owner) {
        uint32_t run = excl;
        int i = 0;
        for (; i < per - 1; ++i) {
            if (k < run + c[i]) break;
            run += c[i];
        }
        b = (uint32_t)(lane * per + i);
        bl = run;
    }
    bin = __shfl_sync(0xffffffffu, b, owner);
    below = __shfl_sync(0xffffffffu, bl, owner);
    if (total) *total = __shfl_sync(0xffffffffu, incl, 31);
}

// PAIR: 4-byte loads of a channel pair (needs a 4-byte aligned base and an
// even leading dimension); otherwise two 2-byte loads.
template <int PASS, bool PAIR>
__global__ void __launch_bounds__(kHistThreads) k_hist(HistArgs a)
{
    constexpr int NB = PASS == 1 ? kBins1 : kBins2;
    extern __shared__ uint32_t h[];                    // [NB][kSlab]
    __shared__ uint32_t target[kSlab];
    const int slab = blockIdx.x % a.nslab;
    const int split = blockIdx.x / a.nslab;
    const int c0 = slab * kSlab;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (a.needed && !a.needed[slab]) return;                 // block-uniform

    for (int i = threadIdx.x; i < NB * kSlab; i += kHistThreads) h[i] = 0;
    if (PASS == 2) {
        for (int j = warp; j < kSlab; j += kHistThreads / 32) {
            uint32_t bin = 0xFFFFFFFFu, below = 0;
            if (c0 + j < a.C) warp_select_bin(a.hist1 + (size_t)(c0 + j) * kBins1, kBins1, a.k, bin, below);
            if (lane == 0) target[j] = bin;
        }
    }
    __syncthreads();

    const int ch0 = 2 * lane, ch1 = 2 * lane + 1;        // local channels of this lane
    const bool v0 = c0 + ch0 < a.C, v1 = c0 + ch1 < a.C;
    uint32_t tb0 = 0, tb1 = 0;
    if (PASS == 2) {
        tb0 = target[ch0];
        tb1 = target[ch1];
    }
    // Conflict-free order: lanes 0-15 touch even channels first, 16-31 odd.
    const bool swap = lane >= 16;
    const int64_t t0 = (int64_t)split * a.rows_per_split;
    int64_t t1 = t0 + a.rows_per_split;
    if (t1 > a.T) t1 = a.T;
    const uint16_t *col = a.acts + c0 + ch0;

    for (int64_t t = t0 + warp; t < t1; t += (int64_t)(kHistThreads / 32) * kRowUnroll) {
        uint32_t w[kRowUnroll];
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            const int64_t r = t + (int64_t)u * (kHistThreads / 32);
            w[u] = 0;
            if (r < t1) {
                const uint16_t *p = col + r * a.lda;
                if (PAIR && v1) w[u] = ldg_nc_u32(p);
                else w[u] = (v0 ? (uint32_t)__ldg(p) : 0u) | (v1 ? (uint32_t)__ldg(p + 1) << 16 : 0u);
            }
        }
#pragma unroll
        for (int u = 0; u < kRowUnroll; ++u) {
            const int64_t r = t + (int64_t)u * (kHistThreads / 32);
            if (r >= t1) break;
            const uint32_t k0 = w[u] & 0x7FFFu, k1 = (w[u] >> 16) & 0x7FFFu;
            const uint32_t ka = swap ? k1 : k0, kb = swap ? k0 : k1;
            const int ca = swap ? ch1 : ch0, cb = swap ? ch0 : ch1;
            const bool va = swap ? v1 : v0, vb = swap ? v0 : v1;
            if (PASS == 1) {
                if (va) atomicAdd(&h[(ka >> 7) * kSlab + ca], 1u);
                if (vb) atomicAdd(&h[(kb >> 7) * kSlab + cb], 1u);
            } else {
                const uint32_t ta = swap ? tb1 : tb0, tbb = swap ? tb0 : tb1;
                if (va && (ka >> 7) == ta) atomicAdd(&h[(ka & 127u) * kSlab + ca], 1u);
                if (vb && (kb >> 7) == tbb) atomicAdd(&h[(kb & 127u) * kSlab + cb], 1u);
            }
        }
    }
    __syncthreads();
    uint32_t *g = PASS == 1 ? a.hist1 : a.hist2;
    for (int i = threadIdx.x; i < NB * kSlab; i += kHistThreads) {
        const uint32_t v = h[i];
        const int bin = i / kSlab, ch = i % kSlab;
        if (v && c0 + ch < a.C) atomicAdd(&g[(size_t)(c0 + ch) * NB + bin], v);
    }
}

// pct[c] = key at rank k: one warp per channel.
__global__ void k_finalize(const uint32_t *hist1, const uint32_t *hist2, int C, uint32_t k, uint16_t *pct,
                           const uint8_t *failed)
{
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (warp >= C) return;
    if (failed && !failed[warp]) return;
    uint32_t b1, below1, b2, below2;
    warp_select_bin(hist1 + (size_t)warp * kBins1, kBins1, k, b1, below1);
    warp_select_bin(hist2 + (size_t)warp * kBins2, kBins2, k - below1, b2, below2);
    if ((threadIdx.x & 31) == 0) pct[warp] = (uint16_t)((b1 << 7) | b2);
}

// ------------------------------------------------------- windowed single pass
//
// A row sample (about 2048 rows) gives each channel a window of 256 keys (at
// least a factor 2 in value) starting at the sample's exact order statistic
// at ten times the target tail mass (its 99th percentile for q = 0.999),
// found by the same two-pass radix select run on the sampled rows.  One
// pass over all tokens then counts the keys at or above the window start
// (`ge`) and histograms the keys inside the window; the target rank k is in
// the window iff T - ge <= k < T - ge + (window count), and then the window
// histogram gives the exact key.  Channels where it is not fall back to the
// exact two-pass radix select (launched always; blocks of slabs without a
// failed channel exit at once), so the result never depends on the sample.
//
// Hot loop: a lane owns 4 channels (one 8-byte load per row); with the keys
// packed in 16-bit halves, (x | 0x80008000) - (lo pair) sets bit 15 of a half
// exactly when key >= lo (lo <= 0x8000, so no borrow crosses halves), so the
// common case — every key below the window — costs four instructions per
// 4-byte word.  The window histogram lives in shared memory as 16-bit counts
// (a block covers at most 65535 rows).

constexpr int kWinSlab = 128;       // channels per block
constexpr int kWinBins = 256;
constexpr int kWinUnroll = 16;

struct WinArgs {
    const uint16_t *acts;
    int64_t T;
    int C;
    int64_t lda;
    int nslab;
    int64_t rows_per_split;
    const uint16_t *lo;     // [C] window start key (a sample order statistic)
    uint32_t *ge;           // [C] keys >= window start
    uint32_t *whist;        // [C][256]
};

template <bool V8>
__global__ void __launch_bounds__(kHistThreads) k_window(WinArgs a)
{
    extern __shared__ uint32_t h[];                    // [256 bins][64 words], u16 count per channel
    __shared__ uint32_t lo_s[kWinSlab];
    __shared__ uint32_t ge_s[kWinSlab];
    const int slab = blockIdx.x % a.nslab;
    const int split = blockIdx.x / a.nslab;
    const int c0 = slab * kWinSlab;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    for (int i = threadIdx.x; i < kWinBins * kWinSlab / 2; i += kHistThreads) h[i] = 0;
    for (int j = threadIdx.x; j < kWinSlab; j += kHistThreads) {
        lo_s[j] = c0 + j < a.C ? (uint32_t)a.lo[c0 + j] : 0x8000u;   // past C: never counted
        ge_s[j] = 0;
    }
    __syncthreads();

    const int ch = 4 * lane;
    const uint32_t LO01 = lo_s[ch] | (lo_s[ch + 1] << 16), LO23 = lo_s[ch + 2] | (lo_s[ch + 3] << 16);
    const bool all4 = c0 + ch + 3 < a.C;
    uint32_t ge[4] = {0, 0, 0, 0};
    uint32_t *hrow = h + 2 * lane;                     // word of channels (ch, ch+1); +1: (ch+2, ch+3)
    const int64_t t0 = (int64_t)split * a.rows_per_split;
    int64_t t1 = t0 + a.rows_per_split;
    if (t1 > a.T) t1 = a.T;
    constexpr int RS = kHistThreads / 32;              // rows between a warp's consecutive rows

    // one row: counts keys at or above the window start, histograms the keys inside it
    auto row = [&](uint32_t w01, uint32_t w23) {
        const uint32_t D01 = (w01 | 0x80008000u) - LO01;
        const uint32_t D23 = (w23 | 0x80008000u) - LO23;
        if ((D01 | D23) & 0x80008000u) {
            const uint32_t d[4] = {D01 & 0xFFFFu, D01 >> 16, D23 & 0xFFFFu, D23 >> 16};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint32_t off = d[j] - 0x8000u;  // key - lo (wraps when key < lo)
                ge[j] += off < 0x8000u;
                if (off < (uint32_t)kWinBins) atomicAdd(hrow + off * (kWinSlab / 2) + (j >> 1), 1u << (16 * (j & 1)));
            }
        }
    };
    auto load = [&](const uint16_t *p, uint32_t &w01, uint32_t &w23) {
        if (V8 && all4) {
            asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(w01), "=r"(w23) : "l"(p));
        } else {
            uint32_t e[4] = {0, 0, 0, 0};
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (c0 + ch + q < a.C) e[q] = __ldg(p + q);
            w01 = e[0] | (e[1] << 16);
            w23 = e[2] | (e[3] << 16);
        }
    };

    const int64_t step = (int64_t)RS * a.lda;           // elements between a warp's rows
    int64_t t = t0 + warp;
    const uint16_t *p = a.acts + (size_t)t * a.lda + c0 + ch;
    // full iterations: kWinUnroll rows in flight, no bounds checks
    for (; t + (int64_t)(kWinUnroll - 1) * RS < t1; t += (int64_t)kWinUnroll * RS) {
        uint32_t w01[kWinUnroll], w23[kWinUnroll];
#pragma unroll
        for (int u = 0; u < kWinUnroll; ++u) {
            load(p, w01[u], w23[u]);
            p += step;
        }
#pragma unroll
        for (int u = 0; u < kWinUnroll; ++u) row(w01[u], w23[u]);
    }
    for (; t < t1; t += RS) {                           // tail
        uint32_t w01, w23;
        load(p, w01, w23);
        p += step;
        row(w01, w23);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j)
        if (ge[j]) atomicAdd(&ge_s[ch + j], ge[j]);
    __syncthreads();
    for (int i = threadIdx.x; i < kWinBins * kWinSlab / 2; i += kHistThreads) {
        const uint32_t v = h[i];
        if (!v) continue;
        const int bin = i / (kWinSlab / 2), c = c0 + 2 * (i % (kWinSlab / 2));
        if ((v & 0xFFFFu) && c < a.C) atomicAdd(&a.whist[(size_t)c * kWinBins + bin], v & 0xFFFFu);
        if ((v >> 16) && c + 1 < a.C) atomicAdd(&a.whist[(size_t)(c + 1) * kWinBins + bin], v >> 16);
    }
    for (int j = threadIdx.x; j < kWinSlab; j += kHistThreads)
        if (ge_s[j] && c0 + j < a.C) atomicAdd(&a.ge[c0 + j], ge_s[j]);
}

// Key at rank k from the window counts (one warp per channel); a channel
// whose rank is outside its window is marked for the exact fallback, and its
// window row is cleared for reuse as the fallback's first histogram.
__global__ void k_window_final(uint32_t *whist, const uint32_t *ge, const uint16_t *lo, int C, uint64_t T, uint32_t k,
                               uint16_t *pct, uint8_t *failed, uint32_t *needed)
{
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (c >= C) return;
    uint32_t *row = whist + (size_t)c * kWinBins;
    const uint64_t below = T - ge[c];
    bool ok = false;
    if ((uint64_t)k >= below) {
        uint32_t bin, cum, total;
        warp_select_bin(row, kWinBins, (uint32_t)((uint64_t)k - below), bin, cum, &total);
        if ((uint64_t)k - below < total) {
            ok = true;
            if (lane == 0) pct[c] = (uint16_t)((uint32_t)lo[c] + bin);
        }
    }
    if (!ok) {
        for (int i = lane; i < kWinBins; i += 32) row[i] = 0;
        if (lane == 0) {
            failed[c] = 1;
            atomicOr(&needed[c / kSlab], 1u);
        }
    }
}

constexpr int kMaskThreads = 1024;
constexpr int kKeys = 32768;

// Block-wide exclusive scan of one value per thread (1024 threads).
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *scratch, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    __syncthreads();
    if (lane == 31) scratch[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = scratch[lane];
        uint32_t si = s;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t t = __shfl_up_sync(0xffffffffu, si, o);
            if (lane >= o) si += t;
        }
        scratch[32 + lane] = si - s;
        if (lane == 31) scratch[64] = si;
    }
    __syncthreads();
    total = scratch[64];
    return scratch[32 + warp] + incl - v;
}

__global__ void __launch_bounds__(kMaskThreads) k_mask(const uint16_t *pct, int C, uint32_t n_top, float *ratio,
                                                      uint8_t *mask, int32_t *mask_idx)
{
    extern __shared__ uint32_t hist[];                 // [kKeys]
    __shared__ uint32_t scratch[72];
    __shared__ uint32_t sel[4];                        // med key, tau key, count above tau
    for (int i = threadIdx.x; i < kKeys; i += kMaskThreads) hist[i] = 0;
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += kMaskThreads) atomicAdd(&hist[pct[c] & 0x7FFFu], 1u);
    __syncthreads();

    // each thread owns 32 consecutive keys
    constexpr int PER = kKeys / kMaskThreads;
    uint32_t local = 0;
    for (int i = 0; i < PER; ++i) local += hist[threadIdx.x * PER + i];
    uint32_t total;
    const uint32_t excl = block_excl_scan(local, scratch, total);
    const uint32_t r_med = (uint32_t)(C - 1) / 2u;
    const uint32_t r_tau = (uint32_t)C - n_top;        // ascending rank of the n_top-th largest
    {
        uint32_t run = excl;
        for (int i = 0; i < PER; ++i) {
            const uint32_t cnt = hist[threadIdx.x * PER + i];
            const uint32_t key = (uint32_t)(threadIdx.x * PER + i);
            if (cnt && run <= r_med && r_med < run + cnt) sel[0] = key;
            if (n_top && cnt && run <= r_tau && r_tau < run + cnt) {
                sel[1] = key;
                sel[2] = (uint32_t)C - (run + cnt);      // channels strictly above tau
            }
            run += cnt;
        }
    }
    __syncthreads();
    const uint32_t med_key = sel[0];
    const uint32_t tau = n_top ? sel[1] : 0x10000u;
    const uint32_t above = n_top ? sel[2] : 0u;
    const uint32_t need_eq = n_top - above;            // ties at tau taken by lowest index
    const float med = __uint_as_float(med_key << 16);

    uint32_t eq_base = 0, m_base = 0;
    for (int c0 = 0; c0 < C; c0 += kMaskThreads) {
        const int c = c0 + threadIdx.x;
        const bool in = c < C;
        const uint32_t key = in ? (pct[c] & 0x7FFFu) : 0u;
        const uint32_t eq = in && n_top && key == tau;
        uint32_t tot_eq;
        const uint32_t eq_rank = eq_base + block_excl_scan(eq, scratch, tot_eq);
        const uint32_t m = in && n_top && (key > tau || (eq && eq_rank < need_eq));
        uint32_t tot_m;
        const uint32_t m_pos = m_base + block_excl_scan(m, scratch, tot_m);
        if (in) {
            mask[c] = (uint8_t)m;
            float rt;
            if (med_key == 0) rt = key ? __int_as_float(0x7F800000) : 0.0f;
            else rt = __fdiv_rn(__uint_as_float(key << 16), med);
            ratio[c] = rt;
            if (m && mask_idx) mask_idx[m_pos] = c;
        }
        eq_base += tot_eq;
        m_base += tot_m;
    }
}

size_t a256(size_t v) { return (v + 255) & ~size_t(255); }

struct CalibLayout {
    size_t hs, hs2, whist, hist2, ge, lo, failed, needed, total;
};

CalibLayout calib_layout(int64_t C)
{
    CalibLayout L{};
    const size_t nslab = (size_t)((C + kSlab - 1) / kSlab);
    L.hs = 0;
    L.hs2 = L.hs + a256((size_t)C * kBins1 * 4);
    L.whist = L.hs2 + a256((size_t)C * kBins2 * 4);
    L.hist2 = L.whist + a256((size_t)C * 256 * 4);
    L.ge = L.hist2 + a256((size_t)C * kBins2 * 4);
    L.lo = L.ge + a256((size_t)C * 4);
    L.failed = L.lo + a256((size_t)C * 2);
    L.needed = L.failed + a256((size_t)C);
    L.total = L.needed + a256(nslab * 4);
    return L;
}

// Token splits so that every SM can hold its resident maximum of blocks.
int64_t splits_for(int64_t rows, int64_t nslab, int per_sm, int64_t min_rows, int64_t max_rows)
{
    const int64_t want = (int64_t)per_sm * sm_count();
    int64_t splits = (want + nslab - 1) / nslab;
    if (splits * min_rows > rows) splits = (rows + min_rows - 1) / min_rows;
    if (splits < 1) splits = 1;
    while ((rows + splits - 1) / splits > max_rows) ++splits;
    return splits;
}

} // namespace
} // namespace hif4

using namespace hif4;

extern "C" size_t hif4_calib_workspace(int64_t tokens, int64_t channels)
{
    (void)tokens;
    if (channels <= 0) return 0;
    return calib_layout(channels).total;
}

extern "C" hif4_status hif4_calib_percentile_mask(const void *acts, int64_t tokens, int64_t channels,
                                                  int64_t lda, uint32_t q_num, uint32_t q_den,
                                                  uint32_t mask_num, uint32_t mask_den, void *pct,
                                                  float *ratio, uint8_t *mask, int32_t *mask_idx_out,
                                                  void *workspace, size_t ws_bytes, hif4_stream_t stream)
{
    if (tokens <= 0 || channels <= 0) return HIF4_ERR_INVALID_ARG;
    if (!acts || !pct || !ratio || !mask) return HIF4_ERR_INVALID_ARG;
    if (q_den == 0 || q_num > q_den || mask_den == 0 || mask_num > mask_den) return HIF4_ERR_INVALID_ARG;
    if (lda < channels) return HIF4_ERR_SHAPE;
    if (tokens > 0xFFFFFFFFll || channels > (1 << 24)) return HIF4_ERR_UNSUPPORTED;
    if (!aligned_to(acts, 2)) return HIF4_ERR_ALIGNMENT;
    const bool pair = aligned_to(acts, 4) && (lda % 2 == 0);
    const bool v8 = aligned_to(acts, 8) && (lda % 4 == 0);
    if (!aligned_to(pct, 2) || !aligned_to(ratio, 4) || (mask_idx_out && !aligned_to(mask_idx_out, 4)))
        return HIF4_ERR_ALIGNMENT;
    const CalibLayout L = calib_layout(channels);
    if (!workspace || ws_bytes < L.total) return HIF4_ERR_WORKSPACE;
    if (!aligned_to(workspace, 256)) return HIF4_ERR_ALIGNMENT;

    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    uint32_t *hs = reinterpret_cast<uint32_t *>(ws + L.hs);
    uint32_t *hs2 = reinterpret_cast<uint32_t *>(ws + L.hs2);
    uint32_t *whist = reinterpret_cast<uint32_t *>(ws + L.whist);
    uint32_t *hist2 = reinterpret_cast<uint32_t *>(ws + L.hist2);
    uint32_t *ge = reinterpret_cast<uint32_t *>(ws + L.ge);
    uint16_t *lo = reinterpret_cast<uint16_t *>(ws + L.lo);
    uint8_t *failed = ws + L.failed;
    uint32_t *needed = reinterpret_cast<uint32_t *>(ws + L.needed);
    if (cudaMemsetAsync(workspace, 0, L.total, s) != cudaSuccess) return HIF4_ERR_CUDA;

    const uint64_t kk = ((uint64_t)q_num * (uint64_t)(tokens - 1)) / q_den;
    const size_t smem1 = (size_t)kBins1 * kSlab * 4, smem2 = (size_t)kBins2 * kSlab * 4;
    const size_t smemw = (size_t)kWinBins * kWinSlab / 2 * 4;
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr[dev & 63]) {
        if (cudaFuncSetAttribute(k_hist<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1) != cudaSuccess ||
            cudaFuncSetAttribute(k_hist<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) != cudaSuccess ||
            cudaFuncSetAttribute(k_hist<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem1) != cudaSuccess ||
            cudaFuncSetAttribute(k_hist<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2) != cudaSuccess ||
            cudaFuncSetAttribute(k_window<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemw) != cudaSuccess ||
            cudaFuncSetAttribute(k_window<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smemw) != cudaSuccess ||
            cudaFuncSetAttribute(k_mask, cudaFuncAttributeMaxDynamicSharedMemorySize, kKeys * 4) != cudaSuccess)
            return HIF4_ERR_CUDA;
        attr[dev & 63] = true;
    }
    const int nslab64 = (int)((channels + kSlab - 1) / kSlab);
    const int per_sm1 = blocks_per_sm(reinterpret_cast<const void *>(k_hist<1, true>), kHistThreads, smem1);
    const int64_t min_rows = (int64_t)(kHistThreads / 32) * kRowUnroll;

    // 1. window starts: exact order statistic of a row sample (every R-th row,
    //    about 2048 rows) at ten times the target tail mass below the top
    const int64_t R = tokens / 2048 > 1 ? tokens / 2048 : 1;
    const int64_t Ts = (tokens + R - 1) / R;
    const uint64_t tail = ((uint64_t)(tokens - kk) * 10ull * (uint64_t)Ts + (uint64_t)tokens - 1) / (uint64_t)tokens;
    const uint32_t r_lo = (uint32_t)((uint64_t)Ts > tail + 1 ? (uint64_t)Ts - 1 - tail : 0);
    HistArgs sa{};
    sa.acts = static_cast<const uint16_t *>(acts);
    sa.T = Ts;
    sa.C = (int)channels;
    sa.lda = lda * R;
    sa.nslab = nslab64;
    sa.hist1 = hs;
    sa.hist2 = hs2;
    sa.k = r_lo;
    sa.needed = nullptr;
    const int64_t sp = splits_for(Ts, nslab64, per_sm1, min_rows, INT64_MAX);
    sa.rows_per_split = (Ts + sp - 1) / sp;
    if (pair) k_hist<1, true><<<(int)(nslab64 * sp), kHistThreads, smem1, s>>>(sa);
    else k_hist<1, false><<<(int)(nslab64 * sp), kHistThreads, smem1, s>>>(sa);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    if (pair) k_hist<2, true><<<(int)(nslab64 * sp), kHistThreads, smem2, s>>>(sa);
    else k_hist<2, false><<<(int)(nslab64 * sp), kHistThreads, smem2, s>>>(sa);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    k_finalize<<<(int)((channels * 32 + 255) / 256), 256, 0, s>>>(hs, hs2, (int)channels, r_lo, lo, nullptr);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;

    // 2. windowed pass over every token
    WinArgs wa{};
    wa.acts = static_cast<const uint16_t *>(acts);
    wa.T = tokens;
    wa.C = (int)channels;
    wa.lda = lda;
    wa.nslab = (int)((channels + kWinSlab - 1) / kWinSlab);
    wa.lo = lo;
    wa.ge = ge;
    wa.whist = whist;
    const int per_smw = blocks_per_sm(reinterpret_cast<const void *>(k_window<true>), kHistThreads, smemw);
    const int64_t spw = splits_for(tokens, wa.nslab, per_smw, (int64_t)(kHistThreads / 32) * kWinUnroll, 65535);
    wa.rows_per_split = (tokens + spw - 1) / spw;
    if (v8) k_window<true><<<(int)(wa.nslab * spw), kHistThreads, smemw, s>>>(wa);
    else k_window<false><<<(int)(wa.nslab * spw), kHistThreads, smemw, s>>>(wa);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    k_window_final<<<(int)((channels * 32 + 255) / 256), 256, 0, s>>>(whist, ge, lo, (int)channels, (uint64_t)tokens,
                                                                       (uint32_t)kk, static_cast<uint16_t *>(pct),
                                                                       failed, needed);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;

    // 3. exact two-pass radix select for the channels outside their window
    HistArgs a{};
    a.acts = static_cast<const uint16_t *>(acts);
    a.T = tokens;
    a.C = (int)channels;
    a.lda = lda;
    a.nslab = nslab64;
    a.hist1 = whist;
    a.hist2 = hist2;
    a.k = (uint32_t)kk;
    a.needed = needed;
    const int64_t splits = splits_for(tokens, nslab64, per_sm1, min_rows, INT64_MAX);
    a.rows_per_split = (tokens + splits - 1) / splits;
    const int grid = (int)(nslab64 * splits);
    if (pair) k_hist<1, true><<<grid, kHistThreads, smem1, s>>>(a);
    else k_hist<1, false><<<grid, kHistThreads, smem1, s>>>(a);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    if (pair) k_hist<2, true><<<grid, kHistThreads, smem2, s>>>(a);
    else k_hist<2, false><<<grid, kHistThreads, smem2, s>>>(a);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;
    k_finalize<<<(int)((channels * 32 + 255) / 256), 256, 0, s>>>(whist, hist2, (int)channels, a.k,
                                                                   static_cast<uint16_t *>(pct), failed);
    if (launch_status() != HIF4_OK) return HIF4_ERR_CUDA;

    // 4. median over channels, ratios, top-n mask
    const uint32_t n_top = (uint32_t)(((uint64_t)channels * mask_num) / mask_den);
    k_mask<<<1, kMaskThreads, kKeys * 4, s>>>(static_cast<const uint16_t *>(pct), (int)channels, n_top, ratio, mask,
                                             mask_idx_out);
    return launch_status();
}
