// hif4_calib.cu — tail-aware percentile calibration and channel mask.
//
// [Tail-Aware HiFloat4 summary on agents-report.net, "Why tail percentiles";
// arXiv abstract: "activation-tail-aware percentile calibration module for
// channel-mask construction".]  Rank rule and mask rule are the library's
// readings: per channel, the |x| key at ascending rank
// k = floor(q_num (T-1) / q_den); mask = top floor(C m_num / m_den) channels
// by (percentile desc, channel asc); ratio = percentile / lower median over
// channels.  Keys are the 15-bit BF16 magnitudes (bits & 0x7FFF), whose
// integer order is the |x| order.
//
// Pipeline (all on the device, one stream):
//   1. sample  — the exact order statistic, per channel, of a row sample
//                (about 4096 rows) at four times the target's tail mass
//                below the top, by a two-pass radix select (pass 1: key >> 7,
//                the exponent byte; pass 2: key & 127 inside the bin that
//                holds the rank);
//   2. window  — one pass over every token: per channel, count the keys at
//                or above that sample value lo (`ge`) and histogram the keys
//                in [lo, lo + 256) (at least a factor 2 in value);
//   3. final   — rank k lies in the window iff T - ge <= k < T - ge + count:
//                then the window histogram gives the exact key;
//   4. fallback— channels where it does not run the exact two-pass radix
//                select over all tokens (always launched; blocks of slabs
//                without such a channel exit at once), so the result never
//                depends on the sample;
//   5. mask    — one block: median, ratios, top-n by (key desc, index asc).
//
// Streaming passes count keys of a 128-channel slab into 16-bit shared
// counters (a lane owns 4 channels).  When the rows start on 16-byte
// boundaries they run as k_pass_tma: TMA-staged tiles, a producer warp, one
// block per SM over equal shares of the slab-major row space.  Otherwise
// (2- or 8-byte aligned rows) they run as k_pass: plain loads, a block per
// (slab, token range of at most 65535 rows), 16 rows in flight per warp.
#include <cuda_bf16.h>

#include "hif4_internal.cuh"
#include "hif4_pdl.cuh"
#include "hif4_sm100.cuh"

namespace hif4 {
namespace {

constexpr int kThreads = 256;      // 8 warps
constexpr int kSlab = 128;         // channels per block (32 lanes x 4)
constexpr int kRS = kThreads / 32; // rows between a warp's consecutive rows
constexpr int kUnroll = 16;        // rows in flight per warp
constexpr int kBins1 = 256;        // key >> 7
constexpr int kBins2 = 128;        // key & 127
constexpr int kWinBins = 256;      // window width in keys
constexpr int64_t kMaxRowsPerBlock = 65535;

struct PassArgs {
    const uint16_t *acts;
    int64_t T;               // rows seen by this pass
    int C;
    int64_t lda;             // elements between the pass's consecutive rows
    int nslab;
    int64_t rows_per_split;
    uint32_t *hist1;         // [C][256]
    uint32_t *hist2;         // [C][128]
    uint32_t k;              // target ascending rank (pass 2)
    const uint16_t *tbin;    // pass 2: [C] bin of hist1 that holds rank k
    const uint32_t *needed;  // null, or per slab: nonzero = process
    const uint16_t *lo;      // window pass: [C] window start key
    uint32_t *ge;            // window pass: [C]
    uint32_t *whist;         // window pass: [C][256]
    uint32_t *timed_out;     // set to 1 when a TMA transfer never lands
    uint32_t withhold;       // TMA passes: block 0 withholds its first copy (failure-handling test)
    uint64_t wait_ns;        // TMA passes: limit of every bounded wait
};

// Bin holding ascending rank k of a histogram of `nbins` (multiple of 32)
// counts, the number of elements in lower bins and (optionally) the total.
// Called by a full warp.
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

// 4 keys of a lane's channels in one row: words (ch, ch+1) and (ch+2, ch+3).
template <bool V8>
__device__ __forceinline__ void load4(const uint16_t *p, bool all4, int valid, uint32_t &w01, uint32_t &w23)
{
    if (V8 && all4) {
        asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(w01), "=r"(w23) : "l"(p));
    } else {
        uint32_t e[4] = {0, 0, 0, 0};
#pragma unroll
        for (int q = 0; q < 4; ++q)
            if (q < valid) e[q] = __ldg(p + q);
        w01 = e[0] | (e[1] << 16);
        w23 = e[2] | (e[3] << 16);
    }
}

// MODE 1: histogram of key >> 7;  MODE 2: histogram of key & 127 for keys in
// the target bin;  MODE 3: the window pass.  Shared histograms hold 16-bit
// counts, two channels per word: word (bin, 2 lane + h) has channel
// 4 lane + 2 h in the low half.  Lanes 16-31 visit their two words in the
// opposite order so that the 32 lanes of an update hit 32 different banks.
template <int MODE, bool V8>
__global__ void __launch_bounds__(kThreads) k_pass(PassArgs a)
{
    pdl_enter();
    constexpr int NB = MODE == 1 ? kBins1 : MODE == 2 ? kBins2 : kWinBins;
    extern __shared__ uint32_t h[];                    // [NB][kSlab / 2]
    __shared__ uint32_t par[kSlab];                    // MODE 2: target bin; MODE 3: window start
    __shared__ uint32_t ge_s[kSlab];
    const int slab = blockIdx.x % a.nslab;
    const int split = blockIdx.x / a.nslab;
    const int c0 = slab * kSlab;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (a.needed && !a.needed[slab]) return;           // block-uniform

    for (int i = threadIdx.x; i < NB * kSlab / 2; i += kThreads) h[i] = 0;
    if (MODE == 2) {
        for (int j = threadIdx.x; j < kSlab; j += kThreads)
            par[j] = c0 + j < a.C ? (uint32_t)a.tbin[c0 + j] : 0u;   // counts past C are dropped
    }
    if (MODE == 3) {
        for (int j = threadIdx.x; j < kSlab; j += kThreads) {
            par[j] = c0 + j < a.C ? (uint32_t)a.lo[c0 + j] : 0x8000u;   // past C: never counted
            ge_s[j] = 0;
        }
    }
    __syncthreads();

    const int ch = 4 * lane;
    const int valid = min(4, max(0, a.C - (c0 + ch)));
    const bool all4 = valid == 4;
    const uint32_t swap = lane >= 16 ? 1u : 0u;
    uint32_t *hrow = h + 2 * lane;
    uint32_t P01 = 0, P23 = 0;                         // packed per-channel parameters
    if (MODE == 2) {                                   // target bin, pre-shifted to key bits 7..14
        P01 = (par[ch] << 7) | (par[ch + 1] << 23);
        P23 = (par[ch + 2] << 7) | (par[ch + 3] << 23);
    }
    if (MODE == 3) {
        P01 = par[ch] | (par[ch + 1] << 16);
        P23 = par[ch + 2] | (par[ch + 3] << 16);
    }
    uint32_t ge[4] = {0, 0, 0, 0};

    auto row = [&](uint32_t w01, uint32_t w23) {
        if (MODE == 1) {
            const uint32_t wa = swap ? w23 : w01, wb = swap ? w01 : w23;
            const uint32_t ha = swap, hb = swap ^ 1u;
            atomicAdd(hrow + ((wa >> 7) & 0xFFu) * (kSlab / 2) + ha, 1u);
            atomicAdd(hrow + ((wa >> 23) & 0xFFu) * (kSlab / 2) + ha, 0x10000u);
            atomicAdd(hrow + ((wb >> 7) & 0xFFu) * (kSlab / 2) + hb, 1u);
            atomicAdd(hrow + ((wb >> 23) & 0xFFu) * (kSlab / 2) + hb, 0x10000u);
        } else if (MODE == 2) {
            const uint32_t x01 = (w01 & 0x7F807F80u) ^ P01, x23 = (w23 & 0x7F807F80u) ^ P23;
            if (!(x01 & 0xFFFFu)) atomicAdd(hrow + (w01 & 127u) * (kSlab / 2), 1u);
            if (!(x01 >> 16)) atomicAdd(hrow + ((w01 >> 16) & 127u) * (kSlab / 2), 0x10000u);
            if (!(x23 & 0xFFFFu)) atomicAdd(hrow + (w23 & 127u) * (kSlab / 2) + 1, 1u);
            if (!(x23 >> 16)) atomicAdd(hrow + ((w23 >> 16) & 127u) * (kSlab / 2) + 1, 0x10000u);
        } else {
            // (key | 0x8000) - lo sets bit 15 exactly when key >= lo (lo <= 0x8000: no borrow)
            const uint32_t D01 = (w01 | 0x80008000u) - P01;
            const uint32_t D23 = (w23 | 0x80008000u) - P23;
            if ((D01 | D23) & 0x80008000u) {
                const uint32_t d[4] = {D01 & 0xFFFFu, D01 >> 16, D23 & 0xFFFFu, D23 >> 16};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t off = d[j] - 0x8000u;          // key - lo, wraps when key < lo
                    ge[j] += off < 0x8000u;
                    if (off < (uint32_t)kWinBins)
                        atomicAdd(hrow + off * (kSlab / 2) + (j >> 1), 1u << (16 * (j & 1)));
                }
            }
        }
    };

    const int64_t t0 = (int64_t)split * a.rows_per_split;
    int64_t t1 = t0 + a.rows_per_split;
    if (t1 > a.T) t1 = a.T;
    const int64_t step = (int64_t)kRS * a.lda;
    int64_t t = t0 + warp;
    const uint16_t *p = a.acts + (size_t)t * a.lda + c0 + ch;
    for (; t + (int64_t)(kUnroll - 1) * kRS < t1; t += (int64_t)kUnroll * kRS) {
        uint32_t w01[kUnroll], w23[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            load4<V8>(p, all4, valid, w01[u], w23[u]);
            p += step;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) row(w01[u], w23[u]);
    }
    for (; t < t1; t += kRS) {
        uint32_t w01, w23;
        load4<V8>(p, all4, valid, w01, w23);
        p += step;
        row(w01, w23);
    }

    if (MODE == 3) {
#pragma unroll
        for (int j = 0; j < 4; ++j)
            if (ge[j]) atomicAdd(&ge_s[ch + j], ge[j]);
    }
    __syncthreads();
    uint32_t *g = MODE == 1 ? a.hist1 : MODE == 2 ? a.hist2 : a.whist;
    for (int i = threadIdx.x; i < NB * kSlab / 2; i += kThreads) {
        const uint32_t v = h[i];
        if (!v) continue;
        const int bin = i / (kSlab / 2), wi = i % (kSlab / 2);
        const int c = c0 + 4 * (wi >> 1) + 2 * (wi & 1);              // word (lane, h) -> channel 4 lane + 2 h
        if ((v & 0xFFFFu) && c < a.C) atomicAdd(&g[(size_t)c * NB + bin], v & 0xFFFFu);
        if ((v >> 16) && c + 1 < a.C) atomicAdd(&g[(size_t)(c + 1) * NB + bin], v >> 16);
    }
    if (MODE == 3)
        for (int j = threadIdx.x; j < kSlab; j += kThreads)
            if (ge_s[j] && c0 + j < a.C) atomicAdd(&a.ge[c0 + j], ge_s[j]);
}

// Bin of the first radix histogram that holds rank k (one warp per channel).
__global__ void k_select1(const uint32_t *hist1, int C, uint32_t k, uint16_t *tbin, const uint8_t *failed)
{
    pdl_enter();
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (c >= C) return;
    if (failed && !failed[c]) return;
    uint32_t b, below;
    warp_select_bin(hist1 + (size_t)c * kBins1, kBins1, k, b, below);
    if ((threadIdx.x & 31) == 0) tbin[c] = (uint16_t)b;
}

// TMA-staged variant of k_pass, warp-specialized, one block per SM.  A 2-D
// tensor map over the (strided) rows lands 128-row x 128-channel tiles
// (32 KB) in a 5-stage shared ring beside the 64 KB counter array.  One
// producer warp issues the copies (cp.async.bulk.tensor, completion on a
// "full" mbarrier per slot) and refills a slot once all sixteen consumer
// warps have released it (an "empty" mbarrier per slot), so consumers never
// wait on one another inside a segment and up to 160 KB per SM stay in
// flight.  A consumer warp takes rows warp, warp + 16, ... (8 per tile): it
// loads them all first (8-byte shared loads, 256 contiguous bytes per warp).
// Passes 1 and 2 count every row with straight-line predicated atomics (the
// bin that holds the target often holds several percent of the keys).  The
// window pass counts few keys (those at or above the window start), so each
// lane first marks its rows holding one (a cheap superset test), then the
// warp visits marked rows one per lane per round: the count is paid per
// marked row instead of per divergent row.
//
// Work split: one block per SM; block b takes units [b share, (b+1) share)
// of the slab-major space u = slab * T + row, so all blocks carry equal
// rows and no wave tail is left.  A share crosses at most a few slab
// boundaries; each slab segment zeroes and flushes the shared counters
// (share <= 65535 rows keeps the 16-bit counters exact).  Rows past a
// segment inside a tile are skipped; channels past C land in counters that
// are never flushed.
constexpr int kTmaRows = 128;
constexpr int kTmaStages = 5;
constexpr int kConsumers = 16;                       // consumer warps
constexpr int kTmaThreads = (kConsumers + 1) * 32;   // + one producer warp
constexpr int kRowsPerWarp = kTmaRows / kConsumers;  // 8
constexpr uint32_t kRowBytes = kSlab * 2;
constexpr uint32_t kTileBytes = kTmaRows * kRowBytes;
constexpr uint64_t kWaitNs = 2000000000ull;

// Shared counter layout of the TMA passes: [bin][64 words], word
// 2 l + col of lane l holding two 16-bit counts.  Lanes below 16 keep
// channels 4l, 4l+1 in col 0 and 4l+2, 4l+3 in col 1; lanes from 16 on keep
// them the other way round, so that lanes l and l + 16 (same bank pair) hit
// different banks in every counting instruction.
__device__ __forceinline__ int slot_channel(int wi)
{
    const int l = wi >> 1;
    return 4 * l + 2 * ((wi & 1) ^ (l >= 16 ? 1 : 0));
}

// One row's four keys of this lane (words w01 = channels ch, ch+1 and
// w23 = ch+2, ch+3) into the shared counters (h01 / h23: this lane's
// columns for the two words).
template <int MODE>
__device__ __forceinline__ void count_row(uint32_t w01, uint32_t w23, uint32_t *h01, uint32_t *h23, uint32_t P01,
                                          uint32_t P23, uint32_t (&ge)[4])
{
    if (MODE == 1) {
        atomicAdd(h01 + ((w01 >> 7) & 0xFFu) * (kSlab / 2), 1u);
        atomicAdd(h01 + ((w01 >> 23) & 0xFFu) * (kSlab / 2), 0x10000u);
        atomicAdd(h23 + ((w23 >> 7) & 0xFFu) * (kSlab / 2), 1u);
        atomicAdd(h23 + ((w23 >> 23) & 0xFFu) * (kSlab / 2), 0x10000u);
    } else if (MODE == 2) {
        const uint32_t x01 = (w01 & 0x7F807F80u) ^ P01, x23 = (w23 & 0x7F807F80u) ^ P23;
        if (!(x01 & 0xFFFFu)) atomicAdd(h01 + (w01 & 127u) * (kSlab / 2), 1u);
        if (!(x01 >> 16)) atomicAdd(h01 + ((w01 >> 16) & 127u) * (kSlab / 2), 0x10000u);
        if (!(x23 & 0xFFFFu)) atomicAdd(h23 + (w23 & 127u) * (kSlab / 2), 1u);
        if (!(x23 >> 16)) atomicAdd(h23 + ((w23 >> 16) & 127u) * (kSlab / 2), 0x10000u);
    } else {
        // D = (w | 0x80008000) - P: bit 15 of each half is set iff that key
        // >= lo, the half then holding 0x8000 + (key - lo)
        const uint32_t D01 = (w01 | 0x80008000u) - P01, D23 = (w23 | 0x80008000u) - P23;
        const uint32_t d[4] = {D01 & 0xFFFFu, D01 >> 16, D23 & 0xFFFFu, D23 >> 16};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t off = d[j] - 0x8000u;
            ge[j] += off < 0x8000u;
            if (off < (uint32_t)kWinBins)
                atomicAdd((j < 2 ? h01 : h23) + off * (kSlab / 2), 1u << (16 * (j & 1)));
        }
    }
}

// Superset test for a row that the window count may count: true whenever
// some key of the row is at or above its channel's window start.
__device__ __forceinline__ bool row_candidate(uint32_t w01, uint32_t w23, uint32_t P01, uint32_t P23)
{
    return ((((w01 | 0x80008000u) - P01) | ((w23 | 0x80008000u) - P23)) & 0x80008000u) != 0u;
}

template <int MODE>
__global__ void __launch_bounds__(kTmaThreads, 1) k_pass_tma(const __grid_constant__ CUtensorMap tm, PassArgs a)
{
    pdl_enter();
    using namespace sm100;
    constexpr int NB = MODE == 1 ? kBins1 : MODE == 2 ? kBins2 : kWinBins;
    extern __shared__ __align__(128) uint8_t smraw[];
    uint8_t *tiles = smraw;                                             // kTmaStages x 32 KB
    uint32_t *h = reinterpret_cast<uint32_t *>(smraw + kTmaStages * kTileBytes);   // [NB][kSlab / 2]
    __shared__ uint64_t full[kTmaStages], empty[kTmaStages];
    __shared__ uint16_t par[kSlab];
    __shared__ uint32_t ge_s[kSlab];
    __shared__ uint32_t abort_flag;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int ch = 4 * lane;
    uint32_t *h01 = h + 2 * lane + (lane >= 16 ? 1 : 0);
    uint32_t *h23 = h + 2 * lane + (lane >= 16 ? 0 : 1);

    const int64_t total = (int64_t)a.nslab * a.T;
    int64_t cur = (int64_t)blockIdx.x * a.rows_per_split;
    const int64_t end = cur + a.rows_per_split < total ? cur + a.rows_per_split : total;
    if (threadIdx.x == 0) {
        for (int st = 0; st < kTmaStages; ++st) {
            mbar_init(&full[st], 1);
            mbar_init(&empty[st], kConsumers);
        }
        abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tm);
    }
    uint32_t g = 0;                                    // tiles consumed: ring slot and phase
    while (cur < end) {                                // block-uniform
        const int slab = (int)(cur / a.T);
        const int64_t t0 = cur - (int64_t)slab * a.T;
        const int64_t t1 = t0 + (end - cur) < a.T ? t0 + (end - cur) : a.T;
        cur += t1 - t0;
        if (a.needed && !a.needed[slab]) continue;
        const int c0 = slab * kSlab;
        __syncthreads();                               // previous segment flushed
        for (int i = threadIdx.x; i < NB * kSlab / 2; i += kTmaThreads) h[i] = 0;
        if (MODE == 2)
            for (int j = threadIdx.x; j < kSlab; j += kTmaThreads)
                par[j] = c0 + j < a.C ? a.tbin[c0 + j] : (uint16_t)0;
        if (MODE == 3)
            for (int j = threadIdx.x; j < kSlab; j += kTmaThreads) {
                par[j] = c0 + j < a.C ? a.lo[c0 + j] : (uint16_t)0x8000u;
                ge_s[j] = 0;
            }
        __syncthreads();
        const int nchunks = (int)((t1 - t0 + kTmaRows - 1) / kTmaRows);
        bool ok = true;
        int issued = 0;
        if (warp == kConsumers) {
            // producer: one lane issues every tile of the segment in order
            if (lane == 0) {
                for (; issued < nchunks; ++issued) {
                    const uint32_t gi = g + (uint32_t)issued, st = gi % kTmaStages;
                    if (gi >= (uint32_t)kTmaStages &&
                        !mbar_wait_bounded(&empty[st], (gi / kTmaStages - 1u) & 1u, &abort_flag, a.wait_ns)) {
                        ok = false;
                        break;
                    }
                    if (a.withhold && blockIdx.x == 0 && gi == 0) continue;   // its wait can only run out
                    mbar_arrive_expect_tx(&full[st], kTileBytes);
                    tma_load_2d(tiles + st * kTileBytes, &tm, c0, (int32_t)(t0 + (int64_t)issued * kTmaRows),
                                &full[st]);
                }
            }
        } else {
            uint32_t P01 = 0, P23 = 0;
            if (MODE == 2) {
                P01 = ((uint32_t)par[ch] << 7) | ((uint32_t)par[ch + 1] << 23);
                P23 = ((uint32_t)par[ch + 2] << 7) | ((uint32_t)par[ch + 3] << 23);
            }
            if (MODE == 3) {
                P01 = (uint32_t)par[ch] | ((uint32_t)par[ch + 1] << 16);
                P23 = (uint32_t)par[ch + 2] | ((uint32_t)par[ch + 3] << 16);
            }
            uint32_t ge[4] = {0, 0, 0, 0};
            for (int ci = 0; ci < nchunks; ++ci) {
                const uint32_t gi = g + (uint32_t)ci, st = gi % kTmaStages;
                ok = __all_sync(0xffffffffu,
                                mbar_wait_bounded(&full[st], (gi / kTmaStages) & 1u, &abort_flag, a.wait_ns));
                if (!ok) break;
                // rows warp + 16 i of this tile that lie inside the segment
                const int64_t left = t1 - (t0 + (int64_t)ci * kTmaRows);
                const int rows_here = left >= kTmaRows ? kTmaRows : (int)left;
                const int nmine = rows_here > warp ? (rows_here - warp + kConsumers - 1) / kConsumers : 0;
                const uint32_t valid = (1u << nmine) - 1u;
                const uint8_t *tile = tiles + st * kTileBytes + ch * 2 + warp * kRowBytes;
                uint2 v[kRowsPerWarp];
#pragma unroll
                for (int i = 0; i < kRowsPerWarp; ++i)
                    v[i] = *reinterpret_cast<const uint2 *>(tile + i * (kConsumers * kRowBytes));
                if (MODE != 3) {
#pragma unroll
                    for (int i = 0; i < kRowsPerWarp; ++i)
                        if (valid >> i & 1u) count_row<MODE>(v[i].x, v[i].y, h01, h23, P01, P23, ge);
                } else {
                    uint32_t marked = 0;
#pragma unroll
                    for (int i = 0; i < kRowsPerWarp; ++i)
                        marked |= (uint32_t)row_candidate(v[i].x, v[i].y, P01, P23) << i;
                    marked &= valid;
                    while (__any_sync(0xffffffffu, marked != 0u)) {
                        if (marked) {
                            const int i = __ffs(marked) - 1;
                            marked &= marked - 1u;
                            const uint2 w = *reinterpret_cast<const uint2 *>(tile + i * (kConsumers * kRowBytes));
                            count_row<MODE>(w.x, w.y, h01, h23, P01, P23, ge);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[st]);
            }
            if (MODE == 3) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    if (ge[j]) atomicAdd(&ge_s[ch + j], ge[j]);
            }
        }
        if (__syncthreads_or(!ok)) {                   // time-out: let issued copies land, flag, stop
            if (warp == kConsumers && lane == 0) {
                for (int cj = issued - kTmaStages < 0 ? 0 : issued - kTmaStages; cj < issued; ++cj) {
                    const uint32_t gj = g + (uint32_t)cj;
                    mbar_wait_bounded(&full[gj % kTmaStages], (gj / kTmaStages) & 1u, nullptr, 100000000ull);
                }
                atomicOr(a.timed_out, 1u);
            }
            return;
        }
        g += (uint32_t)nchunks;
        uint32_t *gh = MODE == 1 ? a.hist1 : MODE == 2 ? a.hist2 : a.whist;
        for (int i = threadIdx.x; i < NB * kSlab / 2; i += kTmaThreads) {
            const uint32_t hv = h[i];
            if (!hv) continue;
            const int bin = i / (kSlab / 2);
            const int c = c0 + slot_channel(i % (kSlab / 2));
            if ((hv & 0xFFFFu) && c < a.C) atomicAdd(&gh[(size_t)c * NB + bin], hv & 0xFFFFu);
            if ((hv >> 16) && c + 1 < a.C) atomicAdd(&gh[(size_t)(c + 1) * NB + bin], hv >> 16);
        }
        if (MODE == 3)
            for (int j = threadIdx.x; j < kSlab; j += kTmaThreads)
                if (ge_s[j] && c0 + j < a.C) atomicAdd(&a.ge[c0 + j], ge_s[j]);
    }
}

// Key at rank k from the two radix histograms (one warp per channel); with
// `failed`, only the channels it marks.
__global__ void k_finalize(const uint32_t *hist1, const uint32_t *hist2, int C, uint32_t k, uint16_t *out,
                           const uint8_t *failed)
{
    pdl_enter();
    const int c = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    if (c >= C) return;
    if (failed && !failed[c]) return;
    uint32_t b1, below1, b2, below2;
    warp_select_bin(hist1 + (size_t)c * kBins1, kBins1, k, b1, below1);
    warp_select_bin(hist2 + (size_t)c * kBins2, kBins2, k - below1, b2, below2);
    if ((threadIdx.x & 31) == 0) out[c] = (uint16_t)((b1 << 7) | b2);
}

// Key at rank k from the window counts (one warp per channel); a channel
// whose rank lies outside its window is marked for the exact fallback and
// its window row is cleared for reuse as the fallback's first histogram.
__global__ void k_window_final(uint32_t *whist, const uint32_t *ge, const uint16_t *lo, int C, uint64_t T, uint32_t k,
                               uint16_t *pct, uint8_t *failed, uint32_t *needed)
{
    pdl_enter();
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
// Key histogram slot with one pad word per 32 keys: thread t's 32 consecutive
// keys then sit in 32 different banks across a warp.
constexpr int kKeySlots = kKeys + kKeys / 32;
__device__ __forceinline__ int key_slot(uint32_t key) { return (int)(key + (key >> 5)); }

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

// A time-out in an earlier pass (timed_out != 0) poisons the outputs instead:
// every ratio NaN, the mask all zero, every mask index -1.
__global__ void __launch_bounds__(kMaskThreads) k_mask(const uint16_t *pct, int C, uint32_t n_top, float *ratio,
                                                      uint8_t *mask, int32_t *mask_idx, const uint32_t *timed_out)
{
    pdl_enter();
    extern __shared__ uint32_t hist[];                 // [kKeySlots]
    if (*timed_out) {                                  // block-uniform
        for (int c = threadIdx.x; c < C; c += kMaskThreads) {
            ratio[c] = __int_as_float(0x7FC00000);
            mask[c] = 0;
        }
        if (mask_idx)
            for (uint32_t i = threadIdx.x; i < n_top; i += kMaskThreads) mask_idx[i] = -1;
        return;
    }
    __shared__ uint32_t scratch[72];
    __shared__ uint32_t sel[4];                        // med key, tau key, count above tau
    for (int i = threadIdx.x; i < kKeySlots; i += kMaskThreads) hist[i] = 0;
    __syncthreads();
    for (int c = threadIdx.x; c < C; c += kMaskThreads) atomicAdd(&hist[key_slot(pct[c] & 0x7FFFu)], 1u);
    __syncthreads();

    // each thread owns 32 consecutive keys
    constexpr int PER = kKeys / kMaskThreads;
    uint32_t local = 0;
    for (int i = 0; i < PER; ++i) local += hist[threadIdx.x * (PER + 1) + i];
    uint32_t total;
    const uint32_t excl = block_excl_scan(local, scratch, total);
    const uint32_t r_med = (uint32_t)(C - 1) / 2u;
    const uint32_t r_tau = (uint32_t)C - n_top;        // ascending rank of the n_top-th largest
    {
        uint32_t run = excl;
        for (int i = 0; i < PER; ++i) {
            const uint32_t cnt = hist[threadIdx.x * (PER + 1) + i];
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

    // Mask and indices in three passes over contiguous per-warp channel
    // ranges (warp w owns [w chunk, (w+1) chunk)), with ballots inside a warp
    // and one prefix over the 32 warp totals between passes: ties at tau go
    // to the lowest channel indices, and mask_idx lists the masked channels
    // in ascending order.
    constexpr int kWarps = kMaskThreads / 32;
    __shared__ uint32_t wsum[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t lt = (1u << lane) - 1u;
    const int chunk = ((C + kWarps - 1) / kWarps + 31) & ~31;
    const int cbeg = warp * chunk, cend = min(C, cbeg + chunk);
    // pass 1: channels tied at tau, per warp
    uint32_t n_eq = 0;
    for (int c0 = cbeg; c0 < cend; c0 += 32) {
        const int c = c0 + lane;
        n_eq += __popc(__ballot_sync(0xffffffffu, c < cend && n_top && (pct[c] & 0x7FFFu) == tau));
    }
    if (lane == 0) wsum[warp] = n_eq;
    __syncthreads();
    uint32_t eq_base = 0;
    for (int w = 0; w < warp; ++w) eq_base += wsum[w];
    __syncthreads();
    // pass 2: masked channels, per warp
    uint32_t n_m = 0;
    for (int c0 = cbeg, er = (int)eq_base; c0 < cend; c0 += 32) {
        const int c = c0 + lane;
        const bool in = c < cend;
        const uint32_t key = in ? (pct[c] & 0x7FFFu) : 0u;
        const bool eq = in && n_top && key == tau;
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        const bool m = in && n_top && (key > tau || (eq && (uint32_t)er + __popc(be & lt) < need_eq));
        n_m += __popc(__ballot_sync(0xffffffffu, m));
        er += __popc(be);
    }
    if (lane == 0) wsum[warp] = n_m;
    __syncthreads();
    uint32_t m_base = 0;
    for (int w = 0; w < warp; ++w) m_base += wsum[w];
    // pass 3: outputs
    for (int c0 = cbeg, er = (int)eq_base, mr = (int)m_base; c0 < cend; c0 += 32) {
        const int c = c0 + lane;
        const bool in = c < cend;
        const uint32_t key = in ? (pct[c] & 0x7FFFu) : 0u;
        const bool eq = in && n_top && key == tau;
        const uint32_t be = __ballot_sync(0xffffffffu, eq);
        const bool m = in && n_top && (key > tau || (eq && (uint32_t)er + __popc(be & lt) < need_eq));
        const uint32_t bm = __ballot_sync(0xffffffffu, m);
        if (in) {
            mask[c] = (uint8_t)m;
            float rt;
            if (med_key == 0) rt = key ? __int_as_float(0x7F800000) : 0.0f;
            else rt = __fdiv_rn(__uint_as_float(key << 16), med);
            ratio[c] = rt;
            if (m && mask_idx) mask_idx[mr + __popc(bm & lt)] = c;
        }
        er += __popc(be);
        mr += __popc(bm);
    }
}

size_t a256(size_t v) { return (v + 255) & ~size_t(255); }

struct CalibLayout {
    size_t hs, hs2, whist, hist2, ge, lo, tbin, failed, needed, timed_out, total;
};

CalibLayout calib_layout(int64_t C)
{
    CalibLayout L{};
    const size_t nslab = (size_t)((C + kSlab - 1) / kSlab);
    L.hs = 0;
    L.hs2 = L.hs + a256((size_t)C * kBins1 * 4);
    L.whist = L.hs2 + a256((size_t)C * kBins2 * 4);
    L.hist2 = L.whist + a256((size_t)C * kWinBins * 4);
    L.ge = L.hist2 + a256((size_t)C * kBins2 * 4);
    L.lo = L.ge + a256((size_t)C * 4);
    L.tbin = L.lo + a256((size_t)C * 2);
    L.failed = L.tbin + a256((size_t)C * 2);
    L.needed = L.failed + a256((size_t)C);
    L.timed_out = L.needed + a256(nslab * 4);
    L.total = L.timed_out + 256;
    return L;
}

// Token splits: enough blocks for every SM to hold its resident maximum,
// at most kMaxRowsPerBlock rows per block (16-bit shared counters).
int64_t splits_for(int64_t rows, int nslab, int per_sm)
{
    const int64_t want = (int64_t)per_sm * sm_count();
    int64_t splits = (want + nslab - 1) / nslab;
    const int64_t min_rows = (int64_t)kRS * kUnroll;
    if (splits * min_rows > rows) splits = (rows + min_rows - 1) / min_rows;
    if (splits < 1) splits = 1;
    while ((rows + splits - 1) / splits > kMaxRowsPerBlock) ++splits;
    return splits;
}

template <int MODE>
hif4_status launch_pass_tma(const PassArgs &a0, cudaStream_t s, bool &done)
{
    constexpr int NB = MODE == 1 ? kBins1 : MODE == 2 ? kBins2 : kWinBins;
    const size_t smem = (size_t)kTmaStages * kTileBytes + (size_t)NB * kSlab / 2 * 4;
    done = false;
    if (a0.T > INT32_MAX - kTmaRows) return HIF4_OK;   // TMA row coordinates are int32
    CUtensorMap tm;
    if (!make_tensor_map_bf16_2d(&tm, a0.acts, (uint64_t)a0.C, (uint64_t)a0.T, (uint64_t)a0.lda * 2, kSlab, kTmaRows,
                                 false))
        return HIF4_OK;
    auto k = k_pass_tma<MODE>;
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr[dev & 63]) {
        if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return HIF4_ERR_CUDA;
        attr[dev & 63] = true;
    }
    PassArgs a = a0;
    a.withhold = wait_test_withhold();
    a.wait_ns = wait_limit_ns(kWaitNs);
    // equal shares of the slab-major (slab, row) space, one block per
    // resident slot, 4..65535 tiles' worth of rows each
    const int64_t slots = (int64_t)blocks_per_sm(reinterpret_cast<const void *>(k), kTmaThreads, smem) * sm_count();
    const int64_t total = (int64_t)a.nslab * a.T;
    int64_t share = (total + slots - 1) / slots;
    if (share < 4 * kTmaRows) share = 4 * kTmaRows;
    if (share > kMaxRowsPerBlock) share = kMaxRowsPerBlock;
    a.rows_per_split = share;
    const hif4_status st = launch_pdl(k, dim3((unsigned)((total + share - 1) / share)), dim3(kTmaThreads), smem, s,
                                      tm, a);
    done = st == HIF4_OK;
    return st;
}

template <int MODE>
hif4_status launch_pass(const PassArgs &a0, bool v8, bool tma, cudaStream_t s)
{
    if (tma) {
        bool done = false;
        const hif4_status st = launch_pass_tma<MODE>(a0, s, done);
        if (done || st != HIF4_OK) return st;
    }
    constexpr int NB = MODE == 1 ? kBins1 : MODE == 2 ? kBins2 : kWinBins;
    const size_t smem = (size_t)NB * kSlab / 2 * 4;
    auto kt = k_pass<MODE, true>;
    auto kf = k_pass<MODE, false>;
    static bool attr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!attr[dev & 63]) {
        if (cudaFuncSetAttribute(kt, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess ||
            cudaFuncSetAttribute(kf, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess)
            return HIF4_ERR_CUDA;
        attr[dev & 63] = true;
    }
    PassArgs a = a0;
    const int per_sm = blocks_per_sm(reinterpret_cast<const void *>(kt), kThreads, smem);
    const int64_t splits = splits_for(a.T, a.nslab, per_sm);
    a.rows_per_split = (a.T + splits - 1) / splits;
    const int grid = (int)(a.nslab * splits);
    return v8 ? launch_pdl(kt, dim3(grid), dim3(kThreads), smem, s, a)
              : launch_pdl(kf, dim3(grid), dim3(kThreads), smem, s, a);
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
    uint16_t *tbin = reinterpret_cast<uint16_t *>(ws + L.tbin);
    uint8_t *failed = ws + L.failed;
    uint32_t *needed = reinterpret_cast<uint32_t *>(ws + L.needed);
    uint32_t *timed_out = reinterpret_cast<uint32_t *>(ws + L.timed_out);
    if (cudaMemsetAsync(workspace, 0, L.total, s) != cudaSuccess) return HIF4_ERR_CUDA;

    const uint64_t kk = ((uint64_t)q_num * (uint64_t)(tokens - 1)) / q_den;
    const int nslab = (int)((channels + kSlab - 1) / kSlab);
    const int fgrid = (int)((channels * 32 + 255) / 256);
    hif4_status st;

    // 1. window start: exact order statistic of every R-th row (about 4096
    //    rows) at four times the target's tail mass below the top
    const int64_t R = tokens / 4096 > 1 ? tokens / 4096 : 1;
    const int64_t Ts = (tokens + R - 1) / R;
    const uint64_t tail = ((uint64_t)(tokens - kk) * 4ull * (uint64_t)Ts + (uint64_t)tokens - 1) / (uint64_t)tokens;
    const uint32_t r_lo = (uint32_t)((uint64_t)Ts > tail + 1 ? (uint64_t)Ts - 1 - tail : 0);
    const bool v8s = aligned_to(acts, 8) && ((lda * R) % 4 == 0);
    PassArgs sa{};
    sa.acts = static_cast<const uint16_t *>(acts);
    sa.T = Ts;
    sa.C = (int)channels;
    sa.lda = lda * R;
    sa.nslab = nslab;
    sa.hist1 = hs;
    sa.hist2 = hs2;
    sa.k = r_lo;
    sa.tbin = tbin;
    sa.timed_out = timed_out;
    // TMA needs a 16-byte aligned base and row stride (the box is 256 bytes wide)
    const bool tmas = aligned16(acts) && ((lda * R * 2) % 16 == 0);
    if ((st = launch_pass<1>(sa, v8s, tmas, s)) != HIF4_OK) return st;
    if (launch_pdl(k_select1, dim3(fgrid), dim3(256), 0, s, (const uint32_t *)hs, (int)channels, r_lo, tbin,
                   (const uint8_t *)nullptr) != HIF4_OK)
        return HIF4_ERR_CUDA;
    if ((st = launch_pass<2>(sa, v8s, tmas, s)) != HIF4_OK) return st;
    if (launch_pdl(k_finalize, dim3(fgrid), dim3(256), 0, s, (const uint32_t *)hs, (const uint32_t *)hs2,
                   (int)channels, r_lo, lo, (const uint8_t *)nullptr) != HIF4_OK)
        return HIF4_ERR_CUDA;

    // 2-3. windowed pass over every token, then the key where rank k falls
    const bool v8 = aligned_to(acts, 8) && (lda % 4 == 0);
    const bool tma = aligned16(acts) && ((lda * 2) % 16 == 0);
    PassArgs a{};
    a.acts = static_cast<const uint16_t *>(acts);
    a.T = tokens;
    a.C = (int)channels;
    a.lda = lda;
    a.nslab = nslab;
    a.lo = lo;
    a.ge = ge;
    a.whist = whist;
    a.timed_out = timed_out;
    if ((st = launch_pass<3>(a, v8, tma, s)) != HIF4_OK) return st;
    if (launch_pdl(k_window_final, dim3(fgrid), dim3(256), 0, s, whist, (const uint32_t *)ge, (const uint16_t *)lo,
                   (int)channels, (uint64_t)tokens, (uint32_t)kk, static_cast<uint16_t *>(pct), failed,
                   needed) != HIF4_OK)
        return HIF4_ERR_CUDA;

    // 4. exact two-pass radix select for the channels outside their window
    a.hist1 = whist;
    a.hist2 = hist2;
    a.k = (uint32_t)kk;
    a.tbin = tbin;
    a.needed = needed;
    if ((st = launch_pass<1>(a, v8, tma, s)) != HIF4_OK) return st;
    if (launch_pdl(k_select1, dim3(fgrid), dim3(256), 0, s, (const uint32_t *)whist, (int)channels, (uint32_t)kk,
                   tbin, (const uint8_t *)failed) != HIF4_OK)
        return HIF4_ERR_CUDA;
    if ((st = launch_pass<2>(a, v8, tma, s)) != HIF4_OK) return st;
    if (launch_pdl(k_finalize, dim3(fgrid), dim3(256), 0, s, (const uint32_t *)whist, (const uint32_t *)hist2,
                   (int)channels, (uint32_t)kk, static_cast<uint16_t *>(pct), (const uint8_t *)failed) != HIF4_OK)
        return HIF4_ERR_CUDA;

    // 5. median over channels, ratios, top-n mask
    static bool mattr[64] = {false};
    int dev = 0;
    cudaGetDevice(&dev);
    if (!mattr[dev & 63]) {
        if (cudaFuncSetAttribute(k_mask, cudaFuncAttributeMaxDynamicSharedMemorySize, kKeySlots * 4) != cudaSuccess)
            return HIF4_ERR_CUDA;
        mattr[dev & 63] = true;
    }
    const uint32_t n_top = (uint32_t)(((uint64_t)channels * mask_num) / mask_den);
    return launch_pdl(k_mask, dim3(1), dim3(kMaskThreads), (size_t)kKeySlots * 4, s,
                      static_cast<const uint16_t *>(pct), (int)channels, n_top, ratio, mask, mask_idx_out,
                      (const uint32_t *)timed_out);
}
