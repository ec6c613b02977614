// hif4_state.cu — the compact post-training-quantization state of one
// linear layer, serialized [TA summary, "Method overview": compact deltas
// that restore the quantized behaviour are stored instead of the full BF16
// weights].  What the quantized layer needs at inference is exactly its HiF4
// codes and metadata, its protected-column indices and those columns' BF16
// weights; the record holds those and nothing else (4.5 bits per weight plus
// 16 bits per protected weight).
//
// Format, version 1 (little-endian; sections start at 64-byte offsets from
// the record start so that each can be mapped or copied to the device as is):
//   offset  0  magic "HIF4PTQS" (8 bytes)
//           8  u32 version = 1
//          12  u32 header bytes = 64
//          16  i64 N (rows = output features)
//          24  i64 K (columns = input features, a multiple of 64)
//          32  i32 n_masked (protected columns, 0 <= n_masked <= K)
//          36  u32 flags = 0 (reserved)
//          40  u64 total bytes of the record, trailer included
//          48  16 zero bytes (reserved)
//          64  mask_idx  n_masked x i32, sorted, distinct, in [0, K)
//   align64    codes     N x K/2 bytes (element 2b in the low nibble of byte b)
//   align64    meta      N x K/64 x u32 (c | e2 << 8 | e3 << 16)
//   align64    w_masked  N x n_masked x u16 (BF16 bit patterns, row-major)
//   align64    u32 CRC-32 (IEEE 802.3: reflected polynomial 0xEDB88320,
//              initial value and final XOR 0xFFFFFFFF) of every byte before it
// Host memory only: no device is touched, so these calls work without a GPU.
#include <cstring>

#include "hif4_internal.cuh"

namespace hif4 {
namespace {

constexpr char kMagic[8] = {'H', 'I', 'F', '4', 'P', 'T', 'Q', 'S'};
constexpr uint32_t kVersion = 1;
constexpr uint64_t kHeader = 64;

uint64_t a64(uint64_t v) { return (v + 63) & ~uint64_t(63); }

struct Layout {
    uint64_t idx, codes, meta, wm, crc, total;
};

// Section offsets for a layer, or false when the sizes overflow 64 bits.
bool layout(int64_t N, int64_t K, int64_t n_masked, Layout &L)
{
    if (N <= 0 || K <= 0 || K % HIF4_UNIT != 0 || n_masked < 0 || n_masked > K) return false;
    const uint64_t n = (uint64_t)N, k = (uint64_t)K, m = (uint64_t)n_masked;
    if (n > (uint64_t)1 << 40 || k > (uint64_t)1 << 40) return false;     // keeps every product below 2^63
    L.idx = kHeader;
    L.codes = a64(L.idx + 4 * m);
    L.meta = a64(L.codes + n * (k / 2));
    L.wm = a64(L.meta + 4 * n * (k / HIF4_UNIT));
    L.crc = a64(L.wm + 2 * n * m);
    L.total = L.crc + 4;
    return true;
}

uint32_t crc_table[256];
bool crc_ready = false;

uint32_t crc32(const uint8_t *p, uint64_t n)
{
    if (!crc_ready) {                       // benign race: every writer stores the same table
        for (uint32_t i = 0; i < 256; ++i) {
            uint32_t c = i;
            for (int b = 0; b < 8; ++b) c = (c & 1u) ? (0xEDB88320u ^ (c >> 1)) : (c >> 1);
            crc_table[i] = c;
        }
        crc_ready = true;
    }
    uint32_t c = 0xFFFFFFFFu;
    for (uint64_t i = 0; i < n; ++i) c = crc_table[(c ^ p[i]) & 0xFFu] ^ (c >> 8);
    return c ^ 0xFFFFFFFFu;
}

template <typename T>
void put(uint8_t *b, uint64_t off, T v)
{
    std::memcpy(b + off, &v, sizeof v);
}
template <typename T>
T get(const uint8_t *b, uint64_t off)
{
    T v;
    std::memcpy(&v, b + off, sizeof v);
    return v;
}

bool indices_ok(const int32_t *idx, int32_t n, int64_t K)
{
    for (int32_t j = 0; j < n; ++j)
        if (idx[j] < 0 || idx[j] >= K || (j > 0 && idx[j - 1] >= idx[j])) return false;
    return true;
}

// Header and checksum checks; on success fills N, K, n_masked and the layout.
hif4_status parse(const void *buf, size_t bytes, int64_t &N, int64_t &K, int32_t &nm, Layout &L)
{
    if (!buf) return HIF4_ERR_INVALID_ARG;
    const uint8_t *b = static_cast<const uint8_t *>(buf);
    if (bytes < kHeader + 4) return HIF4_ERR_FORMAT;
    if (std::memcmp(b, kMagic, 8) != 0) return HIF4_ERR_FORMAT;
    if (get<uint32_t>(b, 8) != kVersion || get<uint32_t>(b, 12) != kHeader) return HIF4_ERR_FORMAT;
    N = get<int64_t>(b, 16);
    K = get<int64_t>(b, 24);
    nm = get<int32_t>(b, 32);
    if (get<uint32_t>(b, 36) != 0) return HIF4_ERR_FORMAT;
    if (!layout(N, K, nm, L)) return HIF4_ERR_FORMAT;
    if (get<uint64_t>(b, 40) != L.total || (uint64_t)bytes < L.total) return HIF4_ERR_FORMAT;
    if (crc32(b, L.crc) != get<uint32_t>(b, L.crc)) return HIF4_ERR_FORMAT;
    if (!indices_ok(reinterpret_cast<const int32_t *>(b + L.idx), nm, K)) return HIF4_ERR_FORMAT;
    return HIF4_OK;
}

} // namespace
} // namespace hif4

using namespace hif4;

extern "C" size_t hif4_ptq_state_bytes(int64_t N, int64_t K, int32_t n_masked)
{
    Layout L;
    return layout(N, K, n_masked, L) ? (size_t)L.total : 0;
}

extern "C" hif4_status hif4_ptq_state_pack(int64_t N, int64_t K, const uint8_t *codes, const uint32_t *meta,
                                           const int32_t *mask_idx, int32_t n_masked, const void *w_masked,
                                           void *out, size_t out_bytes)
{
    Layout L;
    if (N <= 0 || K <= 0 || n_masked < 0) return HIF4_ERR_INVALID_ARG;
    if (K % HIF4_UNIT != 0) return HIF4_ERR_SHAPE;
    if (!layout(N, K, n_masked, L)) return HIF4_ERR_INVALID_ARG;
    if (!codes || !meta || !out || (n_masked > 0 && (!mask_idx || !w_masked))) return HIF4_ERR_INVALID_ARG;
    if ((uint64_t)out_bytes < L.total) return HIF4_ERR_WORKSPACE;
    if (n_masked > 0 && !indices_ok(mask_idx, n_masked, K)) return HIF4_ERR_INVALID_ARG;
    uint8_t *b = static_cast<uint8_t *>(out);
    std::memset(b, 0, (size_t)L.total);
    std::memcpy(b, kMagic, 8);
    put<uint32_t>(b, 8, kVersion);
    put<uint32_t>(b, 12, (uint32_t)kHeader);
    put<int64_t>(b, 16, N);
    put<int64_t>(b, 24, K);
    put<int32_t>(b, 32, n_masked);
    put<uint32_t>(b, 36, 0u);
    put<uint64_t>(b, 40, L.total);
    if (n_masked > 0) std::memcpy(b + L.idx, mask_idx, 4 * (size_t)n_masked);
    std::memcpy(b + L.codes, codes, (size_t)N * (size_t)(K / 2));
    std::memcpy(b + L.meta, meta, 4 * (size_t)N * (size_t)(K / HIF4_UNIT));
    if (n_masked > 0) std::memcpy(b + L.wm, w_masked, 2 * (size_t)N * (size_t)n_masked);
    put<uint32_t>(b, L.crc, crc32(b, L.crc));
    return HIF4_OK;
}

extern "C" hif4_status hif4_ptq_state_info(const void *buf, size_t bytes, int64_t *N, int64_t *K,
                                           int32_t *n_masked)
{
    int64_t n, k;
    int32_t m;
    Layout L;
    const hif4_status st = parse(buf, bytes, n, k, m, L);
    if (st != HIF4_OK) return st;
    if (N) *N = n;
    if (K) *K = k;
    if (n_masked) *n_masked = m;
    return HIF4_OK;
}

extern "C" hif4_status hif4_ptq_state_unpack(const void *buf, size_t bytes, uint8_t *codes, uint32_t *meta,
                                             int32_t *mask_idx, void *w_masked)
{
    int64_t N, K;
    int32_t nm;
    Layout L;
    const hif4_status st = parse(buf, bytes, N, K, nm, L);
    if (st != HIF4_OK) return st;
    if (!codes || !meta || (nm > 0 && (!mask_idx || !w_masked))) return HIF4_ERR_INVALID_ARG;
    const uint8_t *b = static_cast<const uint8_t *>(buf);
    if (nm > 0) std::memcpy(mask_idx, b + L.idx, 4 * (size_t)nm);
    std::memcpy(codes, b + L.codes, (size_t)N * (size_t)(K / 2));
    std::memcpy(meta, b + L.meta, 4 * (size_t)N * (size_t)(K / HIF4_UNIT));
    if (nm > 0) std::memcpy(w_masked, b + L.wm, 2 * (size_t)N * (size_t)nm);
    return HIF4_OK;
}
