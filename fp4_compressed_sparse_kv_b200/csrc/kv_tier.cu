// kv_tier.cu -- the storage half of the persistent KV tier: a sequence's FP4 entries, their E4M3
// scales and its indexer keys copied out of the paged caches into one contiguous buffer (device
// memory, or page-locked host memory the kernel addresses over the bus) and back into pages.
//
// yomxxx.com long-form post on KV-cache compression limits, section 三 (the global KV resident in
// HBM, the persistent KV on SSD or in host memory, fetched back when needed); rebasdaily article on
// DeepSeek-V4.1-Flash KV compression, section "先让长输入少走一半路" (SWA Bounded Replay: the
// sliding-window state is not stored; the most recent tokens are replayed to restore it).  The
// window entries are therefore not exported: after an import the caller re-packs the last
// min(n, 128) tokens with their window slots (csa_kv_pack_fp4 writes the same FP4 and key bytes
// again, and the window).
//
// Record layout, one per 64-token page of the sequence, 26,624 bytes:
//   codes [64][256] | scales [64][32] | keys [64][128]
// i.e. the three per-page arrays of the caches back to back.  Rows past the sequence's end in its
// last page are copied as they are.
#include "common.cuh"

namespace csa {

constexpr int kCodePage = kPage * kCodeBytes;            // 16,384
constexpr int kScalePage = kPage * kScaleBytes;          // 2,048
constexpr int kKeyPage = kPage * kIdxDim;                // 8,192
constexpr int kRecord = kCodePage + kScalePage + kKeyPage;

constexpr int kRecordVecs = kRecord / 16;               // 1,664 16-byte pieces
constexpr int kTierThreads = 416;                        // 13 warps, 4 pieces each
constexpr int kTierPer = kRecordVecs / kTierThreads;
static_assert(kTierPer * kTierThreads == kRecordVecs, "record pieces split evenly");

// One CTA per page.  Thread t moves pieces t + 416 i (i < 4) of the record, all four loads issued
// before the first store.  export: pages -> record; import: record -> pages.
template <bool kExport>
__global__ void __launch_bounds__(kTierThreads) kv_tier_kernel(uint8_t *codes, uint8_t *scales, uint8_t *keys,
                                                               int num_pages, const int32_t *__restrict__ block_table,
                                                               uint8_t *rec, void *ws)
{
    const int i = blockIdx.x;
    const int page = block_table[i];
    if (page < 0 || page >= num_pages) {
        if (threadIdx.x == 0) report(ws, CSA_ERR_DEVICE_DATA, (long long)i);
        return;
    }
    uint4 *r = reinterpret_cast<uint4 *>(rec + (size_t)i * kRecord);
    uint4 *c = reinterpret_cast<uint4 *>(codes + (size_t)page * kCodePage);
    uint4 *s = reinterpret_cast<uint4 *>(scales + (size_t)page * kScalePage);
    uint4 *k = reinterpret_cast<uint4 *>(keys + (size_t)page * kKeyPage);
    constexpr int nc = kCodePage / 16, ns = kScalePage / 16;
    uint4 *cache[kTierPer];
    uint4 v[kTierPer];
#pragma unroll
    for (int u = 0; u < kTierPer; ++u) {
        const int j = threadIdx.x + u * kTierThreads;
        cache[u] = j < nc ? c + j : (j < nc + ns ? s + (j - nc) : k + (j - nc - ns));
    }
#pragma unroll
    for (int u = 0; u < kTierPer; ++u) v[u] = kExport ? *cache[u] : r[threadIdx.x + u * kTierThreads];
#pragma unroll
    for (int u = 0; u < kTierPer; ++u) {
        if (kExport)
            r[threadIdx.x + u * kTierThreads] = v[u];
        else
            *cache[u] = v[u];
    }
}

}  // namespace csa

using namespace csa;

namespace {
inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// The address the kernel uses for `p`: itself for device or managed memory, the mapped device
// address for page-locked host memory; nullptr for host memory the device cannot address.
uint8_t *device_address(uint8_t *p)
{
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return p;
    if (at.type == cudaMemoryTypeHost) return static_cast<uint8_t *>(at.devicePointer);
    return nullptr;
}

csa_status kv_tier(bool exp, const csa_kv_layer *layer, const int32_t *block_table, int32_t n, uint8_t *buf, void *ws,
                   size_t ws_bytes, void *stream)
{
    if (n < 0 || n > CSA_MAX_SEQ_LEN) return CSA_ERR_INVALID_ARG;
    if (n == 0) return CSA_OK;
    if (!layer || !layer->codes || !layer->scales || !layer->keys || layer->num_pages < 1) return CSA_ERR_INVALID_ARG;
    if (!aligned16(layer->codes) || !aligned16(layer->scales) || !aligned16(layer->keys)) return CSA_ERR_INVALID_ARG;
    if (!block_table || !buf || !ws || !aligned16(block_table) || !aligned16(buf) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    buf = device_address(buf);
    if (!buf || !aligned16(buf)) return CSA_ERR_INVALID_ARG;
    const int pages = (n + kPage - 1) / kPage;
    cudaStream_t st = (cudaStream_t)stream;
    if (exp)
        kv_tier_kernel<true><<<pages, kTierThreads, 0, st>>>(layer->codes, layer->scales, layer->keys, layer->num_pages,
                                                    block_table, buf, ws);
    else
        kv_tier_kernel<false><<<pages, kTierThreads, 0, st>>>(layer->codes, layer->scales, layer->keys, layer->num_pages,
                                                     block_table, buf, ws);
    return cudaGetLastError() == cudaSuccess ? CSA_OK : CSA_ERR_CUDA;
}
}  // namespace

extern "C" {

size_t csa_kv_record_bytes(int32_t n)
{
    if (n < 0) return 0;
    return (size_t)((n + kPage - 1) / kPage) * (size_t)kRecord;
}

csa_status csa_kv_export(const csa_kv_layer *layer, const int32_t *block_table, int32_t n, uint8_t *dst, void *ws,
                         size_t ws_bytes, void *stream)
{
    return kv_tier(true, layer, block_table, n, dst, ws, ws_bytes, stream);
}

csa_status csa_kv_import(const csa_kv_layer *layer, const int32_t *block_table, int32_t n, const uint8_t *src,
                         void *ws, size_t ws_bytes, void *stream)
{
    return kv_tier(false, layer, block_table, n, const_cast<uint8_t *>(src), ws, ws_bytes, stream);
}

}  // extern "C"
