// common.cuh -- shared definitions of the CSA2 FP4 sparse-KV kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

#include <mutex>

#include "../../include/csa.h"

namespace csa {

constexpr int kPage = CSA_PAGE_TOKENS;      // tokens per page
constexpr int kBlock = CSA_BLOCK_POSITIONS; // positions per indexer block
constexpr int kBlocksPerPage = kPage / kBlock;
constexpr int kLatent = CSA_LATENT;
constexpr int kCodeBytes = kLatent / 2;     // 256 B of E2M1 codes per entry
constexpr int kScaleBytes = kLatent / 16;   // 32 E4M3 scales per entry
constexpr int kIdxHeads = CSA_INDEX_HEADS;
constexpr int kIdxDim = CSA_INDEX_DIM;
constexpr int kWindow = CSA_WINDOW;

// ------------------------------------------------------------------------------------------------
// Workspace: [0, 256) status header; then block scores; the Full indexer's screening buffers; then
// attention split partials.  Offsets up to the attention partials depend on B, max_seq_len and cap
// only, so indexer calls need not know H.
// ------------------------------------------------------------------------------------------------
constexpr size_t kHeaderBytes = CSA_WORKSPACE_HEADER_BYTES;
constexpr int kNumSms = 148;                // B200 SM count, used to size the attention split
constexpr int kAttnUnit = 8;                // entries per attention work unit (one block)
constexpr int kWindowUnits = kWindow / kAttnUnit;

struct WsLayout {
    size_t scores = 0;       // float [B][score_cap] (the Full selection keeps uint32 score keys here)
    size_t score_cap = 0;
    size_t topk = 0;         // uint32 [B][topk_words] per-sequence select state (words, counts)
    size_t nb = 0;           // blocks of the longest sequence
    size_t lo = 0, hi = 0;   // float [B][lstride] screening bounds of every block
    size_t lstride = 0;      // nb rounded up to 4 (16-byte rows)
    size_t qt = 0;           // uint8 [B][kQtBytes] query-term operand images
    size_t qm = 0;           // [B][kQmBytes] per-sequence screening constants
    size_t status = 0;       // uint8 [B][status_stride] class of every block (out, sure, uncertain, chosen)
    size_t status_stride = 0;   // nb rounded up to 16
    size_t uslice = 0;       // int32 [B][nb] uncertain blocks beyond the selection's shared-memory lists
    size_t hist = 0;         // uint32 [B][kHistBins] histogram of the blocks' lower-bound keys
    size_t hist2 = 0;        // uint32 [B][kHistBins] second level, inside the threshold bin
    size_t screen_end = 0;   // end of the indexer's regions
    size_t part_o = 0;       // float [B][splits][H][512]
    size_t part_ml = 0;      // float2 [B][splits][H]  (running max, running sum)
    int splits = 0;
    size_t total = 0;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Attention split count per sequence: about one wave of CTAs over the GPU (one CTA per SM for the
// tensor-core kernel, whose 128-entry tiles fill the SM; two for the CUDA-core kernel), never more
// than the sequence's largest number of tiles (selected blocks plus the window).
inline int attn_splits(int B, int cap, int units_per_tile)
{
    int max_units = cap + kWindowUnits;
    int max_tiles = (max_units + units_per_tile - 1) / units_per_tile;
    const int target = units_per_tile >= 16 ? kNumSms : 2 * kNumSms;
    int s = target / B;
    if (s < 1) s = 1;
    if (s > max_tiles) s = max_tiles;
    if (s < 1) s = 1;
    return s;
}

constexpr int kTopkWords = 8;
constexpr size_t kQtBytes = 32 * CSA_INDEX_DIM;   // 3 E4M3 terms x 8 heads + 8 zero rows, 128 B each
constexpr size_t kQmBytes = 64;
constexpr int kHistBins = 4096;                   // top 12 bits of a 32-bit order key

inline WsLayout ws_layout(int B, int H, int max_seq_len, int cap, int units_per_tile)
{
    WsLayout w;
    size_t nb = ((size_t)max_seq_len + kBlock - 1) / kBlock;
    w.score_cap = nb > (size_t)cap ? nb : (size_t)cap;
    size_t o = kHeaderBytes;
    w.scores = o;
    o = align_up(o + (size_t)B * w.score_cap * 4, 256);
    w.topk = o;
    o = align_up(o + (size_t)B * kTopkWords * 4, 256);
    w.nb = nb;
    w.lstride = align_up(nb, 4);
    w.lo = o;
    o = align_up(o + (size_t)B * w.lstride * 4, 256);
    w.hi = o;
    o = align_up(o + (size_t)B * w.lstride * 4, 256);
    w.qt = o;
    o = align_up(o + (size_t)B * kQtBytes, 1024);
    w.qm = o;
    o = align_up(o + (size_t)B * kQmBytes, 256);
    w.status = o;
    w.status_stride = align_up(nb, 16);
    o = align_up(o + (size_t)B * w.status_stride, 256);
    w.uslice = o;
    o = align_up(o + (size_t)B * nb * 4, 256);
    w.hist = o;
    o = align_up(o + (size_t)B * kHistBins * 4, 256);
    w.hist2 = o;
    o = align_up(o + (size_t)B * kHistBins * 4, 256);
    w.screen_end = o;
    w.splits = attn_splits(B, cap, units_per_tile);
    w.part_o = o;
    o = align_up(o + (size_t)B * w.splits * H * kLatent * 4, 256);
    w.part_ml = o;
    o = align_up(o + (size_t)B * w.splits * H * 8, 256);
    w.total = o;
    return w;
}

// Allow `bytes` of dynamic shared memory for kernel `fn` on the current device, calling the runtime
// only the first time a kernel needs more than it was last allowed there (the setting persists).
inline cudaError_t allow_dynamic_smem(const void *fn, size_t bytes)
{
    struct Entry {
        const void *fn;
        int dev;
        size_t bytes;
    };
    static std::mutex mu;
    static Entry tab[256];
    static int n = 0;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(mu);
    int i = 0;
    while (i < n && !(tab[i].fn == fn && tab[i].dev == dev)) ++i;
    if (i < n && tab[i].bytes >= bytes) return cudaSuccess;
    e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
    if (e != cudaSuccess) return e;
    if (i == n && n < 256) tab[n++] = Entry{fn, dev, bytes};
    else if (i < n) tab[i].bytes = bytes;
    return cudaSuccess;
}

// Launch `kernel` so that it may start before the previous grid of the stream completes: the
// previous grid lets it be scheduled (grid_dep_launch) and the kernel waits for the previous grid's
// results where it needs them (grid_dep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                     Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args &&>(args)...);
}

// ------------------------------------------------------------------------------------------------
// Device status word: the first error wins; its detail is the offending index.
// ------------------------------------------------------------------------------------------------
struct DevStatus {
    int32_t code;
    int32_t pad;
    long long detail;
};

__device__ __forceinline__ void report(void *ws, int code, long long detail)
{
    DevStatus *st = reinterpret_cast<DevStatus *>(ws);
    if (atomicCAS(&st->code, 0, code) == 0)
        atomicExch(reinterpret_cast<unsigned long long *>(&st->detail), (unsigned long long)detail);
}

// ------------------------------------------------------------------------------------------------
// Small numeric helpers
// ------------------------------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Total order on float bit patterns (larger float -> larger key), -0 folded onto +0.
__device__ __forceinline__ uint32_t order_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Inverse of order_key (a key of 0 or +0 gives +0).
__device__ __forceinline__ float key_to_float(uint32_t u)
{
    return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

}  // namespace csa
