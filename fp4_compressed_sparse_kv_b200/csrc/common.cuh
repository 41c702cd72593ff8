// common.cuh -- shared definitions of the CSA2 FP4 sparse-KV kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <stdint.h>

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
// Workspace: [0, 256) status header; then block scores; then attention split partials.
// ------------------------------------------------------------------------------------------------
constexpr size_t kHeaderBytes = CSA_WORKSPACE_HEADER_BYTES;
constexpr int kNumSms = 148;                // B200 SM count, used to size the attention split
constexpr int kAttnUnit = 8;                // entries per attention work unit (one block)
constexpr int kWindowUnits = kWindow / kAttnUnit;

struct WsLayout {
    size_t scores = 0;       // float [B][score_cap]
    size_t score_cap = 0;
    size_t topk = 0;         // uint32 [B][topk_words] per-sequence select state
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

constexpr int kTopkWords = 4;

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
    w.splits = attn_splits(B, cap, units_per_tile);
    w.part_o = o;
    o = align_up(o + (size_t)B * w.splits * H * kLatent * 4, 256);
    w.part_ml = o;
    o = align_up(o + (size_t)B * w.splits * H * 8, 256);
    w.total = o;
    return w;
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

}  // namespace csa
