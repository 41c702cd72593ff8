// indexer.cu -- steps 2-3: hierarchical sparse indexer (Full / Reindex block scoring, exact Top-K)
// and the Reuse copy.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": a Full
// layer re-selects Top-K positions over the whole range (the decoder's first Full layer scans the
// full range into a 2,048-block x 8-position candidate pool); a Reindex layer searches only inside
// that pool; a Reuse layer takes the earlier layer's positions unchanged.  The position score is
// sum_h w_h * ReLU(q_h . k) over 8 heads of 128-dim E4M3 keys, in binary32 with a fixed operation
// order (see csa.h), so that the selected set is bit-for-bit reproducible.
#include "common.cuh"
#include "convert.cuh"
#include "pipeline.cuh"

namespace csa {

// ------------------------------------------------------------------------------------------------
// Block scoring.  Persistent CTAs; a work item is 8 consecutive "virtual" blocks of one sequence:
// in Full mode virtual block v is block v (8 blocks = one 64-token page); in Reindex mode it is
// pool[b][v].  A producer warp gathers each item's 8 x 1 KB key blocks into a shared-memory ring
// with 1-D bulk copies; 8 consumer warps each score one block.  Consumer lane (g, j) = (lane/8,
// lane%8) holds dims 16j..16j+15 of all 8 query heads in registers and takes key g of each group
// of 4, so one 16-byte shared load feeds 128 FMAs.  The 8 per-lane partials per head are combined
// by a 3-step xor reduce-scatter (distances 4, 2, 1) that forms exactly
// ((p0+p4)+(p2+p6)) + ((p1+p5)+(p3+p7)) in every lane, up to the commutativity of each addition.
// ------------------------------------------------------------------------------------------------
constexpr int kScoreStages = 8;
constexpr int kScoreConsumers = 8;
constexpr int kScoreThreads = (kScoreConsumers + 1) * 32;
constexpr int kBlockBytes = kBlock * kIdxDim;              // 1 KB of keys per block
constexpr int kStageBytes = kScoreConsumers * kBlockBytes;  // 8 KB per stage
constexpr int kBlkEmpty = -2;                               // virtual block past the end
constexpr int kBlkBad = -1;                                 // invalid metadata (reported)

struct ScoreArgs {
    const uint8_t *keys;
    int num_pages;
    const int32_t *seq_len;
    const int32_t *block_table;
    int max_pages;
    int max_seq_len;
    int B;
    const uint16_t *iq;
    const float *iw;
    const int32_t *pool;        // null: Full mode
    const int32_t *pool_count;
    int pool_cap;
    int items_per_seq;
    float *scores;
    int score_stride;
    void *ws;
};

struct StageMeta {
    int b;
    int L;
    int blk[kScoreConsumers];
};

struct ScoreSmem {
    alignas(128) uint8_t stage[kScoreStages][kStageBytes];
    StageMeta meta[kScoreStages];
    uint64_t full[kScoreStages];
    uint64_t empty[kScoreStages];
    int abort_flag;
};

__device__ __forceinline__ float score_key(const float (&q)[8][16], const float (&w)[8], uint4 kr, int lane)
{
    const int j = lane & 7;
    float k[16];
    const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const uint32_t lo = e4m3x2_to_f16x2((uint16_t)(kw[i] & 0xFFFF));
        const uint32_t hi = e4m3x2_to_f16x2((uint16_t)(kw[i] >> 16));
        k[4 * i + 0] = h_lo(lo);
        k[4 * i + 1] = h_hi(lo);
        k[4 * i + 2] = h_lo(hi);
        k[4 * i + 3] = h_hi(hi);
    }
    float part[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
        float p = 0.f;
#pragma unroll
        for (int t = 0; t < 16; ++t) p = __fmaf_rn(q[h][t], k[t], p);
        part[h] = p;
    }
    // reduce-scatter over the 8 lanes of this key: lane j ends with head j
    const bool up4 = j & 4, up2 = j & 2, up1 = j & 1;
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float send = up4 ? part[i] : part[4 + i];
        const float keep = up4 ? part[4 + i] : part[i];
        a[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    }
    float c[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const float send = up2 ? a[i] : a[2 + i];
        const float keep = up2 ? a[2 + i] : a[i];
        c[i] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 2));
    }
    const float send = up1 ? c[0] : c[1];
    const float keep = up1 ? c[1] : c[0];
    const float d = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 1));
    const float r = d > 0.f ? d : 0.f;
    float score = 0.f;
    const int base = lane & ~7;
#pragma unroll
    for (int h = 0; h < 8; ++h) score = __fmaf_rn(w[h], __shfl_sync(0xffffffffu, r, base | h), score);
    return score;
}

__global__ void __launch_bounds__(kScoreThreads, 1) block_score_kernel(ScoreArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    ScoreSmem &sm = *reinterpret_cast<ScoreSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = (long long)a.B * a.items_per_seq;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kScoreStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.empty[s], kScoreConsumers);
        }
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == kScoreConsumers) {
        // ---------------- producer ----------------
        if (lane == 0) {
            long long k = 0;
            for (long long item = blockIdx.x; item < total; item += gridDim.x, ++k) {
                const int st = (int)(k % kScoreStages);
                const uint32_t ph = (uint32_t)((k / kScoreStages) & 1);
                if (!mbar_wait(&sm.empty[st], ph ^ 1u, &sm.abort_flag, a.ws, item)) break;
                const int b = (int)(item / a.items_per_seq);
                const int grp = (int)(item % a.items_per_seq);
                StageMeta &m = sm.meta[st];
                const int L = a.seq_len[b];
                m.b = b;
                m.L = L;
                int blks[kScoreConsumers];
                uint32_t bytes = 0;
                const bool L_ok = L >= 1 && L <= a.max_seq_len;
                if (!L_ok && grp == 0) report(a.ws, CSA_ERR_DEVICE_DATA, b);
                int nvb = 0;
                if (L_ok) {
                    nvb = a.pool ? a.pool_count[b] : (L + kBlock - 1) / kBlock;
                    if (a.pool && (nvb < 0 || nvb > a.pool_cap)) {
                        if (grp == 0) report(a.ws, CSA_ERR_DEVICE_DATA, b);
                        nvb = 0;
                    }
                }
                const int nb = (L + kBlock - 1) / kBlock;
#pragma unroll
                for (int w = 0; w < kScoreConsumers; ++w) {
                    const int v = grp * kScoreConsumers + w;
                    int blk = kBlkEmpty;
                    if (v < nvb) {
                        blk = a.pool ? a.pool[(size_t)b * a.pool_cap + v] : v;
                        if (a.pool && v > 0 && a.pool[(size_t)b * a.pool_cap + v - 1] >= blk)
                            report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b * a.pool_cap + v);
                        if (blk < 0 || blk >= nb) {
                            report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b * a.pool_cap + v);
                            blk = kBlkBad;
                        } else {
                            const int page = a.block_table[(size_t)b * a.max_pages + blk / kBlocksPerPage];
                            if (page < 0 || page >= a.num_pages) {
                                report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b * a.max_pages + blk / kBlocksPerPage);
                                blk = kBlkBad;
                            } else {
                                bytes += kBlockBytes;
                            }
                        }
                    }
                    blks[w] = blk;
                    m.blk[w] = blk;
                }
                if (bytes == 0) {
                    mbar_arrive(&sm.full[st]);
                } else {
                    mbar_arrive_expect_tx(&sm.full[st], bytes);
#pragma unroll
                    for (int w = 0; w < kScoreConsumers; ++w) {
                        const int blk = blks[w];
                        if (blk < 0) continue;
                        const int page = a.block_table[(size_t)b * a.max_pages + blk / kBlocksPerPage];
                        const uint8_t *src =
                            a.keys + ((size_t)page * kPage + (size_t)(blk % kBlocksPerPage) * kBlock) * kIdxDim;
                        bulk_g2s(sm.stage[st] + w * kBlockBytes, src, kBlockBytes, &sm.full[st]);
                    }
                }
            }
            // no copy may still be landing in shared memory when the CTA exits
            const long long first = k > kScoreStages ? k - kScoreStages : 0;
            for (long long kk = first; kk < k; ++kk) {
                volatile int no_abort = 0;
                mbar_wait(&sm.full[kk % kScoreStages], (uint32_t)((kk / kScoreStages) & 1), &no_abort, a.ws, -1);
            }
        }
    } else {
        // ---------------- consumers ----------------
        float q[8][16];
        float w[8];
        int cur_b = -1;
        long long k = 0;
        for (long long item = blockIdx.x; item < total; item += gridDim.x, ++k) {
            const int st = (int)(k % kScoreStages);
            const uint32_t ph = (uint32_t)((k / kScoreStages) & 1);
            if (!mbar_wait(&sm.full[st], ph, &sm.abort_flag, a.ws, item)) break;
            const StageMeta &m = sm.meta[st];
            const int b = m.b, L = m.L;
            const int blk = m.blk[warp];
            if (blk >= 0) {
                if (b != cur_b) {
                    const int j = lane & 7;
#pragma unroll
                    for (int h = 0; h < 8; ++h) {
                        const uint4 *src =
                            reinterpret_cast<const uint4 *>(a.iq + ((size_t)b * kIdxHeads + h) * kIdxDim + 16 * j);
                        const uint4 u0 = src[0], u1 = src[1];
                        const uint32_t uw[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
#pragma unroll
                        for (int i = 0; i < 8; ++i) {
                            q[h][2 * i] = bf16_lo(uw[i]);
                            q[h][2 * i + 1] = bf16_hi(uw[i]);
                        }
                        w[h] = a.iw[(size_t)b * kIdxHeads + h];
                    }
                    cur_b = b;
                }
                const uint8_t *sp = sm.stage[st] + warp * kBlockBytes;
                const int g = lane >> 3, j = lane & 7;
                float best = -INFINITY;
#pragma unroll
                for (int it = 0; it < 2; ++it) {
                    const int kk = it * 4 + g;
                    const uint4 kr = *reinterpret_cast<const uint4 *>(sp + kk * kIdxDim + 16 * j);
                    const float s = score_key(q, w, kr, lane);
                    if (blk * kBlock + kk < L) best = fmaxf(best, s);
                }
                best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 8));
                best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
                if (lane == 0) {
                    const int v = (int)(item % a.items_per_seq) * kScoreConsumers + warp;
                    a.scores[(size_t)b * a.score_stride + v] = best;
                }
            } else if (blk == kBlkBad && lane == 0) {
                const int v = (int)(item % a.items_per_seq) * kScoreConsumers + warp;
                a.scores[(size_t)b * a.score_stride + v] = -INFINITY;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.empty[st]);
        }
    }
    __syncthreads();
}

// ------------------------------------------------------------------------------------------------
// Exact Top-K of one sequence's n candidate scores: radix select of the k-th largest order key in
// four 8-bit passes (keys cached in shared memory when they fit), then one ascending pass that
// keeps every key above the threshold and the lowest-indexed ties, written in index order.
// ------------------------------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkCacheKeys = 16384;

__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_tot, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t t = lane < (int)(blockDim.x >> 5) ? warp_tot[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, t, o);
            if (lane >= o) t += y;
        }
        warp_tot[lane] = t;  // inclusive
    }
    __syncthreads();
    const uint32_t before = (warp > 0 ? warp_tot[warp - 1] : 0u) + x - v;
    *total = warp_tot[(blockDim.x >> 5) - 1];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const float *__restrict__ scores, int score_stride,
                                                               const int32_t *__restrict__ seq_len, int max_seq_len,
                                                               const int32_t *__restrict__ pool,
                                                               const int32_t *__restrict__ pool_count, int pool_cap,
                                                               int k, int32_t *__restrict__ out_blocks,
                                                               int32_t *__restrict__ out_count, void *ws)
{
    extern __shared__ uint32_t skeys[];
    __shared__ uint32_t hist[256];
    __shared__ uint32_t warp_tot[32];
    __shared__ uint32_t sel[2];
    const int b = blockIdx.x, t = threadIdx.x, lane = t & 31;
    const int L = seq_len[b];
    int n;
    if (L < 1 || L > max_seq_len) {
        n = 0;
        if (t == 0) report(ws, CSA_ERR_DEVICE_DATA, b);
    } else if (pool) {
        n = pool_count[b];
        if (n < 0 || n > pool_cap) n = 0;  // reported by the scoring kernel
    } else {
        n = (L + kBlock - 1) / kBlock;
    }
    const float *sc = scores + (size_t)b * score_stride;
    const int32_t *ids = pool ? pool + (size_t)b * pool_cap : nullptr;
    int32_t *out = out_blocks + (size_t)b * k;

    if (n <= k) {
        for (int i = t; i < n; i += kTopkThreads) out[i] = ids ? ids[i] : i;
        if (t == 0) out_count[b] = n;
        return;
    }
    const bool cached = n <= kTopkCacheKeys;
    if (cached) {
        for (int i = t; i < n; i += kTopkThreads) skeys[i] = order_key(sc[i]);
        __syncthreads();
    }
    uint32_t prefix = 0, mask = 0;
    uint32_t remaining = (uint32_t)k;
    for (int pass = 0; pass < 4; ++pass) {
        const int shift = 24 - 8 * pass;
        if (t < 256) hist[t] = 0;
        __syncthreads();
        for (int base = 0; base < n; base += kTopkThreads) {
            const int i = base + t;
            uint32_t digit = 256;
            if (i < n) {
                const uint32_t u = cached ? skeys[i] : order_key(sc[i]);
                if ((u & mask) == prefix) digit = (u >> shift) & 255u;
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, digit);
            if (digit < 256 && lane == __ffs(peers) - 1) atomicAdd(&hist[digit], (uint32_t)__popc(peers));
        }
        __syncthreads();
        // suffix counts from the top bucket down; the threshold bucket is where they reach `remaining`
        uint32_t c = 0;
        if (t < 256) c = hist[255 - t];
        uint32_t x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        if (t < 256 && lane == 31) warp_tot[t >> 5] = x;
        __syncthreads();
        if (t < 256) {
            uint32_t before = 0;
            for (int wi = 0; wi < (t >> 5); ++wi) before += warp_tot[wi];
            const uint32_t incl = before + x;
            if (incl >= remaining && incl - c < remaining) {
                sel[0] = 255u - (uint32_t)t;
                sel[1] = incl - c;
            }
        }
        __syncthreads();
        prefix |= sel[0] << shift;
        mask |= 255u << shift;
        remaining -= sel[1];
        __syncthreads();
    }
    const uint32_t T = prefix, need_eq = remaining;
    uint32_t gt_run = 0, eq_run = 0;
    for (int base = 0; base < n; base += kTopkThreads) {
        const int i = base + t;
        uint32_t u = 0;
        bool gt = false, eq = false;
        if (i < n) {
            u = cached ? skeys[i] : order_key(sc[i]);
            gt = u > T;
            eq = u == T;
        }
        uint32_t tot;
        const uint32_t ex = block_excl_scan((gt ? 1u : 0u) | (eq ? 0x10000u : 0u), warp_tot, &tot);
        const uint32_t gt_b = gt_run + (ex & 0xFFFF), eq_b = eq_run + (ex >> 16);
        if (gt || (eq && eq_b < need_eq)) out[gt_b + min(eq_b, need_eq)] = ids ? ids[i] : i;
        gt_run += tot & 0xFFFF;
        eq_run += tot >> 16;
    }
    if (t == 0) out_count[b] = k;
}

// ------------------------------------------------------------------------------------------------
// Reuse: copy the previous layer's set.
// ------------------------------------------------------------------------------------------------
__global__ void reuse_kernel(const int32_t *__restrict__ prev, const int32_t *__restrict__ prev_count, int prev_cap,
                             int32_t *__restrict__ out, int32_t *__restrict__ out_count, int out_cap, void *ws)
{
    const int b = blockIdx.x;
    int n = prev_count[b];
    if (n < 0 || n > prev_cap || n > out_cap) {
        if (threadIdx.x == 0) report(ws, CSA_ERR_DEVICE_DATA, b);
        n = 0;
    }
    for (int i = threadIdx.x; i < n; i += blockDim.x) out[(size_t)b * out_cap + i] = prev[(size_t)b * prev_cap + i];
    if (threadIdx.x == 0) out_count[b] = n;
}

// ------------------------------------------------------------------------------------------------
// Launchers
// ------------------------------------------------------------------------------------------------
static int g_num_sms[64];

static int num_sms()
{
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64) return 148;
    if (g_num_sms[dev] == 0) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_num_sms[dev] = n > 0 ? n : 148;
    }
    return g_num_sms[dev];
}

cudaError_t launch_block_scores(const ScoreArgs &args, cudaStream_t st)
{
    const size_t smem = sizeof(ScoreSmem);
    cudaError_t e = cudaFuncSetAttribute(block_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const long long total = (long long)args.B * args.items_per_seq;
    if (total == 0) return cudaSuccess;
    const int grid = (int)(total < num_sms() ? total : num_sms());
    block_score_kernel<<<grid, kScoreThreads, smem, st>>>(args);
    return cudaGetLastError();
}

cudaError_t launch_block_scores_full_or_pool(const uint8_t *keys, int num_pages, const csa_batch &bt,
                                             const uint16_t *iq, const float *iw, const int32_t *pool,
                                             const int32_t *pool_count, int pool_cap, float *scores,
                                             int score_stride, void *ws, cudaStream_t st)
{
    ScoreArgs a;
    a.keys = keys;
    a.num_pages = num_pages;
    a.seq_len = bt.seq_len;
    a.block_table = bt.block_table;
    a.max_pages = bt.max_pages;
    a.max_seq_len = bt.max_seq_len;
    a.B = bt.B;
    a.iq = iq;
    a.iw = iw;
    a.pool = pool;
    a.pool_count = pool_count;
    a.pool_cap = pool_cap;
    a.items_per_seq = pool ? (pool_cap + kScoreConsumers - 1) / kScoreConsumers
                           : (bt.max_seq_len + kPage - 1) / kPage;
    a.scores = scores;
    a.score_stride = score_stride;
    a.ws = ws;
    return launch_block_scores(a, st);
}

cudaError_t launch_topk(const float *scores, int score_stride, const int32_t *seq_len, int max_seq_len,
                        const int32_t *pool, const int32_t *pool_count, int pool_cap, int k, int B,
                        int32_t *out_blocks, int32_t *out_count, int max_candidates, void *ws, cudaStream_t st)
{
    const size_t smem = (size_t)(max_candidates < kTopkCacheKeys ? max_candidates : kTopkCacheKeys) * 4;
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    topk_kernel<<<B, kTopkThreads, smem, st>>>(scores, score_stride, seq_len, max_seq_len, pool, pool_count, pool_cap,
                                               k, out_blocks, out_count, ws);
    return cudaGetLastError();
}

cudaError_t launch_reuse(int B, const int32_t *prev, const int32_t *prev_count, int prev_cap, int32_t *out,
                         int32_t *out_count, int out_cap, void *ws, cudaStream_t st)
{
    reuse_kernel<<<B, 256, 0, st>>>(prev, prev_count, prev_cap, out, out_count, out_cap, ws);
    return cudaGetLastError();
}

}  // namespace csa
