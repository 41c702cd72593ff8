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
#include "radix.cuh"
#include "score.cuh"

namespace csa {

// ------------------------------------------------------------------------------------------------
// Block scoring.  Persistent CTAs of 8 warps; a work item is 8 consecutive "virtual" blocks of one
// sequence (in Full mode virtual block v is block v, so an item is one 64-token page; in Reindex
// mode it is pool[b][v]) and warp w always takes virtual block w of each item.  Every warp runs its
// own pipeline: lane 0 resolves the block's page a few items ahead and bulk-copies its 1 KB of keys
// into the warp's shared-memory ring; no warp ever waits for another.
//
// The query pairs of each lane stay in registers; the lane layout and the operation order of the exact
// score are those of score.cuh.
// ------------------------------------------------------------------------------------------------
constexpr int kScoreWarps = 8;
constexpr int kScoreThreads = kScoreWarps * 32;
constexpr int kScoreStages = 6;
constexpr int kBlockBytes = kBlock * kIdxDim;   // 1 KB of keys per block
constexpr int kBlkEmpty = -2;                    // virtual block past the end
constexpr int kBlkBad = -1;                      // invalid metadata (reported)

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

constexpr int kMetaRing = 64;   // per-warp ring of resolved items (>= 32 + kScoreStages)

struct ItemMeta {
    const uint8_t *src;   // the block's 1 KB of keys, or null
    int b;
    int L;
    int blk;
    int v;
};

struct ScoreSmem {
    alignas(128) uint8_t stage[kScoreWarps][kScoreStages][kBlockBytes];
    ItemMeta meta[kScoreWarps][kMetaRing];
    uint64_t full[kScoreWarps][kScoreStages];
    int abort_flag;
};

__global__ void __launch_bounds__(kScoreThreads, 1) block_score_kernel(ScoreArgs a)
{
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    ScoreSmem &sm = *reinterpret_cast<ScoreSmem *>(smem_raw);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long total = (long long)a.B * a.items_per_seq;
    // each CTA takes a contiguous range of items, so consecutive items mostly share a sequence (and
    // its query stays in registers)
    const long long per = (total + gridDim.x - 1) / gridDim.x;
    const long long first = (long long)blockIdx.x * per;
    const long long last = first + per < total ? first + per : total;

    if (threadIdx.x == 0) {
        for (int w = 0; w < kScoreWarps; ++w)
            for (int st = 0; st < kScoreStages; ++st) mbar_init(&sm.full[w][st], 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    // ---- metadata of this warp's block of items k0 .. k0+31, one item per lane, loads in parallel
    // local item counters are 32-bit (stage and ring arithmetic by constants stays cheap)
    auto resolve32 = [&](uint32_t k0) {
        const uint32_t k = k0 + lane;
        const long long item = first + k;
        ItemMeta m{nullptr, 0, 0, kBlkEmpty, 0};
        if (item < last) {
            const int b = (int)(item / a.items_per_seq);
            const int grp = (int)(item % a.items_per_seq);
            const int L = a.seq_len[b];
            int nvb = 0;
            if (L < 1 || L > a.max_seq_len) {
                if (grp == 0 && warp == 0) report(a.ws, CSA_ERR_DEVICE_DATA, b);
            } else {
                nvb = a.pool ? a.pool_count[b] : (L + kBlock - 1) / kBlock;
                if (a.pool && (nvb < 0 || nvb > a.pool_cap)) {
                    if (grp == 0 && warp == 0) report(a.ws, CSA_ERR_DEVICE_DATA, b);
                    nvb = 0;
                }
            }
            const int v = grp * kScoreWarps + warp;
            const int nb = (L + kBlock - 1) / kBlock;
            m.b = b;
            m.L = L;
            m.v = v;
            if (v < nvb) {
                int blk = a.pool ? a.pool[(size_t)b * a.pool_cap + v] : v;
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
                        m.src = a.keys + ((size_t)page * kPage + (size_t)(blk % kBlocksPerPage) * kBlock) * kIdxDim;
                    }
                }
                m.blk = blk;
            }
        }
        sm.meta[warp][k % kMetaRing] = m;
    };
    // lane 0: start the copy of item k's block into stage k % kScoreStages
    auto issue = [&](uint32_t k) {
        const long long item = first + k;
        if (item >= last) return;
        const int st = (int)(k % kScoreStages);
        const ItemMeta &m = sm.meta[warp][k % kMetaRing];
        if (m.src) {
            fence_async_smem();   // this warp's earlier reads of the stage precede the copy into it
            mbar_arrive_expect_tx(&sm.full[warp][st], kBlockBytes);
            bulk_g2s(sm.stage[warp][st], m.src, kBlockBytes, &sm.full[warp][st]);
        } else {
            mbar_arrive(&sm.full[warp][st]);
        }
    };

    resolve32(0);
    __syncwarp();
    if (lane == 0)
        for (uint32_t k = 0; k < kScoreStages - 1; ++k) issue(k);
    __syncwarp();

    unsigned long long q2[4][16];
    float w[8];
    int cur_b = -1;
    const int g = lane >> 3, j = lane & 7;
    uint32_t k = 0;
    for (long long item = first; item < last; ++item, ++k) {
        const uint32_t kn = k + kScoreStages - 1;   // the item whose copy starts now
        if ((kn & 31) == 0) {
            resolve32(kn);
            __syncwarp();
        }
        if (lane == 0) issue(kn);
        const int st = (int)(k % kScoreStages);
        if (!warp_wait(&sm.full[warp][st], (uint32_t)((k / kScoreStages) & 1), &sm.abort_flag, a.ws, item)) break;
        const ItemMeta m = sm.meta[warp][k % kMetaRing];
        if (m.blk >= 0) {
            if (m.b != cur_b) {
                cur_b = m.b;
#pragma unroll
                for (int s2 = 0; s2 < 4; ++s2) {
                    const int h0 = (2 * s2) ^ j, h1 = (2 * s2 + 1) ^ j;
                    const uint4 *r0 =
                        reinterpret_cast<const uint4 *>(a.iq + ((size_t)m.b * kIdxHeads + h0) * kIdxDim + 16 * j);
                    const uint4 *r1 =
                        reinterpret_cast<const uint4 *>(a.iq + ((size_t)m.b * kIdxHeads + h1) * kIdxDim + 16 * j);
                    const uint4 x0 = r0[0], x1 = r0[1], y0 = r1[0], y1 = r1[1];
                    const uint32_t xw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
                    const uint32_t yw[8] = {y0.x, y0.y, y0.z, y0.w, y1.x, y1.y, y1.z, y1.w};
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        q2[s2][2 * i] = f2_pack(bf16_lo(xw[i]), bf16_lo(yw[i]));
                        q2[s2][2 * i + 1] = f2_pack(bf16_hi(xw[i]), bf16_hi(yw[i]));
                    }
                }
#pragma unroll
                for (int h = 0; h < 8; ++h) w[h] = a.iw[(size_t)m.b * kIdxHeads + h];
            }
            const uint8_t *sp = sm.stage[warp][st];
            const uint4 kr0 = *reinterpret_cast<const uint4 *>(sp + g * kIdxDim + 16 * j);
            const uint4 kr1 = *reinterpret_cast<const uint4 *>(sp + (4 + g) * kIdxDim + 16 * j);
            const float s0 = score_key(QRegs{q2}, w, kr0, lane);
            const float s1 = score_key(QRegs{q2}, w, kr1, lane);
            float best = -INFINITY;
            if (m.blk * kBlock + g < m.L) best = fmaxf(best, s0);   // a NaN score never wins
            if (m.blk * kBlock + 4 + g < m.L) best = fmaxf(best, s1);
            best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 8));
            best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
            if (lane == 0) a.scores[(size_t)m.b * a.score_stride + m.v] = best;
        } else if (m.blk == kBlkBad && lane == 0) {
            a.scores[(size_t)m.b * a.score_stride + m.v] = -INFINITY;
        }
        __syncwarp();
    }
    // no copy may still be landing in shared memory when the CTA exits: wait for every stage this
    // warp started (k counts the items consumed; issue() ran up to k + kScoreStages - 2)
    if (lane == 0) {
        for (uint32_t kk = k; kk < k + kScoreStages - 1; ++kk) {
            const long long item = first + kk;
            if (item >= last) break;
            volatile int no_abort = 0;
            mbar_wait(&sm.full[warp][kk % kScoreStages], (uint32_t)((kk / kScoreStages) & 1), &no_abort, a.ws, -1);
        }
    }
    __syncwarp();
}

// ------------------------------------------------------------------------------------------------
// Exact Top-K of one sequence's n candidate scores, one CTA per sequence.  Scores become order keys
// (a total order on floats); keys are cached in shared memory when they fit.  The bits that every
// key shares (the common prefix of the minimum and maximum key) are skipped; the rest are resolved
// MSB first in digits of up to 8 bits with per-warp shared-memory histograms, giving the exact k-th
// largest key T and the number need_eq of keys equal to T that belong to the set (the lowest-indexed
// ones).  A final pass over per-warp contiguous segments writes the chosen ids in index order.
// ------------------------------------------------------------------------------------------------
constexpr int kTopkThreads = 1024;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkCacheKeys = 16384;
constexpr int kTopkHistWords = kTopkWarps * 256;

__global__ void __launch_bounds__(kTopkThreads, 1) topk_kernel(const float *__restrict__ scores, int score_stride,
                                                               const int32_t *__restrict__ seq_len, int max_seq_len,
                                                               const int32_t *__restrict__ pool,
                                                               const int32_t *__restrict__ pool_count, int pool_cap,
                                                               int k, int32_t *__restrict__ out_blocks,
                                                               int32_t *__restrict__ out_count, void *ws)
{
    extern __shared__ uint32_t tk_smem[];
    uint32_t *whist = tk_smem;                    // [32 warps][256]
    uint32_t *skeys = tk_smem + kTopkHistWords;   // cached keys
    __shared__ uint32_t scratch[40];
    __shared__ uint32_t wcount[2][kTopkWarps];
    __shared__ uint32_t sel[2];
    const int b = blockIdx.x, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    // the next kernel (the attention) may start its own preparation while the selection runs; the
    // scores are read only once the previous grid (the block scorer) has finished
    grid_dep_launch();
    grid_dep_wait();
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
    uint32_t T, need_eq;
    radix_select<kTopkThreads>(n, (uint32_t)k, [&](int i) { return cached ? skeys[i] : order_key(sc[i]); }, 0, whist,
                               scratch, sel, T, need_eq);

    // per-warp contiguous segments: counts, then ordered writes
    const int seg = (n + kTopkWarps - 1) / kTopkWarps;
    const int s0 = warp * seg, s1 = min(n, s0 + seg);
    uint32_t gt_cnt = 0, eq_cnt = 0;
    for (int base = s0; base < s1; base += 32) {
        const int i = base + lane;
        uint32_t u = 0;
        if (i < s1) u = cached ? skeys[i] : order_key(sc[i]);
        gt_cnt += __popc(__ballot_sync(0xffffffffu, i < s1 && u > T));
        eq_cnt += __popc(__ballot_sync(0xffffffffu, i < s1 && u == T));
    }
    if (lane == 0) {
        wcount[0][warp] = gt_cnt;
        wcount[1][warp] = eq_cnt;
    }
    __syncthreads();
    uint32_t gt_run = 0, eq_run = 0;
    for (int wi = 0; wi < warp; ++wi) {
        gt_run += wcount[0][wi];
        eq_run += wcount[1][wi];
    }
    const uint32_t lt_mask = (1u << lane) - 1u;
    for (int base = s0; base < s1; base += 32) {
        const int i = base + lane;
        uint32_t u = 0;
        if (i < s1) u = cached ? skeys[i] : order_key(sc[i]);
        const bool gt = i < s1 && u > T, eq = i < s1 && u == T;
        const uint32_t bg = __ballot_sync(0xffffffffu, gt), be = __ballot_sync(0xffffffffu, eq);
        const uint32_t gt_b = gt_run + __popc(bg & lt_mask), eq_b = eq_run + __popc(be & lt_mask);
        if (gt || (eq && eq_b < need_eq)) out[gt_b + min(eq_b, need_eq)] = ids ? ids[i] : i;
        gt_run += __popc(bg);
        eq_run += __popc(be);
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
    // the next kernel (the layer's attention) may start its own preparation while this copy runs;
    // the previous layer's set is read only once the previous grid has finished
    grid_dep_launch();
    grid_dep_wait();
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
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(block_score_kernel), smem);
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
    a.items_per_seq = pool ? (pool_cap + kScoreWarps - 1) / kScoreWarps
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
    const size_t smem =
        (size_t)kTopkHistWords * 4 + (size_t)(max_candidates < kTopkCacheKeys ? max_candidates : kTopkCacheKeys) * 4;
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(topk_kernel), smem);
    if (e != cudaSuccess) return e;
    return launch_overlapped(topk_kernel, dim3(B), dim3(kTopkThreads), smem, st, scores, score_stride, seq_len,
                             max_seq_len, pool, pool_count, pool_cap, k, out_blocks, out_count, ws);
}

cudaError_t launch_reuse(int B, const int32_t *prev, const int32_t *prev_count, int prev_cap, int32_t *out,
                         int32_t *out_count, int out_cap, void *ws, cudaStream_t st)
{
    return launch_overlapped(reuse_kernel, dim3(B), dim3(256), 0, st, prev, prev_count, prev_cap, out, out_count,
                             out_cap, ws);
}

}  // namespace csa
