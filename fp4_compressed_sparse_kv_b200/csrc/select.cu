// select.cu -- the Full indexer's selection after the tensor-core screen: from every block's bounds
// [lower, upper] of its exact score, the exact Top-k blocks of each sequence, in one launch.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": a Full
// layer keeps the Top-K blocks of 8 positions over the whole context (ties toward the lower block).
// The screen (screen.cu) bounds every block's exact score; with T <= the k-th largest lower bound
// and U >= the (k+1)-th largest upper bound a block is
//   out        if upper < T: k blocks have lower >= T, so k scores are >= T, above this one's;
//   sure       if lower > U: only blocks with upper > U, at most k of them and this block among
//              them, can reach its score, so it is in the Top-K whatever the ties;
//   uncertain  otherwise: scored exactly here, and the best k - #sure of them taken.
// The k-th largest lower-bound key X is located to 24 bits: its top 12 bits from the screen's
// per-sequence histogram, the next 12 from a second histogram of the keys in that bin.  T = X with
// the last 8 bits clear; U = (X with them set) + the widest interval of the sequence, rounded up: a
// block with upper > U has lower > X, and fewer than k blocks do.  If some bound of the sequence is
// not finite, U is the largest key and no block is sure.
//
// One cluster of 8 CTAs per sequence (16 for batches of up to 18 sequences), CTA c owning a
// contiguous chunk of its blocks (thread t: 8 consecutive blocks per round of 2,048).  The cluster's
// hardware barrier orders the steps; partial results are exchanged through distributed shared
// memory, the second histogram through global memory.  Every wait is a cluster barrier, which all
// CTAs of the cluster reach on every path (every branch below depends only on per-sequence values),
// so no wait can be left open.
//   1. second histogram and the widest interval over the chunk;            barrier
//   2. T and U; classify the chunk into class bytes, the uncertain blocks listed in block order
//      with their pages; score them exactly (the binary32 chain of csa.h);  barrier
//   3. the k - #sure best uncertain blocks of the sequence (by exact score, then lower block id),
//      each CTA marking its own: ranked by counting against the whole list when there are few, else
//      radix-selected over the cluster;                                    barrier
//   4. the sure and chosen blocks of each chunk written in ascending order at the chunk's offset.
#include <atomic>

#include <cooperative_groups.h>

#include "common.cuh"
#include "convert.cuh"
#include "pipeline.cuh"
#include "radix.cuh"
#include "score.cuh"

namespace cg = cooperative_groups;

namespace csa {

constexpr int kSelThreads = 256;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelPer = 8;               // consecutive blocks per thread in one round
constexpr int kSelRound = kSelThreads * kSelPer;   // blocks per round
constexpr int kSelListCap = 1024;        // uncertain blocks of one CTA kept in shared memory
constexpr int kSelRankCap = 1024;        // up to this many uncertain blocks in a sequence: rank them
constexpr int kSelStatCap = 16384;       // class bytes of a chunk staged in shared memory up to this
constexpr uint8_t kOut = 0, kSure = 1, kUncertain = 2, kChosen = 3;
static_assert(kSelRankCap <= kSelListCap, "the rank path reads every CTA's list from shared memory");

struct SelArgs {
    const float *lo;
    const float *hi;
    int lstride;                // row stride of lo and hi (blocks, a multiple of 4)
    const uint32_t *hist;       // [B][kHistBins]: top 12 bits of the lower-bound keys (the screen)
    uint32_t *hist2;            // [B][kHistBins], zero on entry
    uint8_t *status;            // [B][sstride]: class bytes of chunks too long for shared memory
    int sstride;
    int32_t *uslice;            // [B][ustride]: uncertain blocks beyond a CTA's shared-memory list
    uint32_t *okeys;            //   and their exact-score order keys
    int ustride;
    const int32_t *seq_len;
    int max_seq_len;
    const int32_t *block_table;
    int max_pages;
    const uint8_t *keys;
    int num_pages;
    const uint16_t *iq;
    const float *iw;
    int k;
    int32_t *out_blocks;
    int32_t *out_count;
    void *ws;
};

struct SelSmem {
    unsigned long long qs[8 * kQRowPairs];   // the sequence's query pairs (score.cuh)
    uint32_t ukey[kSelListCap];              // this CTA's uncertain blocks in block order: score keys
    int32_t uid[kSelListCap];                //   block ids
    int32_t upage[kSelListCap];              //   and their pages
    uint32_t gkey[kSelRankCap];              // the sequence's uncertain blocks (rank path)
    int32_t gid[kSelRankCap];
    alignas(16) uint8_t sstat[kSelStatCap];  // class bytes of the chunk
    int32_t cpage[kSelRound / kBlocksPerPage];   // pages of the chunk's first round
    uint32_t rhist[2][256];                  // radix digits of this CTA's keys (read by the cluster)
    uint32_t scratch[40];
    uint32_t wkey;                           // this CTA's widest interval (read by the cluster)
    uint32_t n_sure, n_unc, n_tie, n_take;   // this CTA's counts (read by the cluster)
    uint32_t n_chosen;
    uint32_t sel[2];
};

// Over a kHistBins-bin histogram h (read from L2: other CTAs of the cluster add to it): the bin
// holding the rank-th largest element (1-based) and that element's rank inside the bin; every
// thread gets both.  If the counts fall short of rank: bin 0 (a threshold that keeps everything).
// Thread t reads its 16 bins kHistBins - 16 (t + 1) .. kHistBins - 16 t - 1 with 16-byte loads.
__device__ __forceinline__ void rank_bin(const uint32_t *h, uint32_t rank, uint32_t *scratch, int *bin_out,
                                         uint32_t *rank_out)
{
    constexpr int kPer = kHistBins / kSelThreads;
    static_assert(kPer == 16, "four 16-byte loads per thread");
    const int t = threadIdx.x;
    const int lo_bin = kHistBins - kPer * (t + 1);
    uint32_t v[kPer];
#pragma unroll
    for (int m = 0; m < 4; ++m) {
        const uint4 q = __ldcg(reinterpret_cast<const uint4 *>(h + lo_bin) + m);
        v[4 * m] = q.x;
        v[4 * m + 1] = q.y;
        v[4 * m + 2] = q.z;
        v[4 * m + 3] = q.w;
    }
    uint32_t s = 0;
#pragma unroll
    for (int i = 0; i < kPer; ++i) s += v[i];
    if (t == 0) {
        scratch[33] = 0u;
        scratch[34] = 1u;
    }
    uint32_t total;
    uint32_t run = cta_scan(s, scratch, total);   // elements in larger bins than this thread's
    if (run < rank && rank <= run + s) {
#pragma unroll
        for (int i = kPer - 1; i >= 0; --i) {   // largest bin first
            if (run < rank && rank <= run + v[i]) {
                scratch[33] = (uint32_t)(lo_bin + i);
                scratch[34] = rank - run;
            }
            run += v[i];
        }
    }
    __syncthreads();
    *bin_out = (int)scratch[33];
    *rank_out = scratch[34];
    __syncthreads();
}

// Split cluster barrier: arrive (no memory ordering) ... wait.
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// The 8 values p[i .. i+8) (i a multiple of 8 from a 16-byte aligned row), -inf past `end`.
__device__ __forceinline__ void load8(const float *p, int i, int end, float (&v)[8])
{
    if (i + 8 <= end) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p + i));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(p + i) + 1);
        v[0] = a.x, v[1] = a.y, v[2] = a.z, v[3] = a.w, v[4] = b.x, v[5] = b.y, v[6] = b.z, v[7] = b.w;
    } else {
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = i + q < end ? __ldg(p + i + q) : -INFINITY;
    }
}

template <int kSelCtas>
__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(const SelArgs a)
{
    __shared__ SelSmem sm;
    cg::cluster_group cluster = cg::this_cluster();
    const int c = (int)cluster.block_rank();
    const int b = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;

    // the query does not come from the screen: load it before waiting for the screen's results
    load_query_pairs(a.iq + (size_t)b * kIdxHeads * kIdxDim, sm.qs);
    float w[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) w[h] = a.iw[(size_t)b * kIdxHeads + h];
    grid_dep_wait();
    grid_dep_launch();   // the attention may be scheduled meanwhile

    const int L = a.seq_len[b];
    int32_t *out = a.out_blocks + (size_t)b * a.k;
    if (L < 1 || L > a.max_seq_len) {   // the same for every CTA of the cluster: no barrier is left open
        if (c == 0 && t == 0) {
            a.out_count[b] = 0;
            report(a.ws, CSA_ERR_DEVICE_DATA, b);
        }
        return;
    }
    const int n = (L + kBlock - 1) / kBlock;
    if (n <= a.k) {   // every block is selected
        for (int i = c * kSelThreads + t; i < n; i += kSelCtas * kSelThreads) out[i] = i;
        if (c == 0 && t == 0) a.out_count[b] = n;
        return;
    }
    // chunk [i0, i1) of this CTA: a multiple of 16 blocks; thread t takes 8 consecutive blocks of
    // each round of 2,048
    const int per = (((n + kSelCtas - 1) / kSelCtas) + 15) & ~15;
    const int i0 = min(n, c * per), i1 = min(n, i0 + per);
    const int rounds = (i1 - i0 + kSelRound - 1) / kSelRound;
    const float *lp = a.lo + (size_t)b * a.lstride;
    const float *hp = a.hi + (size_t)b * a.lstride;
    const bool staged = per <= kSelStatCap;
    uint8_t *st8 = staged ? sm.sstat - i0 : a.status + (size_t)b * a.sstride;   // indexed by block id
    uint32_t *h2 = a.hist2 + (size_t)b * kHistBins;
    int32_t *us = a.uslice + (size_t)b * a.ustride;
    uint32_t *ok = a.okeys + (size_t)b * a.ustride;
    const int32_t *btab = a.block_table + (size_t)b * a.max_pages;

    // ---- 1. second histogram (keys in the k-th lower bound's first-level bin) and widest interval
    float l8[8], h8[8];
    load8(lp, i0 + kSelPer * t, i1, l8);   // round 0, in flight during the first rank_bin
    load8(hp, i0 + kSelPer * t, i1, h8);
    static_assert(kSelRound / kBlocksPerPage == kSelThreads, "one page of round 0 per thread");
    if (i0 + kBlocksPerPage * t < i1) sm.cpage[t] = btab[i0 / kBlocksPerPage + t];   // (i0: whole pages)
    int bin1;
    uint32_t r1;
    rank_bin(a.hist + (size_t)b * kHistBins, (uint32_t)a.k, sm.scratch, &bin1, &r1);
    uint32_t wkey = 0u;   // order key of the widest interval (+inf when a bound is not finite)
    for (int r = 0; r < rounds; ++r) {
        const int i = i0 + r * kSelRound + kSelPer * t;
        if (r > 0) {
            load8(lp, i, i1, l8);
            load8(hp, i, i1, h8);
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (i + q < i1) {
                const float wd = __fsub_ru(h8[q], l8[q]);
                wkey = max(wkey, wd == wd ? order_key(wd) : 0xFF800000u);
                const uint32_t kl = order_key(l8[q]);
                if ((int)(kl >> 20) == bin1) atomicAdd(&h2[(kl >> 8) & (kHistBins - 1)], 1u);
            }
        }
    }
    wkey = block_reduce_minmax(wkey, true, sm.scratch);
    if (t == 0) sm.wkey = wkey;
    cluster.sync();

    // ---- 2. thresholds, classification, exact scores of the uncertain blocks
    {
        uint32_t wk[kSelCtas];
#pragma unroll
        for (int r = 0; r < kSelCtas; ++r) wk[r] = *cluster.map_shared_rank(&sm.wkey, r);
#pragma unroll
        for (int r = 0; r < kSelCtas; ++r) wkey = max(wkey, wk[r]);
    }
    int bin2;
    uint32_t r2;
    rank_bin(h2, r1, sm.scratch, &bin2, &r2);
    const uint32_t T = ((uint32_t)bin1 << 20) | ((uint32_t)bin2 << 8);
    const uint32_t U = wkey >= 0xFF800000u ? 0xFFFFFFFFu : order_key(__fadd_ru(key_to_float(T | 0xFFu), key_to_float(wkey)));
    uint32_t n_sure = 0, nu = 0;
    for (int r = 0; r < rounds; ++r) {
        const int i = i0 + r * kSelRound + kSelPer * t;
        load8(lp, i, i1, l8);   // (from L1: read in step 1)
        load8(hp, i, i1, h8);
        uint32_t cls[2] = {0u, 0u}, mine = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            uint32_t cl = kOut;
            if (i + q < i1) {
                const uint32_t hk = order_key(h8[q]), lk = order_key(l8[q]);
                cl = hk < T ? kOut : (lk > U ? kSure : kUncertain);
            }
            cls[q >> 2] |= cl << (8 * (q & 3));
            n_sure += cl == kSure;
            mine += cl == kUncertain;
        }
        if (i < i1) *reinterpret_cast<uint2 *>(st8 + i) = make_uint2(cls[0], cls[1]);
        uint32_t total;
        uint32_t pos = nu + cta_scan(mine, sm.scratch, total);
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            if (((cls[q >> 2] >> (8 * (q & 3))) & 0xFFu) == kUncertain) {
                const int blk = i + q;
                if (pos < (uint32_t)kSelListCap) {
                    sm.uid[pos] = blk;
                    sm.upage[pos] = r == 0 ? sm.cpage[(blk - i0) / kBlocksPerPage] : btab[blk / kBlocksPerPage];
                } else {
                    us[i0 + pos] = blk;
                }
                ++pos;
            }
        }
        nu += total;
    }
    __syncthreads();
    // warp u % 8 scores uncertain block u: 8 positions, lane (g, j) keys g and 4 + g, dims 16j..;
    // the keys of two blocks are in flight at once
    const int g = lane >> 3, j = lane & 7;
    const QSmem q2{sm.qs + j * kQRowPairs};
    for (uint32_t u0 = warp; u0 < nu; u0 += 2 * kSelWarps) {
        uint4 kr[2][2];
        int blk[2];
        bool good[2];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const uint32_t u = u0 + m * kSelWarps;
            blk[m] = -1;
            good[m] = false;
            if (u < nu) {
                int page;
                if (u < (uint32_t)kSelListCap) {
                    blk[m] = sm.uid[u];
                    page = sm.upage[u];
                } else {
                    blk[m] = __ldcg(us + i0 + u);
                    page = btab[blk[m] / kBlocksPerPage];
                }
                good[m] = page >= 0 && page < a.num_pages;
                if (good[m]) {
                    const uint8_t *src =
                        a.keys + ((size_t)page * kPage + (size_t)(blk[m] % kBlocksPerPage) * kBlock) * kIdxDim;
                    kr[m][0] = __ldg(reinterpret_cast<const uint4 *>(src + g * kIdxDim + 16 * j));
                    kr[m][1] = __ldg(reinterpret_cast<const uint4 *>(src + (4 + g) * kIdxDim + 16 * j));
                } else if (lane == 0) {
                    report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b * a.max_pages + blk[m] / kBlocksPerPage);
                }
            }
        }
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const uint32_t u = u0 + m * kSelWarps;
            if (u >= nu) break;
            float best = -INFINITY;
            if (good[m]) {
                const float s0 = score_key(q2, w, kr[m][0], lane);
                const float s1 = score_key(q2, w, kr[m][1], lane);
                if (blk[m] * kBlock + g < L) best = fmaxf(best, s0);   // a NaN score never wins
                if (blk[m] * kBlock + 4 + g < L) best = fmaxf(best, s1);
            }
            best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 8));
            best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
            if (lane == 0) {
                if (u < (uint32_t)kSelListCap) sm.ukey[u] = order_key(best);
                else ok[i0 + u] = order_key(best);
            }
        }
    }
    n_sure = block_reduce_sum(n_sure, sm.scratch);   // (its barriers also publish ukey)
    if (t == 0) {
        sm.n_sure = n_sure;
        sm.n_unc = nu;
        sm.n_chosen = 0;
    }
    cluster.sync();

    // ---- 3. the kk best uncertain blocks of the sequence; each CTA marks its own
    uint32_t N_sure = 0, NU = 0, nu_r[kSelCtas], ns_r[kSelCtas];
#pragma unroll
    for (int r = 0; r < kSelCtas; ++r) {
        ns_r[r] = *cluster.map_shared_rank(&sm.n_sure, r);
        nu_r[r] = *cluster.map_shared_rank(&sm.n_unc, r);
    }
#pragma unroll
    for (int r = 0; r < kSelCtas; ++r) {
        N_sure += ns_r[r];
        NU += nu_r[r];
    }
    const bool consistent = N_sure <= (uint32_t)a.k && (uint32_t)a.k - N_sure <= NU;
    const uint32_t kk = consistent ? (uint32_t)a.k - N_sure : 0u;
    auto own_key = [&](uint32_t e) { return e < (uint32_t)kSelListCap ? sm.ukey[e] : __ldcg(ok + i0 + e); };
    auto own_id = [&](uint32_t e) { return e < (uint32_t)kSelListCap ? sm.uid[e] : __ldcg(us + i0 + e); };
    uint32_t n_chosen = 0;
    if (!consistent) {
        if (c == 0 && t == 0) report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b);
    } else if (kk == NU) {   // every uncertain block
        for (uint32_t e = t; e < nu; e += kSelThreads) st8[own_id(e)] = kChosen;
        n_chosen = nu;
    } else if (kk > 0 && NU <= (uint32_t)kSelRankCap) {
        // gather the sequence's list (block order), then rank this CTA's blocks by counting
        for (uint32_t e = t; e < NU; e += kSelThreads) {
            int r = 0;
            uint32_t off = 0, acc = 0;
#pragma unroll
            for (int q = 0; q < kSelCtas - 1; ++q) {
                acc += nu_r[q];
                if (e >= acc) {
                    r = q + 1;
                    off = acc;
                }
            }
            sm.gkey[e] = cluster.map_shared_rank(sm.ukey, r)[e - off];
            sm.gid[e] = cluster.map_shared_rank(sm.uid, r)[e - off];
        }
        __syncthreads();
        uint32_t mine = 0;
        for (uint32_t e = warp; e < nu; e += kSelWarps) {
            const uint32_t x = sm.ukey[e];
            const int id = sm.uid[e];
            uint32_t rank = 0;
            for (uint32_t f = lane; f < NU; f += 32) {
                const uint32_t y = sm.gkey[f];
                rank += (y > x) || (y == x && sm.gid[f] < id);
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
            if (lane == 0 && rank < kk) {
                st8[id] = kChosen;
                ++mine;
            }
        }
        if (lane == 0 && mine) atomicAdd(&sm.n_chosen, mine);
        __syncthreads();
        n_chosen = sm.n_chosen;
    } else if (kk > 0) {
        // radix selection of the kk-th largest key over the cluster, 8 bits per round, MSB first
        uint32_t prefix = 0, pmask = 0, want = kk;
        for (int round = 0; round < 4; ++round) {
            const int shift = 24 - 8 * round;
            uint32_t *hb = sm.rhist[round & 1];
            hb[t] = 0u;
            __syncthreads();
            for (uint32_t e = t; e < nu; e += kSelThreads) {
                const uint32_t x = own_key(e);
                if ((x & pmask) == prefix) atomicAdd(&hb[(x >> shift) & 255u], 1u);
            }
            cluster.sync();
            const int d = 255 - t;   // thread t: digit 255 - t, largest first
            uint32_t cr[kSelCtas];
#pragma unroll
            for (int r = 0; r < kSelCtas; ++r) cr[r] = cluster.map_shared_rank(hb, r)[d];
            uint32_t cnt = 0;
#pragma unroll
            for (int r = 0; r < kSelCtas; ++r) cnt += cr[r];
            uint32_t total;
            const uint32_t excl = cta_scan(cnt, sm.scratch, total);
            if (excl < want && want <= excl + cnt) {
                sm.sel[0] = (uint32_t)d;
                sm.sel[1] = excl;
            }
            __syncthreads();
            prefix |= sm.sel[0] << shift;
            pmask |= 255u << shift;
            want -= sm.sel[1];
            __syncthreads();
        }
        // keys above the threshold are chosen; of the keys equal to it, the want lowest block ids
        // (the CTAs' lists are in block order and the chunks ascend with the CTA rank)
        uint32_t n_tie = 0, above = 0;
        for (uint32_t e = t; e < nu; e += kSelThreads) {
            const uint32_t x = own_key(e);
            if (x > prefix) {
                st8[own_id(e)] = kChosen;
                ++above;
            }
            n_tie += x == prefix;
        }
        n_tie = block_reduce_sum(n_tie, sm.scratch);
        above = block_reduce_sum(above, sm.scratch);
        if (t == 0) sm.n_tie = n_tie;
        cluster.sync();
        uint32_t tie_base = 0;
        for (int r = 0; r < c; ++r) tie_base += *cluster.map_shared_rank(&sm.n_tie, r);
        uint32_t seen = 0, taken_ties = 0;
        for (uint32_t e0 = 0; e0 < nu; e0 += kSelThreads) {
            const uint32_t e = e0 + t;
            const bool tie = e < nu && own_key(e) == prefix;
            uint32_t total;
            const uint32_t r = seen + cta_scan(tie ? 1u : 0u, sm.scratch, total);
            if (tie && tie_base + r < want) {
                st8[own_id(e)] = kChosen;
                ++taken_ties;
            }
            seen += total;
        }
        n_chosen = above + block_reduce_sum(taken_ties, sm.scratch);
    }
    // blocks this CTA contributes; after reading every CTA's count a CTA only signals the final
    // barrier, writes its part of the result and then waits there (its shared memory must outlive
    // the others' reads)
    if (t == 0) sm.n_take = consistent ? n_sure + n_chosen : 0u;
    cluster.sync();

    // ---- 4. ordered output: the sure and chosen blocks of the chunk at the chunk's offset
    uint32_t cbase = 0, all = 0;
    {
        uint32_t tk[kSelCtas];
#pragma unroll
        for (int r = 0; r < kSelCtas; ++r) tk[r] = *cluster.map_shared_rank(&sm.n_take, r);
#pragma unroll
        for (int r = 0; r < kSelCtas; ++r) {
            cbase += r < c ? tk[r] : 0u;
            all += tk[r];
        }
    }
    cluster_arrive_relaxed();
    if (consistent) {
        uint32_t pos = cbase;
        for (int r = 0; r < rounds; ++r) {
            const int i = i0 + r * kSelRound + kSelPer * t;
            uint2 v = make_uint2(0u, 0u);
            if (i < i1) v = *reinterpret_cast<const uint2 *>(st8 + i);
            const uint32_t cls[2] = {v.x, v.y};
            uint32_t mine = 0;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t x = (cls[q >> 2] >> (8 * (q & 3))) & 0xFFu;
                mine += (i + q < i1) && (x == kSure || x == kChosen);
            }
            uint32_t total;
            uint32_t p = pos + cta_scan(mine, sm.scratch, total);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const uint32_t x = (cls[q >> 2] >> (8 * (q & 3))) & 0xFFu;
                if ((i + q < i1) && (x == kSure || x == kChosen)) {
                    if (p < (uint32_t)a.k) out[p] = i + q;
                    ++p;
                }
            }
            pos += total;
        }
    }
    if (c == 0 && t == 0) {
        a.out_count[b] = consistent ? a.k : 0;
        if (consistent && all != (uint32_t)a.k) report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b);
    }
    cluster_wait();
}

// Launch kernel16 with 16-CTA clusters (non-portable) when the batch is small enough for them to fill
// at most two CTAs per SM and the device can place one, kernel8 with 8-CTA clusters otherwise; grid
// (cluster size, B), programmatic dependent launch.
template <typename Args>
cudaError_t launch_clusters(void (*kernel16)(Args), void (*kernel8)(Args), int B, cudaStream_t st, const Args &a)
{
    static std::atomic<int> cap16[64];   // per device: 0 unknown, 1 yes, 2 no
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    int nsm = 0;
    if ((e = cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    bool use16 = false;
    if (B * 16 <= 2 * nsm && dev >= 0 && dev < 64) {
        if (cap16[dev].load() == 0) {   // first use on this device (concurrent callers may both query)
            int ok = 0;
            if (cudaFuncSetAttribute(kernel16, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess) {
                cudaLaunchConfig_t q = {};
                q.gridDim = dim3(16, 1);
                q.blockDim = dim3(kSelThreads);
                cudaLaunchAttribute qa[1];
                qa[0].id = cudaLaunchAttributeClusterDimension;
                qa[0].val.clusterDim.x = 16;
                qa[0].val.clusterDim.y = 1;
                qa[0].val.clusterDim.z = 1;
                q.attrs = qa;
                q.numAttrs = 1;
                int n = 0;
                ok = cudaOccupancyMaxActiveClusters(&n, kernel16, &q) == cudaSuccess && n >= 1;
            }
            cudaGetLastError();
            cap16[dev].store(ok ? 1 : 2);
        }
        use16 = cap16[dev].load() == 1;
    }
    const int nc = use16 ? 16 : 8;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nc, B);
    cfg.blockDim = dim3(kSelThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = nc;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return use16 ? cudaLaunchKernelEx(&cfg, kernel16, a) : cudaLaunchKernelEx(&cfg, kernel8, a);
}

cudaError_t launch_select(const float *lo, const float *hi, int lstride, const csa_batch &bt, int k,
                          const uint32_t *hist, uint32_t *hist2, uint8_t *status, int sstride, int32_t *uslice,
                          uint32_t *okeys, int ustride, const uint8_t *keys, int num_pages,
                          const uint16_t *iq, const float *iw, int32_t *out_blocks, int32_t *out_count, void *ws,
                          cudaStream_t st)
{
    SelArgs a;
    a.lo = lo;
    a.hi = hi;
    a.lstride = lstride;
    a.hist = hist;
    a.hist2 = hist2;
    a.status = status;
    a.sstride = sstride;
    a.uslice = uslice;
    a.okeys = okeys;
    a.ustride = ustride;
    a.seq_len = bt.seq_len;
    a.max_seq_len = bt.max_seq_len;
    a.block_table = bt.block_table;
    a.max_pages = bt.max_pages;
    a.keys = keys;
    a.num_pages = num_pages;
    a.iq = iq;
    a.iw = iw;
    a.k = k;
    a.out_blocks = out_blocks;
    a.out_count = out_count;
    a.ws = ws;
    return launch_clusters(select_kernel<16>, select_kernel<8>, bt.B, st, a);
}

}  // namespace csa
