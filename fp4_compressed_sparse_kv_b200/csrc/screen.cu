// screen.cu -- the Full-layer indexer's tensor-core screening: per-block bounds of the exact score,
// and from them the candidate blocks that must be scored exactly.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": a Full
// layer selects its Top-K blocks of 8 positions over the whole context, so its scan reads every
// indexer key.  The exact score (csa.h) is a fixed binary32 FMA chain on CUDA cores; here every
// position is first scored approximately on the tensor cores, at the speed of reading the keys, with
// a rigorous bound eps on the distance to the exact score.  The exact Top-K lies among the blocks
// whose upper bound reaches the k-th largest lower bound; only those are scored exactly
// (csa_indexer_full), so the result is identical to the exhaustive exact scan.
//
//  1. qterm_kernel: per sequence and head, q_h * 2^s (largest |q| in [128, 256)) is split into three
//     E4M3 terms t1 + t2 + t3 plus a residual delta, and written as the tensor-core B operand.
//  2. screen_kernel: D_i = t_i . k for all positions from tcgen05 MMAs (kind::f8f6f4, E4M3 x E4M3,
//     fp32 accumulation in TMEM) on key tiles brought in by TMA; the epilogue forms the approximate
//     head values d^_h = ((D_1 + D_2) + D_3) 2^-s, the approximate score t^ = the same weighted ReLU
//     chain as the exact score, the bound eps_p, then per block the largest lower and upper bound,
//     and a per-sequence histogram of the lower bounds.
//  3. (select.cu) from the bounds, the blocks sure to be in the Top-K, those that cannot be, and the
//     uncertain rest, which are scored exactly; the sure blocks plus the best uncertain ones, in
//     ascending block order.

// The bound, with u = 2^-24, gamma_n = n u / (1 - n u), kmax_p the position's largest |key|:
//  * exact chain: 16-term FMA chains then a 3-level tree; every product bf16 x E4M3 is exact in
//    binary32, so |d_h - q_h . k| <= gamma_19 sum_d |q_d k_d| <= gamma_19 kmax Q1_h (Q1_h = sum |q_d|);
//  * screen: the tensor core's fp32 accumulation is taken to err by at most kTcRel times the sum of
//    the magnitudes of its (exact) products -- measured on B200 below 2^-25 for E4M3, taken as 2^-14;
//    then two binary32 adds and an exact power-of-two scale:
//    |d^_h - q_h . k| <= kmax ((kTcRel + gamma_2 (1 + kTcRel)) T1_h + Delta_h), with T1_h the sum of
//    all |t_i,d| 2^-s and Delta_h = sum |delta_d| 2^-s;
//  * so |d^_h - d_h| <= kmax F_h, F_h = (kTcRel + gamma_2 (1 + kTcRel)) T1_h + Delta_h + gamma_19 Q1_h;
//    ReLU is 1-Lipschitz and both weighted chains carry gamma_8 relative error, which gives
//    |score - t^| <= kmax (1 + gamma_8) sum_h |w_h| F_h + 2 gamma_8 (1 + gamma_8) sum_h |w_h| relu(d^_h);
//  * underflow adds at most a few 2^-150 per operation: an absolute slack 2^-100 (1 + sum |w|) covers
//    it; positions where any partial sum could come near overflow (kmax Q1 sum|w| >= 1e37) and
//    non-finite values get no bound (lower = -NaN, upper = +NaN: the two ends of the Top-K order).
// All constants are formed in double and rounded up by a relative 1e-6; the per-position sums use
// round-up arithmetic.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "convert.cuh"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace csa {

constexpr int kScrRows = 128;                             // positions per tile: two pages
constexpr int kScrN = 32;                                 // MMA N: 3 terms x 8 heads + 8 zero rows
constexpr int kScrStages = 9;
constexpr int kScrEpiGroups = 2;                          // epilogue groups, taking tiles in turn
constexpr int kScrAcc = 6;                                // TMEM accumulators (a multiple of the groups)
constexpr int kScrTmemCols = 256;                         // >= 32 * kScrAcc, a power of two
constexpr int kScrMaxGroups = 2;                          // row-max groups, taking tiles in turn
constexpr int kScrThreads = 64 + 128 * kScrMaxGroups + 128 * kScrEpiGroups;   // loader, MMA, row max, epilogues
constexpr int kScrEpiWarp0 = 2 + 4 * kScrMaxGroups;        // first epilogue warp
static_assert(kScrAcc % kScrEpiGroups == 0, "each accumulator belongs to one epilogue group");
static_assert(32 * kScrAcc <= kScrTmemCols, "accumulators must fit the TMEM allocation");
constexpr uint32_t kScrKeyBytes = kScrRows * kIdxDim;     // 16 KB
constexpr uint32_t kScrPageBytes = kPage * kIdxDim;       // 8 KB
constexpr uint32_t kScrQtBytes = (uint32_t)kQtBytes;      // 4 KB
constexpr int kScrRing = 64;                              // resolved-item ring (>= 32 + stages)
constexpr double kTcRel = 6.103515625e-05;                // 2^-14
constexpr double kU = 5.9604644775390625e-08;             // 2^-24
constexpr double kRoundUp = 1.000001;

__host__ __device__ constexpr double gamma_n(int n) { return n * kU / (1.0 - n * kU); }

struct QMeta {
    float inv_scale[8];   // 2^-s_h
    float G;              // (1 + gamma_8) sum_h |w_h| F_h, rounded up
    float chain;          // 2 gamma_8 (1 + gamma_8), rounded up
    float absl;           // absolute slack
    float big;            // max_h Q1_h * max(1, sum |w|): overflow guard
    float pad[4];
};
static_assert(sizeof(QMeta) <= kQmBytes, "QMeta must fit its workspace slot");

// ------------------------------------------------------------------------------------------------
// Step 1: query terms.  One CTA per sequence, warp h = head h, lane l = dims 4l .. 4l+3.
// qt[b] holds the shared-memory image of a 32-row x 128-byte K-major operand in the 128-byte
// swizzle (row n at n*128, its 16-byte unit u at position u ^ (n & 7)): row 8i + h is term i of head
// h, rows 24..31 are zero.  A plain copy into a 1024-byte-aligned buffer gives the MMA's layout.
// ------------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) qterm_kernel(const uint16_t *__restrict__ iq, const float *__restrict__ iw,
                                                    uint8_t *__restrict__ qt, QMeta *__restrict__ qm,
                                                    uint32_t *__restrict__ hist, uint32_t *__restrict__ hist2)
{
    const int b = blockIdx.x, h = threadIdx.x >> 5, l = threadIdx.x & 31;
    // launched so that it may be scheduled while the stream's previous kernel (e.g. the pack of the
    // new tokens, whose keys the screen reads) finishes: wait for it, then let the screen start
    // streaming keys while the query terms are formed
    grid_dep_wait();
    grid_dep_launch();
    // the histograms the later steps accumulate into start from zero on every call
    for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
        hist[(size_t)b * kHistBins + i] = 0u;
        if (hist2) hist2[(size_t)b * kHistBins + i] = 0u;
    }
    const uint2 raw = reinterpret_cast<const uint2 *>(iq + ((size_t)b * kIdxHeads + h) * kIdxDim)[l];
    const float q[4] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) amax = fmaxf(amax, fabsf(q[i]));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    int s = 0;
    if (amax > 0.f && amax <= 3.0e38f) {
        int e;
        frexpf(amax, &e);   // amax in [2^(e-1), 2^e)
        s = 8 - e;          // scaled maximum in [128, 256)
    }
    uint32_t word[3] = {0u, 0u, 0u};
    double t1 = 0.0, dl = 0.0, q1 = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float r = ldexpf(q[i], s);
#pragma unroll
        for (int term = 0; term < 3; ++term) {
            const uint8_t c = (uint8_t)(f32x2_to_e4m3x2(r, 0.f) & 0xFF);
            const float cv = e4m3_to_f32(c);
            r = r - cv;   // exact: cv is r rounded to a coarser grid that r's own grid contains
            t1 += fabs((double)cv);
            word[term] |= (uint32_t)c << (8 * i);
        }
        dl += fabs((double)r);
        q1 += fabs((double)q[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        t1 += __shfl_xor_sync(0xffffffffu, t1, o);
        dl += __shfl_xor_sync(0xffffffffu, dl, o);
        q1 += __shfl_xor_sync(0xffffffffu, q1, o);
    }
    uint8_t *img = qt + (size_t)b * kScrQtBytes;
    const int d = 4 * l, unit = d >> 4, off = d & 15;
#pragma unroll
    for (int term = 0; term < 4; ++term) {
        const int n = term * 8 + h;
        *reinterpret_cast<uint32_t *>(img + n * 128 + ((unit ^ (n & 7)) << 4) + off) = term < 3 ? word[term] : 0u;
    }
    __shared__ double Fh[8], Q1h[8];
    if (l == 0) {
        const double inv = ldexp(1.0, -s);
        Fh[h] = (kTcRel + gamma_n(2) * (1.0 + kTcRel)) * (t1 * inv) + dl * inv + gamma_n(19) * q1;
        Q1h[h] = q1;
        qm[b].inv_scale[h] = ldexpf(1.f, -s);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        double G = 0.0, sw = 0.0, qmax = 0.0;
        for (int hh = 0; hh < 8; ++hh) {
            const double w = fabs((double)iw[(size_t)b * kIdxHeads + hh]);
            G += w * Fh[hh];
            sw += w;
            qmax = fmax(qmax, Q1h[hh]);
        }
        const double g8 = gamma_n(8);
        qm[b].G = (float)(G * (1.0 + g8) * kRoundUp);
        qm[b].chain = (float)(2.0 * g8 * (1.0 + g8) * kRoundUp);
        qm[b].absl = (float)(ldexp(1.0, -100) * (1.0 + sw) * 2.0);
        qm[b].big = (float)(qmax * fmax(1.0, sw) * 1.01);   // NaN or inf when inputs are: no bounds
    }
}

// ------------------------------------------------------------------------------------------------
// Step 2: screen.  Persistent CTAs (one per SM), each taking every grid-th 128-position tile (two
// pages) of the batch.  Warp 0 resolves tiles 32 at a time (one per lane) and issues the TMA loads of
// their two key pages plus, when the sequence changed since that stage's last use, the query-term
// image.  As soon as a stage lands, warp 1 issues the four K=32 MMAs of its tile into one of six
// 32-column TMEM accumulators and one of two row-max groups (warps 2-5, 6-9; thread = row) writes
// each row's largest |key| beside that accumulator; the stage is then free again (the MMA's commit
// and the 128 row-max threads release it), so nearly all stages stay in flight.  Two groups of four
// epilogue warps (thread = tile row = TMEM lane) take the tiles in turn (tile k: accumulator k mod 6,
// group k mod 2) and turn accumulator and row maxima into per-block bounds.
// ------------------------------------------------------------------------------------------------
struct ScreenArgs {
    const int32_t *seq_len;
    const int32_t *block_table;
    int max_pages;
    int max_seq_len;
    int B;
    int num_pages;
    int tiles_per_seq;
    long long total;      // B * tiles_per_seq
    const float *iw;
    const uint8_t *qt;
    const QMeta *qm;
    float *lo;
    float *hi;
    int stride;
    uint32_t *hist;   // [B][kHistBins]: count of blocks per top 12 bits of the lower-bound key
    void *ws;
};

struct ScrItem {
    int b, L, tile;
    int p0, p1;   // page ids of the tile's two pages (-1: none)
};

struct ScrSmem {
    uint8_t keys[kScrStages][kScrKeyBytes];
    uint8_t qt[kScrStages][kScrQtBytes];
    float kmax[kScrAcc][kScrRows];   // largest |key| of each row, beside its accumulator
    ScrItem ring[kScrRing];
    uint64_t full[kScrStages], sfree[kScrStages], dfull[kScrAcc], dfree[kScrAcc], mma_fin;
    int stage_b[kScrStages];
    uint32_t tmem;
    int abort_flag;
};

// kind::f8f6f4 instruction descriptor: D f32, A and B E4M3 (format 0), both K-major, M=128, N=32.
constexpr uint32_t kIdescScreen =
    (1u << 4) | ((uint32_t)(kScrN >> 3) << 17) | ((uint32_t)(kScrRows >> 4) << 24);

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate)
{
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Per 16-bit lane maximum of two words (sm_90+ SIMD integer max).
__device__ __forceinline__ uint32_t vmax_u16x2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Largest E4M3 magnitude code (bits 0-6) of a 128-byte key row in shared memory.  The row is in
// the 128-byte swizzle, so thread r reads its 16-byte units in the order u ^ (r & 7), which spreads
// the 8 threads of a quarter-warp over all 32 banks.  Magnitude codes order like the values they
// encode.  Odd bytes are the high bytes of the 16-bit lanes of the masked words; even bytes become
// high bytes after a shift by 8; a 16-bit max then keeps each high-byte maximum.
__device__ __forceinline__ uint32_t row_max_code(const uint8_t *row, int r)
{
    const uint4 *p = reinterpret_cast<const uint4 *>(row);
    uint32_t hi[8], lo[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {   // per 16-byte unit: a 2-level tree over its 4 words
        const uint4 v = p[u ^ (r & 7)];
        const uint32_t w0 = v.x & 0x7F7F7F7Fu, w1 = v.y & 0x7F7F7F7Fu, w2 = v.z & 0x7F7F7F7Fu, w3 = v.w & 0x7F7F7F7Fu;
        hi[u] = vmax_u16x2(vmax_u16x2(w0, w1), vmax_u16x2(w2, w3));
        lo[u] = vmax_u16x2(vmax_u16x2(w0 << 8, w1 << 8), vmax_u16x2(w2 << 8, w3 << 8));
    }
#pragma unroll
    for (int s = 4; s > 0; s >>= 1)   // then a 3-level tree over the units
#pragma unroll
        for (int u = 0; u < s; ++u) {
            hi[u] = vmax_u16x2(hi[u], hi[u + s]);
            lo[u] = vmax_u16x2(lo[u], lo[u + s]);
        }
    return max(max(hi[0] >> 24, (hi[0] >> 8) & 0xFFu), max(lo[0] >> 24, (lo[0] >> 8) & 0xFFu));
}

__device__ __forceinline__ float no_lower() { return __uint_as_float(0xFFFFFFFFu); }   // -NaN: orders first
__device__ __forceinline__ float no_upper() { return __uint_as_float(0x7FFFFFFFu); }   // +NaN: orders last

__global__ void __launch_bounds__(kScrThreads, 1) screen_kernel(const __grid_constant__ CUtensorMap tmap,
                                                                const ScreenArgs a)
{
    extern __shared__ uint8_t scr_raw[];
    ScrSmem &sm = *reinterpret_cast<ScrSmem *>((reinterpret_cast<uintptr_t>(scr_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // CTA c takes tiles c, c + grid, c + 2 grid, ... of the batch's (sequence, tile) slots, so that the
    // real tiles (slots below each sequence's own length) spread evenly over the CTAs whatever the mix
    // of lengths; consecutive tiles of a CTA still mostly share a sequence
    const long long first = blockIdx.x, step = gridDim.x;
    // local tile counters are 32-bit (at most 2^31 tiles per CTA): stage and phase arithmetic by
    // constants then stays a few instructions
    const uint32_t n_items = a.total > first ? (uint32_t)((a.total - first + step - 1) / step) : 0u;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kScrStages; ++s) {
            mbar_init(&sm.full[s], 1);
            mbar_init(&sm.sfree[s], 1 + 128);   // the MMA's commit and the row-max threads
            sm.stage_b[s] = -1;
        }
        for (int d = 0; d < kScrAcc; ++d) {
            mbar_init(&sm.dfull[d], 1 + 128);   // the MMA's commit and the row-max threads
            mbar_init(&sm.dfree[d], 128);       // the epilogue group of accumulator d
        }
        mbar_init(&sm.mma_fin, 1);
        sm.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tc_alloc(smem_addr(&sm.tmem), kScrTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sm.tmem;

    if (warp == 0) {
        // ---------------- loader ----------------
        auto resolve32 = [&](uint32_t k0) {
            const uint32_t k = k0 + lane;
            ScrItem it{-1, 0, 0, -1, -1};
            if (k < n_items) {
                const long long item = first + (long long)k * step;
                const int b = (int)(item / a.tiles_per_seq), tile = (int)(item % a.tiles_per_seq);
                const int L = a.seq_len[b];
                it.b = b;
                it.L = L;
                it.tile = tile;
                if (L < 1 || L > a.max_seq_len) {
                    if (tile == 0) report(a.ws, CSA_ERR_DEVICE_DATA, b);
                } else if (tile * kScrRows < L) {
                    const int pg = 2 * tile;
                    const int p0 = a.block_table[(size_t)b * a.max_pages + pg];
                    if (p0 < 0 || p0 >= a.num_pages) {
                        report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b * a.max_pages + pg);
                    } else {
                        it.p0 = p0;
                        if ((pg + 1) * kPage < L) {
                            const int p1 = a.block_table[(size_t)b * a.max_pages + pg + 1];
                            if (p1 < 0 || p1 >= a.num_pages) {
                                report(a.ws, CSA_ERR_DEVICE_DATA, (long long)b * a.max_pages + pg + 1);
                                it.p0 = -1;
                            } else {
                                it.p1 = p1;
                            }
                        }
                    }
                }
            }
            sm.ring[k % kScrRing] = it;
        };
        uint32_t issued = 0;
        bool q_visible = false;   // the query terms of the previous grid have been waited for
        for (uint32_t k = 0; k < n_items; ++k) {
            if ((k & 31) == 0) {
                resolve32(k);
                __syncwarp();
            }
            const int st = (int)(k % kScrStages);
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait(&sm.sfree[st], (uint32_t)(((k / kScrStages) & 1) ^ 1), &sm.abort_flag, a.ws, 20) ? 1 : 0;
                if (ok) {
                    const ScrItem it = sm.ring[k % kScrRing];
                    if (it.p0 >= 0) {
                        const bool need_q = sm.stage_b[st] != it.b;
                        const uint32_t bytes = (it.p1 >= 0 ? kScrKeyBytes : kScrPageBytes) + (need_q ? kScrQtBytes : 0u);
                        mbar_arrive_expect_tx(&sm.full[st], bytes);
                        tma_load_2d(sm.keys[st], &tmap, 0, it.p0 * kPage, &sm.full[st]);
                        if (it.p1 >= 0) tma_load_2d(sm.keys[st] + kScrPageBytes, &tmap, 0, it.p1 * kPage, &sm.full[st]);
                        if (need_q) {
                            if (!q_visible) {
                                grid_dep_wait();
                                q_visible = true;
                            }
                            bulk_g2s(sm.qt[st], a.qt + (size_t)it.b * kScrQtBytes, kScrQtBytes, &sm.full[st]);
                            sm.stage_b[st] = it.b;
                        }
                    } else {
                        mbar_arrive(&sm.full[st]);
                    }
                }
            }
            if (!__shfl_sync(0xffffffffu, ok, 0)) break;
            issued = k + 1;
        }
        // no copy may still be landing in shared memory when the CTA exits
        if (lane == 0) {
            for (uint32_t kk = issued > kScrStages ? issued - kScrStages : 0u; kk < issued; ++kk) {
                volatile int no_abort = 0;
                mbar_wait(&sm.full[kk % kScrStages], (uint32_t)((kk / kScrStages) & 1), &no_abort, a.ws, 25);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            bool any_mma = false;
            for (uint32_t k = 0; k < n_items; ++k) {
                const int st = (int)(k % kScrStages), d = (int)(k % kScrAcc);
                if (!mbar_wait(&sm.full[st], (uint32_t)((k / kScrStages) & 1), &sm.abort_flag, a.ws, 21)) break;
                if (!mbar_wait(&sm.dfree[d], (uint32_t)(((k / kScrAcc) & 1) ^ 1), &sm.abort_flag, a.ws, 22)) break;
                tc_fence_after();
                if (sm.ring[k % kScrRing].p0 >= 0) {
                    const uint32_t ka = smem_addr(sm.keys[st]), kb = smem_addr(sm.qt[st]);
#pragma unroll
                    for (int kk = 0; kk < kIdxDim / 32; ++kk)
                        tc_mma_f8(tmem + 32 * d, umma_sdesc_sw128(ka + kk * 32, 16, 1024),
                                  umma_sdesc_sw128(kb + kk * 32, 16, 1024), kIdescScreen, kk > 0);
                    tc_commit(smem_addr(&sm.dfull[d]));
                    tc_commit(smem_addr(&sm.sfree[st]));
                    any_mma = true;
                } else {
                    mbar_arrive(&sm.dfull[d]);
                    mbar_arrive(&sm.sfree[st]);
                }
            }
            if (any_mma) {   // every MMA this thread issued has finished before TMEM is released
                tc_commit(smem_addr(&sm.mma_fin));
                volatile int no_abort = 0;
                mbar_wait(&sm.mma_fin, 0, &no_abort, a.ws, 26);
            }
        }
        __syncwarp();
    } else if (warp < kScrEpiWarp0) {
        // ---------------- row maxima, group mg: tiles k = mg, mg + 2, ...; thread = tile row ----------
        const int mg = (warp - 2) >> 2;
        const int r = threadIdx.x - 64 - 128 * mg;
        for (uint32_t k = mg; k < n_items; k += kScrMaxGroups) {
            const int st = (int)(k % kScrStages), d = (int)(k % kScrAcc);
            if (!warp_wait(&sm.full[st], (uint32_t)((k / kScrStages) & 1), &sm.abort_flag, a.ws, 27)) break;
            if (!warp_wait(&sm.dfree[d], (uint32_t)(((k / kScrAcc) & 1) ^ 1), &sm.abort_flag, a.ws, 28)) break;
            if (sm.ring[k % kScrRing].p0 >= 0)
                sm.kmax[d][r] = e4m3_to_f32((uint8_t)row_max_code(sm.keys[st] + r * kIdxDim, r));
            mbar_arrive(&sm.dfull[d]);
            mbar_arrive(&sm.sfree[st]);
        }
    } else {
        // ---------------- epilogue group g: tiles k = g, g + 2, ...; thread = tile row = TMEM lane ----
        const int g = (warp - kScrEpiWarp0) >> 2;
        grid_dep_wait();   // the screening constants and the zeroed histogram
        const int quad = warp & 3;
        const int r = 32 * quad + lane;
        const uint32_t tl = tmem + ((uint32_t)(32 * quad) << 16);
        int cur_b = -1;
        QMeta qm{};
        float w[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (uint32_t k = g; k < n_items; k += kScrEpiGroups) {
            const int d = (int)(k % kScrAcc);
            if (!warp_wait(&sm.dfull[d], (uint32_t)((k / kScrAcc) & 1), &sm.abort_flag, a.ws, 24)) break;
            tc_fence_after();
            const ScrItem it = sm.ring[k % kScrRing];
            if (it.p0 >= 0) {
                if (it.b != cur_b) {
                    cur_b = it.b;
                    qm = a.qm[it.b];
#pragma unroll
                    for (int h = 0; h < 8; ++h) w[h] = a.iw[(size_t)it.b * kIdxHeads + h];
                }
                const float kmax = sm.kmax[d][r];
                float D[32];
                tc_ld32_sync(tl + 32 * d, D);
                float t = 0.f, wr = 0.f;
#pragma unroll
                for (int h = 0; h < 8; ++h) {
                    const float dh = __fmul_rn(__fadd_rn(__fadd_rn(D[h], D[8 + h]), D[16 + h]), qm.inv_scale[h]);
                    const float rh = dh > 0.f ? dh : 0.f;
                    t = __fmaf_rn(w[h], rh, t);
                    wr = __fmaf_ru(fabsf(w[h]), rh, wr);
                }
                const float eps = __fmaf_ru(kmax, qm.G, __fmaf_ru(qm.chain, wr, qm.absl));
                float lo, hi;
                const int p = it.tile * kScrRows + r;
                if (p >= it.L) {
                    lo = -INFINITY;   // not a position: leaves the block's maxima alone
                    hi = -INFINITY;
                } else if (!(__fmul_ru(kmax, qm.big) < 1e37f) || !(fabsf(t) <= 3.0e38f) || !(eps <= 3.0e38f)) {
                    lo = no_lower();
                    hi = no_upper();
                } else {
                    lo = __fsub_rd(t, eps);
                    hi = __fadd_ru(t, eps);
                }
                // block = 8 consecutive rows = 8 consecutive lanes.  The block score is the max of its
                // positions' scores, so the max of their lower bounds and the max of their upper bounds
                // bound it (a position without bounds has the smallest lower and largest upper key).
                uint32_t klo = order_key(lo), khi = order_key(hi);
#pragma unroll
                for (int o = 1; o < 8; o <<= 1) {
                    klo = max(klo, __shfl_xor_sync(0xffffffffu, klo, o));
                    khi = max(khi, __shfl_xor_sync(0xffffffffu, khi, o));
                }
                const int blk = it.tile * (kScrRows / kBlock) + r / kBlock;
                if ((lane & 7) == 0 && blk * kBlock < it.L) {
                    const size_t o = (size_t)it.b * a.stride + blk;
                    a.lo[o] = __uint_as_float(klo & 0x80000000u ? klo & 0x7FFFFFFFu : ~klo);
                    a.hi[o] = __uint_as_float(khi & 0x80000000u ? khi & 0x7FFFFFFFu : ~khi);
                    atomicAdd(&a.hist[(size_t)it.b * kHistBins + (klo >> 20)], 1u);
                }
            }
            tc_fence_before();
            mbar_arrive(&sm.dfree[d]);
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tc_dealloc(tmem, kScrTmemCols);
}

// ------------------------------------------------------------------------------------------------
// Host side
// ------------------------------------------------------------------------------------------------
namespace {

std::mutex g_encode_mu;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// The driver's tensor-map encoder, looked up once through the runtime (no link against libcuda).
cudaError_t tensor_map_encoder(PFN_cuTensorMapEncodeTiled_v12000 *out)
{
    std::lock_guard<std::mutex> lock(g_encode_mu);
    if (!g_encode) {
        void *fn = nullptr;
        cudaDriverEntryPointQueryResult q;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
        if (e != cudaSuccess) return e;
        if (q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = g_encode;
    return cudaSuccess;
}

// The keys' tensor map, re-encoded only when the key pool changes (the last one per device is kept).
cudaError_t keys_tensor_map(const uint8_t *keys, int num_pages, CUtensorMap *out)
{
    struct Cached {
        const uint8_t *keys;
        int num_pages;
        CUtensorMap map;
    };
    static std::mutex mu;
    static Cached cache[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lock(mu);
        if (cache[dev].keys == keys && cache[dev].num_pages == num_pages) {
            *out = cache[dev].map;
            return cudaSuccess;
        }
    }
    PFN_cuTensorMapEncodeTiled_v12000 encode;
    if ((e = tensor_map_encoder(&encode)) != cudaSuccess) return e;
    const cuuint64_t dims[2] = {(cuuint64_t)kIdxDim, (cuuint64_t)num_pages * kPage};
    const cuuint64_t strides[1] = {(cuuint64_t)kIdxDim};
    const cuuint32_t box[2] = {(cuuint32_t)kIdxDim, (cuuint32_t)kPage};
    const cuuint32_t estr[2] = {1, 1};
    if (encode(out, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(keys), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    if (dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lock(mu);
        cache[dev].keys = keys;
        cache[dev].num_pages = num_pages;
        cache[dev].map = *out;
    }
    return cudaSuccess;
}

int g_sm_count[64];

int sm_count()
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return kNumSms;
    if (!g_sm_count[dev]) {
        int n = 0;
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        g_sm_count[dev] = n > 0 ? n : kNumSms;
    }
    return g_sm_count[dev];
}

}  // namespace

// Keys as a 2-D tensor [num_pages * 64 rows][128 bytes], boxes of one page, 128-byte swizzle.
bool screen_supported(int num_pages) { return (long long)num_pages * kPage <= 0xFFFFFFFFll; }

cudaError_t launch_screen_bounds(const uint8_t *keys, int num_pages, const csa_batch &bt, const uint16_t *iq,
                                 const float *iw, uint8_t *qt, void *qm, uint32_t *hist, uint32_t *hist2, float *lo,
                                 float *hi, int stride, void *ws, cudaStream_t st)
{
    cudaError_t e;
    CUtensorMap map;
    if ((e = keys_tensor_map(keys, num_pages, &map)) != cudaSuccess) return e;

    if ((e = launch_overlapped(qterm_kernel, dim3(bt.B), dim3(256), 0, st, iq, iw, qt, reinterpret_cast<QMeta *>(qm),
                               hist, hist2)) != cudaSuccess)
        return e;

    ScreenArgs sa;
    sa.seq_len = bt.seq_len;
    sa.block_table = bt.block_table;
    sa.max_pages = bt.max_pages;
    sa.max_seq_len = bt.max_seq_len;
    sa.B = bt.B;
    sa.num_pages = num_pages;
    sa.tiles_per_seq = (bt.max_seq_len + kScrRows - 1) / kScrRows;
    sa.total = (long long)bt.B * sa.tiles_per_seq;
    const int grid = (int)(sa.total < sm_count() ? sa.total : sm_count());
    sa.iw = iw;
    sa.qt = qt;
    sa.qm = reinterpret_cast<const QMeta *>(qm);
    sa.lo = lo;
    sa.hi = hi;
    sa.stride = stride;
    sa.hist = hist;
    sa.ws = ws;
    const size_t smem = sizeof(ScrSmem) + 1024;
    if ((e = allow_dynamic_smem(reinterpret_cast<const void *>(screen_kernel), smem)) != cudaSuccess)
        return e;
    return launch_overlapped(screen_kernel, dim3(grid), dim3(kScrThreads), smem, st, map, sa);
}

}  // namespace csa
