// attention_tc.cu -- step 4 on the sm_100a tensor cores (tcgen05, TMEM) for 64 query heads per CTA.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用" (sparse
// attention over the selected positions of the FP4 main KV) and section "先让长输入少走一半路" (the
// FP8 sliding window); yomxxx.com long-form post, section 五 (fixed-stride entries dequantised in
// the kernel, in parallel).  The 512-channel latent serves as both key and value.
//
// With 64 heads sharing one latent, QK^T and PV are dense contractions: 4 x 64 x 512 FLOP per 288-B
// entry, above the fp16 tensor ridge of B200, so they run on the tensor cores.  Dequantisation of
// the FP4 entries is exact in fp16 (an E2M1 value times an E4M3 scale has at most 6 significant bits
// and lies in [2^-10, 2688]); a window entry's E4M3 values times its binary32 scale are rounded to
// fp16 (relative error 2^-11); Q is scaled per head by a power of two into fp16's range; P is rounded
// to fp16 (relative error 2^-11); accumulation is fp32 in TMEM.
//
// Tile = 128 entries.  Both MMAs put the entries / channels on M = 128 ("swap AB"):
//   QK:  S^T[128 entries x 64 heads]  = V[128 x 512] . Q^T          (A = V K-major, B = Q K-major)
//   PV:  O^T[128 ch x 64 heads] (x4)  = V^T[128 ch x 128 entries] . P^T   (A = V^T MN-major, B = P^T MN-major)
//   L :  L^T[128 x 64 heads]          = ones[128 x 128 entries] . P^T      (every row = the column sums of P)
// so TMEM holds S^T in 64 columns, O^T in 256 and L^T in 64, and one 128-byte-swizzled fp16 copy of
// the tile in shared memory is read as K-major V by QK and as MN-major V^T by PV.  The all-ones
// operand is one 128-byte block read through a zero-stride descriptor; summing the same fp16 P on the
// tensor core keeps the normaliser consistent with the numerator.
//
// Warp roles (288 threads).  Warp 8 owns the TMEM allocation and its lane 0 issues every MMA: QK of
// tile t chunk by chunk as its 64-channel chunks are dequantised, then PV and L of tile t once P is
// in shared memory.  Warps 0-7 form two groups of four (TMEM lanes 0-127 each; thread = tile row):
// group 1 = warps 0-3 takes heads 0-31 of the softmax and the epilogue, group 0 = warps 4-7 heads
// 32-63 and also writes each tile's entry metadata; the two halves are independent, each with its own
// named barrier.  Both groups load Q and dequantise: thread e of a group takes tile row e and the
// group's four 64-channel chunks (0, 1, 4, 5 for group 0; 2, 3, 6, 7 for group 1) from raw entries
// prefetched into registers a tile ahead.  The V buffer is single; the chunks of tile t+1 are written
// as soon as PV(t) has finished the M-tile reading them, so dequantisation and the QK of tile t+1
// overlap the end of PV(t).  Softmax rescales lazily: O^T and L^T are rescaled in TMEM only when a
// head's running maximum grows by more than 2^8; the new maxima come from one warp max-reduction per
// head (redux.sync on order-preserving integer keys).
#include "attention_common.cuh"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace csa {

constexpr int kTcHeads = 64;
constexpr int kTcRows = 128;
constexpr int kTcUnits = kTcRows / kAttnUnit;
constexpr int kTcChunks = kLatent / 64;
constexpr int kTcThreads = 288;   // 4 softmax warps, 4 dequant warps, 1 MMA warp
constexpr uint32_t kVChunk = kTcRows * 128;   // 16 KB: 128 rows x 64 fp16
constexpr uint32_t kQChunk = kTcHeads * 128;  // 8 KB: 64 rows x 64 fp16
constexpr uint32_t kOffV = 0;
constexpr uint32_t kOffQ = kOffV + kTcChunks * kVChunk;
constexpr uint32_t kOffP = kOffQ + kTcChunks * kQChunk;
constexpr uint32_t kOffOnes = kOffP + kTcRows * 128;   // 128 B of fp16 ones
constexpr uint32_t kOffMisc = kOffOnes + 1024;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 64;
constexpr uint32_t kColL = 320;
constexpr float kLazy = 8.f;      // log2-domain growth of a head maximum tolerated without rescaling
constexpr float kPOffset = 7.f;   // p = exp2(z - m + 7) <= 2^15 keeps small p out of fp16 subnormals
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcMisc {
    uint64_t s_full, p_full, q_ready, o_done, final_bar;
    uint64_t v_ready[kTcChunks];
    uint64_t v_free[kTcChunks / 2];
    uint32_t tmem_base;
    int abort_flag;
    float vmeta[2][kTcRows];    // per entry: 1 valid, -1 masked
    float zscale[kTcHeads];     // tau * 2^-k_h * log2(e)
    float m[kTcHeads];          // running max, log2 domain
    float alpha[kTcHeads];
    float red[4][kTcHeads];
};

constexpr size_t kTcSmem = kOffMisc + sizeof(TcMisc) + 1024;

constexpr uint32_t kIdescQK = umma_idesc_f16(128, kTcHeads, false, false);
constexpr uint32_t kIdescPV = umma_idesc_f16(128, kTcHeads, true, true);
constexpr uint32_t kIdescL = umma_idesc_f16(128, kTcHeads, false, true);

__device__ __forceinline__ uint32_t swz(uint32_t row, uint32_t unit) { return row * 128u + ((unit ^ (row & 7u)) << 4); }


__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b)
{
    __half2 x = *reinterpret_cast<__half2 *>(&a), y = *reinterpret_cast<__half2 *>(&b);
    __half2 r = __hmul2(x, y);
    return *reinterpret_cast<uint32_t *>(&r);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi)
{
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Warpgroup barriers (named barrier `id`, the 128 threads of one group: 1 for warps 0-3, 2 for warps
// 4-7).  Every thread of the group executes each of them once per tile, also after a failed wait, so
// none can be left waiting.
__device__ __forceinline__ bool group_and(int id, bool v)
{
    int r;
    asm volatile("{\n.reg .pred p, q;\nsetp.ne.b32 q, %2, 0;\nbar.red.and.pred p, %1, 128, q;\nselp.b32 %0, 1, 0, p;\n}"
                 : "=r"(r)
                 : "r"(id), "r"((int)v)
                 : "memory");
    return r != 0;
}

__device__ __forceinline__ bool group_or(int id, bool v)
{
    int r;
    asm volatile("{\n.reg .pred p, q;\nsetp.ne.b32 q, %2, 0;\nbar.red.or.pred p, %1, 128, q;\nselp.b32 %0, 1, 0, p;\n}"
                 : "=r"(r)
                 : "r"(id), "r"((int)v)
                 : "memory");
    return r != 0;
}

__device__ __forceinline__ void group_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }

// One thread's share of a tile's dequantisation: entry e (tile row) and the four 64-channel chunks of
// its thread group (group 0: chunks 0, 1, 4, 5; group 1: chunks 2, 3, 6, 7), raw bytes prefetched
// into registers.
struct TileRows {
    EntryRef r;
    bool valid;
    uint4 code[8];     // FP4 entry: code bytes of the group's chunks (64 B at 64*g, 64 B at 128 + 64*g);
                       // window entry: the 128 values of the chunk pair being written
    uint2 scl[2];      // their scale words

    // Window entry: start loading the values of chunk pair `pair` (chunks 2g + 4 pair and the next).
    __device__ __forceinline__ void fetch_window_pair(int pair, int g)
    {
        if (valid && r.swa) {
            const uint4 *src = reinterpret_cast<const uint4 *>(r.p + 64 * (2 * g + 4 * pair));
#pragma unroll
            for (int q = 0; q < 8; ++q) code[q] = src[q];
        }
    }

    __device__ __forceinline__ void load(const AttnArgs &a, const SeqView &sv, int u_begin, int u_end, int t, int e,
                                         int g)
    {
        const int u = u_begin + t * kTcUnits + e / kAttnUnit, j = e % kAttnUnit;
        valid = u < u_end && entry_ref(a, sv, u, j, r);
        if (valid && !r.swa) {
            const uint4 *cp = reinterpret_cast<const uint4 *>(r.p);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                code[q] = cp[4 * g + q];
                code[4 + q] = cp[8 + 4 * g + q];
            }
            const uint2 *sp = reinterpret_cast<const uint2 *>(r.sc);
            scl[0] = sp[g];
            scl[1] = sp[2 + g];
        }
    }

    // Chunk slot cs (0..3) of this group: channels 64c .. 64c+63, c = 2g + (cs & 1) + 4 (cs >> 1).
    __device__ __forceinline__ void write(uint8_t *V, int e, int c, int cs) const
    {
        uint4 out[8];
        if (!valid) {
#pragma unroll
            for (int jj = 0; jj < 8; ++jj) out[jj] = make_uint4(0u, 0u, 0u, 0u);
        } else if (!r.swa) {
            const uint32_t sw = (cs & 1) ? scl[cs >> 1].y : scl[cs >> 1].x;
#pragma unroll
            for (int gg = 0; gg < 4; ++gg) {
                const uint32_t sh = e4m3x2_to_f16x2((uint16_t)((sw >> (8 * gg)) & 0xFF));
                const uint32_t s2 = (sh & 0xFFFFu) | (sh << 16);
                const uint4 cw = code[2 * cs + (gg >> 1)];
                const uint32_t w0 = (gg & 1) ? cw.z : cw.x, w1 = (gg & 1) ? cw.w : cw.y;
                uint32_t v[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    v[q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w0 >> (8 * q))), s2);
                    v[4 + q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w1 >> (8 * q))), s2);
                }
                out[2 * gg] = make_uint4(v[0], v[1], v[2], v[3]);
                out[2 * gg + 1] = make_uint4(v[4], v[5], v[6], v[7]);
            }
        } else {
            // window entry: 64 E4M3 values (fetched with its chunk pair) times the entry's binary32
            // scale, rounded to fp16
            const float fs = r.fscale;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = code[4 * (cs & 1) + q];
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                uint32_t v[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t lo = e4m3x2_to_f16x2((uint16_t)(ww[k] & 0xFFFF));
                    const uint32_t hi = e4m3x2_to_f16x2((uint16_t)(ww[k] >> 16));
                    v[2 * k] = pack_f16x2(h_lo(lo) * fs, h_hi(lo) * fs);
                    v[2 * k + 1] = pack_f16x2(h_lo(hi) * fs, h_hi(hi) * fs);
                }
                out[2 * q] = make_uint4(v[0], v[1], v[2], v[3]);
                out[2 * q + 1] = make_uint4(v[4], v[5], v[6], v[7]);
            }
        }
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) *reinterpret_cast<uint4 *>(V + c * kVChunk + swz((uint32_t)e, (uint32_t)jj)) = out[jj];
    }
};

// Dequantise this group's four chunks of tile t into V (waiting for PV(t-1) to release each pair).
__device__ __forceinline__ bool dequant_group(TcMisc &ms, uint8_t *V, TileRows &rows, const AttnArgs &a, int t, int e,
                                              int g)
{
    bool ok = true;
#pragma unroll
    for (int cs = 0; cs < 4; ++cs) {
        const int c = 2 * g + (cs & 1) + 4 * (cs >> 1);
        if ((cs & 1) == 0) {
            rows.fetch_window_pair(cs >> 1, g);   // in flight while PV(t-1) releases the pair
            if (t > 0) ok = ok && warp_wait(&ms.v_free[c >> 1], (t - 1) & 1, &ms.abort_flag, a.ws, 5);
        }
        if (ok) rows.write(V, e, c, cs);
        fence_async_smem();
        mbar_arrive(&ms.v_ready[c]);
    }
    return ok;
}

// Q of heads h0..h0+63 into shared memory as fp16, 128B-swizzled K-major, each head scaled by a power
// of two 2^k_h that puts its largest |q| in [2^13, 2^14); the softmax undoes it through zscale.
// Thread t of the 256 dequantising threads converts a quarter row (128 channels) of head t/4.
__device__ __forceinline__ void load_q(const AttnArgs &a, TcMisc &ms, uint8_t *Q, int b, int h0, int t)
{
    const int h = t >> 2, quarter = t & 3;
    const uint4 *qrow = reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.H + h0 + h) * kLatent + quarter * 128);
    uint4 qw[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) qw[c] = qrow[c];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        const uint32_t ww[4] = {qw[c].x, qw[c].y, qw[c].z, qw[c].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(ww[k])), fabsf(bf16_hi(ww[k]))));
    }
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    int k = 0;
    if (amax > 0.f) {
        const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
        k = 13 - ex;
        k = k < -60 ? -60 : (k > 60 ? 60 : k);
    }
    const float sc = exp2f((float)k);
    if (quarter == 0) ms.zscale[h] = a.sm_scale * exp2f((float)-k) * kLog2e;
#pragma unroll
    for (int c = 0; c < 16; ++c) {
        uint4 o;
        o.x = pack_f16x2(bf16_lo(qw[c].x) * sc, bf16_hi(qw[c].x) * sc);
        o.y = pack_f16x2(bf16_lo(qw[c].y) * sc, bf16_hi(qw[c].y) * sc);
        o.z = pack_f16x2(bf16_lo(qw[c].z) * sc, bf16_hi(qw[c].z) * sc);
        o.w = pack_f16x2(bf16_lo(qw[c].w) * sc, bf16_hi(qw[c].w) * sc);
        const int ch = quarter * 128 + 8 * c;
        *reinterpret_cast<uint4 *>(Q + (ch >> 6) * kQChunk + swz(h, (ch & 63) >> 3)) = o;
    }
    fence_async_smem();
    mbar_arrive(&ms.q_ready);
}

__global__ void __launch_bounds__(kTcThreads, 1) attn_split_tc_kernel(AttnArgs a, int head_groups)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *V = base + kOffV;
    uint8_t *Q = base + kOffQ;
    uint8_t *P = base + kOffP;
    uint8_t *ONES = base + kOffOnes;
    TcMisc &ms = *reinterpret_cast<TcMisc *>(base + kOffMisc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_launch();   // the combine may be scheduled as splits finish
    const int s = blockIdx.x, b = blockIdx.y / head_groups, hg = blockIdx.y % head_groups;
    const int h0 = hg * kTcHeads;

    if (threadIdx.x == 0) {
        mbar_init(&ms.s_full, 1);
        mbar_init(&ms.p_full, 256);   // both groups' halves of P
        mbar_init(&ms.q_ready, 256);
        mbar_init(&ms.o_done, 1);
        mbar_init(&ms.final_bar, 1);
        for (int c = 0; c < kTcChunks; ++c) mbar_init(&ms.v_ready[c], 128);
        for (int c = 0; c < kTcChunks / 2; ++c) mbar_init(&ms.v_free[c], 1);
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kTcHeads) ms.m[threadIdx.x] = -INFINITY;
    if (threadIdx.x < 32) reinterpret_cast<uint32_t *>(ONES)[threadIdx.x] = 0x3C003C00u;   // fp16 1.0 pairs
    __syncthreads();
    // Q is an input of the step, not a result of the previous grid: load it while that grid finishes
    if (warp < 8) load_q(a, ms, Q, b, h0, threadIdx.x);
    grid_dep_wait();   // the selected blocks of the previous grid

    SeqView sv;
    const bool seq_ok = seq_view(a, b, sv);
    int u_begin = 0, u_end = 0;
    if (seq_ok) split_range(sv.units, s, a.splits, u_begin, u_end);
    const int ntiles = (u_end - u_begin + kTcUnits - 1) / kTcUnits;
    if (warp == 8 && ntiles > 0) {
        tc_alloc(smem_addr(&ms.tmem_base), kTmemCols);
        tc_relinquish();
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;

    if (ntiles == 0) {
        // empty split: a neutral partial
        if (warp < 4) {
            float *po = a.part_o + (((size_t)b * a.splits + s) * a.H + h0) * kLatent;
            for (int h = 0; h < kTcHeads; ++h)
                for (int c = threadIdx.x; c < kLatent; c += 128) po[(size_t)h * kLatent + c] = 0.f;
            if (threadIdx.x < kTcHeads)
                reinterpret_cast<float2 *>(a.part_ml)[((size_t)b * a.splits + s) * a.H + h0 + threadIdx.x] =
                    make_float2(-INFINITY, 0.f);
        }
        return;
    }

    if (warp == 8) {
        // ------------------------------- MMA issuer -------------------------------
        if (lane == 0) {
            const uint32_t sV = smem_addr(V), sQ = smem_addr(Q), sP = smem_addr(P), sOnes = smem_addr(ONES);
            const uint64_t ones_desc = umma_sdesc_noswz(sOnes, 0, 0);
            bool ok = mbar_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
            tc_fence_after();
            for (int t = 0; ok && t < ntiles; ++t) {
                const uint32_t ph = t & 1;
                for (int c = 0; c < kTcChunks; ++c) {
                    if (!(ok = mbar_wait(&ms.v_ready[c], ph, &ms.abort_flag, a.ws, 2))) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = umma_sdesc_sw128(sV + c * kVChunk + kk * 32, 16, 1024);
                        const uint64_t bd = umma_sdesc_sw128(sQ + c * kQChunk + kk * 32, 16, 1024);
                        tc_mma_f16(tmem + kColS, ad, bd, kIdescQK, (c | kk) != 0);
                    }
                }
                if (!ok) break;
                tc_commit(smem_addr(&ms.s_full));
                if (!(ok = mbar_wait(&ms.p_full, ph, &ms.abort_flag, a.ws, 3))) break;
                tc_fence_after();
                for (int m = 0; m < 4; ++m) {
#pragma unroll
                    for (int kk = 0; kk < kTcRows / 16; ++kk) {
                        const uint64_t ad = umma_sdesc_sw128(sV + 2 * m * kVChunk + kk * 2048, kVChunk, 1024);
                        const uint64_t bd = umma_sdesc_sw128(sP + kk * 2048, kVChunk, 1024);
                        tc_mma_f16(tmem + kColO + 64 * m, ad, bd, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
                    }
                    tc_commit(smem_addr(&ms.v_free[m]));
                }
#pragma unroll
                for (int kk = 0; kk < kTcRows / 16; ++kk) {
                    const uint64_t bd = umma_sdesc_sw128(sP + kk * 2048, kVChunk, 1024);
                    tc_mma_f16(tmem + kColL, ones_desc, bd, kIdescL, (t > 0 || kk > 0) ? 1u : 0u);
                }
                if (t == ntiles - 1) tc_commit(smem_addr(&ms.o_done));
            }
            // every MMA this thread issued has completed before TMEM is released
            tc_commit(smem_addr(&ms.final_bar));
            volatile int no_abort = 0;
            mbar_wait(&ms.final_bar, 0, &no_abort, a.ws, 4);
        }
        __syncwarp();
    } else {
        // --------------- softmax groups: group 1 = warps 0-3 (heads 0-31, chunks 2, 3, 6, 7), ---------
        // --------------- group 0 = warps 4-7 (heads 32-63, chunks 0, 1, 4, 5, tile metadata) ---------
        const int grp = warp >= 4 ? 0 : 1;
        const int hh = 1 - grp;              // this group's half of the heads
        const int bar_id = 2 - grp;          // named barrier of the group
        const int e = threadIdx.x & 127;     // TMEM lane = tile row (entry); channel in the epilogue
        const int wq = warp & 3;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
        TileRows rows;
        rows.load(a, sv, u_begin, u_end, 0, e, grp);
        if (grp == 0) ms.vmeta[0][e] = rows.valid ? 1.f : -1.f;
        bool ok = dequant_group(ms, V, rows, a, 0, e, grp);
        ok = warp_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1) && ok;   // every head's score scale
        ok = group_and(bar_id, ok);
        for (int t = 0; ok && t < ntiles; ++t) {
            const uint32_t ph = t & 1;
            bool tok = warp_wait(&ms.s_full, ph, &ms.abort_flag, a.ws, 6) &&
                       warp_wait(&ms.v_ready[0], ph, &ms.abort_flag, a.ws, 7);
            if (!(ok = group_and(bar_id, tok))) break;
            tc_fence_after();
            const bool valid = ms.vmeta[ph][e] >= 0.f;
            // scores of this group's 32 heads, in the log2 domain (masked rows: -inf)
            float zt[32];
            tc_ld32_sync(tl + kColS + 32 * hh, zt);
#pragma unroll
            for (int q = 0; q < 32; ++q) zt[q] = valid ? zt[q] * ms.zscale[32 * hh + q] : -INFINITY;
            bool need = false;
#pragma unroll
            for (int q = 0; q < 32; ++q) need |= zt[q] > ms.m[32 * hh + q] + kLazy;
            if (group_or(bar_id, need)) {
                // new maxima: per head one warp max-reduction on order keys, then over the four warps
#pragma unroll
                for (int q = 0; q < 32; ++q) {
                    const uint32_t u = __reduce_max_sync(0xffffffffu, order_key(zt[q]));
                    if (lane == 0) ms.red[wq][32 * hh + q] = key_to_float(u);
                }
                group_sync(bar_id);
                if (e < 32) {
                    const int h = 32 * hh + e;
                    const float mt = fmaxf(fmaxf(ms.red[0][h], ms.red[1][h]), fmaxf(ms.red[2][h], ms.red[3][h]));
                    const float mo = ms.m[h];
                    const float mn = fmaxf(mo, mt);
                    ms.alpha[h] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
                    ms.m[h] = mn;
                }
                group_sync(bar_id);
                if (t > 0) {
                    // this group's head columns of O^T (4 M-tiles) and of L^T
#pragma unroll 1
                    for (int m = 0; m < 5; ++m) {
                        float o[32];
                        const uint32_t col = (m < 4 ? kColO + 64 * m : kColL) + 32 * hh;
                        tc_ld32_sync(tl + col, o);
#pragma unroll
                        for (int q = 0; q < 32; ++q) o[q] *= ms.alpha[32 * hh + q];
                        tc_st32(tl + col, o);
                    }
                    tc_wait_st();
                }
            }
            uint32_t pk[16];
#pragma unroll
            for (int q = 0; q < 32; q += 2) {
                const float p0 = exp2f(zt[q] - ms.m[32 * hh + q] + kPOffset);
                const float p1 = exp2f(zt[q + 1] - ms.m[32 * hh + q + 1] + kPOffset);
                pk[q / 2] = pack_f16x2(p0, p1);
            }
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                *reinterpret_cast<uint4 *>(P + swz((uint32_t)e, (uint32_t)(4 * hh + jj))) =
                    make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&ms.p_full);
            // this group's chunks of the next tile, as PV(t) releases them
            if (t + 1 < ntiles) {
                rows.load(a, sv, u_begin, u_end, t + 1, e, grp);
                if (grp == 0) ms.vmeta[(t + 1) & 1][e] = rows.valid ? 1.f : -1.f;
                dequant_group(ms, V, rows, a, t + 1, e, grp);
            }
        }
        // ---- epilogue: this group's heads of the split's partial (o, m, l)
        float *po = a.part_o + (((size_t)b * a.splits + s) * a.H + h0) * kLatent;
        float2 *pml = reinterpret_cast<float2 *>(a.part_ml) + ((size_t)b * a.splits + s) * a.H + h0;
        bool eok = ok && warp_wait(&ms.o_done, 0, &ms.abort_flag, a.ws, 8);
        eok = group_and(bar_id, eok);
        if (eok) {
            tc_fence_after();
            for (int m = 0; m < 4; ++m) {
                float o[32];
                tc_ld32_sync(tl + kColO + 64 * m + 32 * hh, o);
#pragma unroll
                for (int q = 0; q < 32; ++q) po[(size_t)(32 * hh + q) * kLatent + 128 * m + e] = o[q];
            }
            if (wq == 0) {
                // every row of L^T holds the sums; lane 0's row is shared through shared memory
                float l[32];
                tc_ld32_sync(tl + kColL + 32 * hh, l);
                if (lane == 0) {
#pragma unroll
                    for (int q = 0; q < 32; ++q) ms.red[0][32 * hh + q] = l[q];
                }
            }
            group_sync(bar_id);
            if (e < 32) {
                const int h = 32 * hh + e;
                pml[h] = make_float2((ms.m[h] - kPOffset) * kLn2, ms.red[0][h]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 8) tc_dealloc(tmem, kTmemCols);
}

bool attn_tc_supported(int H) { return H == 64 || H == 128; }

int attn_units_per_tile(int H) { return attn_tc_supported(H) ? kTcUnits : 4; }

cudaError_t launch_attn_tc(const AttnArgs &a, cudaStream_t st)
{
    static_assert(kTcSmem <= 232448, "shared memory budget");
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void *>(attn_split_tc_kernel), kTcSmem);
    if (e != cudaSuccess) return e;
    const int groups = a.H / kTcHeads;
    dim3 grid(a.splits, a.B * groups);
    return launch_overlapped(attn_split_tc_kernel, grid, dim3(kTcThreads), kTcSmem, st, a, groups);
}

}  // namespace csa
