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
// fp16 (relative error 2^-11); Q is scaled by one power of two into fp16's range; P is rounded to
// fp16 (relative error 2^-11); accumulation is fp32 in TMEM.  The softmax denominators are summed
// in fp32 on the CUDA cores from the unrounded probabilities (at most 2^-12 relative apart from the
// fp16 numerators).
//
// Tile = 128 entries.  Both MMAs put the entries / channels on M = 128 ("swap AB"):
//   QK:  S^T[128 entries x 64 heads]  = V[128 x 512] . Q^T               (A = V K-major, B = Q K-major)
//   PV:  O^T[128 ch x 64 heads] (x4)  = V^T[128 ch x 128 entries] . P^T  (A = V^T MN-major, B = P^T MN-major)
// One 128-byte-swizzled fp16 copy of the tile in shared memory is read as K-major V by QK and as
// MN-major V^T by PV.  TMEM: O^T in 4 x 64 columns, S^T as two partial accumulators (even and odd
// chunks, one per QK issuer, summed by the softmax) in 2 x 64 columns, and each row's softmax sums
// in 64 columns.
//
// Warp roles (640 threads).  Warps 16-19 issue the MMAs (lane 0 each; warp 16 also owns the TMEM
// allocation): one thread issues a tcgen05.mma only every ~100 cycles, so QK of the even and of the
// odd chunks and PV of M-tiles 0-1 and 2-3 each have their own issuer.  Warps 0-15 form four groups of
// four warps; thread e of a group is tile row e (TMEM lane e).  Group g owns heads 16g .. 16g+15 of
// the softmax and channels 128g + e of the epilogue.  The V buffer is single; as PV(t) releases
// M-tile m (V chunks 2m, 2m+1), all 512 threads dequantise those 128 channels of tile t+1 (thread
// (g, e): 32 channels of entry e), from raw bytes loaded into registers a tile earlier.  Entry
// addresses come from a table in shared memory that all threads fill after the grid dependency
// (16 tiles at a time), so no dependent global load stalls a tile.  Softmax rescales lazily: O^T is
// rescaled in TMEM only when a head's running maximum grows by more than 2^8.
#include "attention_common.cuh"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace csa {

constexpr int kTcHeads = 64;
constexpr int kTcRows = 128;
constexpr int kTcUnits = kTcRows / kAttnUnit;    // 16 units of 8 entries per tile
constexpr int kTcChunks = kLatent / 64;          // 8 chunks of 64 channels
constexpr int kTcGroups = 4;                     // compute groups of 4 warps
constexpr int kTcHeadsPerGroup = kTcHeads / kTcGroups;
constexpr int kTcIssuers = 4;                    // MMA-issuing warps: QK even / odd chunks, PV M-tiles 0-1 / 2-3
constexpr int kTcThreads = 32 * (4 * kTcGroups + kTcIssuers);
constexpr int kTcCompute = 128 * kTcGroups;
constexpr int kSAcc = 2;
constexpr int kTabTiles = 16;                    // tiles of entry addresses resolved at a time                         // partial QK accumulators (independent MMA chains)
constexpr uint32_t kVChunk = kTcRows * 128;      // 16 KB: 128 rows x 64 fp16
constexpr uint32_t kQChunk = kTcHeads * 128;     // 8 KB: 64 rows x 64 fp16
constexpr uint32_t kOffV = 0;
constexpr uint32_t kOffQ = kOffV + kTcChunks * kVChunk;
constexpr uint32_t kOffP = kOffQ + kTcChunks * kQChunk;
constexpr uint32_t kOffMisc = kOffP + kTcRows * 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;                    // O^T: M-tile m in columns 64m .. 64m+63
constexpr uint32_t kColS = 256;                  // S^T partial a in columns 256 + 64a ..
constexpr uint32_t kColL = kColS + 64 * kSAcc;   // per-row softmax sums: group g in 16 columns at 16g
constexpr float kLazy = 8.f;      // log2-domain growth of a head maximum tolerated without rescaling
constexpr float kPOffset = 7.f;   // p = exp2(z - m + 7) <= 2^15 keeps small p out of fp16 subnormals
constexpr float kNoMax = -1e30f;  // running maximum before any finite score (exp2 of it minus a finite value is 0)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcMisc {
    uint64_t s_full, p_full, q_ready, o_done;
    uint64_t final_bar[kTcIssuers];
    uint64_t v_ready[4];          // per PV M-tile: its 128 channels of the next tile are written
    uint64_t v_free[4];           // per PV M-tile: PV has finished reading them
    uint32_t tmem_base;
    int abort_flag;
    float qmax[16];                              // per compute warp: largest |q| of its rows
    float red[kTcGroups][4][kTcHeadsPerGroup];   // per group, per warp: a per-head partial
    float mx[kTcGroups][kTcHeadsPerGroup];       // running maximum of each head (log2 domain)
    int32_t rows[kTabTiles][kTcRows];            // entry of (tile, row): FP4 cache row >= 0, window slot
                                                 // -(slot + 2), or -1 (masked)
    float alpha[kTcGroups][kTcHeadsPerGroup];    // rescale factor of each head at a maximum update
    SeqView sv;                                  // the sequence, read from here by every thread
    int u_begin, u_end;                          // this split's units
};

constexpr size_t kTcSmem = kOffMisc + sizeof(TcMisc) + 1024;

constexpr uint32_t kIdescQK = umma_idesc_f16(128, kTcHeads, false, false);
constexpr uint32_t kIdescPV = umma_idesc_f16(128, kTcHeads, true, true);

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

// Group barriers (named barrier `id` over the 128 threads of one group).  Every thread of the group
// executes each of them once per tile, also after a failed wait, so none can be left waiting.
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

// Barrier over the 512 compute threads (the MMA warp does not take part).
__device__ __forceinline__ void compute_sync() { asm volatile("bar.sync 5, %0;" ::"n"(kTcCompute) : "memory"); }

// 32 lanes x 16 consecutive 32-bit columns, waited for in the same statement.
__device__ __forceinline__ void tc_ld16_sync(uint32_t taddr, float *v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_st16(uint32_t taddr, const float *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
        "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
        "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
        "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
        "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
        "r"(__float_as_uint(v[15]))
        : "memory");
}

// This thread's row of the group's 16 scores in the log2 domain: the sum of the partial QK
// accumulators times zs; a masked row gives -inf.
__device__ __forceinline__ void load_scores(uint32_t taddr, bool valid, float zs, float *z)
{
    tc_ld16_sync(taddr, z);
#pragma unroll
    for (int aa = 1; aa < kSAcc; ++aa) {
        float z2[kTcHeadsPerGroup];
        tc_ld16_sync(taddr + 64 * aa, z2);
#pragma unroll
        for (int q = 0; q < kTcHeadsPerGroup; ++q) z[q] += z2[q];
    }
#pragma unroll
    for (int q = 0; q < kTcHeadsPerGroup; ++q) z[q] = valid ? z[q] * zs : -INFINITY;
}

// Tile-aligned split of a sequence's units: split s of `splits` gets whole 16-unit tiles, so every
// tile but the sequence's last is full.
__device__ __forceinline__ void split_tiles(int units, int s, int splits, int &ub, int &ue)
{
    const int tiles = (units + kTcUnits - 1) / kTcUnits;
    const int tb = (int)((long long)tiles * s / splits), te = (int)((long long)tiles * (s + 1) / splits);
    ub = tb * kTcUnits;
    ue = te * kTcUnits < units ? te * kTcUnits : units;
}

// Table code of (tile t, row e) of this split: the FP4 cache row (page * 64 + offset) of the entry,
// -(slot + 2) for a window entry, -1 for a masked row (past the split or the sequence).
__device__ __forceinline__ int32_t entry_code(const AttnArgs &a, const SeqView &sv, int u_begin, int u_end, int t, int e)
{
    const int u = u_begin + t * kTcUnits + e / kAttnUnit, j = e % kAttnUnit;
    if (u >= u_end) return -1;
    if (u < sv.nE) {
        const int blk = sv.blocks[u];
        if (blk < 0 || blk >= sv.nb) {
            report(a.ws, CSA_ERR_DEVICE_DATA, u);
            return -1;
        }
        const int p = blk * kBlock + j;
        if (p >= sv.L) return -1;
        const int page = sv.bt[blk / kBlocksPerPage];
        if (page < 0 || page >= a.num_pages) {
            report(a.ws, CSA_ERR_DEVICE_DATA, blk);
            return -1;
        }
        return page * kPage + (blk % kBlocksPerPage) * kBlock + j;
    }
    const int p = sv.w0 + (u - sv.nE) * kAttnUnit + j;
    if (p >= sv.L) return -1;
    return -(sv.row * kWindow + (p % kWindow) + 2);
}

// One thread's share of one tile: entry e, and in each M-tile m the 32 channels 128m + 32g .. +31.
// The raw bytes of an FP4 entry (16 B of codes and 2 scale bytes per M-tile) are loaded into
// registers a tile before they are dequantised; a window entry (32 E4M3 values per M-tile) is read
// when it is written, since the window is at most one tile of a sequence.
struct RawTile {
    uint4 code[4];
    uint32_t sc[4];
    int32_t row;

    __device__ __forceinline__ void fetch(const AttnArgs &a, int32_t code_row, int g)
    {
        row = code_row;
        if (row >= 0) {
            const uint8_t *cp = a.codes + (size_t)row * kCodeBytes + 16 * g;
            const uint8_t *sp = a.scales + (size_t)row * kScaleBytes + 2 * g;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                code[m] = *reinterpret_cast<const uint4 *>(cp + 64 * m);
                sc[m] = *reinterpret_cast<const uint16_t *>(sp + 8 * m);
            }
        }
    }

    // Dequantise this thread's 32 channels of M-tile m (V chunk 2m + g/2, 16-byte units 4(g%2) ..
    // 4(g%2)+3 of row e).
    __device__ __forceinline__ void write(const AttnArgs &a, uint8_t *V, int m, int e, int g) const
    {
        uint8_t *dst = V + (2 * m + (g >> 1)) * kVChunk;
        const uint32_t u0 = 4u * (uint32_t)(g & 1);
        if (row == -1) {
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, u0 + jj)) = make_uint4(0u, 0u, 0u, 0u);
        } else if (row >= 0) {
#pragma unroll
            for (int gg = 0; gg < 2; ++gg) {
                const uint32_t sh = e4m3x2_to_f16x2((uint16_t)((sc[m] >> (8 * gg)) & 0xFF));
                const uint32_t s2 = (sh & 0xFFFFu) | (sh << 16);
                const uint32_t w0 = gg ? code[m].z : code[m].x, w1 = gg ? code[m].w : code[m].y;
                uint32_t v[8];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    v[q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w0 >> (8 * q))), s2);
                    v[4 + q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w1 >> (8 * q))), s2);
                }
                *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, u0 + 2 * gg)) = make_uint4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, u0 + 2 * gg + 1)) = make_uint4(v[4], v[5], v[6], v[7]);
            }
        } else {
            // window entry: 32 E4M3 values times the entry's binary32 scale, rounded to fp16
            const size_t slot = (size_t)(-row - 2);
            const float fs = a.swa_scale[slot];
            const uint4 *src = reinterpret_cast<const uint4 *>(a.swa + slot * kLatent + 128 * m + 32 * g);
#pragma unroll
            for (int q = 0; q < 2; ++q) {
                const uint4 w = src[q];
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                uint32_t v[8];
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const uint32_t lo = e4m3x2_to_f16x2((uint16_t)(ww[k] & 0xFFFF));
                    const uint32_t hi = e4m3x2_to_f16x2((uint16_t)(ww[k] >> 16));
                    v[2 * k] = pack_f16x2(h_lo(lo) * fs, h_hi(lo) * fs);
                    v[2 * k + 1] = pack_f16x2(h_lo(hi) * fs, h_hi(hi) * fs);
                }
                *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, u0 + 2 * q)) = make_uint4(v[0], v[1], v[2], v[3]);
                *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, u0 + 2 * q + 1)) = make_uint4(v[4], v[5], v[6], v[7]);
            }
        }
    }
};

// Fill the entry table with tiles t0 .. t0 + kTabTiles - 1 (every compute thread takes a share).
__device__ __forceinline__ void fill_table(const AttnArgs &a, TcMisc &ms, int t0, int ntiles, int tid)
{
    const int n = (ntiles - t0 < kTabTiles ? ntiles - t0 : kTabTiles) * kTcRows;
    for (int i = tid; i < n; i += kTcCompute)
        ms.rows[i / kTcRows][i % kTcRows] = entry_code(a, ms.sv, ms.u_begin, ms.u_end, t0 + i / kTcRows, i % kTcRows);
}

// Q of heads h0..h0+63 into shared memory as fp16, 128B-swizzled K-major, scaled by one power of two
// 2^k that puts the largest |q| of the 64 heads in [2^13, 2^14); returns tau * log2(e) * 2^-k, the
// factor that turns an accumulated score into the log2 domain.  Compute thread t converts channels
// 64(t/64) .. 64(t/64)+63 of head t%64 (consecutive threads write different rows of one chunk, so
// the 16-byte stores do not collide in shared-memory banks).
__device__ __forceinline__ float load_q(const AttnArgs &a, TcMisc &ms, uint8_t *Q, int b, int h0, int t)
{
    const int h = t & 63, part = t >> 6;
    const uint4 *qrow = reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.H + h0 + h) * kLatent + part * 64);
    uint4 qw[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) qw[c] = qrow[c];
    float amax = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint32_t ww[4] = {qw[c].x, qw[c].y, qw[c].z, qw[c].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(ww[k])), fabsf(bf16_hi(ww[k]))));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    if ((t & 31) == 0) ms.qmax[t >> 5] = amax;
    compute_sync();
    amax = 0.f;
#pragma unroll
    for (int w = 0; w < 16; ++w) amax = fmaxf(amax, ms.qmax[w]);
    int k = 0;
    if (amax > 0.f) {
        const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
        k = 13 - ex;
        k = k < -60 ? -60 : (k > 60 ? 60 : k);
    }
    const float sc = exp2f((float)k);
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        uint4 o;
        o.x = pack_f16x2(bf16_lo(qw[c].x) * sc, bf16_hi(qw[c].x) * sc);
        o.y = pack_f16x2(bf16_lo(qw[c].y) * sc, bf16_hi(qw[c].y) * sc);
        o.z = pack_f16x2(bf16_lo(qw[c].z) * sc, bf16_hi(qw[c].z) * sc);
        o.w = pack_f16x2(bf16_lo(qw[c].w) * sc, bf16_hi(qw[c].w) * sc);
        *reinterpret_cast<uint4 *>(Q + part * kQChunk + swz(h, c)) = o;
    }
    fence_async_smem();
    mbar_arrive(&ms.q_ready);
    return a.sm_scale * exp2f((float)-k) * kLog2e;
}

// M-tiles in the order PV releases them (issuer 2 does M-tile 0 then 1, issuer 3 M-tile 2 then 3).
__device__ __forceinline__ int release_order(int i) { return (i & 1) * 2 + (i >> 1); }

__global__ void __launch_bounds__(kTcThreads, 1) attn_split_tc_kernel(AttnArgs a, int head_groups)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *V = base + kOffV;
    uint8_t *Q = base + kOffQ;
    uint8_t *P = base + kOffP;
    TcMisc &ms = *reinterpret_cast<TcMisc *>(base + kOffMisc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_launch();   // the combine may be scheduled as splits finish
    const int s = blockIdx.x, b = blockIdx.y / head_groups, hg = blockIdx.y % head_groups;
    const int h0 = hg * kTcHeads;

    if (threadIdx.x == 0) {
        mbar_init(&ms.s_full, 2);     // both QK issuers
        mbar_init(&ms.p_full, kTcCompute);
        mbar_init(&ms.q_ready, kTcCompute);
        mbar_init(&ms.o_done, 2);     // both PV issuers
        for (int r = 0; r < kTcIssuers; ++r) mbar_init(&ms.final_bar[r], 1);
        for (int m = 0; m < 4; ++m) {
            mbar_init(&ms.v_ready[m], kTcCompute);
            mbar_init(&ms.v_free[m], 1);
        }
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();
    // Q is an input of the step, not a result of the previous grid: load it while that grid finishes
    float zs = 0.f;
    if (warp < 16) zs = load_q(a, ms, Q, b, h0, threadIdx.x);
    grid_dep_wait();   // the selected blocks of the previous grid

    if (threadIdx.x == 0) {
        int ub = 0, ue = 0;
        if (seq_view(a, b, ms.sv)) split_tiles(ms.sv.units, s, a.splits, ub, ue);
        ms.u_begin = ub;
        ms.u_end = ue;
    }
    __syncthreads();
    const int ntiles = (ms.u_end - ms.u_begin + kTcUnits - 1) / kTcUnits;
    if (warp == 16 && ntiles > 0) {
        tc_alloc(smem_addr(&ms.tmem_base), kTmemCols);
        tc_relinquish();
    }
    if (warp < 16 && ntiles > 0) fill_table(a, ms, 0, ntiles, threadIdx.x);
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

    if (warp >= 16) {
        // ------------------------------- MMA issuers -------------------------------
        // One thread issues a tcgen05.mma only every ~100 cycles, longer than an M=128, N=64, K=16
        // MMA takes, so four warps issue: QK of the even chunks into S partial 0 and of the odd
        // chunks into partial 1 (M-tile by M-tile as the dequantisation finishes them), and PV of
        // M-tiles 0, 1 and of M-tiles 2, 3, one M-tile after the other so that the first two are
        // released early.
        const int r = warp - 16;
        if (lane == 0) {
            const uint32_t sV = smem_addr(V), sQ = smem_addr(Q), sP = smem_addr(P);
            bool ok = true;
            if (r < 2) {
                ok = mbar_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
                for (int t = 0; ok && t < ntiles; ++t) {
                    // S is read by every group's softmax of the previous tile
                    if (t > 0 && !(ok = mbar_wait(&ms.p_full, (t - 1) & 1, &ms.abort_flag, a.ws, 3))) break;
                    for (int i = 0; i < 4; ++i) {
                        const int m = release_order(i);
                        if (!(ok = mbar_wait(&ms.v_ready[m], t & 1, &ms.abort_flag, a.ws, 2))) break;
                        tc_fence_after();
                        const int c = 2 * m + r;
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = umma_sdesc_sw128(sV + c * kVChunk + kk * 32, 16, 1024);
                            const uint64_t bd = umma_sdesc_sw128(sQ + c * kQChunk + kk * 32, 16, 1024);
                            tc_mma_f16(tmem + kColS + 64 * r, ad, bd, kIdescQK, (i > 0 || kk > 0) ? 1u : 0u);
                        }
                    }
                    if (!ok) break;
                    tc_commit(smem_addr(&ms.s_full));
                }
            } else {
                for (int t = 0; ok && t < ntiles; ++t) {
                    if (!(ok = mbar_wait(&ms.p_full, t & 1, &ms.abort_flag, a.ws, 3))) break;
                    tc_fence_after();
                    for (int m = 2 * (r - 2); m < 2 * (r - 2) + 2; ++m) {
#pragma unroll
                        for (int kk = 0; kk < kTcRows / 16; ++kk) {
                            const uint64_t ad = umma_sdesc_sw128(sV + 2 * m * kVChunk + kk * 2048, kVChunk, 1024);
                            const uint64_t bd = umma_sdesc_sw128(sP + kk * 2048, kVChunk, 1024);
                            tc_mma_f16(tmem + kColO + 64 * m, ad, bd, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
                        }
                        tc_commit(smem_addr(&ms.v_free[m]));
                    }
                    if (t == ntiles - 1) tc_commit(smem_addr(&ms.o_done));
                }
            }
            // every MMA this thread issued has completed before TMEM is released
            tc_commit(smem_addr(&ms.final_bar[r]));
            volatile int no_abort = 0;
            mbar_wait(&ms.final_bar[r], 0, &no_abort, a.ws, 4);
        }
        __syncwarp();
    } else {
        // ------------------- compute groups: group g = warps 4g .. 4g+3 -------------------
        const int g = warp >> 2;
        const int bar_id = 1 + g;            // named barrier of the group
        const int e = threadIdx.x & 127;     // TMEM lane = tile row (entry); channel in the epilogue
        const int wq = warp & 3;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
        const int hb = kTcHeadsPerGroup * g;  // this group's first head
        const uint32_t tcol_l = tl + kColL + hb;   // this thread's row of per-head sums
        if (e < kTcHeadsPerGroup) ms.mx[g][e] = kNoMax;
        {
            float zero[kTcHeadsPerGroup];
#pragma unroll
            for (int q = 0; q < kTcHeadsPerGroup; ++q) zero[q] = 0.f;
            tc_st16(tcol_l, zero);
            tc_wait_st();
        }
        RawTile raw;
        // tile 0 straight in; tile 1's bytes in flight while the loop starts
        raw.fetch(a, ms.rows[0][e], g);
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            raw.write(a, V, m, e, g);
            fence_async_smem();
            mbar_arrive(&ms.v_ready[m]);
        }
        bool valid_cur = raw.row != -1;
        if (ntiles > 1) raw.fetch(a, ms.rows[1][e], g);
        bool ok = warp_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
        ok = group_and(bar_id, ok);   // also orders the maxima's initial values before their first use
        // After a failed wait the loop still runs to the end, skipping the work, so that every thread
        // takes the same compute-wide barriers (the entry-table refills); ok is uniform in a group.
        for (int t = 0; t < ntiles; ++t) {
            const uint32_t ph = t & 1;
            ok = group_and(bar_id, ok && warp_wait(&ms.s_full, ph, &ms.abort_flag, a.ws, 6));
            if (ok) {
                tc_fence_after();
                // scores of this group's 16 heads: the sum of the partial accumulators
                float z[kTcHeadsPerGroup];
                load_scores(tl + kColS + hb, valid_cur, zs, z);
                bool need = false;
#pragma unroll
                for (int q = 0; q < kTcHeadsPerGroup; ++q) need |= z[q] > ms.mx[g][q] + kLazy;
                if (group_or(bar_id, need)) {
                    // new maxima: per head one warp max-reduction on order keys, then over the group's warps
#pragma unroll
                    for (int q = 0; q < kTcHeadsPerGroup; ++q) {
                        const uint32_t u = __reduce_max_sync(0xffffffffu, order_key(z[q]));
                        if (lane == 0) ms.red[g][wq][q] = key_to_float(u);
                    }
                    group_sync(bar_id);
                    if (e < kTcHeadsPerGroup) {
                        const float mt = fmaxf(fmaxf(ms.red[g][0][e], ms.red[g][1][e]), fmaxf(ms.red[g][2][e], ms.red[g][3][e]));
                        const float mo = ms.mx[g][e];
                        const float mn = fmaxf(mo, mt);
                        ms.alpha[g][e] = exp2f(mo - mn);   // 0 while mo is kNoMax
                        ms.mx[g][e] = mn;
                    }
                    group_sync(bar_id);   // new maxima and factors visible; ms.red free again
                    // this thread's sums, and (after the first tile) this group's head columns of the four
                    // O^T M-tiles.  PV(t-1) has completed: QK(t) was issued only after every M-tile of
                    // tile t had been written, each after PV(t-1) had released it (v_free)
                    {
                        float lv[kTcHeadsPerGroup];
                        tc_ld16_sync(tcol_l, lv);
#pragma unroll
                        for (int q = 0; q < kTcHeadsPerGroup; ++q) lv[q] *= ms.alpha[g][q];
                        tc_st16(tcol_l, lv);
                    }
                    if (t > 0) {
#pragma unroll 1
                        for (int mt = 0; mt < 4; ++mt) {
                            float o[kTcHeadsPerGroup];
                            const uint32_t col = kColO + 64 * mt + hb;
                            tc_ld16_sync(tl + col, o);
#pragma unroll
                            for (int q = 0; q < kTcHeadsPerGroup; ++q) o[q] *= ms.alpha[g][q];
                            tc_st16(tl + col, o);
                        }
                    }
                    tc_wait_st();
                    load_scores(tl + kColS + hb, valid_cur, zs, z);   // again, rather than kept live
                }
                float lv[kTcHeadsPerGroup];
                tc_ld16_sync(tcol_l, lv);
                uint32_t pk[kTcHeadsPerGroup / 2];
#pragma unroll
                for (int q = 0; q < kTcHeadsPerGroup; q += 2) {
                    const float p0 = exp2f(z[q] - ms.mx[g][q] + kPOffset);
                    const float p1 = exp2f(z[q + 1] - ms.mx[g][q + 1] + kPOffset);
                    lv[q] += p0;
                    lv[q + 1] += p1;
                    pk[q / 2] = pack_f16x2(p0, p1);
                }
                tc_st16(tcol_l, lv);
                *reinterpret_cast<uint4 *>(P + swz((uint32_t)e, (uint32_t)(2 * g))) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
                *reinterpret_cast<uint4 *>(P + swz((uint32_t)e, (uint32_t)(2 * g + 1))) =
                    make_uint4(pk[4], pk[5], pk[6], pk[7]);
                fence_async_smem();
                tc_wait_st();
                tc_fence_before();
            }
            mbar_arrive(&ms.p_full);
            if (t + 1 < ntiles) {
                // every M-tile of tile t+1 as PV(t) releases it; then the bytes of tile t+2 are
                // requested, to arrive while tile t+1 is processed
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int m = release_order(i);
                    ok = group_and(bar_id, ok && warp_wait(&ms.v_free[m], ph, &ms.abort_flag, a.ws, 5));
                    if (ok) raw.write(a, V, m, e, g);
                    fence_async_smem();
                    mbar_arrive(&ms.v_ready[m]);
                }
                valid_cur = raw.row != -1;
                if (t + 2 < ntiles) {
                    if ((t + 2) % kTabTiles == 0) {
                        // the next tiles' entry addresses (every thread has fetched from the old ones)
                        compute_sync();
                        fill_table(a, ms, t + 2, ntiles, threadIdx.x);
                        compute_sync();
                    }
                    raw.fetch(a, ms.rows[(t + 2) % kTabTiles][e], g);
                }
            }
        }
        // ---- epilogue: this group's share of the split's partial (o, m, l): channels 128g + e of
        // every head (O^T M-tile g, lane e) and the (m, l) of heads hb .. hb+15
        float *po = a.part_o + (((size_t)b * a.splits + s) * a.H + h0) * kLatent;
        float2 *pml = reinterpret_cast<float2 *>(a.part_ml) + ((size_t)b * a.splits + s) * a.H + h0;
        bool eok = ok && warp_wait(&ms.o_done, 0, &ms.abort_flag, a.ws, 8);
        eok = group_and(bar_id, eok);
        if (eok) {
            tc_fence_after();
#pragma unroll
            for (int hq = 0; hq < kTcHeads; hq += 16) {
                float o[16];
                tc_ld16_sync(tmem + ((uint32_t)(wq * 32) << 16) + kColO + 64 * g + hq, o);
#pragma unroll
                for (int q = 0; q < 16; ++q) po[(size_t)(hq + q) * kLatent + 128 * g + e] = o[q];
            }
            // softmax denominators: sum of the per-row sums over the group's 128 rows
            float lv[kTcHeadsPerGroup];
            tc_ld16_sync(tcol_l, lv);
#pragma unroll
            for (int q = 0; q < kTcHeadsPerGroup; ++q) {
                float v = lv[q];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) ms.red[g][wq][q] = v;
            }
            group_sync(bar_id);
            if (e < kTcHeadsPerGroup) {
                const float lsum = (ms.red[g][0][e] + ms.red[g][1][e]) + (ms.red[g][2][e] + ms.red[g][3][e]);
                pml[hb + e] = make_float2((ms.mx[g][e] - kPOffset) * kLn2, lsum);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 16) tc_dealloc(tmem, kTmemCols);
}

bool attn_tc_supported(int H) { return H == 64 || H == 128; }

int attn_units_per_tile(int H) { return attn_tc_supported(H) ? kTcUnits : 4; }

bool attn_tc_layer_ok(int num_pages, int num_rows)
{
    // the entry table holds FP4 cache rows and window slots as int32
    return (long long)num_pages * kPage < (1ll << 31) && (long long)num_rows * kWindow < (1ll << 30);
}

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
