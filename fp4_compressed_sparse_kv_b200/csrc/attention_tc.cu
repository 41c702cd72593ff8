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
// Work unit: a half-tile of 64 entries.  Two half-tiles are in flight, each with its own V and P
// buffer, so the dequantisation of one overlaps the MMAs and the softmax of the other.
//   QK:  S^T[64 entries x 64 heads] = V[64 x 512] . Q^T        (M = 64; A = V K-major, B = Q K-major)
//   PV:  O^T[128 ch x 64 heads] (x4) += V^T[128 ch x 64 entries] . P^T  (A = V^T MN-major, B = P^T MN-major)
// The same 128-byte-swizzled fp16 copy of a half-tile is read as K-major V by QK and as MN-major V^T
// by PV.  TMEM: O^T in 4 x 64 columns; S^T as four partial accumulators (one per MMA issuer, summed
// by the softmax) in 4 x 64 columns, an M=64 accumulator taking 16 lanes of every 32: half-tile t
// in the lower 16 lanes of each quarter when t is even, the upper 16 when odd.
//
// Warp roles (640 threads).
//   warps 0-7   producers: thread (e, cp) dequantises channels 128cp .. 128cp+127 of entry e from raw
//               bytes it loaded two half-tiles earlier, once PV has released the buffer;
//   warps 8-15  softmax: two groups of four warps, heads 32s .. 32s+31; a warp reads the 16 score rows
//               of its TMEM quarter with 16-lane loads (thread t: rows t/4 and t/4+8, 8 heads);
//   warps 16-19 MMA issuers (lane 0; warp 16 also owns the TMEM allocation).  One thread issues a
//               tcgen05.mma only every ~100 cycles, longer than these MMAs take, so issuer r does QK
//               of chunks r and r+4 (into S partial r) and PV of M-tile r, QK one half-tile ahead.
// Softmax rescales lazily: O^T is rescaled in TMEM only when a head's running maximum grows by more
// than 2^8 (after waiting for the previous half-tile's PV).
#include "attention_common.cuh"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace csa {

constexpr int kTcHeads = 64;
constexpr int kHalf = 64;                        // entries per half-tile
constexpr int kHalfUnits = kHalf / kAttnUnit;    // 8 units of 8 entries
constexpr int kTcUnits = 2 * kHalfUnits;         // units per 128-entry tile (split sizing)
constexpr int kTcChunks = kLatent / 64;          // 8 chunks of 64 channels
constexpr int kProducers = 256;                  // warps 0-7
constexpr int kSoftmax = 256;                    // warps 8-15
constexpr int kTcThreads = 640;
constexpr int kTcCompute = kProducers + kSoftmax;
constexpr uint32_t kVChunk = kHalf * 128;        // 8 KB: 64 rows x 64 fp16
constexpr uint32_t kVBuf = kTcChunks * kVChunk;  // 64 KB per half-tile buffer
constexpr uint32_t kQChunk = kTcHeads * 128;     // 8 KB: 64 rows x 64 fp16
constexpr uint32_t kPBuf = kHalf * 128;          // 8 KB: 64 entry rows x 64 heads fp16
constexpr int kTabHalves = 32;                   // half-tiles of entry addresses resolved at a time
constexpr uint32_t kOffV = 0;
constexpr uint32_t kOffQ = kOffV + 2 * kVBuf;
constexpr uint32_t kOffP = kOffQ + kTcChunks * kQChunk;
constexpr uint32_t kOffTab = kOffP + 2 * kPBuf;
constexpr uint32_t kOffMisc = kOffTab + kTabHalves * kHalf * 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;                    // O^T: M-tile m in columns 64m .. 64m+63
constexpr uint32_t kColS = 256;                  // S^T partial r in columns 256 + 64r ..
constexpr float kLazy = 8.f;      // log2-domain growth of a head maximum tolerated without rescaling
constexpr float kPOffset = 7.f;   // p = exp2(z - m + 7) <= 2^15 keeps small p out of fp16 subnormals
constexpr float kNoMax = -1e30f;  // running maximum before any finite score (exp2 of it minus a finite value is 0)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcMisc {
    uint64_t q_ready, o_done;
    uint64_t v_ready[2], v_free[2], s_full[2], p_full[2];
    uint64_t final_bar[4];
    uint32_t tmem_base;
    int abort_flag;
    int u_begin, u_end;                          // this split's units
    SeqView sv;                                  // the sequence, read from here by every thread
    float qmax[16];                              // per Q-loading warp: largest |q| of its rows
    float mx[kTcHeads];                          // running maximum of each head (log2 domain)
    float alpha[kTcHeads];                       // rescale factor of each head at a maximum update
    float red[2][4][32];                         // per softmax group and warp: a per-head partial
    uint64_t vmask[2];                           // valid rows of the half-tile in each V buffer
};

constexpr size_t kTcSmem = kOffMisc + sizeof(TcMisc) + 1024;

constexpr uint32_t kIdescQK = umma_idesc_f16(64, kTcHeads, false, false);
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

// Named barriers: 1, 2 = the two softmax groups (128 threads each); 3 = the producers (256);
// 4 = producers and softmax warps (512).  Every participant executes each of them the same number of
// times, also after a failed wait.
__device__ __forceinline__ bool bar_and(int id, int n, bool v)
{
    int r;
    asm volatile("{\n.reg .pred p, q;\nsetp.ne.b32 q, %3, 0;\nbar.red.and.pred p, %1, %2, q;\nselp.b32 %0, 1, 0, p;\n}"
                 : "=r"(r)
                 : "r"(id), "r"(n), "r"((int)v)
                 : "memory");
    return r != 0;
}

__device__ __forceinline__ bool bar_or(int id, int n, bool v)
{
    int r;
    asm volatile("{\n.reg .pred p, q;\nsetp.ne.b32 q, %3, 0;\nbar.red.or.pred p, %1, %2, q;\nselp.b32 %0, 1, 0, p;\n}"
                 : "=r"(r)
                 : "r"(id), "r"(n), "r"((int)v)
                 : "memory");
    return r != 0;
}

__device__ __forceinline__ void bar_sync(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// 16 lanes x (4 x 8) columns: thread t gets rows t/4 and t/4 + 8 of the 16 lanes at taddr, columns
// 8j + 2(t%4) and 8j + 2(t%4) + 1 for j = 0..3: v[4j] (row t/4, even column), v[4j+1] (row t/4, odd),
// v[4j+2], v[4j+3] (row t/4 + 8).  Waited for in the same statement.
__device__ __forceinline__ void tc_ld16x256_x4_sync(uint32_t taddr, float *v)
{
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive 32-bit columns (thread i: lane i), waited for in the same statement.
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

// Half-tile-aligned split of a sequence's units: split s of `splits` gets whole 8-unit half-tiles,
// so every half-tile but the sequence's last is full.
__device__ __forceinline__ void split_halves(int units, int s, int splits, int &ub, int &ue)
{
    const int halves = (units + kHalfUnits - 1) / kHalfUnits;
    const int hb = (int)((long long)halves * s / splits), he = (int)((long long)halves * (s + 1) / splits);
    ub = hb * kHalfUnits;
    ue = he * kHalfUnits < units ? he * kHalfUnits : units;
}

// Entry table: for each row e of each half-tile, the FP4 cache row (page * 64 + offset) of the entry,
// -(slot + 2) for a window entry, or -1 for a masked row (past the split or the sequence).

// A producer thread's share of one half-tile: entry e, channels 128cp .. 128cp+127 (V chunks 2cp,
// 2cp+1).  The raw bytes of an FP4 entry (64 B of codes, 8 scale bytes, contiguous) are loaded
// into registers two half-tiles before they are dequantised; a window entry (128 E4M3 values) is
// read when it is written, since the window is at most two half-tiles of a sequence.  (A mapping in
// which one warp-wide load covers two whole entries loads fewer lines but writes the swizzled
// V rows with 4-way bank conflicts, which costs more.)
struct RawHalf {
    uint4 code[4];
    uint2 sc;
    int32_t row;

    __device__ __forceinline__ void fetch(const AttnArgs &a, int32_t code_row, int cp)
    {
        row = code_row;
        if (row >= 0) {
            const uint4 *cp4 = reinterpret_cast<const uint4 *>(a.codes + (size_t)row * kCodeBytes + 64 * cp);
#pragma unroll
            for (int q = 0; q < 4; ++q) code[q] = cp4[q];
            sc = *reinterpret_cast<const uint2 *>(a.scales + (size_t)row * kScaleBytes + 8 * cp);
        }
    }

    // Dequantise into V chunks 2cp + h (h = 0, 1), row e.
    __device__ __forceinline__ void write(const AttnArgs &a, uint8_t *Vb, int e, int cp) const
    {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            uint8_t *dst = Vb + (2 * cp + h) * kVChunk;
            if (row == -1) {
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, (uint32_t)jj)) = make_uint4(0u, 0u, 0u, 0u);
            } else if (row >= 0) {
                const uint32_t sw = h ? sc.y : sc.x;
#pragma unroll
                for (int gg = 0; gg < 4; ++gg) {
                    const uint32_t sh = e4m3x2_to_f16x2((uint16_t)((sw >> (8 * gg)) & 0xFF));
                    const uint32_t s2 = (sh & 0xFFFFu) | (sh << 16);
                    const uint4 cw = code[2 * h + (gg >> 1)];
                    const uint32_t w0 = (gg & 1) ? cw.z : cw.x, w1 = (gg & 1) ? cw.w : cw.y;
                    uint32_t v[8];
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        v[q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w0 >> (8 * q))), s2);
                        v[4 + q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w1 >> (8 * q))), s2);
                    }
                    *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, (uint32_t)(2 * gg))) =
                        make_uint4(v[0], v[1], v[2], v[3]);
                    *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, (uint32_t)(2 * gg + 1))) =
                        make_uint4(v[4], v[5], v[6], v[7]);
                }
            } else {
                // window entry: 64 E4M3 values times the entry's binary32 scale, rounded to fp16
                const size_t slot = (size_t)(-row - 2);
                const float fs = a.swa_scale[slot];
                const uint4 *src = reinterpret_cast<const uint4 *>(a.swa + slot * kLatent + 128 * cp + 64 * h);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
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
                    *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, (uint32_t)(2 * q))) = make_uint4(v[0], v[1], v[2], v[3]);
                    *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, (uint32_t)(2 * q + 1))) =
                        make_uint4(v[4], v[5], v[6], v[7]);
                }
            }
        }
    }
};

// Fill the entry table with half-tiles t0 .. t0 + kTabHalves - 1: producer thread i takes unit i of
// the range (8 entries: one selected block, or 8 window positions), so the block id and the page
// table are read once per unit, in two rounds of independent loads.
static_assert(kTabHalves * kHalfUnits == kProducers, "one unit of the table per producer thread");
__device__ __forceinline__ void fill_table(const AttnArgs &a, TcMisc &ms, int32_t *tab, int t0, int tid)
{
    const SeqView &sv = ms.sv;
    const int u = ms.u_begin + t0 * kHalfUnits + tid;
    int32_t *out = tab + tid * kAttnUnit;
    int32_t code = -1;         // code of position 0 of the unit, or -1 for none
    int limit = 0;             // positions j < limit of the unit are valid
    if (u < ms.u_end) {
        if (u < sv.nE) {
            const int blk = sv.blocks[u];
            if (blk < 0 || blk >= sv.nb) {
                report(a.ws, CSA_ERR_DEVICE_DATA, u);
            } else {
                const int page = sv.bt[blk / kBlocksPerPage];
                if (page < 0 || page >= a.num_pages) {
                    report(a.ws, CSA_ERR_DEVICE_DATA, blk);
                } else {
                    code = page * kPage + (blk % kBlocksPerPage) * kBlock;
                    limit = sv.L - blk * kBlock;
                }
            }
#pragma unroll
            for (int j = 0; j < kAttnUnit; ++j) out[j] = (code >= 0 && j < limit) ? code + j : -1;
        } else {
            const int p0 = sv.w0 + (u - sv.nE) * kAttnUnit;
#pragma unroll
            for (int j = 0; j < kAttnUnit; ++j)
                out[j] = (p0 + j < sv.L) ? -(sv.row * kWindow + ((p0 + j) % kWindow) + 2) : -1;
        }
    } else {
#pragma unroll
        for (int j = 0; j < kAttnUnit; ++j) out[j] = -1;
    }
}

// Q of heads h0..h0+63 into shared memory as fp16, 128B-swizzled K-major, scaled by one power of two
// 2^k that puts the largest |q| of the 64 heads in [2^13, 2^14); returns tau * log2(e) * 2^-k, the
// factor that turns an accumulated score into the log2 domain.  Thread t (of the 512 producer and
// softmax threads) converts channels 64(t/64) .. 64(t/64)+63 of head t%64 (consecutive threads write
// different rows of one chunk, so the 16-byte stores do not collide in shared-memory banks).
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
    bar_sync(4, kTcCompute);
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

// This thread's 16 scores (rows t/4 and t/4 + 8 of its warp's quarter, 8 heads of its group) in the
// log2 domain: the sum of the four partial accumulators times zs; a masked row gives -inf.
__device__ __forceinline__ void load_scores(uint32_t taddr, bool v0, bool v1, float zs, float *z)
{
    tc_ld16x256_x4_sync(taddr, z);
#pragma unroll
    for (int r = 1; r < 4; ++r) {
        float z2[16];
        tc_ld16x256_x4_sync(taddr + 64 * r, z2);
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] += z2[i];
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const bool valid = (i & 2) ? v1 : v0;
        z[i] = valid ? z[i] * zs : -INFINITY;
    }
}

__global__ void __launch_bounds__(kTcThreads, 1) attn_split_tc_kernel(AttnArgs a, int head_groups)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *V = base + kOffV;
    uint8_t *Q = base + kOffQ;
    uint8_t *P = base + kOffP;
    int32_t *tab = reinterpret_cast<int32_t *>(base + kOffTab);
    TcMisc &ms = *reinterpret_cast<TcMisc *>(base + kOffMisc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_launch();   // the combine may be scheduled as splits finish
    const int s = blockIdx.x, b = blockIdx.y / head_groups, hg = blockIdx.y % head_groups;
    const int h0 = hg * kTcHeads;

    if (threadIdx.x == 0) {
        mbar_init(&ms.q_ready, kTcCompute);
        mbar_init(&ms.o_done, 4);
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ms.v_ready[i], kProducers);
            mbar_init(&ms.v_free[i], 4);
            mbar_init(&ms.s_full[i], 4);
            mbar_init(&ms.p_full[i], kSoftmax);
        }
        for (int r = 0; r < 4; ++r) mbar_init(&ms.final_bar[r], 1);
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kTcHeads) ms.mx[threadIdx.x] = kNoMax;
    __syncthreads();
    // Q is an input of the step, not a result of the previous grid: load it while that grid finishes
    float zs = 0.f;
    if (warp < 16) zs = load_q(a, ms, Q, b, h0, threadIdx.x);
    grid_dep_wait();   // the selected blocks of the previous grid

    if (threadIdx.x == 0) {
        int ub = 0, ue = 0;
        if (seq_view(a, b, ms.sv)) split_halves(ms.sv.units, s, a.splits, ub, ue);
        ms.u_begin = ub;
        ms.u_end = ue;
    }
    __syncthreads();
    const int nh = (ms.u_end - ms.u_begin + kHalfUnits - 1) / kHalfUnits;   // half-tiles of this split
    if (warp == 16 && nh > 0) {
        tc_alloc(smem_addr(&ms.tmem_base), kTmemCols);
        tc_relinquish();
    }
    if (warp < 8 && nh > 0) fill_table(a, ms, tab, 0, threadIdx.x);
    fence_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;

    if (nh == 0) {
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

    bool ok = true;
    if (warp >= 16) {
        // ------------------------------- MMA issuers -------------------------------
        const int r = warp - 16;
        if (lane == 0) {
            const uint32_t sV = smem_addr(V), sQ = smem_addr(Q), sP = smem_addr(P);
            ok = mbar_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
            tc_fence_after();
            // QK of chunks r and r + 4 of half-tile t into S partial r, lanes of parity t % 2
            auto issue_qk = [&](int t) {
                const int p = t & 1;
                const uint32_t dS = tmem + ((uint32_t)(16 * p) << 16) + kColS + 64 * r;
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    const int c = r + 4 * i;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint64_t ad = umma_sdesc_sw128(sV + p * kVBuf + c * kVChunk + kk * 32, 16, 1024);
                        const uint64_t bd = umma_sdesc_sw128(sQ + c * kQChunk + kk * 32, 16, 1024);
                        tc_mma_f16(dS, ad, bd, kIdescQK, (i > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                tc_commit(smem_addr(&ms.s_full[p]));
            };
            // PV of M-tile r of half-tile t
            auto issue_pv = [&](int t) {
                const int p = t & 1;
#pragma unroll
                for (int kk = 0; kk < kHalf / 16; ++kk) {
                    const uint64_t ad = umma_sdesc_sw128(sV + p * kVBuf + 2 * r * kVChunk + kk * 2048, kVChunk, 1024);
                    const uint64_t bd = umma_sdesc_sw128(sP + p * kPBuf + kk * 2048, kVChunk, 1024);
                    tc_mma_f16(tmem + kColO + 64 * r, ad, bd, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
                }
                tc_commit(smem_addr(&ms.v_free[p]));
                if (t == nh - 1) tc_commit(smem_addr(&ms.o_done));
            };
            // Issue whichever is ready first: PV(pv) once the softmax has written P(pv), QK(qk) once the
            // producers have written half-tile qk, so that the chains of the even and of the odd
            // half-tiles overlap.  (QK(t) precedes PV(t) through the softmax; QK(t+2) follows PV(t)
            // through the producers, who wait for it before reusing the buffer.)  The waits are
            // polled together with non-blocking tests (a suspended test of one could miss the other's
            // completion), under the same limit as every other wait.
            int qk = 0, pv = 0;
            unsigned long long t0 = 0;
            for (uint32_t it = 0; ok && pv < nh; ++it) {
                if (pv < qk && mbar_test_wait(&ms.p_full[pv & 1], (pv >> 1) & 1)) {
                    tc_fence_after();
                    issue_pv(pv++);
                    t0 = 0;
                    continue;
                }
                if (qk < nh && mbar_test_wait(&ms.v_ready[qk & 1], (qk >> 1) & 1)) {
                    tc_fence_after();
                    issue_qk(qk++);
                    t0 = 0;
                    continue;
                }
                if ((it & 63u) == 0) {
                    volatile int *abort_flag = &ms.abort_flag;
                    if (*abort_flag) {
                        ok = false;
                    } else {
                        const unsigned long long now = global_ns();
                        if (t0 == 0) {
                            t0 = now;
                        } else if (now - t0 > kWaitLimitNs) {
                            *abort_flag = 1;
                            report(a.ws, CSA_ERR_TIMEOUT, 2);
                            ok = false;
                        }
                    }
                }
            }
            // every MMA this thread issued has completed before TMEM is released
            tc_commit(smem_addr(&ms.final_bar[r]));
            volatile int no_abort = 0;
            mbar_wait(&ms.final_bar[r], 0, &no_abort, a.ws, 4);
        }
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------- producers -------------------------------
        // After a failed wait the loop still runs to the end, skipping the work, so that every
        // producer takes the same barriers (the entry-table refills).
        const int d = threadIdx.x, e = d & (kHalf - 1), cp = d >> 6;
        RawHalf raw0, raw1;   // half-tiles of even and of odd index
        raw0.fetch(a, tab[e], cp);
        if (nh > 1) raw1.fetch(a, tab[kHalf + e], cp);
        auto step = [&](int t, RawHalf &rw) {
            const int p = t & 1;
            if (t >= 2) ok = ok && warp_wait(&ms.v_free[p], ((t >> 1) - 1) & 1, &ms.abort_flag, a.ws, 5);
            if (ok) rw.write(a, V + p * kVBuf, e, cp);
            if (cp == 0) {
                const unsigned int vb = __ballot_sync(0xffffffffu, rw.row != -1);
                if (lane == 0) reinterpret_cast<volatile uint32_t *>(&ms.vmask[p])[warp] = vb;
            }
            fence_async_smem();
            mbar_arrive(&ms.v_ready[p]);
            if (t + 2 < nh) {
                if ((t + 2) % kTabHalves == 0) {
                    // the next half-tiles' entry addresses (every producer has fetched from the old ones)
                    bar_sync(3, kProducers);
                    fill_table(a, ms, tab, t + 2, d);
                    bar_sync(3, kProducers);
                }
                rw.fetch(a, tab[((t + 2) % kTabHalves) * kHalf + e], cp);
            }
        };
#pragma unroll 1
        for (int t = 0; t < nh; t += 2) {
            step(t, raw0);
            if (t + 1 < nh) step(t + 1, raw1);
        }
    } else {
        // ------------------------------- softmax -------------------------------
        const int sg = (warp - 8) >> 2;         // group: heads 32sg .. 32sg+31
        const int q = warp & 3;                 // TMEM quarter: lanes 32q .. 32q+31
        const int gt = threadIdx.x & 127;       // thread within the group
        const int bar_id = 1 + sg;
        const int R0 = 16 * q + (lane >> 2);    // half-tile rows of this thread: R0 and R0 + 8
        const int hc = 2 * (lane & 3);          // head columns: 32sg + 8j + hc, +1 (j = 0..3)
        float l[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) l[i] = 0.f;
        ok = warp_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
        for (int t = 0; t < nh; ++t) {
            const int p = t & 1;
            const uint32_t ph = (t >> 1) & 1;
            // v_ready: the producers' valid-row mask of this half-tile; s_full: its scores
            ok = bar_and(bar_id, 128, ok && warp_wait(&ms.v_ready[p], ph, &ms.abort_flag, a.ws, 9) &&
                                          warp_wait(&ms.s_full[p], ph, &ms.abort_flag, a.ws, 6));
            if (ok) {
                tc_fence_after();
                const uint64_t vm = ms.vmask[p];
                const bool v0 = (vm >> R0) & 1, v1 = (vm >> (R0 + 8)) & 1;
                const uint32_t taddr = tmem + ((uint32_t)(32 * q + 16 * p) << 16) + kColS + 32 * sg;
                float z[16];
                load_scores(taddr, v0, v1, zs, z);
                // z[4j + c]: row R0, z[4j + 2 + c]: row R0 + 8; head 32sg + 8j + hc + c
                bool need = false;
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        const float mo = ms.mx[32 * sg + 8 * j + hc + c] + kLazy;
                        need |= z[4 * j + c] > mo || z[4 * j + 2 + c] > mo;
                    }
                if (bar_or(bar_id, 128, need)) {
                    // new maxima: over this thread's two rows, the warp's 8 row pairs, then the 4 warps
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            float m2 = fmaxf(z[4 * j + c], z[4 * j + 2 + c]);
                            m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, 4));
                            m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, 8));
                            m2 = fmaxf(m2, __shfl_xor_sync(0xffffffffu, m2, 16));
                            if (lane < 4) ms.red[sg][q][8 * j + hc + c] = m2;
                        }
                    bar_sync(bar_id, 128);
                    if (gt < 32) {
                        const int h = 32 * sg + gt;
                        const float mt = fmaxf(fmaxf(ms.red[sg][0][gt], ms.red[sg][1][gt]),
                                               fmaxf(ms.red[sg][2][gt], ms.red[sg][3][gt]));
                        const float mo = ms.mx[h];
                        const float mn = fmaxf(mo, mt);
                        ms.alpha[h] = exp2f(mo - mn);   // 0 while mo is kNoMax
                        ms.mx[h] = mn;
                    }
                    bar_sync(bar_id, 128);   // new maxima and factors visible; ms.red free again
#pragma unroll
                    for (int j = 0; j < 4; ++j)
#pragma unroll
                        for (int c = 0; c < 2; ++c) l[2 * j + c] *= ms.alpha[32 * sg + 8 * j + hc + c];
                    if (t > 0) {
                        // this group's head columns of the four O^T M-tiles, once PV(t-1) has completed
                        const bool pv_ok = warp_wait(&ms.v_free[(t - 1) & 1], ((t - 1) >> 1) & 1, &ms.abort_flag, a.ws, 7);
                        if (pv_ok) {
                            tc_fence_after();
                            const uint32_t tl = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
                            for (int k = 0; k < 8; ++k) {
                                float o[16];
                                const uint32_t col = kColO + 64 * (k >> 1) + 32 * sg + 16 * (k & 1);
                                tc_ld16_sync(tl + col, o);
#pragma unroll
                                for (int i = 0; i < 16; ++i) o[i] *= ms.alpha[32 * sg + 16 * (k & 1) + i];
                                tc_st16(tl + col, o);
                            }
                            tc_wait_st();
                        }
                        ok = pv_ok;
                    }
                    load_scores(taddr, v0, v1, zs, z);   // again, rather than kept live
                }
                // P^T rows R0, R0 + 8 (entries), this thread's 8 heads: 4-byte pairs
                uint8_t *Pb = P + p * kPBuf;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int hh = 32 * sg + 8 * j + hc;
                    const float m0 = ms.mx[hh] - kPOffset, m1 = ms.mx[hh + 1] - kPOffset;
                    const float p00 = exp2f(z[4 * j] - m0), p01 = exp2f(z[4 * j + 1] - m1);
                    const float p10 = exp2f(z[4 * j + 2] - m0), p11 = exp2f(z[4 * j + 3] - m1);
                    l[2 * j] += p00 + p10;
                    l[2 * j + 1] += p01 + p11;
                    const uint32_t unit = (uint32_t)(4 * sg + j), off = 4u * (uint32_t)(lane & 3);
                    *reinterpret_cast<uint32_t *>(Pb + swz((uint32_t)R0, unit) + off) = pack_f16x2(p00, p01);
                    *reinterpret_cast<uint32_t *>(Pb + swz((uint32_t)(R0 + 8), unit) + off) = pack_f16x2(p10, p11);
                }
                fence_async_smem();
                tc_fence_before();
            }
            mbar_arrive(&ms.p_full[p]);
        }
        // softmax denominators: per head, the sum over the group's threads
        if (bar_and(bar_id, 128, ok)) {
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                float v = l[i];
                v += __shfl_xor_sync(0xffffffffu, v, 4);
                v += __shfl_xor_sync(0xffffffffu, v, 8);
                v += __shfl_xor_sync(0xffffffffu, v, 16);
                l[i] = v;
            }
            if (lane < 4) {
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    ms.red[sg][q][8 * j + hc] = l[2 * j];
                    ms.red[sg][q][8 * j + hc + 1] = l[2 * j + 1];
                }
            }
            bar_sync(bar_id, 128);
            if (gt < 32) {
                const int h = 32 * sg + gt;
                const float lsum = (ms.red[sg][0][gt] + ms.red[sg][1][gt]) + (ms.red[sg][2][gt] + ms.red[sg][3][gt]);
                float2 *pml = reinterpret_cast<float2 *>(a.part_ml) + ((size_t)b * a.splits + s) * a.H + h0;
                pml[h] = make_float2((ms.mx[h] - kPOffset) * kLn2, lsum);
            }
        }
    }
    // ---- epilogue: O^T, M-tile w/4, quarter w%4, by every producer and softmax warp
    if (warp < 16) {
        const bool eok = bar_and(4, kTcCompute, ok && warp_wait(&ms.o_done, 0, &ms.abort_flag, a.ws, 8));
        if (eok) {
            tc_fence_after();
            const int m = warp >> 2, qq = warp & 3;
            float *po = a.part_o + (((size_t)b * a.splits + s) * a.H + h0) * kLatent + 128 * m + 32 * qq + lane;
#pragma unroll
            for (int hq = 0; hq < kTcHeads; hq += 16) {
                float o[16];
                tc_ld16_sync(tmem + ((uint32_t)(32 * qq) << 16) + kColO + 64 * m + hq, o);
#pragma unroll
                for (int i = 0; i < 16; ++i) po[(size_t)(hq + i) * kLatent] = o[i];
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
