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
// Work unit: a tile of 64 entries.  Three tiles are in flight, each with its own 64 KB fp16 V buffer
// (128-byte swizzle) and 8 KB P buffer in shared memory; Q lives in TMEM, which is what leaves room
// for the third buffer.
//   QK:  S_x[64 heads x 64 entries] = Q_x . V_x^T for the channel halves x = 0, 1 (M = 64; A = Q_x
//        read from TMEM, B = V K-major).  An MMA that reads A from TMEM writes D at the same lanes, so
//        half x keeps Q_x and its two S_x buffers in the 16-lane half x of every TMEM lane quarter:
//        head m in lane 32(m/16) + 16x + m%16; Q_x in columns 256..383 (two fp16 channels per column,
//        the even channel low), S_x of tile t in columns 384 + 64(t%2).
//   PV:  O^T[128 ch x 64 heads] (x4) += V^T[128 ch x 64 entries] . P^T  (M = 128; A = V^T MN-major,
//        B = P^T K-major: one 128-byte row of 64 entries per head), O^T in columns 0..255 of all lanes.
// The same swizzled fp16 copy of a tile is read as K-major V by QK and as MN-major V^T by PV.
//
// Warp roles (768 threads).
//   warps 0-15  producers: thread (e, cp) dequantises channels 64cp .. 64cp+63 of entry e (V chunk
//               cp) into registers one tile ahead and stores them once PV has released the
//               buffer; they also load Q and write O^T at the end;
//   warps 16-19 softmax, warp 16+q on TMEM quarter q (heads 16q .. 16q+15): lane l owns entries
//               32(l/16) .. 32(l/16)+31 of head 16q + l%16 and reads both channel halves' scores of
//               them with 16-lane loads split between the half-warps, so a head's maximum and sum
//               need one shuffle (with lane l^16, which owns the head's other 32 entries);
//   warps 20-23 MMA issuers (lane 0): 20, 21 = QK of channel half 0, 1 (warp 20 also owns the TMEM
//               allocation); 22, 23 = PV of M-tiles 0-1, 2-3.  Two issuers per product, because one
//               thread issues a tcgen05.mma only every ~65 cycles, twice what an M=64 MMA takes.
// Softmax rescales lazily: O^T is rescaled in TMEM only when a head's running maximum grows by more
// than 2^8 (after waiting for the previous tile's PV).
#include "attention_common.cuh"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace csa {

constexpr int kTcHeads = 64;
constexpr int kTile = 64;                        // entries per tile
constexpr int kTileUnits = kTile / kAttnUnit;    // 8 units of 8 entries
constexpr int kTcUnits = 2 * kTileUnits;         // units per 128 entries (split sizing)
constexpr int kTcChunks = kLatent / 64;          // 8 chunks of 64 channels
constexpr int kStages = 3;                       // tiles in flight
constexpr int kProducers = 512;                  // warps 0-15
constexpr int kSoftmax = 128;                    // warps 16-19
constexpr int kSoftmaxWarp = 16;
constexpr int kIssuerWarp = 20;                  // warps 20-23
constexpr int kTcThreads = 768;
constexpr uint32_t kVChunk = kTile * 128;        // 8 KB: 64 rows x 64 fp16
constexpr uint32_t kVBuf = kTcChunks * kVChunk;  // 64 KB per tile buffer
constexpr uint32_t kPBuf = kTcHeads * 128;       // 8 KB: 64 head rows x 64 entries fp16
constexpr int kTabTiles = 32;                    // tiles of entry addresses resolved at a time
constexpr uint32_t kOffV = 0;
constexpr uint32_t kOffP = kOffV + kStages * kVBuf;
constexpr uint32_t kOffTab = kOffP + kStages * kPBuf;
constexpr uint32_t kOffMisc = kOffTab + kTabTiles * kTile * 4;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0;                    // O^T: M-tile m in columns 64m .. 64m+63
constexpr uint32_t kColQ = 256;                  // Q_x: 128 columns in lane half x
constexpr uint32_t kColS = 384;                  // S_x of tile t: columns 384 + 64(t%2) in lane half x
constexpr float kLazy = 8.f;      // log2-domain growth of a head maximum tolerated without rescaling
constexpr float kPOffset = 7.f;   // p = exp2(z - m + 7) <= 2^15 keeps small p out of fp16 subnormals
constexpr float kNoMax = -1e30f;  // running maximum before any finite score (exp2 of it minus a finite value is 0)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcMisc {
    uint64_t q_ready, o_done;
    uint64_t v_ready[kStages], v_free[kStages], p_full[kStages];
    uint64_t s_full[2], s_free[2];
    uint64_t final_bar[4];
    uint32_t tmem_base;
    int abort_flag;
    int u_begin, u_end;                          // this split's units
    SeqView sv;                                  // the sequence, read from here by every thread
    float qmax[16];                              // per Q-loading warp: largest |q| of its part of Q
    float alpha[kTcHeads];                       // rescale factor of each head at a maximum update
    uint64_t vmask[kStages];                     // valid rows of the tile in each V buffer
};

constexpr size_t kTcSmem = kOffMisc + sizeof(TcMisc) + 1024;

constexpr uint32_t kIdescQK = umma_idesc_f16(64, kTile, false, false);
constexpr uint32_t kIdescPV = umma_idesc_f16(128, kTcHeads, true, false);

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

// Named barriers: 1 = the softmax warps (128 threads); 3 = the producers (512); 4 = every warp (768).
// Every participant executes each of them the same number of times, also after a failed wait.
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

// Tile-aligned split of a sequence's units: split s of `splits` gets whole 8-unit tiles, so every
// tile but the sequence's last is full.
__device__ __forceinline__ void split_tiles(int units, int s, int splits, int &ub, int &ue)
{
    const int tiles = (units + kTileUnits - 1) / kTileUnits;
    const int hb = (int)((long long)tiles * s / splits), he = (int)((long long)tiles * (s + 1) / splits);
    ub = hb * kTileUnits;
    ue = he * kTileUnits < units ? he * kTileUnits : units;
}

// Entry table: for each row e of each tile, the FP4 cache row (page * 64 + offset) of the entry,
// -(slot + 2) for a window entry, or -1 for a masked row (past the split or the sequence).

// A producer thread's share of one tile: entry e, channels 64cp .. 64cp+63 (V chunk cp).  The raw
// bytes of an FP4 entry (32 B of codes, 4 scale bytes) are loaded into registers two tiles ahead
// and dequantised one tile ahead, so that once PV releases the buffer only the stores remain; a
// window entry (64 E4M3 values) is read when it is dequantised, since the window is at most two
// tiles of a sequence.
struct RawEntry {
    uint4 code[2];
    uint32_t sc;
    int32_t row;

    __device__ __forceinline__ void fetch(const AttnArgs &a, int32_t code_row, int cp)
    {
        row = code_row;
        if (row >= 0) {
            const uint4 *cp4 = reinterpret_cast<const uint4 *>(a.codes + (size_t)row * kCodeBytes + 32 * cp);
            code[0] = cp4[0];
            code[1] = cp4[1];
            sc = *reinterpret_cast<const uint32_t *>(a.scales + (size_t)row * kScaleBytes + 4 * cp);
        }
    }

    // Dequantise into v: channels 64cp .. 64cp+63 as 32 fp16 pairs (zeros for a masked row).
    __device__ __forceinline__ void dequant(const AttnArgs &a, int cp, uint32_t *v) const
    {
        if (row == -1) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0u;
        } else if (row >= 0) {
            uint32_t sh[2];   // the four group scales as (s0, s1), (s2, s3)
            e4m3x4_to_f16x2x2(sc, sh);
#pragma unroll
            for (int gg = 0; gg < 4; ++gg) {
                // group gg's scale in both halves
                const uint32_t s2 = __byte_perm(sh[gg >> 1], 0u, (gg & 1) ? 0x3232u : 0x1010u);
                const uint4 cw = code[gg >> 1];
                uint32_t c0[4], c1[4];
                e2m1x8_to_f16x2x4((gg & 1) ? cw.z : cw.x, c0);
                e2m1x8_to_f16x2x4((gg & 1) ? cw.w : cw.y, c1);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    v[8 * gg + q] = hmul2_u32(c0[q], s2);
                    v[8 * gg + 4 + q] = hmul2_u32(c1[q], s2);
                }
            }
        } else {
            // window entry: 64 E4M3 values times the entry's binary32 scale, rounded to fp16
            const size_t slot = (size_t)(-row - 2);
            const float fs = a.swa_scale[slot];
            const uint4 *src = reinterpret_cast<const uint4 *>(a.swa + slot * kLatent + 64 * cp);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const uint4 w = src[q];
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    uint32_t hv[2];
                    e4m3x4_to_f16x2x2(ww[k], hv);
                    v[8 * q + 2 * k] = pack_f16x2(h_lo(hv[0]) * fs, h_hi(hv[0]) * fs);
                    v[8 * q + 2 * k + 1] = pack_f16x2(h_lo(hv[1]) * fs, h_hi(hv[1]) * fs);
                }
            }
        }
    }
};

// Row e of V chunk cp: 8 swizzled 16-byte units.
__device__ __forceinline__ void store_row(uint8_t *Vb, int e, int cp, const uint32_t *v)
{
    uint8_t *dst = Vb + cp * kVChunk;
#pragma unroll
    for (int j = 0; j < 8; ++j)
        *reinterpret_cast<uint4 *>(dst + swz((uint32_t)e, (uint32_t)j)) =
            make_uint4(v[4 * j], v[4 * j + 1], v[4 * j + 2], v[4 * j + 3]);
}

// Fill the entry table with tiles t0 .. t0 + kTabTiles - 1: thread i (of the first kTabFill
// producers) takes unit i of the range (8 entries: one selected block, or 8 window positions), so
// the block id and the page table are read once per unit, in two rounds of independent loads.
constexpr int kTabFill = kTabTiles * kTileUnits;
static_assert(kTabFill <= kProducers, "one unit of the table per filling thread");
__device__ __forceinline__ void fill_table(const AttnArgs &a, TcMisc &ms, int32_t *tab, int t0, int tid)
{
    const SeqView &sv = ms.sv;
    const int u = ms.u_begin + t0 * kTileUnits + tid;
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

__device__ __forceinline__ void tc_st16_u(uint32_t taddr, const uint32_t *v)
{
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
        "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns (thread i: lane i), waited for in the same statement; and
// the matching store.
__device__ __forceinline__ void tc_ld8_sync(uint32_t taddr, float *v)
{
    uint32_t r[8];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tc_st8(uint32_t taddr, const float *v)
{
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
}

// Two loads of 16 lanes x 16 columns with a half-warp split: thread i < 16 gets lane base+i, columns
// [col, col+16) and thread i >= 16 lane base+i-16, columns [col+32, col+48), from each address; one
// wait for both in the same statement.
__device__ __forceinline__ void tc_ld16x32bx2_x16_pair(uint32_t ta, uint32_t tb, float *a, float *b)
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%32], 32;\n"
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%33], 32;\n"
        "tcgen05.wait::ld.sync.aligned;"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(ta), "r"(tb)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        a[i] = __uint_as_float(r[i]);
        b[i] = __uint_as_float(r[16 + i]);
    }
}

// One arrival per warp: every lane's earlier writes (and its proxy or tcgen05 fences) are ordered
// before lane 0's arrive by the warp barrier.  Barriers that warps arrive on count warps.
__device__ __forceinline__ void warp_arrive(uint64_t *bar)
{
    __syncwarp();
    if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

// Q of heads h0..h0+63 into TMEM as the A operand of the QK MMAs, scaled by one power of two 2^k that
// puts the largest |q| of the 64 heads in [2^13, 2^14); returns tau * log2(e) * 2^-k, the factor that
// turns an accumulated score into the log2 domain (every thread gets it).  Warp w < 16 writes TMEM
// quarter w%4 (heads 16(w%4) .. +15) and channel block w/4 of each half: lane l converts channels
// 256(l/16) + 64(w/4) .. +63 of head 16(w%4) + l%16 into 32 columns of lane 32(w%4) + l.
__device__ __forceinline__ float load_q(const AttnArgs &a, TcMisc &ms, uint32_t tmem, int b, int h0, int t)
{
    const int w = t >> 5, lane = t & 31, q = w & 3, j = (w >> 2) & 3;
    const bool loader = w < 16;
    const int h = 16 * q + (lane & 15);
    const int c0 = 256 * (lane >> 4) + 64 * j;
    uint4 qw[8];
    float amax = 0.f;
    if (loader) {
        const uint4 *qrow = reinterpret_cast<const uint4 *>(a.q + ((size_t)b * a.H + h0 + h) * kLatent + c0);
#pragma unroll
        for (int c = 0; c < 8; ++c) qw[c] = qrow[c];
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const uint32_t ww[4] = {qw[c].x, qw[c].y, qw[c].z, qw[c].w};
#pragma unroll
            for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(ww[k])), fabsf(bf16_hi(ww[k]))));
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (lane == 0) ms.qmax[w] = amax;
    }
    bar_sync(4, kTcThreads);
    amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, ms.qmax[i]);
    int k = 0;
    if (amax > 0.f) {
        const int ex = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
        k = 13 - ex;
        k = k < -60 ? -60 : (k > 60 ? 60 : k);
    }
    if (loader) {
        const float sc = exp2f((float)k);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
            uint32_t v[16];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const uint4 x = qw[4 * hh + c];
                v[4 * c] = pack_f16x2(bf16_lo(x.x) * sc, bf16_hi(x.x) * sc);
                v[4 * c + 1] = pack_f16x2(bf16_lo(x.y) * sc, bf16_hi(x.y) * sc);
                v[4 * c + 2] = pack_f16x2(bf16_lo(x.z) * sc, bf16_hi(x.z) * sc);
                v[4 * c + 3] = pack_f16x2(bf16_lo(x.w) * sc, bf16_hi(x.w) * sc);
            }
            tc_st16_u(tmem + ((uint32_t)(32 * q) << 16) + kColQ + 32 * j + 16 * hh, v);
        }
        tc_wait_st();
        tc_fence_before();
        warp_arrive(&ms.q_ready);
    }
    return a.sm_scale * exp2f((float)-k) * kLog2e;
}

__global__ void __launch_bounds__(kTcThreads, 1) attn_split_tc_kernel(AttnArgs a, int head_groups)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *V = base + kOffV;
    uint8_t *P = base + kOffP;
    int32_t *tab = reinterpret_cast<int32_t *>(base + kOffTab);
    TcMisc &ms = *reinterpret_cast<TcMisc *>(base + kOffMisc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    grid_dep_launch();   // the combine may be scheduled as splits finish
    const int s = blockIdx.x, b = blockIdx.y / head_groups, hg = blockIdx.y % head_groups;
    const int h0 = hg * kTcHeads;

    if (threadIdx.x == 0) {
        mbar_init(&ms.q_ready, 16);    // the Q-loading warps 0-15
        mbar_init(&ms.o_done, 2);
        for (int i = 0; i < kStages; ++i) {
            mbar_init(&ms.v_ready[i], kProducers / 32);
            mbar_init(&ms.v_free[i], 2);
            mbar_init(&ms.p_full[i], kSoftmax / 32);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&ms.s_full[i], 2);
            mbar_init(&ms.s_free[i], kSoftmax / 32);
        }
        for (int r = 0; r < 4; ++r) mbar_init(&ms.final_bar[r], 1);
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == kIssuerWarp) {
        tc_alloc(smem_addr(&ms.tmem_base), kTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;
    // Q is an input of the step, not a result of the previous grid: load it while that grid finishes
    const float zs = load_q(a, ms, tmem, b, h0, threadIdx.x);
    bool ok = true;

    // One tile of the softmax (warps 16-19): scores of tile t from TMEM, the running maxima (O^T
    // rescaled when one grows by more than 2^8), P^T into the tile's P buffer.  A dry call (before
    // the previous grid has finished) runs the same code on whatever the S and O^T columns hold,
    // with no waits or arrivals and the rescale forced, so that the first real tile runs warm; it
    // writes only the P buffer of tile 2, O^T and the rescale factors, all rewritten before use.
    const int q = warp - kSoftmaxWarp;       // TMEM quarter: heads 16q .. 16q+15
    const int u = lane >> 4;                 // this thread's entries 32u .. 32u+31 of a tile
    const int hl = 16 * q + (lane & 15);     // this thread's head
    const uint32_t tq = tmem + ((uint32_t)((32 * q) & 127) << 16);
    auto softmax_tile = [&](int t, bool dry, float &m_run, float &lsum) {
        const int p = dry ? 2 : t % kStages, sb = dry ? 0 : t & 1;
        // v_ready: the producers' valid-row mask of this tile; s_full: both halves of its scores
        if (!dry)
            ok = bar_and(1, kSoftmax, ok && warp_wait(&ms.v_ready[p], (uint32_t)(t / kStages) & 1u, &ms.abort_flag, a.ws, 9) &&
                                          warp_wait(&ms.s_full[sb], (uint32_t)(t >> 1) & 1u, &ms.abort_flag, a.ws, 6));
        if (ok) {
            tc_fence_after();
            // z[j] = S_0 + S_1 of entry 32u + j of head hl (unscaled): 16-lane loads whose first
            // half-warp reads columns c.. and second half-warp columns c + 32.. of the same lanes
            float z[32];
#pragma unroll
            for (int pc = 0; pc < 2; ++pc) {
                float s0[16], s1[16];
                tc_ld16x32bx2_x16_pair(tq + kColS + 64 * sb + 16 * pc, tq + (16u << 16) + kColS + 64 * sb + 16 * pc,
                                       s0, s1);
#pragma unroll
                for (int i = 0; i < 16; ++i) z[16 * pc + i] = s0[i] + s1[i];
            }
            tc_fence_before();
            if (!dry) warp_arrive(&ms.s_free[sb]);   // QK of tile t + 2 may overwrite these columns
            const uint32_t vbits = dry ? 0xFFFFFFFFu : (uint32_t)(ms.vmask[p] >> (32 * u));
            if (vbits != 0xFFFFFFFFu) {
                // a tile with masked entries (the sequence's last): their scores drop out
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (!((vbits >> i) & 1u)) z[i] = -INFINITY;
            }
            float mt = -INFINITY;
#pragma unroll
            for (int i = 0; i < 32; ++i) mt = fmaxf(mt, z[i]);
            // the head's maximum over the tile, log2 domain (zs > 0: the scaled maximum is the
            // maximum of the scaled scores)
            mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 16)) * zs;
            const bool need = dry || mt > m_run + kLazy;
            if (bar_or(1, kSoftmax, need)) {
                // some head's maximum grew: new maxima, and O^T rescaled column by column
                const float mn = need ? fmaxf(m_run, mt) : m_run;
                const float al = exp2f(m_run - mn);   // 0 while m_run is kNoMax, 1 if unchanged
                if (u == 0) ms.alpha[hl] = al;
                lsum *= al;
                m_run = mn;
                bar_sync(1, kSoftmax);   // every head's factor visible
                if (t > 0 || dry) {
                    // this warp's lanes of the four O^T M-tiles, once PV(t-1) has completed
                    const int tp = t - 1;
                    const bool pv_ok = dry || warp_wait(&ms.v_free[tp % kStages], (uint32_t)(tp / kStages) & 1u,
                                                        &ms.abort_flag, a.ws, 7);
                    if (pv_ok) {
                        tc_fence_after();
#pragma unroll 1
                        for (int k = 0; k < 32; ++k) {
                            float o[8];
                            const uint32_t col = kColO + 8 * k;   // M-tile k/8, heads 8(k%8) ..
                            tc_ld8_sync(tq + col, o);
#pragma unroll
                            for (int i = 0; i < 8; ++i) o[i] *= ms.alpha[8 * (k & 7) + i];
                            tc_st8(tq + col, o);
                        }
                        tc_wait_st();
                    }
                    ok = pv_ok;
                }
            }
            // P^T row hl, entries 32u .. 32u+31: four 16-byte units of the 128-byte swizzled row;
            // p = 2^(z zs - m + 7), 0 for a masked entry (z = -inf)
            const float mref = m_run - kPOffset;
            float ls = 0.f;
            uint8_t *Pb = P + p * kPBuf;
#pragma unroll
            for (int g = 0; g < 4; ++g) {
                uint32_t pk[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float p0 = exp2f(fmaf(z[8 * g + 2 * i], zs, -mref));
                    const float p1 = exp2f(fmaf(z[8 * g + 2 * i + 1], zs, -mref));
                    ls += p0 + p1;
                    pk[i] = pack_f16x2(p0, p1);
                }
                *reinterpret_cast<uint4 *>(Pb + swz((uint32_t)hl, (uint32_t)(4 * u + g))) =
                    make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
            lsum += ls;
            fence_async_smem();
            tc_fence_before();
        } else if (!dry) {
            warp_arrive(&ms.s_free[sb]);
        }
        if (!dry) warp_arrive(&ms.p_full[p]);
    };

    // warm the first-pass code of the softmax and of the producers while the previous grid finishes
    if (warp >= kSoftmaxWarp && warp < kIssuerWarp) {
        float dm = kNoMax, dl = 0.f;
        softmax_tile(0, true, dm, dl);
    } else if (warp < kSoftmaxWarp) {
        RawEntry dummy;
        dummy.row = 0;
        dummy.code[0] = dummy.code[1] = make_uint4(0u, 0u, 0u, 0u);
        dummy.sc = 0x38383838u;   // E4M3 1.0
        uint32_t v[32];
        dummy.dequant(a, threadIdx.x >> 6, v);
        store_row(V + 2 * kVBuf, threadIdx.x & (kTile - 1), threadIdx.x >> 6, v);
    }
    grid_dep_wait();   // the selected blocks of the previous grid

    if (threadIdx.x == 0) {
        int ub = 0, ue = 0;
        if (seq_view(a, b, ms.sv)) split_tiles(ms.sv.units, s, a.splits, ub, ue);
        ms.u_begin = ub;
        ms.u_end = ue;
    }
    __syncthreads();
    const int nh = (ms.u_end - ms.u_begin + kTileUnits - 1) / kTileUnits;   // tiles of this split
    if (threadIdx.x < kTabFill && nh > 0) fill_table(a, ms, tab, 0, threadIdx.x);
    __syncthreads();

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
        tc_fence_before();
        __syncthreads();
        tc_fence_after();
        if (warp == kIssuerWarp) tc_dealloc(tmem, kTmemCols);
        return;
    }

    if (warp >= kIssuerWarp) {
        // ------------------------------- MMA issuers -------------------------------
        const int r = warp - kIssuerWarp;
        if (lane == 0) {
            const uint32_t sV = smem_addr(V), sP = smem_addr(P);
            ok = mbar_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
            tc_fence_after();
            if (r < 2) {
                // QK of channel half r into S_r of tile t (lanes of half r, columns of parity t % 2),
                // once the producers have written tile t and the softmax has read tile t - 2's scores
                const uint32_t lanes = (uint32_t)(16 * r) << 16;
                for (int t = 0; ok && t < nh; ++t) {
                    const int p = t % kStages, sb = t & 1;
                    ok = mbar_wait(&ms.v_ready[p], (uint32_t)(t / kStages) & 1u, &ms.abort_flag, a.ws, 3);
                    if (ok && t >= 2) ok = mbar_wait(&ms.s_free[sb], (uint32_t)((t >> 1) - 1) & 1u, &ms.abort_flag, a.ws, 10);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int k = 0; k < 16; ++k) {
                        const int c = 4 * r + (k >> 2);   // V chunk of channels 256r + 16k ..
                        const uint64_t bd = umma_sdesc_sw128(sV + p * kVBuf + c * kVChunk + (k & 3) * 32, 16, 1024);
                        tc_mma_f16_ts(tmem + lanes + kColS + 64 * sb, tmem + lanes + kColQ + 8 * k, bd, kIdescQK,
                                      k > 0 ? 1u : 0u);
                    }
                    tc_commit(smem_addr(&ms.s_full[sb]));
                }
            } else {
                // PV of M-tiles 2(r-2), 2(r-2)+1 once the softmax has written P of tile t; the commit
                // releases the tile's V and P buffers
                const int m0 = 2 * (r - 2);
                for (int t = 0; ok && t < nh; ++t) {
                    const int p = t % kStages;
                    ok = mbar_wait(&ms.p_full[p], (uint32_t)(t / kStages) & 1u, &ms.abort_flag, a.ws, 2);
                    if (!ok) break;
                    tc_fence_after();
#pragma unroll
                    for (int mi = 0; mi < 2; ++mi)
#pragma unroll
                        for (int kk = 0; kk < kTile / 16; ++kk) {
                            const int m = m0 + mi;
                            const uint64_t ad = umma_sdesc_sw128(sV + p * kVBuf + 2 * m * kVChunk + kk * 2048, kVChunk, 1024);
                            const uint64_t bd = umma_sdesc_sw128(sP + p * kPBuf + kk * 32, 16, 1024);
                            tc_mma_f16(tmem + kColO + 64 * m, ad, bd, kIdescPV, (t > 0 || kk > 0) ? 1u : 0u);
                        }
                    tc_commit(smem_addr(&ms.v_free[p]));
                    if (t == nh - 1) tc_commit(smem_addr(&ms.o_done));
                }
            }
            // every MMA this thread issued has completed before TMEM is released
            tc_commit(smem_addr(&ms.final_bar[r]));
            volatile int no_abort = 0;
            mbar_wait(&ms.final_bar[r], 0, &no_abort, a.ws, 4);
        }
        ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
    } else if (warp < kSoftmaxWarp) {
        // ------------------------------- producers -------------------------------
        // After a failed wait the loop still runs to the end, skipping the work, so that every
        // producer takes the same barriers (the entry-table refills).
        const int d = threadIdx.x, e = d & (kTile - 1), cp = d >> 6;
        RawEntry raw0, raw1;   // tiles of even and of odd index
        raw0.fetch(a, tab[e], cp);
        if (nh > 1) raw1.fetch(a, tab[kTile + e], cp);
        uint32_t v[32];       // the next tile's row, dequantised before its buffer is free
        raw0.dequant(a, cp, v);
        // rw holds tile t, already dequantised into v, so it takes tile t + 2 at once; rn holds t + 1
        auto step = [&](int t, RawEntry &rw, const RawEntry &rn) {
            const int p = t % kStages;
            const unsigned int vb = __ballot_sync(0xffffffffu, rw.row != -1);   // tile t's valid rows
            if (t + 2 < nh) {
                if ((t + 2) % kTabTiles == 0) {
                    // the next tiles' entry addresses (every producer has fetched from the old ones)
                    bar_sync(3, kProducers);
                    if (d < kTabFill) fill_table(a, ms, tab, t + 2, d);
                    bar_sync(3, kProducers);
                }
                rw.fetch(a, tab[((t + 2) % kTabTiles) * kTile + e], cp);
            }
            if (t >= kStages) ok = ok && warp_wait(&ms.v_free[p], (uint32_t)(t / kStages - 1) & 1u, &ms.abort_flag, a.ws, 5);
            if (ok) store_row(V + p * kVBuf, e, cp, v);
            if (cp == 0 && lane == 0) reinterpret_cast<volatile uint32_t *>(&ms.vmask[p])[warp] = vb;
            fence_async_smem();
            warp_arrive(&ms.v_ready[p]);
            if (t + 1 < nh) rn.dequant(a, cp, v);
        };
#pragma unroll 1
        for (int t = 0; t < nh; t += 2) {
            step(t, raw0, raw1);
            if (t + 1 < nh) step(t + 1, raw1, raw0);
        }
    } else {
        // ------------------------------- softmax -------------------------------
        float m_run = kNoMax;                    // the head's running maximum (log2 domain), as the partner has it
        float lsum = 0.f;                        // this thread's share of the head's denominator
        for (int t = 0; t < nh; ++t) softmax_tile(t, false, m_run, lsum);
        // softmax denominators: the two halves of each head
        if (bar_and(1, kSoftmax, ok)) {
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 16);
            if (u == 0) {
                float2 *pml = reinterpret_cast<float2 *>(a.part_ml) + ((size_t)b * a.splits + s) * a.H + h0;
                pml[hl] = make_float2((m_run - kPOffset) * kLn2, lsum);
            }
        }
    }
    // ---- epilogue: O^T, M-tile w/4, quarter w%4, by warps 0-15
    {
        const bool eok = bar_and(4, kTcThreads, ok && warp_wait(&ms.o_done, 0, &ms.abort_flag, a.ws, 8));
        if (eok && warp < 16) {
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
    if (warp == kIssuerWarp) tc_dealloc(tmem, kTmemCols);
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
