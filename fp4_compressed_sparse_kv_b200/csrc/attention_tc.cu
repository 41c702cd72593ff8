// attention_tc.cu -- step 4 on the sm_100a tensor cores (tcgen05, TMEM) for 64 query heads per CTA.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用" (sparse
// attention over the selected positions of the FP4 main KV) and section "先让长输入少走一半路" (the
// FP8 sliding window); yomxxx.com long-form post, section 五 (fixed-stride entries dequantised in
// the kernel, in parallel).  The 512-channel latent serves as both key and value.
//
// With 64 heads sharing one latent, QK^T and PV are dense contractions: 4 x 64 x 512 FLOP per 288-B
// entry, above the fp16 tensor ridge of B200, so they run on the tensor cores.  Dequantisation is
// exact in fp16 (an E2M1 value times an E4M3 scale has at most 6 significant bits and lies in
// [2^-10, 2688]); Q is scaled per head by a power of two into fp16's range; P is rounded to fp16
// (relative error 2^-11); accumulation is fp32 in TMEM.
//
// Tile = 128 entries.  Both MMAs put the entries / channels on M = 128 ("swap AB"):
//   QK:  S^T[128 entries x 64 heads]  = V[128 x 512] . Q^T          (A = V K-major, B = Q K-major)
//   PV:  O^T[128 ch x 64 heads] (x4)  = V^T[128 ch x 128 entries] . P^T   (A = V^T MN-major, B = P^T MN-major)
// so TMEM holds S^T in 64 columns and O^T in 256, and one 128-byte-swizzled fp16 copy of the tile in
// shared memory is read as K-major V by QK and as MN-major V^T by PV.
//
// Warp roles (256 threads): warps 0-3 (TMEM lanes 0-127) run the softmax and the epilogue, warp 0
// owns the TMEM allocation and its lane 0 issues the MMAs between softmax steps (QK of tile t before
// softmax(t), PV of tile t after it); warps 4-7 load Q once, then dequantise each tile chunk by
// chunk (64 channels) from raw entries they prefetch into registers.
// The V buffer is single: chunks of tile t+1 are written as soon as PV(t) has finished the 128-channel
// M-tile that reads them.  Softmax rescales lazily: O^T in TMEM is rescaled only when a head's
// running maximum grows by more than 2^8.
#include "attention_common.cuh"
#include "pipeline.cuh"
#include "tcgen05.cuh"

namespace csa {

constexpr int kTcHeads = 64;
constexpr int kTcRows = 128;
constexpr int kTcUnits = kTcRows / kAttnUnit;
constexpr int kTcChunks = kLatent / 64;
constexpr int kTcThreads = 256;   // 4 softmax/MMA warps, 4 dequant warps
constexpr uint32_t kVChunk = kTcRows * 128;   // 16 KB: 128 rows x 64 fp16
constexpr uint32_t kQChunk = kTcHeads * 128;  // 8 KB: 64 rows x 64 fp16
constexpr uint32_t kOffV = 0;
constexpr uint32_t kOffQ = kOffV + kTcChunks * kVChunk;
constexpr uint32_t kOffP = kOffQ + kTcChunks * kQChunk;
constexpr uint32_t kOffMisc = kOffP + kTcRows * 128;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 64;
constexpr float kLazy = 8.f;      // log2-domain growth of a head maximum tolerated without rescaling
constexpr float kPOffset = 7.f;   // p = exp2(z - m + 7) <= 2^15 keeps small p out of fp16 subnormals
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TcMisc {
    uint64_t s_full, p_full, q_ready, o_done, final_bar;
    uint64_t v_ready[kTcChunks];
    uint64_t v_free[kTcChunks / 2];
    uint64_t sm_bar;            // softmax warpgroup sync (bounded, unlike a named barrier)
    uint32_t tmem_base;
    int abort_flag;
    int vote[4];
    float vmeta[2][kTcRows];    // per entry: -1 masked, else its value scale (1 for FP4, window scale)
    float zscale[kTcHeads];     // tau * 2^-k_h * log2(e)
    float m[kTcHeads];          // running max, log2 domain
    float alpha[kTcHeads];
    float red[4][kTcHeads];
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

__global__ void __launch_bounds__(kTcThreads, 1) attn_split_tc_kernel(AttnArgs a, int head_groups)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *V = base + kOffV;
    uint8_t *Q = base + kOffQ;
    uint8_t *P = base + kOffP;
    TcMisc &ms = *reinterpret_cast<TcMisc *>(base + kOffMisc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int s = blockIdx.x, b = blockIdx.y / head_groups, hg = blockIdx.y % head_groups;
    const int h0 = hg * kTcHeads;

    SeqView sv;
    const bool seq_ok = seq_view(a, b, sv);
    int u_begin = 0, u_end = 0;
    if (seq_ok) split_range(sv.units, s, a.splits, u_begin, u_end);
    const int ntiles = (u_end - u_begin + kTcUnits - 1) / kTcUnits;

    if (threadIdx.x == 0) {
        mbar_init(&ms.s_full, 1);
        mbar_init(&ms.p_full, 128);
        mbar_init(&ms.q_ready, 128);
        mbar_init(&ms.o_done, 1);
        mbar_init(&ms.final_bar, 1);
        for (int c = 0; c < kTcChunks; ++c) mbar_init(&ms.v_ready[c], 128);
        for (int c = 0; c < kTcChunks / 2; ++c) mbar_init(&ms.v_free[c], 1);
        mbar_init(&ms.sm_bar, 128);
        ms.abort_flag = 0;
        fence_mbar_init();
    }
    if (threadIdx.x < kTcHeads) ms.m[threadIdx.x] = -INFINITY;
    if (warp == 0 && ntiles > 0) {
        tc_alloc(smem_addr(&ms.tmem_base), kTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = ms.tmem_base;

    if (warp >= 4) {
        // ------------------------------- Q load, then dequantisation ------------------------
        const int i = threadIdx.x - 128;   // 0..127
        {
            // Q: thread i converts half a head row (256 channels); per-head power-of-two scale
            const int h = i >> 1, half = i & 1;
            const uint16_t *qrow = a.q + ((size_t)b * a.H + h0 + h) * kLatent + half * 256;
            float amax = 0.f;
            for (int c = 0; c < 256; c += 8) {
                const uint4 w = *reinterpret_cast<const uint4 *>(qrow + c);
                const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                for (int k = 0; k < 4; ++k) amax = fmaxf(amax, fmaxf(fabsf(bf16_lo(ww[k])), fabsf(bf16_hi(ww[k]))));
            }
            amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
            int k = 0;
            if (amax > 0.f) {
                const int e = (int)((__float_as_uint(amax) >> 23) & 0xFF) - 127;
                k = 13 - e;
                k = k < -60 ? -60 : (k > 60 ? 60 : k);
            }
            const float sc = exp2f((float)k);
            if (half == 0) ms.zscale[h] = a.sm_scale * exp2f((float)-k) * kLog2e;
            for (int c = 0; c < 256; c += 8) {
                const uint4 w = *reinterpret_cast<const uint4 *>(qrow + c);
                uint4 o;
                o.x = pack_f16x2(bf16_lo(w.x) * sc, bf16_hi(w.x) * sc);
                o.y = pack_f16x2(bf16_lo(w.y) * sc, bf16_hi(w.y) * sc);
                o.z = pack_f16x2(bf16_lo(w.z) * sc, bf16_hi(w.z) * sc);
                o.w = pack_f16x2(bf16_lo(w.w) * sc, bf16_hi(w.w) * sc);
                const int ch = half * 256 + c;
                *reinterpret_cast<uint4 *>(Q + (ch >> 6) * kQChunk + swz(h, (ch & 63) >> 3)) = o;
            }
            fence_async_smem();
            mbar_arrive(&ms.q_ready);
        }
        bool ok = true;
        for (int t = 0; ok && t < ntiles; ++t) {
            const int u = u_begin + t * kTcUnits + i / kAttnUnit, j = i % kAttnUnit;
            EntryRef r;
            const bool valid = u < u_end && entry_ref(a, sv, u, j, r);
            uint4 craw[16];
            uint4 sraw[2];
            if (valid && !r.swa) {
#pragma unroll
                for (int q = 0; q < 16; ++q) craw[q] = reinterpret_cast<const uint4 *>(r.p)[q];
                sraw[0] = reinterpret_cast<const uint4 *>(r.sc)[0];
                sraw[1] = reinterpret_cast<const uint4 *>(r.sc)[1];
            }
            ms.vmeta[t & 1][i] = valid ? (r.swa ? r.fscale : 1.f) : -1.f;
#pragma unroll
            for (int c = 0; c < kTcChunks; ++c) {
                if (t > 0 && (c & 1) == 0) {
                    ok = warp_wait(&ms.v_free[c >> 1], (t - 1) & 1, &ms.abort_flag, a.ws, 5);
                    if (!ok) break;
                }
                uint4 out[8];
                if (!valid) {
#pragma unroll
                    for (int jj = 0; jj < 8; ++jj) out[jj] = make_uint4(0u, 0u, 0u, 0u);
                } else if (!r.swa) {
                    // channels 64c .. 64c+63: code bytes 32c .. 32c+31, scale groups 4c .. 4c+3
                    const uint32_t sw = (c < 4) ? (&sraw[0].x)[c] : (&sraw[1].x)[c - 4];
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const uint32_t sh = e4m3x2_to_f16x2((uint16_t)((sw >> (8 * g)) & 0xFF));
                        const uint32_t s2 = (sh & 0xFFFFu) | (sh << 16);
                        const uint4 cw = craw[2 * c + (g >> 1)];
                        const uint32_t w0 = (g & 1) ? cw.z : cw.x, w1 = (g & 1) ? cw.w : cw.y;
                        uint32_t v[8];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            v[q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w0 >> (8 * q))), s2);
                            v[4 + q] = hmul2_u32(e2m1x2_to_f16x2((uint8_t)(w1 >> (8 * q))), s2);
                        }
                        out[2 * g] = make_uint4(v[0], v[1], v[2], v[3]);
                        out[2 * g + 1] = make_uint4(v[4], v[5], v[6], v[7]);
                    }
                } else {
                    // window entry: 64 E4M3 values, exact in fp16; its scale is applied in the softmax
                    const uint4 *src = reinterpret_cast<const uint4 *>(r.p + 64 * c);
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        const uint4 w = src[q];
                        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
                        uint32_t v[8];
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            v[2 * k] = e4m3x2_to_f16x2((uint16_t)(ww[k] & 0xFFFF));
                            v[2 * k + 1] = e4m3x2_to_f16x2((uint16_t)(ww[k] >> 16));
                        }
                        out[2 * q] = make_uint4(v[0], v[1], v[2], v[3]);
                        out[2 * q + 1] = make_uint4(v[4], v[5], v[6], v[7]);
                    }
                }
#pragma unroll
                for (int jj = 0; jj < 8; ++jj)
                    *reinterpret_cast<uint4 *>(V + c * kVChunk + swz((uint32_t)i, (uint32_t)jj)) = out[jj];
                fence_async_smem();
                mbar_arrive(&ms.v_ready[c]);
            }
        }
    } else if (warp < 4) {
        // ------------------------------- softmax + epilogue -------------------------------
        const int e = threadIdx.x;              // TMEM lane = tile row (entry) / channel in epilogue
        const int wq = warp & 3;
        const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
        float lsum[kTcHeads];
#pragma unroll
        for (int h = 0; h < kTcHeads; ++h) lsum[h] = 0.f;
        bool ok = ntiles > 0;
        uint32_t sync_phase = 0;
        // all 128 softmax threads arrive, then wait with a time limit; false on timeout or abort
        auto sync128 = [&]() -> bool {
            mbar_arrive(&ms.sm_bar);
            const bool r = warp_wait(&ms.sm_bar, sync_phase & 1, &ms.abort_flag, a.ws, 9);
            ++sync_phase;
            return r;
        };
        const uint32_t sV = smem_addr(V), sQ = smem_addr(Q), sP = smem_addr(P);
        const bool issuer = warp == 0 && lane == 0;
        // Q and the per-head score scales are in shared memory (written by the dequant warps)
        if (ntiles > 0) {
            ok = warp_wait(&ms.q_ready, 0, &ms.abort_flag, a.ws, 1);
            tc_fence_after();
        }
        for (int t = 0; ok && t < ntiles; ++t) {
            const uint32_t ph = t & 1;
            if (warp == 0) {
                // QK of tile t, chunk by chunk as the dequantisation lands
                int iok = 1;
                if (issuer) {
                    for (int c = 0; c < kTcChunks; ++c) {
                        if (!mbar_wait(&ms.v_ready[c], ph, &ms.abort_flag, a.ws, 2)) {
                            iok = 0;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = umma_sdesc_sw128(sV + c * kVChunk + kk * 32, 16, 1024);
                            const uint64_t bd = umma_sdesc_sw128(sQ + c * kQChunk + kk * 32, 16, 1024);
                            tc_mma_f16(tmem + kColS, ad, bd, kIdescQK, (c | kk) != 0);
                        }
                    }
                    if (iok) tc_commit(smem_addr(&ms.s_full));
                }
                if (!__shfl_sync(0xffffffffu, iok, 0)) {
                    ok = false;
                    break;
                }
            }
            ok = warp_wait(&ms.s_full, ph, &ms.abort_flag, a.ws, 6) &&
                 warp_wait(&ms.v_ready[kTcChunks - 1], ph, &ms.abort_flag, a.ws, 7);
            if (!ok) break;
            tc_fence_after();
            float z[kTcHeads];
            tc_ld32(tl + kColS, z);
            tc_ld32(tl + kColS + 32, z + 32);
            tc_wait_ld();
            const float em = ms.vmeta[ph][e];
            const bool valid = em >= 0.f;
            bool need = false;
#pragma unroll
            for (int h = 0; h < kTcHeads; ++h) {
                z[h] = valid ? z[h] * (em * ms.zscale[h]) : -INFINITY;
                need |= z[h] > ms.m[h] + kLazy;
            }
            const bool wneed = __any_sync(0xffffffffu, need);
            if (lane == 0) ms.vote[wq] = wneed ? 1 : 0;
            if (!(ok = sync128())) break;
            const bool rescale = ms.vote[0] | ms.vote[1] | ms.vote[2] | ms.vote[3];
            if (rescale) {
#pragma unroll
                for (int h = 0; h < kTcHeads; ++h) {
                    float v = z[h];
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
                    if (lane == 0) ms.red[wq][h] = v;
                }
                if (!(ok = sync128())) break;
                if (e < kTcHeads) {
                    const float mt = fmaxf(fmaxf(ms.red[0][e], ms.red[1][e]), fmaxf(ms.red[2][e], ms.red[3][e]));
                    const float mo = ms.m[e];
                    const float mn = fmaxf(mo, mt);
                    ms.alpha[e] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
                    ms.m[e] = mn;
                }
                if (!(ok = sync128())) break;
#pragma unroll
                for (int h = 0; h < kTcHeads; ++h) lsum[h] *= ms.alpha[h];
                if (t > 0) {
                    for (int m = 0; m < 4; ++m) {
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            float o[32];
                            const uint32_t col = kColO + 64 * m + 32 * half;
                            tc_ld32(tl + col, o);
                            tc_wait_ld();
#pragma unroll
                            for (int q = 0; q < 32; ++q) o[q] *= ms.alpha[32 * half + q];
                            tc_st32(tl + col, o);
                        }
                    }
                    tc_wait_st();
                }
            }
            const float pv_scale = valid ? em : 0.f;
            uint32_t pk[kTcHeads / 2];
#pragma unroll
            for (int h = 0; h < kTcHeads; h += 2) {
                const float p0 = exp2f(z[h] - ms.m[h] + kPOffset);
                const float p1 = exp2f(z[h + 1] - ms.m[h + 1] + kPOffset);
                lsum[h] += p0;
                lsum[h + 1] += p1;
                pk[h / 2] = pack_f16x2(p0 * pv_scale, p1 * pv_scale);
            }
#pragma unroll
            for (int jj = 0; jj < 8; ++jj)
                *reinterpret_cast<uint4 *>(P + swz((uint32_t)e, (uint32_t)jj)) =
                    make_uint4(pk[4 * jj], pk[4 * jj + 1], pk[4 * jj + 2], pk[4 * jj + 3]);
            fence_async_smem();
            tc_fence_before();
            mbar_arrive(&ms.p_full);
            if (warp == 0) {
                // PV of tile t once all 128 rows of P are in shared memory
                int iok = 1;
                if (issuer) {
                    if (!mbar_wait(&ms.p_full, ph, &ms.abort_flag, a.ws, 3)) {
                        iok = 0;
                    } else {
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
                        if (t == ntiles - 1) tc_commit(smem_addr(&ms.o_done));
                    }
                }
                if (!__shfl_sync(0xffffffffu, iok, 0)) {
                    ok = false;
                    break;
                }
            }
        }
        if (issuer && ntiles > 0) {
            // every MMA this thread issued has completed before TMEM is released
            tc_commit(smem_addr(&ms.final_bar));
            volatile int no_abort = 0;
            mbar_wait(&ms.final_bar, 0, &no_abort, a.ws, 4);
        }
        __syncwarp();
        // ---- epilogue: partial (o, m, l) of this split
        float *po = a.part_o + (((size_t)b * a.splits + s) * a.H + h0) * kLatent;
        float2 *pml = reinterpret_cast<float2 *>(a.part_ml) + ((size_t)b * a.splits + s) * a.H + h0;
        if (ntiles == 0) {
            for (int h = 0; h < kTcHeads; ++h) {
                po[(size_t)h * kLatent + e] = 0.f;
                po[(size_t)h * kLatent + 128 + e] = 0.f;
                po[(size_t)h * kLatent + 256 + e] = 0.f;
                po[(size_t)h * kLatent + 384 + e] = 0.f;
            }
            if (e < kTcHeads) pml[e] = make_float2(-INFINITY, 0.f);
        } else if (ok) {
            ok = warp_wait(&ms.o_done, 0, &ms.abort_flag, a.ws, 8);
            tc_fence_after();
#pragma unroll
            for (int h = 0; h < kTcHeads; ++h) {
                float v = lsum[h];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
                if (lane == 0) ms.red[wq][h] = v;
            }
            ok = ok && sync128();
            if (ok) {
                for (int m = 0; m < 4; ++m) {
#pragma unroll
                    for (int half = 0; half < 2; ++half) {
                        float o[32];
                        tc_ld32(tl + kColO + 64 * m + 32 * half, o);
                        tc_wait_ld();
#pragma unroll
                        for (int q = 0; q < 32; ++q) po[(size_t)(32 * half + q) * kLatent + 128 * m + e] = o[q];
                    }
                }
                if (e < kTcHeads) {
                    const float l = ms.red[0][e] + ms.red[1][e] + ms.red[2][e] + ms.red[3][e];
                    pml[e] = make_float2((ms.m[e] - kPOffset) * kLn2, l);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 0 && ntiles > 0) tc_dealloc(tmem, kTmemCols);
}

bool attn_tc_supported(int H) { return H == 64 || H == 128; }

int attn_units_per_tile(int H) { return attn_tc_supported(H) ? kTcUnits : 4; }

cudaError_t launch_attn_tc(const AttnArgs &a, cudaStream_t st)
{
    static_assert(kTcSmem <= 232448, "shared memory budget");
    cudaError_t e = cudaFuncSetAttribute(attn_split_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kTcSmem);
    if (e != cudaSuccess) return e;
    const int groups = a.H / kTcHeads;
    dim3 grid(a.splits, a.B * groups);
    attn_split_tc_kernel<<<grid, kTcThreads, kTcSmem, st>>>(a, groups);
    return cudaGetLastError();
}

}  // namespace csa
