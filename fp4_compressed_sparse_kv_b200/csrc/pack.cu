// pack.cu -- step 1: pack new tokens' latents into the FP4 main cache, the E4M3 indexer-key cache
// and the FP8 sliding-window ring.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": the
// main KV is FP4 while the more quantisation-sensitive SWA KV stays FP8.  ailily.cc article
// "每个 token 只占 890 字节", section 二: one E4M3 scale per 16 channels holds the value range.
//
// One warp per token at a time; for long calls, four consecutive tokens per warp with all their loads
// issued first.
// Lane g owns 16-channel group g of the 512-channel latent, which is exactly one E4M3 scale: its amax
// needs no cross-lane step, and its 16 codes are one 8-byte store.  The window entry needs the
// token's amax, a 5-step warp max.  Loads are 2 x 16 B per lane (latent) and 8 B per lane (key), all
// coalesced; HBM-bound streaming.
//
// The norm variant starts from the pre-norm latent (ailily.cc article, section 三: the KV latent is
// RMS-normalised, with weights of magnitude about 1, and rotated by RoPE, which keeps its norm): in
// binary32, lane g forms the FMA chain of its 16 squares, an xor butterfly (16, 8, 4, 2, 1) sums the
// lanes, r = 1 / sqrt(sum / 512 + 1e-6) with correctly rounded operations, y = (v * r) * weight; lanes
// 28-31 then rotate their channel pairs (448 + 2i, 449 + 2i) with the caller's (cos_i, sin_i), every
// product and sum rounded on its own; the result is rounded to bf16 and packed as above.
#include <cuda_bf16.h>

#include "common.cuh"
#include "convert.cuh"
#include "pipeline.cuh"

namespace csa {

// A token's inputs, loaded ahead of its arithmetic.
struct PackIn {
    uint4 a, b;     // latent channels 16 lane .. 16 lane + 15 (bf16)
    uint2 kw;       // indexer-key channels 4 lane .. 4 lane + 3 (bf16)
    int64_t s;      // main slot
    int32_t ss;     // window slot
};

template <bool kNorm>
__device__ __forceinline__ void pack_token(const csa_kv_layer &layer, const PackIn &in, int tok, int lane, void *ws,
                                           const float *__restrict__ norm_w, const float *__restrict__ rope_cs)
{
    const int64_t s = in.s;
    const int32_t ss = in.ss;
    const bool main_ok = s >= 0 && s < (int64_t)layer.num_pages * kPage;
    const bool swa_ok = ss >= 0 && ss < layer.num_rows * kWindow;
    if (lane == 0 && (!main_ok || (ss >= 0 && !swa_ok))) report(ws, CSA_ERR_DEVICE_DATA, tok);

    // 16 channels of group `lane`
    const uint32_t w[8] = {in.a.x, in.a.y, in.a.z, in.a.w, in.b.x, in.b.y, in.b.z, in.b.w};
    float x[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = bf16_lo(w[i]);
        x[2 * i + 1] = bf16_hi(w[i]);
    }
    if (kNorm) {
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc = __fmaf_rn(x[i], x[i], acc);
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) acc = __fadd_rn(acc, __shfl_xor_sync(0xffffffffu, acc, d));
        const float r = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(__fdiv_rn(acc, 512.0f), 1e-6f)));
        const float4 *wp = reinterpret_cast<const float4 *>(norm_w + 16 * lane);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float4 wv = wp[q];
            x[4 * q] = __fmul_rn(__fmul_rn(x[4 * q], r), wv.x);
            x[4 * q + 1] = __fmul_rn(__fmul_rn(x[4 * q + 1], r), wv.y);
            x[4 * q + 2] = __fmul_rn(__fmul_rn(x[4 * q + 2], r), wv.z);
            x[4 * q + 3] = __fmul_rn(__fmul_rn(x[4 * q + 3], r), wv.w);
        }
        if (lane >= 28) {   // channels 448..511: pairs 8 (lane - 28) .. 8 (lane - 28) + 7
            const float4 *cp = reinterpret_cast<const float4 *>(rope_cs + (size_t)tok * 64 + 16 * (lane - 28));
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float4 c2 = cp[q];   // (cos, sin) of two pairs
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const float co = h ? c2.z : c2.x, si = h ? c2.w : c2.y;
                    const int m = 2 * q + h;
                    const float a = x[2 * m], b = x[2 * m + 1];
                    x[2 * m] = __fsub_rn(__fmul_rn(a, co), __fmul_rn(b, si));
                    x[2 * m + 1] = __fadd_rn(__fmul_rn(a, si), __fmul_rn(b, co));
                }
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) x[i] = __bfloat162float(__float2bfloat16_rn(x[i]));
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));

    if (main_ok) {
        // s = E4M3(amax / 6); codes = E2M1(x / s), or 0 when s decodes to 0
        const uint8_t sc = (uint8_t)(f32x2_to_e4m3x2(__fdiv_rn(amax, 6.0f), 0.f) & 0xFF);
        const float sd = e4m3_to_f32(sc);
        uint2 codes = make_uint2(0u, 0u);
        if (sd != 0.f) {
            float y[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) y[i] = __fdiv_rn(x[i], sd);
            codes.x = f32x8_to_e2m1x8(y);
            codes.y = f32x8_to_e2m1x8(y + 8);
        }
        reinterpret_cast<uint2 *>(layer.codes + s * kCodeBytes)[lane] = codes;
        layer.scales[s * kScaleBytes + lane] = sc;

        // indexer key: channels 4*lane .. 4*lane+3, plain E4M3 cast
        const uint2 kw = in.kw;
        const uint32_t k01 = f32x2_to_e4m3x2(bf16_lo(kw.x), bf16_hi(kw.x));
        const uint32_t k23 = f32x2_to_e4m3x2(bf16_lo(kw.y), bf16_hi(kw.y));
        reinterpret_cast<uint32_t *>(layer.keys + s * kIdxDim)[lane] = k01 | (k23 << 16);
    }

    if (ss >= 0) {  // warp-uniform
        float m = amax;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        if (swa_ok) {
            const float scale = __fdiv_rn(m, 448.0f);
            uint32_t v[4] = {0u, 0u, 0u, 0u};
            if (scale != 0.f) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const uint32_t lo = f32x2_to_e4m3x2(__fdiv_rn(x[4 * i], scale), __fdiv_rn(x[4 * i + 1], scale));
                    const uint32_t hi = f32x2_to_e4m3x2(__fdiv_rn(x[4 * i + 2], scale), __fdiv_rn(x[4 * i + 3], scale));
                    v[i] = lo | (hi << 16);
                }
            }
            reinterpret_cast<uint4 *>(layer.swa + (size_t)ss * kLatent)[lane] = make_uint4(v[0], v[1], v[2], v[3]);
            if (lane == 0) layer.swa_scale[ss] = scale;
        }
    }
}


// Each warp packs kTok consecutive tokens: their loads are issued together, then each token's
// arithmetic runs on registers, so every warp keeps several tokens' bytes in flight (prefill chunks);
// a decode batch of a few tokens takes one token per warp, its latency being one token's.
constexpr int kPackTokLarge = 4;
constexpr int kPackLargeFrom = 4096;   // tokens per call from which warps take kPackTokLarge tokens

template <bool kNorm, int kPackTok>
__global__ void __launch_bounds__(256) kv_pack_kernel(csa_kv_layer layer, const uint16_t *__restrict__ latent,
                                                      const uint16_t *__restrict__ idx_key,
                                                      const int64_t *__restrict__ slot,
                                                      const int32_t *__restrict__ swa_slot, int n, void *ws,
                                                      const float *__restrict__ norm_w,
                                                      const float *__restrict__ rope_cs)
{
    // a dependent kernel launched after this one (the indexer's query terms, an attention) may be
    // scheduled now: each waits for this grid before it reads anything this grid writes
    grid_dep_launch();
    const int tok0 = (blockIdx.x * 8 + (threadIdx.x >> 5)) * kPackTok;
    const int lane = threadIdx.x & 31;
    PackIn in[kPackTok];
#pragma unroll
    for (int i = 0; i < kPackTok; ++i) {
        const int tok = tok0 + i;
        if (tok < n) {
            const uint4 *src = reinterpret_cast<const uint4 *>(latent + (size_t)tok * kLatent) + 2 * lane;
            in[i].a = src[0];
            in[i].b = src[1];
            in[i].kw = reinterpret_cast<const uint2 *>(idx_key + (size_t)tok * kIdxDim)[lane];
            in[i].s = slot[tok];
            in[i].ss = swa_slot ? swa_slot[tok] : -1;
        }
    }
#pragma unroll
    for (int i = 0; i < kPackTok; ++i)
        if (tok0 + i < n) pack_token<kNorm>(layer, in[i], tok0 + i, lane, ws, norm_w, rope_cs);
}

cudaError_t launch_kv_pack(const csa_kv_layer &layer, const uint16_t *latent, const uint16_t *idx_key,
                           const int64_t *slot, const int32_t *swa_slot, int n, void *ws, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    if (n >= kPackLargeFrom)
        kv_pack_kernel<false, kPackTokLarge><<<(n + 8 * kPackTokLarge - 1) / (8 * kPackTokLarge), 256, 0, st>>>(
            layer, latent, idx_key, slot, swa_slot, n, ws, nullptr, nullptr);
    else
        kv_pack_kernel<false, 1><<<(n + 7) / 8, 256, 0, st>>>(layer, latent, idx_key, slot, swa_slot, n, ws, nullptr,
                                                             nullptr);
    return cudaGetLastError();
}

cudaError_t launch_kv_norm_rope_pack(const csa_kv_layer &layer, const uint16_t *latent, const float *norm_w,
                                     const float *rope_cs, const uint16_t *idx_key, const int64_t *slot,
                                     const int32_t *swa_slot, int n, void *ws, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    if (n >= kPackLargeFrom)
        kv_pack_kernel<true, kPackTokLarge><<<(n + 8 * kPackTokLarge - 1) / (8 * kPackTokLarge), 256, 0, st>>>(
            layer, latent, idx_key, slot, swa_slot, n, ws, norm_w, rope_cs);
    else
        kv_pack_kernel<true, 1><<<(n + 7) / 8, 256, 0, st>>>(layer, latent, idx_key, slot, swa_slot, n, ws, norm_w,
                                                            rope_cs);
    return cudaGetLastError();
}

}  // namespace csa
