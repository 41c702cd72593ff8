// pack.cu -- step 1: pack new tokens' latents into the FP4 main cache, the E4M3 indexer-key cache
// and the FP8 sliding-window ring.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": the
// main KV is FP4 while the more quantisation-sensitive SWA KV stays FP8.  ailily.cc article
// "每个 token 只占 890 字节", section 二: one E4M3 scale per 16 channels holds the value range.
//
// One warp per token.  Lane g owns 16-channel group g of the 512-channel latent, which is exactly
// one E4M3 scale: its amax needs no cross-lane step, and its 16 codes are one 8-byte store.  The
// window entry needs the token's amax, a 5-step warp max.  Loads are 2 x 16 B per lane (latent) and
// 8 B per lane (key), all coalesced; HBM-bound streaming.
#include "common.cuh"
#include "convert.cuh"

namespace csa {

__global__ void __launch_bounds__(256) kv_pack_kernel(csa_kv_layer layer, const uint16_t *__restrict__ latent,
                                                      const uint16_t *__restrict__ idx_key,
                                                      const int64_t *__restrict__ slot,
                                                      const int32_t *__restrict__ swa_slot, int n, void *ws)
{
    const int tok = blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (tok >= n) return;

    const int64_t s = slot[tok];
    const int32_t ss = swa_slot ? swa_slot[tok] : -1;
    const bool main_ok = s >= 0 && s < (int64_t)layer.num_pages * kPage;
    const bool swa_ok = ss >= 0 && ss < layer.num_rows * kWindow;
    if (lane == 0 && (!main_ok || (ss >= 0 && !swa_ok))) report(ws, CSA_ERR_DEVICE_DATA, tok);

    // 16 channels of group `lane`
    const uint4 *src = reinterpret_cast<const uint4 *>(latent + (size_t)tok * kLatent) + 2 * lane;
    const uint4 a = src[0], b = src[1];
    const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
    float x[16];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        x[2 * i] = bf16_lo(w[i]);
        x[2 * i + 1] = bf16_hi(w[i]);
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
        const uint2 kw = reinterpret_cast<const uint2 *>(idx_key + (size_t)tok * kIdxDim)[lane];
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

cudaError_t launch_kv_pack(const csa_kv_layer &layer, const uint16_t *latent, const uint16_t *idx_key,
                           const int64_t *slot, const int32_t *swa_slot, int n, void *ws, cudaStream_t st)
{
    if (n == 0) return cudaSuccess;
    kv_pack_kernel<<<(n + 7) / 8, 256, 0, st>>>(layer, latent, idx_key, slot, swa_slot, n, ws);
    return cudaGetLastError();
}

}  // namespace csa
