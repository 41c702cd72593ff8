// attention_cc.cu -- step 4 on CUDA cores: split-KV sparse decode attention over the selected FP4
// entries and the FP8 sliding window, one softmax over both, plus the split combine.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用" (sparse
// attention over the selected positions; FP4 main KV) and section "先让长输入少走一半路" (the
// sliding-window branch, whose KV stays FP8).  yomxxx.com long-form post, section 五: the kernel
// computes each entry's address from its token index (fixed 288-byte entries) and dequantises
// in-kernel, in parallel.
//
// This kernel computes in fp32 on CUDA cores and serves every head count; the tensor-core kernel
// (attention_tc.cu) is the fast path for H = 64.  A work item is (sequence b, split s, head
// group); the sequence's entries are a list of 8-entry units (its selected blocks, then the window
// in 8-position chunks) cut into `splits` contiguous ranges.  Each split writes an unnormalised
// partial (o, m, l) that attn_combine_kernel merges.
#include "attention_common.cuh"
#include "pipeline.cuh"

namespace csa {

constexpr int kCcThreads = 256;
constexpr int kCcTile = 32;                  // entries per tile (4 units)
constexpr int kCcRow = kLatent + 4;          // padded fp32 row (breaks bank aliasing across rows)

template <int HG>
__global__ void __launch_bounds__(kCcThreads, 1) attn_split_cc_kernel(AttnArgs a, int head_groups)
{
    extern __shared__ __align__(16) float sm_f[];
    float *Qs = sm_f;                              // [HG][kCcRow]
    float *Vs = Qs + HG * kCcRow;                  // [kCcTile][kCcRow]
    float *Ps = Vs + kCcTile * kCcRow;             // [kCcTile][HG]  scores, then probabilities
    float *alpha_s = Ps + kCcTile * HG;            // [HG]
    float *m_s = alpha_s + HG;                     // [HG]
    float *l_s = m_s + HG;                         // [HG]

    const int s = blockIdx.x, b = blockIdx.y / head_groups, hg = blockIdx.y % head_groups;
    const int h0 = hg * HG;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;

    SeqView sv;
    const bool ok = seq_view(a, b, sv);
    int u_begin = 0, u_end = 0;
    if (ok) split_range(sv.units, s, a.splits, u_begin, u_end);

    for (int i = t; i < HG * kLatent; i += kCcThreads) {
        const int h = i / kLatent, c = i % kLatent;
        const uint16_t v = a.q[((size_t)b * a.H + h0 + h) * kLatent + c];
        Qs[h * kCcRow + c] = __uint_as_float((uint32_t)v << 16);
    }
    if (t < HG) {
        m_s[t] = -INFINITY;
        l_s[t] = 0.f;
    }
    float acc[HG][2];
#pragma unroll
    for (int h = 0; h < HG; ++h) acc[h][0] = acc[h][1] = 0.f;
    __syncthreads();

    for (int u0 = u_begin; u0 < u_end; u0 += kCcTile / kAttnUnit) {
        // ---- dequantise the tile: warp w fills entries 4w .. 4w+3, lane owns 16 channels
        bool valid[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int e = warp * 4 + i;
            const int u = u0 + e / kAttnUnit, j = e % kAttnUnit;
            EntryRef r;
            valid[i] = u < u_end && entry_ref(a, sv, u, j, r);
            float v[16];
            if (valid[i]) {
                dequant16(r, lane, v);
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) v[c] = 0.f;
            }
            float4 *dst = reinterpret_cast<float4 *>(Vs + e * kCcRow + 16 * lane);
#pragma unroll
            for (int c = 0; c < 4; ++c) dst[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
        }
        __syncthreads();
        // ---- scores: warp w, entries 4w..4w+3, every head; lanes split the 512 channels
        {
            float v[4][16];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float4 *src = reinterpret_cast<const float4 *>(Vs + (warp * 4 + i) * kCcRow + 16 * lane);
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 f = src[c];
                    v[i][4 * c] = f.x;
                    v[i][4 * c + 1] = f.y;
                    v[i][4 * c + 2] = f.z;
                    v[i][4 * c + 3] = f.w;
                }
            }
            for (int h = 0; h < HG; ++h) {
                const float4 *qs = reinterpret_cast<const float4 *>(Qs + h * kCcRow + 16 * lane);
                float qv[16];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const float4 f = qs[c];
                    qv[4 * c] = f.x;
                    qv[4 * c + 1] = f.y;
                    qv[4 * c + 2] = f.z;
                    qv[4 * c + 3] = f.w;
                }
                float d[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float x = 0.f;
#pragma unroll
                    for (int c = 0; c < 16; ++c) x = fmaf(qv[c], v[i][c], x);
                    d[i] = x;
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) d[i] += __shfl_xor_sync(0xffffffffu, d[i], o);
                }
                if (lane == 0) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) Ps[(warp * 4 + i) * HG + h] = valid[i] ? a.sm_scale * d[i] : -INFINITY;
                }
            }
        }
        __syncthreads();
        // ---- online softmax per head
        if (t < HG) {
            float mt = -INFINITY;
            for (int e = 0; e < kCcTile; ++e) mt = fmaxf(mt, Ps[e * HG + t]);
            const float m_old = m_s[t];
            const float m_new = fmaxf(m_old, mt);
            float alpha = 1.f, sum = 0.f;
            if (m_new != -INFINITY) {
                alpha = expf(m_old - m_new);
                for (int e = 0; e < kCcTile; ++e) {
                    const float z = Ps[e * HG + t];
                    const float p = z == -INFINITY ? 0.f : expf(z - m_new);
                    Ps[e * HG + t] = p;
                    sum += p;
                }
            } else {
                for (int e = 0; e < kCcTile; ++e) Ps[e * HG + t] = 0.f;
            }
            alpha_s[t] = alpha;
            m_s[t] = m_new;
            l_s[t] = l_s[t] * alpha + sum;
        }
        __syncthreads();
        // ---- o += P^T V: thread t owns channels 2t, 2t+1 of every head
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            const float al = alpha_s[h];
            acc[h][0] *= al;
            acc[h][1] *= al;
        }
        for (int e = 0; e < kCcTile; ++e) {
            const float2 v = *reinterpret_cast<const float2 *>(Vs + e * kCcRow + 2 * t);
#pragma unroll
            for (int h = 0; h < HG; ++h) {
                const float p = Ps[e * HG + h];
                acc[h][0] = fmaf(p, v.x, acc[h][0]);
                acc[h][1] = fmaf(p, v.y, acc[h][1]);
            }
        }
        __syncthreads();
    }
    // ---- unnormalised partial of this split
    float *po = a.part_o + (((size_t)b * a.splits + s) * a.H + h0) * kLatent;
#pragma unroll
    for (int h = 0; h < HG; ++h)
        *reinterpret_cast<float2 *>(po + (size_t)h * kLatent + 2 * t) = make_float2(acc[h][0], acc[h][1]);
    if (t < HG) {
        float2 *pml = reinterpret_cast<float2 *>(a.part_ml) + ((size_t)b * a.splits + s) * a.H + h0 + t;
        *pml = make_float2(m_s[t], l_s[t]);
    }
}

template <int HG>
static cudaError_t launch_cc(const AttnArgs &a, cudaStream_t st)
{
    const size_t smem = (size_t)(HG * kCcRow + kCcTile * kCcRow + kCcTile * HG + 3 * HG) * 4;
    cudaError_t e =
        allow_dynamic_smem(reinterpret_cast<const void *>(attn_split_cc_kernel<HG>), smem);
    if (e != cudaSuccess) return e;
    const int groups = a.H / HG;
    dim3 grid(a.splits, a.B * groups);
    attn_split_cc_kernel<HG><<<grid, kCcThreads, smem, st>>>(a, groups);
    return cudaGetLastError();
}

cudaError_t launch_attn_cc(const AttnArgs &a, cudaStream_t st)
{
    if (a.H == 16) return launch_cc<16>(a, st);
    return launch_cc<32>(a, st);
}

// ------------------------------------------------------------------------------------------------
// Split combine: out = sum_s e^{m_s - M} o_s / sum_s e^{m_s - M} l_s, lse = M + ln(sum ...).
// One CTA per (head, sequence): the split weights are computed once into shared memory, then each
// thread accumulates 4 channels with its loads of consecutive splits independent of one another.
// ------------------------------------------------------------------------------------------------
constexpr int kCombineMaxSplits = 1024;

__global__ void __launch_bounds__(128) attn_combine_kernel(const float *__restrict__ part_o,
                                                          const float2 *__restrict__ part_ml, int splits, int H,
                                                          float *__restrict__ out, float *__restrict__ lse)
{
    __shared__ float wgt[kCombineMaxSplits];
    __shared__ float red[8];
    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x, lane = t & 31, warp = t >> 5;
    grid_dep_wait();   // every split's partial
    grid_dep_launch();   // a dependent kernel launched after this one waits for it before reading
    // the partials of the first kPre splits are loaded at once, before (and independently of) the
    // split weights, so that the whole read is one round trip
    constexpr int kPre = 24;
    const float4 *po = reinterpret_cast<const float4 *>(part_o + ((size_t)b * splits * H + h) * kLatent) + t;
    const size_t stride = (size_t)H * kLatent / 4;
    float4 pre[kPre];
#pragma unroll
    for (int q = 0; q < kPre; ++q)
        if (q < splits) pre[q] = po[(size_t)q * stride];
    const float2 *ml = part_ml + (size_t)b * splits * H + h;
    float M = -INFINITY;
    for (int s = t; s < splits; s += 128) M = fmaxf(M, ml[(size_t)s * H].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    if (lane == 0) red[warp] = M;
    __syncthreads();
    M = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    float den = 0.f;
    for (int s = t; s < splits; s += 128) {
        const float2 v = ml[(size_t)s * H];
        const float wv = (v.x == -INFINITY || M == -INFINITY) ? 0.f : expf(v.x - M);
        wgt[s] = wv;
        den = fmaf(wv, v.y, den);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    __syncthreads();
    if (lane == 0) red[4 + warp] = den;
    __syncthreads();
    den = red[4] + red[5] + red[6] + red[7];
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int q = 0; q < kPre; ++q) {
        if (q < splits) {
            const float wv = wgt[q];
            acc.x = fmaf(wv, pre[q].x, acc.x);
            acc.y = fmaf(wv, pre[q].y, acc.y);
            acc.z = fmaf(wv, pre[q].z, acc.z);
            acc.w = fmaf(wv, pre[q].w, acc.w);
        }
    }
    for (int s = kPre; s < splits; ++s) {
        const float4 o = po[(size_t)s * stride];
        const float wv = wgt[s];
        acc.x = fmaf(wv, o.x, acc.x);
        acc.y = fmaf(wv, o.y, acc.y);
        acc.z = fmaf(wv, o.z, acc.z);
        acc.w = fmaf(wv, o.w, acc.w);
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    reinterpret_cast<float4 *>(out + ((size_t)b * H + h) * kLatent)[t] =
        make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (t == 0) lse[(size_t)b * H + h] = den > 0.f ? M + logf(den) : -INFINITY;
}

cudaError_t launch_attn_combine(const AttnArgs &a, float *out, float *lse, cudaStream_t st)
{
    dim3 grid(a.H, a.B);
    return launch_overlapped(attn_combine_kernel, grid, dim3(128), 0, st, a.part_o,
                             reinterpret_cast<const float2 *>(a.part_ml), a.splits, a.H, out, lse);
}

}  // namespace csa
