// context_parallel.cu -- the exchange steps of context-parallel decode of long sequences: each rank
// holds a contiguous, page-aligned slice of a sequence's positions, runs the Full indexer and the
// attention on its slice, and the ranks combine their results exactly.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": the Full
// layer's hierarchical indexer scans the whole range for the Top-K blocks; sharding that range by
// position keeps the result exact because every block of the global Top-K is in the Top-K of its
// own shard (fewer than K blocks of that shard beat it), so the global Top-K is the Top-K of the
// union of the shards' Top-K candidates under the same (score, lower block id) order.  Attention
// over the union of the shards' selected entries (plus the window, on the shard that holds the last
// positions) is the log-sum-exp merge of the shards' attentions, since every shard's output is its
// own normalised softmax average with its log-sum-exp.
//
//   candidates_concat: the shards' candidate lists (local block ids, exact scores) into one list of
//                      global block ids, ascending (shards hold ascending, disjoint ranges);
//   shard_blocks:      the part of a global block set that falls in a shard, as local block ids;
//   attn_merge:        out = sum_r e^{lse_r - LSE} out_r, LSE = log sum_r e^{lse_r}.
#include "common.cuh"

namespace csa {

__global__ void __launch_bounds__(256) cand_concat_kernel(int R, int cap, const int32_t *__restrict__ ids,
                                                          const float *__restrict__ scores,
                                                          const int32_t *__restrict__ counts,
                                                          const int32_t *__restrict__ offsets, int B,
                                                          int32_t *__restrict__ out_ids, float *__restrict__ out_scores,
                                                          int32_t *__restrict__ out_count, void *ws)
{
    __shared__ int base[65];
    const int b = blockIdx.x, t = threadIdx.x;
    if (t == 0) {
        int run = 0;
        for (int r = 0; r < R; ++r) {
            int n = counts[(size_t)r * B + b];
            if (n < 0 || n > cap) {
                report(ws, CSA_ERR_DEVICE_DATA, (long long)r);
                n = 0;
            }
            base[r] = run;
            run += n;
        }
        base[R] = run;
        out_count[b] = run;
    }
    __syncthreads();
    for (int r = 0; r < R; ++r) {
        const int n = base[r + 1] - base[r];
        const int off = offsets[(size_t)r * B + b];
        const int32_t *src = ids + ((size_t)r * B + b) * cap;
        const float *ssrc = scores + ((size_t)r * B + b) * cap;
        int32_t *dst = out_ids + (size_t)b * R * cap + base[r];
        float *sdst = out_scores + (size_t)b * R * cap + base[r];
        for (int i = t; i < n; i += blockDim.x) {
            dst[i] = src[i] + off;
            sdst[i] = ssrc[i];
        }
    }
}

// One warp per sequence: the entries of blocks[b][0 .. count[b]) in [lo[b], hi[b]), minus lo[b], in
// order.
__global__ void __launch_bounds__(32) shard_blocks_kernel(const int32_t *__restrict__ blocks,
                                                          const int32_t *__restrict__ count, int cap,
                                                          const int32_t *__restrict__ lo, const int32_t *__restrict__ hi,
                                                          int32_t *__restrict__ out_blocks, int32_t *__restrict__ out_count,
                                                          int out_cap, void *ws)
{
    const int b = blockIdx.x, lane = threadIdx.x;
    int n = count[b];
    if (n < 0 || n > cap) {
        if (lane == 0) report(ws, CSA_ERR_DEVICE_DATA, (long long)b);
        n = 0;
    }
    const int l = lo[b], h = hi[b];
    const int32_t *src = blocks + (size_t)b * cap;
    int32_t *dst = out_blocks + (size_t)b * out_cap;
    int written = 0;
    for (int i0 = 0; i0 < n; i0 += 32) {
        const int i = i0 + lane;
        const int v = i < n ? src[i] : 0;
        const bool in = i < n && v >= l && v < h;
        const uint32_t m = __ballot_sync(0xffffffffu, in);
        const int pos = written + __popc(m & ((1u << lane) - 1u));
        if (in && pos < out_cap) dst[pos] = v - l;
        written += __popc(m);
    }
    if (lane == 0) {
        if (written > out_cap) {
            report(ws, CSA_ERR_DEVICE_DATA, (long long)b);
            written = out_cap;
        }
        out_count[b] = written;
    }
}

// One CTA per (head, sequence); thread t merges channels 4t .. 4t+3.
__global__ void __launch_bounds__(128) attn_merge_kernel(int R, int B, int H, const float *__restrict__ out_parts,
                                                         const float *__restrict__ lse_parts, float *__restrict__ out,
                                                         float *__restrict__ lse)
{
    const int h = blockIdx.x, b = blockIdx.y, t = threadIdx.x;
    const size_t stride_l = (size_t)B * H, idx = (size_t)b * H + h;
    float M = -INFINITY;
    for (int r = 0; r < R; ++r) M = fmaxf(M, lse_parts[r * stride_l + idx]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;
    if (M > -INFINITY) {
        for (int r = 0; r < R; ++r) {
            const float lr = lse_parts[r * stride_l + idx];
            const float wr = lr == -INFINITY ? 0.f : expf(lr - M);
            if (wr == 0.f) continue;
            const float4 o = reinterpret_cast<const float4 *>(out_parts + (r * stride_l + idx) * kLatent)[t];
            acc.x = fmaf(wr, o.x, acc.x);
            acc.y = fmaf(wr, o.y, acc.y);
            acc.z = fmaf(wr, o.z, acc.z);
            acc.w = fmaf(wr, o.w, acc.w);
            den += wr;
        }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    reinterpret_cast<float4 *>(out + idx * kLatent)[t] = make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
    if (t == 0) lse[idx] = den > 0.f ? M + logf(den) : -INFINITY;
}

}  // namespace csa

using namespace csa;

namespace {
inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }
inline csa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }
}  // namespace

extern "C" {

csa_status csa_candidates_concat(int32_t R, int32_t B, int32_t cap, const int32_t *ids, const float *scores,
                                 const int32_t *counts, const int32_t *offsets, int32_t *out_ids, float *out_scores,
                                 int32_t *out_count, void *ws, size_t ws_bytes, void *stream)
{
    if (R < 1 || R > CSA_MAX_SHARDS || B < 1 || B > 16384 || cap < 1 || cap > CSA_MAX_TOPK) return CSA_ERR_INVALID_ARG;
    if (!ids || !scores || !counts || !offsets || !out_ids || !out_scores || !out_count || !ws)
        return CSA_ERR_INVALID_ARG;
    if (!aligned16(ids) || !aligned16(scores) || !aligned16(counts) || !aligned16(offsets) || !aligned16(out_ids) ||
        !aligned16(out_scores) || !aligned16(out_count) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    cand_concat_kernel<<<B, 256, 0, (cudaStream_t)stream>>>(R, cap, ids, scores, counts, offsets, B, out_ids, out_scores,
                                                           out_count, ws);
    return cuda_status(cudaGetLastError());
}

csa_status csa_shard_blocks(int32_t B, const int32_t *blocks, const int32_t *count, int32_t cap, const int32_t *lo,
                            const int32_t *hi, int32_t *out_blocks, int32_t *out_count, int32_t out_cap, void *ws,
                            size_t ws_bytes, void *stream)
{
    if (B < 1 || B > 16384 || cap < 1 || out_cap < 1) return CSA_ERR_INVALID_ARG;
    if (!blocks || !count || !lo || !hi || !out_blocks || !out_count || !ws) return CSA_ERR_INVALID_ARG;
    if (!aligned16(blocks) || !aligned16(count) || !aligned16(lo) || !aligned16(hi) || !aligned16(out_blocks) ||
        !aligned16(out_count) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    shard_blocks_kernel<<<B, 32, 0, (cudaStream_t)stream>>>(blocks, count, cap, lo, hi, out_blocks, out_count, out_cap,
                                                            ws);
    return cuda_status(cudaGetLastError());
}

csa_status csa_attn_merge(int32_t R, int32_t B, int32_t H, const float *out_parts, const float *lse_parts, float *out,
                          float *lse, void *stream)
{
    if (R < 1 || R > CSA_MAX_SHARDS || B < 1 || B > 16384) return CSA_ERR_INVALID_ARG;
    if (!(H == 16 || H == 32 || H == 64 || H == 128)) return CSA_ERR_UNSUPPORTED;
    if (!out_parts || !lse_parts || !out || !lse) return CSA_ERR_INVALID_ARG;
    if (!aligned16(out_parts) || !aligned16(lse_parts) || !aligned16(out) || !aligned16(lse)) return CSA_ERR_INVALID_ARG;
    attn_merge_kernel<<<dim3(H, B), 128, 0, (cudaStream_t)stream>>>(R, B, H, out_parts, lse_parts, out, lse);
    return cuda_status(cudaGetLastError());
}

}  // extern "C"
