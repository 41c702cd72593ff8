// attention_common.cuh -- work decomposition and entry addressing shared by the attention kernels.
//
// A sequence's attention entries form a list of 8-entry units: first its count[b] selected blocks
// (positions 8*blk .. 8*blk+7, those >= seq_len masked), then the sliding window
// max(0, L-128) .. L-1 in 8-position chunks.  Addresses follow from the token index alone (fixed
// 288-byte FP4 entries and 516-byte window entries), as the yomxxx.com long-form post (section 五)
// requires of a kernel-friendly KV format.
#pragma once

#include "common.cuh"
#include "convert.cuh"

namespace csa {

struct AttnArgs {
    const uint8_t *codes;
    const uint8_t *scales;
    const uint8_t *swa;
    const float *swa_scale;
    int num_pages;
    int num_rows;
    int B;
    const int32_t *seq_len;
    const int32_t *block_table;
    int max_pages;
    const int32_t *swa_row;
    int max_seq_len;
    const uint16_t *q;
    int H;
    float sm_scale;
    const int32_t *blocks;
    const int32_t *count;
    int cap;
    float *part_o;
    float *part_ml;
    int splits;
    void *ws;
};

struct SeqView {
    int L;
    int nb;
    int nE;      // selected blocks
    int nF;      // window entries
    int units;   // nE + ceil(nF / 8)
    int w0;      // first window position
    int row;     // SWA ring row
    const int32_t *bt;
    const int32_t *blocks;
};

__device__ __forceinline__ bool seq_view(const AttnArgs &a, int b, SeqView &v)
{
    v.L = a.seq_len[b];
    if (v.L < 1 || v.L > a.max_seq_len) {
        report(a.ws, CSA_ERR_DEVICE_DATA, b);
        return false;
    }
    v.nb = (v.L + kBlock - 1) / kBlock;
    v.nE = a.count[b];
    if (v.nE < 0 || v.nE > a.cap) {
        report(a.ws, CSA_ERR_DEVICE_DATA, b);
        v.nE = 0;
    }
    v.row = a.swa_row[b];
    v.nF = v.L < kWindow ? v.L : kWindow;
    if (v.row == -1) {
        v.nF = 0;   // no window segment: a shard that does not hold the sequence's last positions
    } else if (v.row < 0 || v.row >= a.num_rows) {
        report(a.ws, CSA_ERR_DEVICE_DATA, b);
        v.nF = 0;
    }
    v.w0 = v.L - (v.L < kWindow ? v.L : kWindow);
    v.units = v.nE + (v.nF + kAttnUnit - 1) / kAttnUnit;
    v.bt = a.block_table + (size_t)b * a.max_pages;
    v.blocks = a.blocks + (size_t)b * a.cap;
    return true;
}

__device__ __forceinline__ void split_range(int units, int s, int splits, int &ub, int &ue)
{
    ub = (int)((long long)units * s / splits);
    ue = (int)((long long)units * (s + 1) / splits);
}

struct EntryRef {
    bool swa;
    const uint8_t *p;    // 256 B of codes, or 512 B of window values
    const uint8_t *sc;   // 32 E4M3 scales (FP4 entry)
    float fscale;        // window entry scale
};

// Entry j of unit u; false if masked (position >= L) or if its metadata is out of range (reported).
__device__ __forceinline__ bool entry_ref(const AttnArgs &a, const SeqView &v, int u, int j, EntryRef &r)
{
    if (u < v.nE) {
        const int blk = v.blocks[u];
        if (blk < 0 || blk >= v.nb) {
            report(a.ws, CSA_ERR_DEVICE_DATA, u);
            return false;
        }
        const int p = blk * kBlock + j;
        if (p >= v.L) return false;
        const int page = v.bt[blk / kBlocksPerPage];
        if (page < 0 || page >= a.num_pages) {
            report(a.ws, CSA_ERR_DEVICE_DATA, blk);
            return false;
        }
        const size_t row = (size_t)page * kPage + (size_t)(blk % kBlocksPerPage) * kBlock + j;
        r.swa = false;
        r.p = a.codes + row * kCodeBytes;
        r.sc = a.scales + row * kScaleBytes;
        r.fscale = 0.f;
        return true;
    }
    const int p = v.w0 + (u - v.nE) * kAttnUnit + j;
    if (p >= v.L) return false;
    const size_t slot = (size_t)v.row * kWindow + (p % kWindow);
    r.swa = true;
    r.p = a.swa + slot * kLatent;
    r.sc = nullptr;
    r.fscale = a.swa_scale[slot];
    return true;
}

// Channels 16*lane .. 16*lane+15 of an entry, dequantised to fp32 (exact for FP4 entries).
__device__ __forceinline__ void dequant16(const EntryRef &r, int lane, float *v)
{
    if (!r.swa) {
        const uint2 c = reinterpret_cast<const uint2 *>(r.p)[lane];
        const float s = e4m3_to_f32(r.sc[lane]);
        uint32_t h2[8];
        e2m1x8_to_f16x2x4(c.x, h2);
        e2m1x8_to_f16x2x4(c.y, h2 + 4);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[2 * i] = h_lo(h2[i]) * s;
            v[2 * i + 1] = h_hi(h2[i]) * s;
        }
    } else {
        const uint4 c = reinterpret_cast<const uint4 *>(r.p)[lane];
        const uint32_t cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint32_t hv[2];
            e4m3x4_to_f16x2x2(cw[i], hv);
            v[4 * i] = h_lo(hv[0]) * r.fscale;
            v[4 * i + 1] = h_hi(hv[0]) * r.fscale;
            v[4 * i + 2] = h_lo(hv[1]) * r.fscale;
            v[4 * i + 3] = h_hi(hv[1]) * r.fscale;
        }
    }
}

cudaError_t launch_attn_cc(const AttnArgs &a, cudaStream_t st);
cudaError_t launch_attn_combine(const AttnArgs &a, float *out, float *lse, cudaStream_t st);

}  // namespace csa
