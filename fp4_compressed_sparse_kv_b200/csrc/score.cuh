// score.cuh -- the exact indexer score of one position, shared by every exact scorer.
//
// rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": the
// position score is sum_h w_h * ReLU(q_h . k) over 8 heads of 128-dim E4M3 keys.  csa.h fixes the
// binary32 operation order: per head, 8 chains of 16 FMAs from +0 (dims 16j .. 16j+15), combined as
// ((p0 + p4) + (p2 + p6)) + ((p1 + p5) + (p3 + p7)), then ReLU, then an FMA chain over h = 0..7 from
// +0.  A warp scores 4 keys at a time: lane (g, j) = (lane / 8, lane % 8) holds dims 16j .. 16j+15 of
// key g and of all 8 query heads; lane j keeps head s ^ j in slot s, so the 3-step xor reduction
// (distances 4, 2, 1) leaves head j's sum in lane j with the order above (up to commutativity).  The
// 16-term chains run as packed fma.rn.f32x2 over head pairs: two independent IEEE FMAs each.
#pragma once

#include <stdint.h>

#include "common.cuh"
#include "convert.cuh"

namespace csa {

__device__ __forceinline__ unsigned long long f2_pack(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}

__device__ __forceinline__ void f2_unpack(unsigned long long v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

__device__ __forceinline__ unsigned long long ffma2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}

// Query pairs q2(s2, t) = (q[h(2 s2)][16j+t], q[h(2 s2+1)][16j+t]), h(s) = s ^ j, of this lane's j:
// held in registers ...
struct QRegs {
    const unsigned long long (&q2)[4][16];
    __device__ __forceinline__ unsigned long long operator()(int s2, int t) const { return q2[s2][t]; }
};

// ... or in shared memory, one row of 4 x 16 pairs per j, rows kQRowPairs pairs apart (the odd pad
// puts the 8 rows' same pair in 8 different bank pairs).  The loads are volatile so that they are
// issued where the chain needs them instead of being hoisted into 128 registers.
constexpr int kQRowPairs = 4 * 16 + 1;
struct QSmem {
    const volatile unsigned long long *row;   // this lane's row
    __device__ __forceinline__ unsigned long long operator()(int s2, int t) const { return row[16 * s2 + t]; }
};

// The 8 query heads of one sequence (bf16 [8][128]) as the pairs of lane j = 0..7: row j of qs.
// Called by all threads of a CTA (any count); the caller synchronises before use.
__device__ __forceinline__ void load_query_pairs(const uint16_t *iq, unsigned long long *qs)
{
    for (int e = threadIdx.x; e < 8 * 64; e += blockDim.x) {
        const int j = e >> 6, s2 = (e >> 4) & 3, t = e & 15;
        const int h0 = (2 * s2) ^ j, h1 = (2 * s2 + 1) ^ j;
        const uint16_t a = iq[h0 * kIdxDim + 16 * j + t], b = iq[h1 * kIdxDim + 16 * j + t];
        qs[j * kQRowPairs + 16 * s2 + t] = f2_pack(__uint_as_float((uint32_t)a << 16), __uint_as_float((uint32_t)b << 16));
    }
}

// Score of the key whose dims 16j..16j+15 this lane holds in kr.
template <typename Q>
__device__ __forceinline__ float score_key(const Q &q2, const float (&w)[8], uint4 kr, int lane)
{
    unsigned long long k2[16];
    const uint32_t kw[4] = {kr.x, kr.y, kr.z, kr.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        uint32_t hv[2];
        e4m3x4_to_f16x2x2(kw[i], hv);
        const float k0 = h_lo(hv[0]), k1 = h_hi(hv[0]), k2v = h_lo(hv[1]), k3 = h_hi(hv[1]);
        k2[4 * i + 0] = f2_pack(k0, k0);
        k2[4 * i + 1] = f2_pack(k1, k1);
        k2[4 * i + 2] = f2_pack(k2v, k2v);
        k2[4 * i + 3] = f2_pack(k3, k3);
    }
    float p[8];
#pragma unroll
    for (int s2 = 0; s2 < 4; ++s2) {
        unsigned long long acc = 0ull;   // (+0, +0)
#pragma unroll
        for (int t = 0; t < 16; ++t) acc = ffma2(q2(s2, t), k2[t], acc);
        f2_unpack(acc, p[2 * s2], p[2 * s2 + 1]);
    }
    float a[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) a[i] = __fadd_rn(p[i], __shfl_xor_sync(0xffffffffu, p[4 + i], 4));
    float c[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) c[i] = __fadd_rn(a[i], __shfl_xor_sync(0xffffffffu, a[2 + i], 2));
    const float d = __fadd_rn(c[0], __shfl_xor_sync(0xffffffffu, c[1], 1));
    const float r = d > 0.f ? d : 0.f;
    float score = 0.f;
    const int base = lane & ~7;
#pragma unroll
    for (int h = 0; h < 8; ++h) score = __fmaf_rn(w[h], __shfl_sync(0xffffffffu, r, base | h), score);
    return score;
}

}  // namespace csa
