// radix.cuh -- block-wide radix selection over 32-bit order keys (one CTA per problem).
#pragma once

#include <stdint.h>

namespace csa {

// Min or max of v over the CTA (blockDim.x a multiple of 32, at most 1024 threads).  scratch holds
// at least 33 words.  Every thread gets the result.
__device__ __forceinline__ uint32_t block_reduce_minmax(uint32_t v, bool is_max, uint32_t *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const uint32_t y = __shfl_xor_sync(0xffffffffu, v, o);
        v = is_max ? max(v, y) : min(v, y);
    }
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? scratch[lane] : (is_max ? 0u : 0xFFFFFFFFu);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            const uint32_t y = __shfl_xor_sync(0xffffffffu, v, o);
            v = is_max ? max(v, y) : min(v, y);
        }
        if (lane == 0) scratch[32] = v;
    }
    __syncthreads();
    v = scratch[32];
    __syncthreads();
    return v;
}

// Sum of v over the CTA (same rules as block_reduce_minmax).
__device__ __forceinline__ uint32_t block_reduce_sum(uint32_t v, uint32_t *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? scratch[lane] : 0u;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) scratch[32] = v;
    }
    __syncthreads();
    v = scratch[32];
    __syncthreads();
    return v;
}

// Exclusive prefix of v over the CTA in thread order (blockDim.x a multiple of 32, at most 1024
// threads; scratch holds at least 32 words); every thread also gets the total.  Two barriers.
__device__ __forceinline__ uint32_t cta_scan(uint32_t v, uint32_t *scratch, uint32_t &total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (int)(blockDim.x >> 5);
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) scratch[warp] = x;
    __syncthreads();
    uint32_t before = 0;
    total = 0;
    for (int w = 0; w < nw; ++w) {
        const uint32_t c = scratch[w];
        before += w < warp ? c : 0u;
        total += c;
    }
    __syncthreads();
    return before + x - v;
}

// The k-th largest of n keys (1 <= k <= n), MSB first in digits of up to 8 bits with per-warp
// shared-memory histograms (whist: kWarps x 256 words).  The bits every key shares (the common
// prefix of the smallest and largest key) are skipped.  Bits below stop_bit may stay unresolved:
// the k-th largest key X then satisfies (X & resolved) == T with T's unresolved bits clear, so
// T <= X <= T | ~resolved (resolved is all ones, and T == X, when stop_bit == 0).  need_eq, exact
// only when everything is resolved, is how many keys equal to T belong to the k largest (the rest
// of the k are > T).  key(i) must return the same value on every call.
template <int kThreads, typename KeyFn>
__device__ __forceinline__ void radix_select(int n, uint32_t k, KeyFn key, int stop_bit, uint32_t *whist,
                                             uint32_t *scratch, uint32_t *sel, uint32_t &T, uint32_t &need_eq,
                                             uint32_t *resolved = nullptr)
{
    constexpr int kWarps = kThreads / 32;
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int i = t; i < n; i += kThreads) {
        const uint32_t u = key(i);
        kmin = min(kmin, u);
        kmax = max(kmax, u);
    }
    kmin = block_reduce_minmax(kmin, false, scratch);
    kmax = block_reduce_minmax(kmax, true, scratch);

    uint32_t prefix = kmax, mask = 0xFFFFFFFFu, remaining = k;
    if (kmin != kmax) {
        int hi = 31 - __clz(kmin ^ kmax);   // highest bit that differs between keys
        mask = hi == 31 ? 0u : ~((2u << hi) - 1u);
        prefix = kmax & mask;
        while (hi >= stop_bit) {
            const int width = hi + 1 < 8 ? hi + 1 : 8;
            const int shift = hi + 1 - width;
            const uint32_t dmask = (1u << width) - 1u;
            for (int i = t; i < kWarps * 256; i += kThreads) whist[i] = 0u;
            __syncthreads();
            for (int i = t; i < n; i += kThreads) {
                const uint32_t u = key(i);
                if ((u & mask) == prefix) atomicAdd(&whist[warp * 256 + ((u >> shift) & dmask)], 1u);
            }
            __syncthreads();
            // bin totals, then counts from the top bin down; the threshold bin is where they reach
            // `remaining`
            uint32_t c = 0;
            if (t < 256) {
                const int bin = 255 - t;
#pragma unroll 8
                for (int w = 0; w < kWarps; ++w) c += whist[w * 256 + bin];
            }
            uint32_t x = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (t < 256 && lane == 31) scratch[warp] = x;
            __syncthreads();
            if (t < 256) {
                uint32_t before = 0;
                for (int wi = 0; wi < warp; ++wi) before += scratch[wi];
                const uint32_t incl = before + x;
                if (incl >= remaining && incl - c < remaining) {
                    sel[0] = 255u - (uint32_t)t;
                    sel[1] = incl - c;
                }
            }
            __syncthreads();
            prefix |= sel[0] << shift;
            mask |= dmask << shift;
            remaining -= sel[1];
            hi = shift - 1;
            __syncthreads();
        }
    }
    T = prefix;
    need_eq = remaining;
    if (resolved) *resolved = mask;
}

}  // namespace csa
