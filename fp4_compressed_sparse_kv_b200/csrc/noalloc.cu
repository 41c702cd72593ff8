// noalloc.cu -- csa_indexer_full_noalloc: the Full-layer indexer (block scores + exact Top-K) for
// callers that cannot hand the library a workspace.
//
// Some callers have no way to obtain device memory at the point where they run the indexer: a runtime
// with a fixed, pre-reserved memory budget that forbids allocation after start-up, a plugin living
// inside a host framework that owns the allocator and does not expose it, or code paths that must not
// call into an allocator for latency or determinism reasons.  For them the scratch this call needs (a
// 256-byte status word and one float per block of every sequence) lives in a fixed array compiled
// into the library, so the call itself allocates nothing.
#include <mutex>

#include "common.cuh"

namespace csa {

cudaError_t launch_block_scores_full_or_pool(const uint8_t *keys, int num_pages, const csa_batch &bt,
                                             const uint16_t *iq, const float *iw, const int32_t *pool,
                                             const int32_t *pool_count, int pool_cap, float *scores,
                                             int score_stride, void *ws, cudaStream_t st);
cudaError_t launch_topk(const float *scores, int score_stride, const int32_t *seq_len, int max_seq_len,
                        const int32_t *pool, const int32_t *pool_count, int pool_cap, int k, int B,
                        int32_t *out_blocks, int32_t *out_count, int max_candidates, void *ws, cudaStream_t st);

}  // namespace csa

using namespace csa;

namespace {

// 4 MiB per GPU, held by every device that loads this library for the life of the process.
constexpr size_t kNoAllocBytes = (size_t)CSA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocBytes];

// The array's name in host code is only a host-side handle; the kernels need its device address,
// looked up once per device (with that device current) and cached.
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kMaxDevices];

cudaError_t noalloc_scratch(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return cudaSuccess;
}

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

}  // namespace

extern "C" csa_status csa_indexer_full_noalloc(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq,
                                               const float *iw, int32_t k, int32_t *out_blocks, int32_t *out_count,
                                               int32_t *dev_status, void *stream)
{
    if (!layer || !layer->keys || layer->num_pages < 1 || !aligned16(layer->keys)) return CSA_ERR_INVALID_ARG;
    if (!batch || batch->B < 1 || batch->B > 16384 || !batch->seq_len || !batch->block_table || !batch->swa_row)
        return CSA_ERR_INVALID_ARG;
    if (batch->max_seq_len < 1 || batch->max_seq_len > CSA_MAX_SEQ_LEN) return CSA_ERR_INVALID_ARG;
    if (batch->max_pages < (batch->max_seq_len + kPage - 1) / kPage) return CSA_ERR_INVALID_ARG;
    if (!aligned16(batch->seq_len) || !aligned16(batch->block_table) || !aligned16(batch->swa_row))
        return CSA_ERR_INVALID_ARG;
    if (!iq || !iw || !out_blocks || !out_count || !aligned16(iq) || !aligned16(iw) || !aligned16(out_blocks) ||
        !aligned16(out_count))
        return CSA_ERR_INVALID_ARG;
    if (dev_status && !aligned16(dev_status)) return CSA_ERR_INVALID_ARG;
    if (k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID_ARG;

    // scratch: status header, then one float per block of every sequence
    const int nb_max = (batch->max_seq_len + kBlock - 1) / kBlock;
    const int stride = nb_max > k ? nb_max : k;
    const size_t need = kHeaderBytes + (size_t)batch->B * (size_t)stride * 4;
    if (need > kNoAllocBytes) return CSA_ERR_WORKSPACE;

    void *ws = nullptr;
    if (noalloc_scratch(&ws) != cudaSuccess) return CSA_ERR_CUDA;
    cudaStream_t st = (cudaStream_t)stream;
    // the status word must start at zero; the scores are written before they are read
    if (cudaMemsetAsync(ws, 0, kHeaderBytes, st) != cudaSuccess) return CSA_ERR_CUDA;
    float *scores = reinterpret_cast<float *>((char *)ws + kHeaderBytes);
    if (launch_block_scores_full_or_pool(layer->keys, layer->num_pages, *batch, iq, iw, nullptr, nullptr, 0, scores,
                                         stride, ws, st) != cudaSuccess)
        return CSA_ERR_CUDA;
    if (launch_topk(scores, stride, batch->seq_len, batch->max_seq_len, nullptr, nullptr, 0, k, batch->B, out_blocks,
                    out_count, nb_max, ws, st) != cudaSuccess)
        return CSA_ERR_CUDA;
    if (dev_status && cudaMemcpyAsync(dev_status, ws, sizeof(int32_t), cudaMemcpyDeviceToDevice, st) != cudaSuccess)
        return CSA_ERR_CUDA;
    return CSA_OK;
}
