// abi.cu -- the extern "C" entry points declared in include/csa.h: argument validation, workspace
// carving and kernel launches.  No allocation, no synchronisation (except csa_check_device_error).
#include <string.h>

#include "attention_common.cuh"
#include "common.cuh"

namespace csa {

struct ScoreArgs;
cudaError_t launch_kv_pack(const csa_kv_layer &layer, const uint16_t *latent, const uint16_t *idx_key,
                           const int64_t *slot, const int32_t *swa_slot, int n, void *ws, cudaStream_t st);
cudaError_t launch_kv_norm_rope_pack(const csa_kv_layer &layer, const uint16_t *latent, const float *norm_w,
                                     const float *rope_cs, const uint16_t *idx_key, const int64_t *slot,
                                     const int32_t *swa_slot, int n, void *ws, cudaStream_t st);
cudaError_t launch_topk(const float *scores, int score_stride, const int32_t *seq_len, int max_seq_len,
                        const int32_t *pool, const int32_t *pool_count, int pool_cap, int k, int B,
                        int32_t *out_blocks, int32_t *out_count, int max_candidates, void *ws, cudaStream_t st);
cudaError_t launch_reuse(int B, const int32_t *prev, const int32_t *prev_count, int prev_cap, int32_t *out,
                         int32_t *out_count, int out_cap, void *ws, cudaStream_t st);
cudaError_t launch_block_scores_full_or_pool(const uint8_t *keys, int num_pages, const csa_batch &bt,
                                             const uint16_t *iq, const float *iw, const int32_t *pool,
                                             const int32_t *pool_count, int pool_cap, float *scores,
                                             int score_stride, void *ws, cudaStream_t st);
bool screen_supported(int num_pages);
cudaError_t launch_screen_bounds(const uint8_t *keys, int num_pages, const csa_batch &bt, const uint16_t *iq,
                                 const float *iw, uint8_t *qt, void *qm, uint32_t *hist, uint32_t *hist2, float *lo,
                                 float *hi, int stride, void *ws, cudaStream_t st);
cudaError_t launch_select(const float *lo, const float *hi, int lstride, const csa_batch &bt, int k,
                          const uint32_t *hist, uint32_t *hist2, uint8_t *status, int sstride, int32_t *uslice,
                          uint32_t *okeys, int ustride, const uint8_t *keys, int num_pages,
                          const uint16_t *iq, const float *iw, int32_t *out_blocks, int32_t *out_count, void *ws,
                          cudaStream_t st);
cudaError_t launch_attn_tc(const AttnArgs &a, cudaStream_t st);
bool attn_tc_supported(int H);
bool attn_tc_layer_ok(int num_pages, int num_rows);
int attn_units_per_tile(int H);

}  // namespace csa

using namespace csa;

namespace {

inline bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

inline csa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? CSA_OK : CSA_ERR_CUDA; }

bool layer_ok(const csa_kv_layer *l, bool need_swa)
{
    if (!l || !l->codes || !l->scales || !l->keys || l->num_pages < 1) return false;
    if (!aligned16(l->codes) || !aligned16(l->scales) || !aligned16(l->keys)) return false;
    if (need_swa) {
        if (!l->swa || !l->swa_scale || l->num_rows < 1) return false;
        if (!aligned16(l->swa) || !aligned16(l->swa_scale)) return false;
    }
    if ((long long)l->num_pages * kPage > (1ll << 40)) return false;
    return true;
}

bool batch_ok(const csa_batch *b)
{
    if (!b || b->B < 1 || b->B > 16384 || !b->seq_len || !b->block_table || !b->swa_row) return false;
    if (b->max_seq_len < 1 || b->max_seq_len > CSA_MAX_SEQ_LEN) return false;
    if (b->max_pages < (b->max_seq_len + kPage - 1) / kPage) return false;
    if (!aligned16(b->seq_len) || !aligned16(b->block_table) || !aligned16(b->swa_row)) return false;
    return true;
}

bool heads_ok(int H) { return H == 16 || H == 32 || H == 64 || H == 128; }

WsLayout layout_for(int B, int H, int max_seq_len, int cap)
{
    return ws_layout(B, H, max_seq_len, cap, attn_units_per_tile(H));
}

}  // namespace

extern "C" {

size_t csa_workspace_bytes(int32_t B, int32_t H, int32_t max_seq_len, int32_t cap)
{
    if (B < 1 || !heads_ok(H) || max_seq_len < 1 || max_seq_len > CSA_MAX_SEQ_LEN || cap < 1 || cap > CSA_MAX_TOPK)
        return 0;
    return layout_for(B, H, max_seq_len, cap).total;
}

csa_status csa_workspace_init(void *ws, size_t ws_bytes, void *stream)
{
    if (!ws || !aligned16(ws) || ws_bytes < kHeaderBytes) return CSA_ERR_INVALID_ARG;
    return cuda_status(cudaMemsetAsync(ws, 0, kHeaderBytes, (cudaStream_t)stream));
}

csa_status csa_kv_pack_fp4(const csa_kv_layer *layer, const uint16_t *latent, const uint16_t *idx_key,
                           const int64_t *slot, const int32_t *swa_slot, int32_t n, void *ws, size_t ws_bytes,
                           void *stream)
{
    if (n < 0) return CSA_ERR_INVALID_ARG;
    if (n == 0) return CSA_OK;
    if (!layer_ok(layer, swa_slot != nullptr)) return CSA_ERR_INVALID_ARG;
    if (!latent || !idx_key || !slot || !aligned16(latent) || !aligned16(idx_key) || !aligned16(slot))
        return CSA_ERR_INVALID_ARG;
    if (swa_slot && !aligned16(swa_slot)) return CSA_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws)) return CSA_ERR_INVALID_ARG;
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    return cuda_status(launch_kv_pack(*layer, latent, idx_key, slot, swa_slot, n, ws, (cudaStream_t)stream));
}

csa_status csa_kv_norm_rope_pack_fp4(const csa_kv_layer *layer, const uint16_t *latent_prenorm,
                                     const float *norm_weight, const float *rope_cos_sin, const uint16_t *idx_key,
                                     const int64_t *slot, const int32_t *swa_slot, int32_t n, void *ws,
                                     size_t ws_bytes, void *stream)
{
    if (n < 0) return CSA_ERR_INVALID_ARG;
    if (n == 0) return CSA_OK;
    if (!layer_ok(layer, swa_slot != nullptr)) return CSA_ERR_INVALID_ARG;
    if (!latent_prenorm || !norm_weight || !rope_cos_sin || !idx_key || !slot || !aligned16(latent_prenorm) ||
        !aligned16(norm_weight) || !aligned16(rope_cos_sin) || !aligned16(idx_key) || !aligned16(slot))
        return CSA_ERR_INVALID_ARG;
    if (swa_slot && !aligned16(swa_slot)) return CSA_ERR_INVALID_ARG;
    if (!ws || !aligned16(ws)) return CSA_ERR_INVALID_ARG;
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    return cuda_status(launch_kv_norm_rope_pack(*layer, latent_prenorm, norm_weight, rope_cos_sin, idx_key, slot,
                                                swa_slot, n, ws, (cudaStream_t)stream));
}

csa_status csa_indexer_block_scores(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq,
                                    const float *iw, const int32_t *pool, const int32_t *pool_count,
                                    int32_t pool_cap, float *scores, int32_t score_stride, void *ws, size_t ws_bytes,
                                    void *stream)
{
    if (!layer_ok(layer, false) || !batch_ok(batch)) return CSA_ERR_INVALID_ARG;
    if (!iq || !iw || !scores || !ws || !aligned16(iq) || !aligned16(iw) || !aligned16(scores) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (pool) {
        if (!pool_count || !aligned16(pool) || !aligned16(pool_count)) return CSA_ERR_INVALID_ARG;
        if (pool_cap < 1 || pool_cap > CSA_MAX_TOPK || score_stride < pool_cap) return CSA_ERR_INVALID_ARG;
    } else if (score_stride < (batch->max_seq_len + kBlock - 1) / kBlock) {
        return CSA_ERR_INVALID_ARG;
    }
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    return cuda_status(launch_block_scores_full_or_pool(layer->keys, layer->num_pages, *batch, iq, iw, pool,
                                                        pool ? pool_count : nullptr, pool ? pool_cap : 0, scores,
                                                        score_stride, ws, (cudaStream_t)stream));
}

csa_status csa_topk_blocks(const csa_batch *batch, const float *scores, int32_t score_stride, const int32_t *pool,
                           const int32_t *pool_count, int32_t pool_cap, int32_t k, int32_t *out_blocks,
                           int32_t *out_count, void *ws, size_t ws_bytes, void *stream)
{
    if (!batch_ok(batch)) return CSA_ERR_INVALID_ARG;
    if (!scores || !out_blocks || !out_count || !ws || !aligned16(scores) || !aligned16(out_blocks) ||
        !aligned16(out_count) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID_ARG;
    int max_candidates;
    if (pool) {
        if (!pool_count || !aligned16(pool) || !aligned16(pool_count)) return CSA_ERR_INVALID_ARG;
        if (pool_cap < 1 || pool_cap > CSA_MAX_SHARDS * CSA_MAX_TOPK || score_stride < pool_cap)
            return CSA_ERR_INVALID_ARG;
        max_candidates = pool_cap;
    } else {
        max_candidates = (batch->max_seq_len + kBlock - 1) / kBlock;
        if (score_stride < max_candidates) return CSA_ERR_INVALID_ARG;
    }
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    return cuda_status(launch_topk(scores, score_stride, batch->seq_len, batch->max_seq_len, pool,
                                   pool ? pool_count : nullptr, pool ? pool_cap : 0, k, batch->B, out_blocks,
                                   out_count, max_candidates, ws, (cudaStream_t)stream));
}

static csa_status check_indexer_common(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq,
                                       const float *iw, int32_t *out_blocks, int32_t *out_count, void *ws)
{
    if (!layer_ok(layer, false) || !batch_ok(batch)) return CSA_ERR_INVALID_ARG;
    if (!iq || !iw || !out_blocks || !out_count || !ws) return CSA_ERR_INVALID_ARG;
    if (!aligned16(iq) || !aligned16(iw) || !aligned16(out_blocks) || !aligned16(out_count) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    return CSA_OK;
}

csa_status csa_indexer_full(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq, const float *iw,
                            int32_t k, int32_t *out_blocks, int32_t *out_count, void *ws, size_t ws_bytes,
                            void *stream)
{
    csa_status s = check_indexer_common(layer, batch, iq, iw, out_blocks, out_count, ws);
    if (s != CSA_OK) return s;
    if (k < 1 || k > CSA_MAX_TOPK) return CSA_ERR_INVALID_ARG;
    const WsLayout w = ws_layout(batch->B, 16, batch->max_seq_len, k, 1);
    if (ws_bytes < w.screen_end) return CSA_ERR_WORKSPACE;
    cudaStream_t st = (cudaStream_t)stream;
    char *base = (char *)ws;
    float *scores = reinterpret_cast<float *>(base + w.scores);
    const int nb = (int)w.nb;
    if (nb <= k) {   // every sequence selects all of its blocks: no score is needed
        return cuda_status(launch_topk(scores, (int)w.score_cap, batch->seq_len, batch->max_seq_len, nullptr, nullptr,
                                       0, k, batch->B, out_blocks, out_count, nb, ws, st));
    }
    if (!screen_supported(layer->num_pages)) {   // exhaustive exact scan
        s = csa_indexer_block_scores(layer, batch, iq, iw, nullptr, nullptr, 0, scores, (int32_t)w.score_cap, ws,
                                     ws_bytes, stream);
        if (s != CSA_OK) return s;
        return csa_topk_blocks(batch, scores, (int32_t)w.score_cap, nullptr, nullptr, 0, k, out_blocks, out_count,
                               ws, ws_bytes, stream);
    }
    // screen every position on the tensor cores; blocks sure to be in the Top-k are kept, blocks that
    // cannot reach it dropped, the uncertain rest scored exactly and the best of them taken
    float *lo = reinterpret_cast<float *>(base + w.lo);
    float *hi = reinterpret_cast<float *>(base + w.hi);
    uint32_t *hist = reinterpret_cast<uint32_t *>(base + w.hist);
    uint32_t *hist2 = reinterpret_cast<uint32_t *>(base + w.hist2);
    uint8_t *status = reinterpret_cast<uint8_t *>(base + w.status);
    int32_t *uslice = reinterpret_cast<int32_t *>(base + w.uslice);
    const int lstride = (int)w.lstride;
    cudaError_t e = launch_screen_bounds(layer->keys, layer->num_pages, *batch, iq, iw,
                                         reinterpret_cast<uint8_t *>(base + w.qt), base + w.qm, hist, hist2, lo, hi,
                                         lstride, ws, st);
    if (e == cudaSuccess)   // the score region (B x score_cap >= B x nb words) keeps the overflow keys
        e = launch_select(lo, hi, lstride, *batch, k, hist, hist2, status, (int)w.status_stride, uslice,
                          reinterpret_cast<uint32_t *>(scores), nb, layer->keys, layer->num_pages, iq, iw,
                          out_blocks, out_count, ws, st);
    return cuda_status(e);
}

csa_status csa_indexer_screen_bounds(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq,
                                     const float *iw, float *lower, float *upper, int32_t stride, void *ws,
                                     size_t ws_bytes, void *stream)
{
    if (!layer_ok(layer, false) || !batch_ok(batch)) return CSA_ERR_INVALID_ARG;
    if (!iq || !iw || !lower || !upper || !ws || !aligned16(iq) || !aligned16(iw) || !aligned16(lower) ||
        !aligned16(upper) || !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    const WsLayout w = ws_layout(batch->B, 16, batch->max_seq_len, 1, 1);
    if (stride < (int32_t)w.nb) return CSA_ERR_INVALID_ARG;
    if (!screen_supported(layer->num_pages)) return CSA_ERR_UNSUPPORTED;
    if (ws_bytes < w.screen_end) return CSA_ERR_WORKSPACE;
    char *base = (char *)ws;
    return cuda_status(launch_screen_bounds(layer->keys, layer->num_pages, *batch, iq, iw,
                                            reinterpret_cast<uint8_t *>(base + w.qt), base + w.qm,
                                            reinterpret_cast<uint32_t *>(base + w.hist), nullptr, lower, upper, stride,
                                            ws, (cudaStream_t)stream));
}

csa_status csa_indexer_reindex(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq,
                               const float *iw, const int32_t *pool, const int32_t *pool_count, int32_t pool_cap,
                               int32_t k_r, int32_t *out_blocks, int32_t *out_count, void *ws, size_t ws_bytes,
                               void *stream)
{
    csa_status s = check_indexer_common(layer, batch, iq, iw, out_blocks, out_count, ws);
    if (s != CSA_OK) return s;
    if (!pool || !pool_count) return CSA_ERR_INVALID_ARG;
    if (pool_cap < 1 || pool_cap > CSA_MAX_TOPK || k_r < 1 || k_r > CSA_MAX_TOPK) return CSA_ERR_INVALID_ARG;
    const WsLayout w = ws_layout(batch->B, 16, batch->max_seq_len, pool_cap, 1);
    if (ws_bytes < w.topk) return CSA_ERR_WORKSPACE;
    float *scores = reinterpret_cast<float *>((char *)ws + w.scores);
    s = csa_indexer_block_scores(layer, batch, iq, iw, pool, pool_count, pool_cap, scores, (int32_t)w.score_cap, ws,
                                 ws_bytes, stream);
    if (s != CSA_OK) return s;
    return csa_topk_blocks(batch, scores, (int32_t)w.score_cap, pool, pool_count, pool_cap, k_r, out_blocks,
                           out_count, ws, ws_bytes, stream);
}

csa_status csa_index_reuse(int32_t B, const int32_t *prev_blocks, const int32_t *prev_count, int32_t prev_cap,
                           int32_t *out_blocks, int32_t *out_count, int32_t out_cap, void *ws, size_t ws_bytes,
                           void *stream)
{
    if (B < 1 || prev_cap < 1 || out_cap < 1 || !prev_blocks || !prev_count || !out_blocks || !out_count || !ws)
        return CSA_ERR_INVALID_ARG;
    if (!aligned16(prev_blocks) || !aligned16(prev_count) || !aligned16(out_blocks) || !aligned16(out_count) ||
        !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (ws_bytes < kHeaderBytes) return CSA_ERR_WORKSPACE;
    return cuda_status(launch_reuse(B, prev_blocks, prev_count, prev_cap, out_blocks, out_count, out_cap, ws,
                                    (cudaStream_t)stream));
}

csa_status csa_sparse_decode_attn(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *q, int32_t H,
                                  float sm_scale, const int32_t *blocks, const int32_t *count, int32_t cap,
                                  float *out, float *lse, void *ws, size_t ws_bytes, void *stream)
{
    if (!layer_ok(layer, true) || !batch_ok(batch)) return CSA_ERR_INVALID_ARG;
    if (!q || !blocks || !count || !out || !lse || !ws) return CSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(blocks) || !aligned16(count) || !aligned16(out) || !aligned16(lse) ||
        !aligned16(ws))
        return CSA_ERR_INVALID_ARG;
    if (cap < 1 || cap > CSA_MAX_TOPK) return CSA_ERR_INVALID_ARG;
    if (!heads_ok(H)) return CSA_ERR_UNSUPPORTED;
    if (attn_tc_supported(H) && !attn_tc_layer_ok(layer->num_pages, layer->num_rows)) return CSA_ERR_UNSUPPORTED;
    if (!(sm_scale > 0.f) || sm_scale > 1e30f) return CSA_ERR_INVALID_ARG;
    const WsLayout w = layout_for(batch->B, H, batch->max_seq_len, cap);
    if (ws_bytes < w.total) return CSA_ERR_WORKSPACE;
    AttnArgs a;
    a.codes = layer->codes;
    a.scales = layer->scales;
    a.swa = layer->swa;
    a.swa_scale = layer->swa_scale;
    a.num_pages = layer->num_pages;
    a.num_rows = layer->num_rows;
    a.B = batch->B;
    a.seq_len = batch->seq_len;
    a.block_table = batch->block_table;
    a.max_pages = batch->max_pages;
    a.swa_row = batch->swa_row;
    a.max_seq_len = batch->max_seq_len;
    a.q = q;
    a.H = H;
    a.sm_scale = sm_scale;
    a.blocks = blocks;
    a.count = count;
    a.cap = cap;
    a.part_o = reinterpret_cast<float *>((char *)ws + w.part_o);
    a.part_ml = reinterpret_cast<float *>((char *)ws + w.part_ml);
    a.splits = w.splits;
    a.ws = ws;
    cudaStream_t st = (cudaStream_t)stream;
    cudaError_t e = attn_tc_supported(H) ? launch_attn_tc(a, st) : launch_attn_cc(a, st);
    if (e != cudaSuccess) return CSA_ERR_CUDA;
    return cuda_status(launch_attn_combine(a, out, lse, st));
}

csa_status csa_decode_layer(const csa_kv_layer *layer, const csa_batch *batch, const csa_layer_step *p, void *ws,
                            size_t ws_bytes, void *stream)
{
    if (!p || !batch_ok(batch)) return CSA_ERR_INVALID_ARG;
    csa_status s;
    switch (p->mode) {
    case CSA_FULL:
        if (p->k != p->cap) return CSA_ERR_INVALID_ARG;
        s = csa_indexer_full(layer, batch, p->iq, p->iw, p->k, p->blocks, p->count, ws, ws_bytes, stream);
        break;
    case CSA_REINDEX:
        if (p->k != p->cap) return CSA_ERR_INVALID_ARG;
        s = csa_indexer_reindex(layer, batch, p->iq, p->iw, p->prev_blocks, p->prev_count, p->prev_cap, p->k,
                                p->blocks, p->count, ws, ws_bytes, stream);
        break;
    case CSA_REUSE:
        s = csa_index_reuse(batch->B, p->prev_blocks, p->prev_count, p->prev_cap, p->blocks, p->count, p->cap, ws,
                            ws_bytes, stream);
        break;
    default:
        return CSA_ERR_INVALID_ARG;
    }
    if (s != CSA_OK) return s;
    return csa_sparse_decode_attn(layer, batch, p->q, p->H, p->sm_scale, p->blocks, p->count, p->cap, p->out,
                                  p->lse, ws, ws_bytes, stream);
}

csa_status csa_check_device_error(void *ws, void *stream, int64_t *detail)
{
    if (!ws || !aligned16(ws)) return CSA_ERR_INVALID_ARG;
    DevStatus h;
    cudaStream_t st = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&h, ws, sizeof h, cudaMemcpyDeviceToHost, st) != cudaSuccess) return CSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return CSA_ERR_CUDA;
    if (detail) *detail = h.detail;
    if (h.code != 0 && cudaMemsetAsync(ws, 0, sizeof h, st) != cudaSuccess) return CSA_ERR_CUDA;
    if (h.code == 0) return CSA_OK;
    return h.code == CSA_ERR_TIMEOUT ? CSA_ERR_TIMEOUT : CSA_ERR_DEVICE_DATA;
}

const char *csa_status_string(csa_status s)
{
    switch (s) {
    case CSA_OK: return "ok";
    case CSA_ERR_INVALID_ARG: return "invalid argument";
    case CSA_ERR_UNSUPPORTED: return "unsupported configuration";
    case CSA_ERR_WORKSPACE: return "workspace too small";
    case CSA_ERR_CUDA: return "CUDA error";
    case CSA_ERR_DEVICE_DATA: return "device metadata out of range";
    case CSA_ERR_TIMEOUT: return "device wait timed out";
    }
    return "unknown status";
}

}  // extern "C"
