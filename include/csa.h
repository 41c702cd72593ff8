/*
 * csa.h -- C-ABI of the CSA2 FP4 compressed sparse-KV decode path (sm_100a).
 *
 * The method is the Compressed Sparse Attention 2 (CSA2) KV path of DeepSeek-V4.1-Flash, as three
 * web pages describe it:
 *   [rebasdaily] rebasdaily.com article on DeepSeek-V4.1-Flash KV compression, section
 *                "同一份笔记，多层一起用" (layer modes Full / Reindex / Reuse; hierarchical sparse
 *                indexer with a 2,048 x 8 = 16,384-position candidate pool; main KV in FP4, SWA KV
 *                in FP8) and section "先让长输入少走一半路" (sliding-window attention branch).
 *   [ailily]     ailily.cc article "每个 token 只占 890 字节", section 二 (mode table; one E4M3 scale
 *                per 16 channels) and section 三 (range argument: sqrt(512) and 448 x 6 = 2688).
 *   [yomxxx]     yomxxx.com long-form post on KV-cache compression limits, section 五 (attention
 *                kernels need a fixed layout with addresses computed from the token index and
 *                in-kernel parallel dequantisation).
 *
 * Conventions for every entry point
 *   - All array arguments are DEVICE pointers unless marked "host".  The caller allocates and owns
 *     every buffer; the library never allocates, frees or synchronises (except
 *     csa_check_device_error, which synchronises the given stream).
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the legacy default stream)
 *     and runs on the calling thread's current CUDA device.
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - Every device pointer must be 16-byte aligned.
 *   - Errors the host can see (null or misaligned pointers, unsupported sizes, too small a
 *     workspace) return before anything is launched.  Launch failures return CSA_ERR_CUDA.
 *     Errors in device-resident data (a page id, block id, slot or SWA row out of range, a
 *     sequence longer than max_seq_len, an unsorted pool) are recorded in the workspace's status
 *     word, the offending item is skipped, and csa_check_device_error reports them.
 *   - Non-finite inputs give undefined (but memory-safe) results.
 *
 * KV layout (one per KV-producing Full layer), pages of 64 tokens:
 *   codes     uint8 [num_pages][64][256]  E2M1 codes, channel 2i in the low nibble of byte i
 *   scales    uint8 [num_pages][64][32]   E4M3 scale of channels 16g..16g+15
 *   keys      uint8 [num_pages][64][128]  E4M3 indexer key
 *   swa       uint8 [num_rows][128][512]  E4M3 sliding-window entry, position p at slot p % 128
 *   swa_scale float [num_rows][128]       per-entry scale of the window entry
 * A block is 8 consecutive positions; block b of a sequence lives in its page
 * block_table[b / 8] at offsets 8*(b % 8) .. 8*(b % 8) + 7.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, size out of range */
    CSA_ERR_UNSUPPORTED = 2,  /* valid but unsupported configuration (e.g. H not in {16,32,64,128}) */
    CSA_ERR_WORKSPACE = 3,    /* ws_bytes smaller than csa_workspace_bytes() requires */
    CSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    CSA_ERR_DEVICE_DATA = 5,  /* device-resident metadata out of range (see csa_check_device_error) */
    CSA_ERR_TIMEOUT = 6       /* a bounded device-side wait gave up */
} csa_status;

typedef enum { CSA_FULL = 0, CSA_REINDEX = 1, CSA_REUSE = 2 } csa_layer_mode;

#define CSA_PAGE_TOKENS 64
#define CSA_BLOCK_POSITIONS 8
#define CSA_LATENT 512
#define CSA_INDEX_HEADS 8
#define CSA_INDEX_DIM 128
#define CSA_WINDOW 128
#define CSA_MAX_SEQ_LEN (1 << 24)
#define CSA_MAX_TOPK 8192
#define CSA_MAX_SHARDS 64

/* One KV-producing layer's caches.  All pointers device, caller-owned. */
typedef struct {
    uint8_t *codes;
    uint8_t *scales;
    uint8_t *keys;
    uint8_t *swa;
    float *swa_scale;
    int32_t num_pages;
    int32_t num_rows;
} csa_kv_layer;

/* One decode batch.  seq_len[b] >= 1 counts the current token; positions are 0 .. seq_len-1. */
typedef struct {
    int32_t B;                   /* host: number of sequences, 1 <= B <= 16384 */
    const int32_t *seq_len;      /* device int32 [B], 1 <= seq_len[b] <= max_seq_len */
    const int32_t *block_table;  /* device int32 [B][max_pages]: page id of each 64-token page */
    int32_t max_pages;           /* host: row stride of block_table, >= ceil(max_seq_len / 64) */
    const int32_t *swa_row;      /* device int32 [B]: the sequence's row of the SWA ring; -1 = no window
                                    segment (attention of a context shard without the last positions) */
    int32_t max_seq_len;         /* host: upper bound of seq_len[], sizes grids and workspace */
} csa_batch;

/* Size in bytes of the workspace the decode calls need for a batch of B sequences with H query
 * heads, contexts up to max_seq_len, and selected-set capacities up to `cap` blocks (the largest
 * Full Top-K or Reindex pool capacity used with this workspace).  Returns 0 for invalid sizes. */
size_t csa_workspace_bytes(int32_t B, int32_t H, int32_t max_seq_len, int32_t cap);

/* Bytes needed by calls that only report device-data errors (csa_kv_pack_fp4). */
#define CSA_WORKSPACE_HEADER_BYTES 256

/* Zero the workspace's status word.  Call once after allocating a workspace. */
csa_status csa_workspace_init(void *ws, size_t ws_bytes, void *stream);

/*
 * Step 1 -- pack n tokens into one layer's caches ([rebasdaily] 同一份笔记，多层一起用: main KV in
 * FP4, SWA KV stays FP8; [ailily] 二: one E4M3 scale per 16 channels).
 *   latent   bf16 [n][512]  post-RMSNorm/RoPE latent (the value that serves as key and value)
 *   idx_key  bf16 [n][128]  indexer key
 *   slot     int64 [n]      destination page*64 + offset; must address a page < num_pages
 *   swa_slot int32 [n]      row*128 + (position % 128) of the token's SWA entry, or -1 for none
 * Per 16-channel group: a = max|x|, s = E4M3(a/6) (binary32 division, round-to-nearest-even,
 * saturating), code = E2M1(x / s) (binary32 division, RNE, saturating, sign kept); s = 0 gives
 * codes 0.  Key: E4M3 of each bf16 channel.  SWA: scale = max|x| / 448 (binary32),
 * value = E4M3(x / scale).  ws needs CSA_WORKSPACE_HEADER_BYTES; a bad slot is skipped and
 * recorded.  The results are bit-for-bit defined.
 */
csa_status csa_kv_pack_fp4(const csa_kv_layer *layer, const uint16_t *latent,
                           const uint16_t *idx_key, const int64_t *slot, const int32_t *swa_slot,
                           int32_t n, void *ws, size_t ws_bytes, void *stream);

/*
 * Step 1 from the pre-norm latent -- RMSNorm, RoPE, then the pack of csa_kv_pack_fp4 ([ailily] 三:
 * the latent is RMS-normalised, with weights of magnitude about 1, and rotated by RoPE, which keeps
 * its norm).  The pages give no arithmetic; this call fixes it, in binary32, in this order:
 *   v = bf16 latent; per 16-channel group g, s_g = FMA chain of v_c^2 (c = 16g .. 16g+15) from 0;
 *   for d = 16, 8, 4, 2, 1: s_g <- s_g + s_(g xor d); r = 1 / sqrt(s_0 / 512 + 1e-6) (correctly
 *   rounded); y_c = (v_c * r) * norm_weight_c; for pair i = 0..31 of channels (448 + 2i, 449 + 2i):
 *   (a, b) -> (a*cos_i - b*sin_i, a*sin_i + b*cos_i), each product and sum rounded on its own;
 *   the latent that is packed is bf16(y) (round to nearest even).
 *   latent_prenorm bf16 [n][512]; norm_weight float [512]; rope_cos_sin float [n][32][2] =
 *   (cos_i, sin_i) of each token's rotation; idx_key, slot, swa_slot as for csa_kv_pack_fp4.
 * Results are bit-for-bit defined for finite inputs; ws needs CSA_WORKSPACE_HEADER_BYTES.
 */
csa_status csa_kv_norm_rope_pack_fp4(const csa_kv_layer *layer, const uint16_t *latent_prenorm,
                                     const float *norm_weight, const float *rope_cos_sin,
                                     const uint16_t *idx_key, const int64_t *slot,
                                     const int32_t *swa_slot, int32_t n, void *ws, size_t ws_bytes,
                                     void *stream);

/*
 * Steps 2-3, Full layer -- score every block of every sequence and select its Top-k
 * ([rebasdaily] 同一份笔记，多层一起用: a Full layer re-selects Top-K over the whole range; the
 * first Full layer's scan builds the 2,048 x 8 candidate pool).
 *   iq   bf16 [B][8][128]  indexer query, 8 heads
 *   iw   float [B][8]      head weights
 *   k    host, 1 <= k <= CSA_MAX_TOPK
 *   out_blocks int32 [B][k]  selected block ids, ascending; entries past out_count are untouched
 *   out_count  int32 [B]     min(k, ceil(seq_len/8))
 * Score of position p: sum over heads h of w_h * ReLU(q_h . k_p), in binary32 in this order:
 * per head, eight 16-dim FMA chains part_j, then ((p0+p4)+(p2+p6)) + ((p1+p5)+(p3+p7)), ReLU, and
 * an FMA chain over h = 0..7.  Block score = max over its positions < seq_len.  Order: larger
 * score first, then lower block id.  The selected set is bit-for-bit defined.
 * How: every position is first screened on the tensor cores (csa_indexer_screen_bounds); only
 * the blocks whose upper bound reaches the k-th largest lower bound are scored exactly, which
 * provably contains the exact Top-k, so the result equals an exhaustive exact scan.  ws: at least
 * csa_workspace_bytes(B, any H, max_seq_len, k) bytes.
 */
csa_status csa_indexer_full(const csa_kv_layer *layer, const csa_batch *batch, const uint16_t *iq,
                            const float *iw, int32_t k, int32_t *out_blocks, int32_t *out_count,
                            void *ws, size_t ws_bytes, void *stream);

/*
 * Screening bounds of the Full-layer score (no counterpart in the pages: this exposes the first
 * stage of csa_indexer_full for checking).  For every block v < ceil(seq_len/8) of every sequence,
 *   lower[b][v] <= exact block score <= upper[b][v]
 * in the order Top-K uses (a total order on binary32 with -0 = +0, NaN with the sign bit clear above
 * +inf and with it set below -inf).  A block whose bound cannot be formed (non-finite inputs, or
 * magnitudes near binary32 overflow) gets lower = -NaN and upper = +NaN, the two ends of that order.
 * The approximate score comes from E4M3 x E4M3 tensor-core products of the keys with a 3-term E4M3
 * split of q; the half-width is a rigorous bound on its distance to the exact binary32 chain.
 *   lower, upper float [B][stride], stride >= ceil(max_seq_len/8); entries past each row's count are
 *   untouched.  ws: csa_workspace_bytes(B, any H, max_seq_len, 1) bytes.
 * Returns CSA_ERR_UNSUPPORTED if num_pages * 64 >= 2^32 (the keys' tensor-map limit).
 */
csa_status csa_indexer_screen_bounds(const csa_kv_layer *layer, const csa_batch *batch,
                                     const uint16_t *iq, const float *iw, float *lower, float *upper,
                                     int32_t stride, void *ws, size_t ws_bytes, void *stream);

/*
 * Steps 2-3, Reindex layer -- re-score only the pool's blocks with this layer's own query and
 * select the Top-k_r inside the pool ([rebasdaily] 同一份笔记，多层一起用: Reindex reuses the
 * earlier layer's KV but re-evaluates which positions matter; later layers search only inside the
 * pool).  `layer` is the KV of the Full layer that built the pool.
 *   pool       int32 [B][pool_cap]  ascending block ids (a Full layer's output)
 *   pool_count int32 [B]            valid entries per row, <= pool_cap
 *   out_blocks int32 [B][k_r], out_count int32 [B] = min(k_r, pool_count)
 * Same score, order and tie rule as csa_indexer_full.
 */
csa_status csa_indexer_reindex(const csa_kv_layer *layer, const csa_batch *batch,
                               const uint16_t *iq, const float *iw, const int32_t *pool,
                               const int32_t *pool_count, int32_t pool_cap, int32_t k_r,
                               int32_t *out_blocks, int32_t *out_count, void *ws, size_t ws_bytes,
                               void *stream);

/*
 * Step 2 alone -- block scores into a caller buffer (csa_indexer_full and csa_indexer_reindex run
 * this and then csa_topk_blocks on workspace memory).  Full mode when pool is NULL: scores[b][v] for
 * blocks v < ceil(seq_len/8); Reindex mode: scores[b][v] of pool[b][v] for v < pool_count[b].
 *   scores float [B][score_stride], score_stride >= ceil(max_seq_len/8) (Full) or pool_cap (Reindex)
 * Same score as csa_indexer_full; bit-for-bit defined.  Entries past each row's count are untouched.
 */
csa_status csa_indexer_block_scores(const csa_kv_layer *layer, const csa_batch *batch,
                                    const uint16_t *iq, const float *iw, const int32_t *pool,
                                    const int32_t *pool_count, int32_t pool_cap, float *scores,
                                    int32_t score_stride, void *ws, size_t ws_bytes, void *stream);

/*
 * Step 3 alone -- exact Top-k of block scores from csa_indexer_block_scores (same pool arguments):
 * larger score first, then lower block id; the min(k, n) chosen block ids are written ascending.
 * In pool mode pool_cap may be up to CSA_MAX_SHARDS * CSA_MAX_TOPK (a concatenation of candidate
 * lists, csa_candidates_concat).  Bit-for-bit defined.  ws needs CSA_WORKSPACE_HEADER_BYTES.
 */
csa_status csa_topk_blocks(const csa_batch *batch, const float *scores, int32_t score_stride,
                           const int32_t *pool, const int32_t *pool_count, int32_t pool_cap,
                           int32_t k, int32_t *out_blocks, int32_t *out_count, void *ws,
                           size_t ws_bytes, void *stream);

/*
 * Step 3, Reuse layer -- take the previous layer's selected set unchanged ([rebasdaily]
 * 同一份笔记，多层一起用: Reuse keeps both the global KV and the earlier layer's Top-K positions).
 * Copies prev_count[b] entries of each row and the counts; bytewise identical.
 *   prev_blocks int32 [B][prev_cap], prev_count int32 [B] (each <= out_cap)
 *   out_blocks  int32 [B][out_cap],  out_count  int32 [B]
 */
csa_status csa_index_reuse(int32_t B, const int32_t *prev_blocks, const int32_t *prev_count,
                           int32_t prev_cap, int32_t *out_blocks, int32_t *out_count,
                           int32_t out_cap, void *ws, size_t ws_bytes, void *stream);

/*
 * Step 4 -- sparse decode attention over the selected FP4 entries and the FP8 window, merged
 * through one softmax ([rebasdaily] 同一份笔记，多层一起用 and 先让长输入少走一半路; [yomxxx] 五:
 * fixed layout, in-kernel parallel dequantisation).
 *   q        bf16 [B][H][512], H in {16, 32, 64, 128}
 *   sm_scale host, softmax temperature tau (1/sqrt(512) is the usual choice)
 *   blocks   int32 [B][cap] selected block ids (< ceil(seq_len/8)), count int32 [B] <= cap
 *   out      float [B][H][512], lse float [B][H]
 * Segment E: the positions < seq_len of the selected blocks, value e2m1(code) * e4m3(scale)
 * (exact).  Segment F: positions max(0, seq_len-128) .. seq_len-1 from the SWA ring row, value
 * e4m3 * swa_scale.  A position in both segments counts once in each.  z = tau * q_h . value;
 * out_h = softmax-weighted sum of values; lse_h = log-sum-exp of z.  Computed with fp16 operands
 * (exact for these values) and fp32 accumulation; agrees with exact arithmetic to within
 * 2e-3 of max|out| per sequence.  With H = 64 or 128 the caches may hold at most 2^31 FP4 entries
 * (num_pages * 64) and 2^30 window entries (num_rows * 128); larger layers return CSA_ERR_UNSUPPORTED.
 * Stream order: the call may begin while the stream's previous kernel is still running, when that
 * kernel releases its dependents early (this library's kernels do), and it reads q at that point;
 * everything else it reads only after the previous kernel has completed.  So q must not be written
 * by an immediately preceding kernel that releases its dependents early (a plain launch does not).
 */
csa_status csa_sparse_decode_attn(const csa_kv_layer *layer, const csa_batch *batch,
                                  const uint16_t *q, int32_t H, float sm_scale,
                                  const int32_t *blocks, const int32_t *count, int32_t cap,
                                  float *out, float *lse, void *ws, size_t ws_bytes, void *stream);

/* One decode step of one layer. */
typedef struct {
    csa_layer_mode mode;
    const uint16_t *iq;          /* Full / Reindex: bf16 [B][8][128] */
    const float *iw;             /* Full / Reindex: float [B][8] */
    int32_t k;                   /* Full: Top-K; Reindex: k_r; ignored for Reuse */
    const int32_t *prev_blocks;  /* Reindex: the pool; Reuse: the previous set */
    const int32_t *prev_count;
    int32_t prev_cap;
    int32_t *blocks;             /* this layer's set, int32 [B][cap] (written) */
    int32_t *count;              /* int32 [B] (written) */
    int32_t cap;                 /* row stride of blocks; Full and Reindex require cap == k */
    const uint16_t *q;           /* bf16 [B][H][512] */
    int32_t H;
    float sm_scale;
    float *out;                  /* float [B][H][512] */
    float *lse;                  /* float [B][H] */
} csa_layer_step;

/*
 * Steps 2-4 for one layer in the given mode ([rebasdaily] 同一份笔记，多层一起用; [ailily] 二 mode
 * table): Full = csa_indexer_full(k); Reindex = csa_indexer_reindex(prev, k); Reuse =
 * csa_index_reuse(prev); then csa_sparse_decode_attn over this layer's set.  Reindex and Reuse
 * layers pass the KV of the most recent Full layer.
 */
csa_status csa_decode_layer(const csa_kv_layer *layer, const csa_batch *batch,
                            const csa_layer_step *step, void *ws, size_t ws_bytes, void *stream);

/*
 * Full-layer indexer that allocates nothing (the pages have no counterpart to this entry point: it is
 * an interface convenience).  Same inputs, outputs and results as csa_indexer_full, but the scratch it
 * needs lives in a fixed array inside the library instead of a caller workspace, for callers that
 * cannot obtain device memory where they run the indexer: runtimes with a fixed memory budget that
 * forbid allocation after start-up, plugins inside a framework that owns the allocator, or paths that
 * must not call an allocator at all.
 *   dev_status  optional int32 device pointer (may be NULL): receives the device-data status code of
 *               this call (0, or CSA_ERR_DEVICE_DATA / CSA_ERR_TIMEOUT), written asynchronously.
 * Limit: 256 + 4 * B * max(ceil(max_seq_len / 8), k) bytes must fit in CSA_NOALLOC_SCRATCH_BYTES
 * (4 MiB; e.g. 8 sequences of 131,072 tokens use 512 KiB); larger calls return CSA_ERR_WORKSPACE.
 * Every GPU that loads the library holds that array until the process exits.  The first call on each
 * device looks up the array's device address (cudaGetSymbolAddress, with that device current) and keeps
 * it for the life of the process; make that first call before any stream capture, and do not reset the
 * device (cudaDeviceReset, or a primary-context reset) after it, since the kept address would then be
 * stale.  All calls on a device share the one array and each call overwrites it: calls that overlap
 * on the GPU (different streams without ordering between them) race and give undefined results.  No
 * allocation or free happens in any call.
 */
#define CSA_NOALLOC_SCRATCH_BYTES (4 << 20)
csa_status csa_indexer_full_noalloc(const csa_kv_layer *layer, const csa_batch *batch,
                                    const uint16_t *iq, const float *iw, int32_t k,
                                    int32_t *out_blocks, int32_t *out_count, int32_t *dev_status,
                                    void *stream);

/*
 * Context-parallel decode of a long sequence: its positions split into R contiguous slices, rank r
 * holding slice [s_r, e_r) (page-aligned, ascending in r) in its own caches, with a batch view of the
 * slice (seq_len = e_r - s_r, swa_row = -1 except on the rank holding the last positions).  Each rank
 * runs csa_indexer_full(k) on its slice and csa_indexer_block_scores on the chosen blocks (their
 * exact scores); the ranks exchange those lists; the Top-k of the concatenated list (csa_topk_blocks
 * in pool mode, over the whole sequence's batch view) is the Full layer's exact Top-k ([rebasdaily]
 * 同一份笔记，多层一起用: the full-range scan, here sharded by position), since every block of the
 * global Top-k is in its own slice's Top-k.  Each rank attends over its part of that set
 * (csa_shard_blocks, then csa_sparse_decode_attn on its slice), and the ranks' (out, lse) merge
 * exactly (csa_attn_merge).  The exchanges themselves (all-gathers) are the caller's, e.g. NCCL.
 *
 * csa_candidates_concat -- per sequence b, the R lists ids[r][b][0 .. counts[r][b]) (local block
 *   ids, ascending) plus offsets[r][b] (the slice's first block) with their scores, into one list
 *   out_ids[b][0 .. out_count[b]) of global ids (ascending when the slices are) and out_scores.
 *     ids int32 [R][B][cap], scores float [R][B][cap], counts int32 [R][B] (<= cap), offsets int32 [R][B]
 *     out_ids int32 [B][R * cap], out_scores float [B][R * cap], out_count int32 [B]
 *   1 <= R <= CSA_MAX_SHARDS.  ws needs CSA_WORKSPACE_HEADER_BYTES (a count out of range is reported).
 */
csa_status csa_candidates_concat(int32_t R, int32_t B, int32_t cap, const int32_t *ids, const float *scores,
                                 const int32_t *counts, const int32_t *offsets, int32_t *out_ids,
                                 float *out_scores, int32_t *out_count, void *ws, size_t ws_bytes, void *stream);

/*
 * csa_shard_blocks -- per sequence b, the entries v of blocks[b][0 .. count[b]) with
 * lo[b] <= v < hi[b], as v - lo[b], in their order, into out_blocks[b][0 .. out_count[b]).
 *     blocks int32 [B][cap], count int32 [B], lo, hi int32 [B], out_blocks int32 [B][out_cap]
 *   More than out_cap entries in range are reported and cut at out_cap.
 */
csa_status csa_shard_blocks(int32_t B, const int32_t *blocks, const int32_t *count, int32_t cap,
                            const int32_t *lo, const int32_t *hi, int32_t *out_blocks, int32_t *out_count,
                            int32_t out_cap, void *ws, size_t ws_bytes, void *stream);

/*
 * csa_attn_merge -- attention over the union of R disjoint entry sets from the attention over each:
 * lse = log sum_r e^{lse_r}, out = sum_r e^{lse_r - lse} out_r (a set with lse_r = -inf, i.e. no
 * entry, takes no part; if every set is empty, out = 0 and lse = -inf).
 *     out_parts float [R][B][H][512], lse_parts float [R][B][H]; out float [B][H][512], lse float [B][H]
 *   1 <= R <= CSA_MAX_SHARDS, H in {16, 32, 64, 128}.
 */
csa_status csa_attn_merge(int32_t R, int32_t B, int32_t H, const float *out_parts, const float *lse_parts,
                          float *out, float *lse, void *stream);

/*
 * Persistent KV tier ([yomxxx] 三 "让 KV 不必一直待在 HBM 里": the global KV stays in HBM, the
 * persistent KV goes to SSD or host memory and is fetched back when needed; [rebasdaily]
 * 先让长输入少走一半路, SWA Bounded Replay: the sliding-window state is not stored, the most recent
 * tokens are replayed to restore it).  A sequence's persistent record holds its FP4 codes, E4M3
 * scales and E4M3 indexer keys and nothing of the window: one 26,624-byte record per 64-token page
 * (416 B per token), laid out
 *     codes [64][256] | scales [64][32] | keys [64][128]
 * for page i of the sequence (block_table[i]), i = 0 .. ceil(n / 64) - 1, back to back.  Rows of the
 * last page past n are copied as they are.  To restore a sequence: csa_kv_import into any pages,
 * then csa_kv_pack_fp4 of its last min(n, 128) tokens with their window slots (the replay; it writes
 * those tokens' FP4 and key bytes again, identically, and the window).
 *
 * csa_kv_record_bytes -- ceil(n / 64) * 26,624 (0 for n < 0).
 * csa_kv_export / csa_kv_import -- copy the record out of / into the pages block_table[0 ..
 *   ceil(n / 64)) (device int32) of `layer`.  dst / src is device memory or page-locked host memory
 *   (cudaHostAlloc, cudaMallocHost, or cudaHostRegister'd); any other host pointer returns
 *   CSA_ERR_INVALID_ARG before any launch.  The copy runs as one kernel on `stream`: a host buffer is
 *   written or read over the bus by the kernel itself.  A page id out of [0, num_pages) is reported
 *   and its record skipped.  0 <= n <= CSA_MAX_SEQ_LEN; n = 0 is a no-op.  ws needs
 *   CSA_WORKSPACE_HEADER_BYTES.  Bit-for-bit.
 */
size_t csa_kv_record_bytes(int32_t n);
csa_status csa_kv_export(const csa_kv_layer *layer, const int32_t *block_table, int32_t n, uint8_t *dst,
                         void *ws, size_t ws_bytes, void *stream);
csa_status csa_kv_import(const csa_kv_layer *layer, const int32_t *block_table, int32_t n, const uint8_t *src,
                         void *ws, size_t ws_bytes, void *stream);

/* Synchronise `stream`, read and clear the workspace status word.  Returns CSA_OK,
 * CSA_ERR_DEVICE_DATA or CSA_ERR_TIMEOUT; *detail (host, may be NULL) receives the first
 * offending index recorded. */
csa_status csa_check_device_error(void *ws, void *stream, int64_t *detail);

const char *csa_status_string(csa_status s);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H */
