"""Context-parallel decode of one long sequence: its positions split by rank, one process per GPU.

rebasdaily article on DeepSeek-V4.1-Flash KV compression, section "同一份笔记，多层一起用": a Full
layer's hierarchical indexer scans the whole context into its Top-K candidate pool.  For a context
too long for one GPU's step time, rank r holds positions [start_r, end_r) (page-aligned, ascending in
r) in its own caches and runs the indexer and the attention on that slice.  The result is exact:

  * every block of the global Top-K is in its own slice's Top-K (fewer than K blocks of the slice
    beat it in the (score, lower block id) order), so the global Top-K is the Top-K of the union of
    the slices' Top-K lists, each with its exact score;
  * attention over the union of the slices' entry sets (the window on the rank that holds the last
    positions) is the log-sum-exp merge of the per-slice attentions.

Two exchanges per Full layer, both all-gathers of small tensors: the slices' (block id, exact score)
candidate lists (8 B per candidate) and the slices' (out, lse) partials (H x 512 x 4 B + H x 4 B).
Every compute step is a C-ABI call (csa.*); the exchanges go through a `Comm` (torch.distributed,
NCCL on GPUs).  full_layer_all_slices runs every slice of a sequence in one process, the exchanges
becoming stacks; the one-GPU tests use it.
"""
import torch

from . import csa


class Shard:
    """Rank r's slice [start, end) of one sequence of total length L: its own caches (KVLayer), the
    block table of its pages and, if it holds the sequence's last position, its window row."""

    def __init__(self, layer, start, end, L, block_table, swa_row, device="cuda"):
        if start % csa.PAGE or (end != L and end % csa.PAGE) or not (0 <= start < end <= L):
            raise ValueError("a slice is a page-aligned [start, end) inside [0, L)")
        self.layer, self.start, self.end, self.L = layer, start, end, L
        self.holds_last = end == L
        self.block_lo = start // csa.BLOCK
        self.block_hi = (end + csa.BLOCK - 1) // csa.BLOCK
        n = end - start
        dev = torch.device(device)
        self.batch = csa.Batch(torch.tensor([n], dtype=torch.int32, device=dev),
                               block_table.reshape(1, -1).to(dev, torch.int32),
                               torch.tensor([swa_row if self.holds_last else -1], dtype=torch.int32, device=dev), n)


class CudaOps:
    """The compute steps on the GPU through the C-ABI, with the workspaces they need."""

    def __init__(self, heads, k, device="cuda"):
        self.H, self.k, self.device = heads, k, device
        self._ws = {}

    def _workspace(self, max_seq_len):
        if max_seq_len not in self._ws:
            self._ws[max_seq_len] = csa.workspace(1, self.H, max_seq_len, self.k, self.device)
        return self._ws[max_seq_len]

    def select_local(self, shard, iq, iw):
        """The slice's Top-k (local block ids) and their exact scores."""
        ws = self._workspace(shard.batch.max_seq_len)
        blocks = torch.zeros((1, self.k), dtype=torch.int32, device=self.device)
        count = torch.zeros((1,), dtype=torch.int32, device=self.device)
        csa.indexer_full(shard.layer, shard.batch, iq, iw, self.k, blocks, count, ws)
        scores = torch.zeros((1, self.k), dtype=torch.float32, device=self.device)
        csa.indexer_block_scores(shard.layer, shard.batch, iq, iw, scores, ws, pool=blocks, pool_count=count)
        return blocks, scores, count

    def select_global(self, L, ids, scores, counts, offsets):
        """Top-k of the concatenated candidate lists ([R, 1, k] each): global block ids, ascending."""
        R = int(ids.shape[0])
        ws = self._workspace(L)
        cat_ids = torch.zeros((1, R * self.k), dtype=torch.int32, device=self.device)
        cat_scores = torch.zeros((1, R * self.k), dtype=torch.float32, device=self.device)
        cat_count = torch.zeros((1,), dtype=torch.int32, device=self.device)
        csa.candidates_concat(ids, scores, counts, offsets, cat_ids, cat_scores, cat_count, ws)
        full = csa.Batch(torch.tensor([L], dtype=torch.int32, device=self.device),
                         torch.zeros((1, (L + csa.PAGE - 1) // csa.PAGE), dtype=torch.int32, device=self.device),
                         torch.tensor([-1], dtype=torch.int32, device=self.device), L)
        blocks = torch.zeros((1, self.k), dtype=torch.int32, device=self.device)
        count = torch.zeros((1,), dtype=torch.int32, device=self.device)
        csa.topk_blocks(full, cat_scores, self.k, blocks, count, ws, pool=cat_ids, pool_count=cat_count)
        return blocks, count

    def attend_local(self, shard, q, blocks, count, sm_scale):
        """Attention of the slice over its part of the global set (and the window, if it holds it)."""
        ws = self._workspace(shard.batch.max_seq_len)
        mine = torch.zeros((1, self.k), dtype=torch.int32, device=self.device)
        mine_count = torch.zeros((1,), dtype=torch.int32, device=self.device)
        lo = torch.tensor([shard.block_lo], dtype=torch.int32, device=self.device)
        hi = torch.tensor([shard.block_hi], dtype=torch.int32, device=self.device)
        csa.shard_blocks(blocks, count, lo, hi, mine, mine_count, ws)
        out = torch.zeros((1, self.H, csa.LATENT), dtype=torch.float32, device=self.device)
        lse = torch.zeros((1, self.H), dtype=torch.float32, device=self.device)
        csa.sparse_decode_attn(shard.layer, shard.batch, q, sm_scale, mine, mine_count, out, lse, ws)
        return out, lse

    def merge(self, out_parts, lse_parts):
        out = torch.zeros(out_parts.shape[1:], dtype=torch.float32, device=self.device)
        lse = torch.zeros(lse_parts.shape[1:], dtype=torch.float32, device=self.device)
        csa.attn_merge(out_parts, lse_parts, out, lse)
        return out, lse


class DistComm:
    """All-gathers over a torch.distributed process group (NCCL between GPUs)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        self.world = dist.get_world_size(group)

    def all_gather(self, t):
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.stack(parts)


def gather_candidates(comm, blocks, scores, count, shard):
    """[R, 1, k] ids and scores, [R, 1] counts and offsets (each slice's first block), by rank."""
    offset = torch.tensor([shard.block_lo], dtype=torch.int32, device=blocks.device)
    return comm.all_gather(blocks), comm.all_gather(scores), comm.all_gather(count), comm.all_gather(offset)


def full_layer(ops, comm, shard, iq, iw, q, sm_scale=None):
    """One Full layer's decode step of this rank's slice; every rank returns the same (out, lse) of the
    whole sequence and the same global Top-k block set."""
    sm_scale = csa.default_sm_scale() if sm_scale is None else sm_scale
    blocks, scores, count = ops.select_local(shard, iq, iw)
    ids, sc, counts, offsets = gather_candidates(comm, blocks, scores, count, shard)
    gblocks, gcount = ops.select_global(shard.L, ids, sc, counts, offsets)
    out, lse = ops.attend_local(shard, q, gblocks, gcount, sm_scale)
    out, lse = ops.merge(comm.all_gather(out), comm.all_gather(lse))
    return out, lse, gblocks, gcount


def full_layer_all_slices(ops, shards, iq, iw, q, sm_scale=None):
    """The same step for every slice of a sequence in one process (the exchanges become stacks)."""
    sm_scale = csa.default_sm_scale() if sm_scale is None else sm_scale
    local = [ops.select_local(s, iq, iw) for s in shards]
    dev = local[0][0].device
    ids = torch.stack([b for b, _, _ in local])
    sc = torch.stack([s for _, s, _ in local])
    counts = torch.stack([c for _, _, c in local])
    offsets = torch.stack([torch.tensor([s.block_lo], dtype=torch.int32, device=dev) for s in shards])
    gblocks, gcount = ops.select_global(shards[0].L, ids, sc, counts, offsets)
    parts = [ops.attend_local(s, q, gblocks, gcount, sm_scale) for s in shards]
    out, lse = ops.merge(torch.stack([o for o, _ in parts]), torch.stack([l for _, l in parts]))
    return out, lse, gblocks, gcount


def page_aligned_slices(L, R):
    """R contiguous page-aligned slices [start, end) covering [0, L), as even as the pages allow."""
    pages = (L + csa.PAGE - 1) // csa.PAGE
    if R < 1 or R > pages:
        raise ValueError("need 1 <= R <= number of pages")
    bounds = [min(L, (pages * r // R) * csa.PAGE) for r in range(R + 1)]
    bounds[-1] = L
    return [(bounds[r], bounds[r + 1]) for r in range(R)]

