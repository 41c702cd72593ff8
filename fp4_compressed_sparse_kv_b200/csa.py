"""Thin Python binding of libcsa.so (include/csa.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels.  PyTorch provides device memory and
streams; tensors must live on the current CUDA device.  There is no CPU fallback: if the shared
library is missing or a tensor is not on the GPU, these functions raise.
"""
import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcsa.so")

PAGE = 64
BLOCK = 8
LATENT = 512
WINDOW = 128
IDX_HEADS = 8
IDX_DIM = 128
HEADER_BYTES = 256
MAX_TOPK = 8192
MAX_SHARDS = 64
FULL, REINDEX, REUSE = 0, 1, 2

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "workspace too small",
          4: "CUDA error", 5: "device metadata out of range", 6: "device wait timed out"}


class CsaError(RuntimeError):
    def __init__(self, status, where):
        super().__init__("%s: %s (status %d)" % (where, STATUS.get(status, "unknown"), status))
        self.status = status


class KVLayerC(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("keys", ctypes.c_void_p),
                ("swa", ctypes.c_void_p), ("swa_scale", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("num_rows", ctypes.c_int32)]


class BatchC(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("seq_len", ctypes.c_void_p), ("block_table", ctypes.c_void_p),
                ("max_pages", ctypes.c_int32), ("swa_row", ctypes.c_void_p),
                ("max_seq_len", ctypes.c_int32)]


class LayerStepC(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int), ("iq", ctypes.c_void_p), ("iw", ctypes.c_void_p),
                ("k", ctypes.c_int32), ("prev_blocks", ctypes.c_void_p),
                ("prev_count", ctypes.c_void_p), ("prev_cap", ctypes.c_int32),
                ("blocks", ctypes.c_void_p), ("count", ctypes.c_void_p), ("cap", ctypes.c_int32),
                ("q", ctypes.c_void_p), ("H", ctypes.c_int32), ("sm_scale", ctypes.c_float),
                ("out", ctypes.c_void_p), ("lse", ctypes.c_void_p)]


EXPORTS = ["csa_workspace_bytes", "csa_workspace_init", "csa_kv_pack_fp4", "csa_indexer_full",
           "csa_indexer_reindex", "csa_indexer_block_scores", "csa_topk_blocks", "csa_index_reuse", "csa_sparse_decode_attn", "csa_decode_layer",
           "csa_check_device_error", "csa_status_string", "csa_indexer_full_noalloc",
           "csa_indexer_screen_bounds", "csa_kv_norm_rope_pack_fp4", "csa_candidates_concat",
           "csa_shard_blocks", "csa_attn_merge", "csa_kv_record_bytes", "csa_kv_export", "csa_kv_import"]

_lib = None


def lib():
    """Load libcsa.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError("libcsa.so not found at %s; build it with "
                          "`python -m fp4_compressed_sparse_kv_b200.build`" % LIB_PATH)
    L = ctypes.CDLL(LIB_PATH)
    P, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    st = ctypes.c_int
    L.csa_workspace_bytes.restype = sz
    L.csa_workspace_bytes.argtypes = [i32, i32, i32, i32]
    L.csa_workspace_init.restype = st
    L.csa_workspace_init.argtypes = [P, sz, P]
    L.csa_kv_pack_fp4.restype = st
    L.csa_kv_pack_fp4.argtypes = [ctypes.POINTER(KVLayerC), P, P, P, P, i32, P, sz, P]
    L.csa_kv_norm_rope_pack_fp4.restype = st
    L.csa_kv_norm_rope_pack_fp4.argtypes = [ctypes.POINTER(KVLayerC), P, P, P, P, P, P, i32, P, sz, P]
    L.csa_indexer_full.restype = st
    L.csa_indexer_full.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC), P, P, i32, P, P,
                                   P, sz, P]
    L.csa_indexer_reindex.restype = st
    L.csa_indexer_reindex.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC), P, P, P, P,
                                      i32, i32, P, P, P, sz, P]
    L.csa_indexer_block_scores.restype = st
    L.csa_indexer_block_scores.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC), P, P, P, P,
                                           i32, P, i32, P, sz, P]
    L.csa_indexer_screen_bounds.restype = st
    L.csa_indexer_screen_bounds.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC), P, P, P, P,
                                            i32, P, sz, P]
    L.csa_topk_blocks.restype = st
    L.csa_topk_blocks.argtypes = [ctypes.POINTER(BatchC), P, i32, P, P, i32, i32, P, P, P, sz, P]
    L.csa_index_reuse.restype = st
    L.csa_index_reuse.argtypes = [i32, P, P, i32, P, P, i32, P, sz, P]
    L.csa_sparse_decode_attn.restype = st
    L.csa_sparse_decode_attn.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC), P, i32,
                                         ctypes.c_float, P, P, i32, P, P, P, sz, P]
    L.csa_decode_layer.restype = st
    L.csa_decode_layer.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC),
                                   ctypes.POINTER(LayerStepC), P, sz, P]
    L.csa_indexer_full_noalloc.restype = st
    L.csa_indexer_full_noalloc.argtypes = [ctypes.POINTER(KVLayerC), ctypes.POINTER(BatchC), P, P, i32, P, P,
                                           P, P]
    L.csa_candidates_concat.restype = st
    L.csa_candidates_concat.argtypes = [i32, i32, i32, P, P, P, P, P, P, P, P, sz, P]
    L.csa_shard_blocks.restype = st
    L.csa_shard_blocks.argtypes = [i32, P, P, i32, P, P, P, P, i32, P, sz, P]
    L.csa_attn_merge.restype = st
    L.csa_attn_merge.argtypes = [i32, i32, i32, P, P, P, P, P]
    L.csa_kv_record_bytes.restype = sz
    L.csa_kv_record_bytes.argtypes = [i32]
    L.csa_kv_export.restype = st
    L.csa_kv_export.argtypes = [ctypes.POINTER(KVLayerC), P, i32, P, P, sz, P]
    L.csa_kv_import.restype = st
    L.csa_kv_import.argtypes = [ctypes.POINTER(KVLayerC), P, i32, P, P, sz, P]
    L.csa_check_device_error.restype = st
    L.csa_check_device_error.argtypes = [P, P, ctypes.POINTER(ctypes.c_int64)]
    L.csa_status_string.restype = ctypes.c_char_p
    L.csa_status_string.argtypes = [ctypes.c_int]
    _lib = L
    return L


def _check(status, where):
    if status != 0:
        raise CsaError(status, where)


def _ptr(t, name):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor (the library has no CPU path)" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _buf_ptr(t, name):
    """A device tensor, or a page-locked host tensor (the kernel reads or writes it over the bus)."""
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch tensor" % name)
    if not (t.is_cuda or t.is_pinned()):
        raise ValueError("%s must be a CUDA tensor or a pinned host tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t.data_ptr()


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def default_sm_scale():
    return 1.0 / math.sqrt(LATENT)


# ------------------------------------------------------------------------------------------------
# Buffers
# ------------------------------------------------------------------------------------------------
class KVLayer:
    """One Full layer's caches: FP4 codes + E4M3 scales + E4M3 indexer keys (pages of 64 tokens)
    and the FP8 sliding-window ring (one 128-slot row per sequence)."""

    def __init__(self, num_pages, num_rows, device="cuda"):
        u8 = dict(dtype=torch.uint8, device=device)
        self.codes = torch.zeros((num_pages, PAGE, LATENT // 2), **u8)
        self.scales = torch.zeros((num_pages, PAGE, LATENT // 16), **u8)
        self.keys = torch.zeros((num_pages, PAGE, IDX_DIM), **u8)
        self.swa = torch.zeros((num_rows, WINDOW, LATENT), **u8)
        self.swa_scale = torch.zeros((num_rows, WINDOW), dtype=torch.float32, device=device)
        self.num_pages, self.num_rows = num_pages, num_rows

    def c(self):
        return KVLayerC(_ptr(self.codes, "codes"), _ptr(self.scales, "scales"),
                        _ptr(self.keys, "keys"), _ptr(self.swa, "swa"),
                        _ptr(self.swa_scale, "swa_scale"), self.num_pages, self.num_rows)


class Batch:
    """Decode-batch metadata: seq_len [B], block_table [B][max_pages], swa_row [B] (int32, device)
    and the host bound max_seq_len."""

    def __init__(self, seq_len, block_table, swa_row, max_seq_len):
        self.seq_len, self.block_table, self.swa_row = seq_len, block_table, swa_row
        self.B = int(seq_len.numel())
        self.max_pages = int(block_table.shape[1])
        self.max_seq_len = int(max_seq_len)

    def c(self):
        return BatchC(self.B, _ptr(self.seq_len, "seq_len"), _ptr(self.block_table, "block_table"),
                      self.max_pages, _ptr(self.swa_row, "swa_row"), self.max_seq_len)


def workspace_bytes(B, H, max_seq_len, cap):
    n = lib().csa_workspace_bytes(B, H, max_seq_len, cap)
    if n == 0:
        raise CsaError(1, "csa_workspace_bytes")
    return n


def workspace(B, H, max_seq_len, cap, device="cuda", stream=None):
    """Allocate (with torch) and initialise a workspace for these sizes."""
    ws = torch.empty(workspace_bytes(B, H, max_seq_len, cap), dtype=torch.uint8, device=device)
    workspace_init(ws, stream)
    return ws


def workspace_init(ws, stream=None):
    _check(lib().csa_workspace_init(_ptr(ws, "ws"), ws.numel(), _stream(stream)), "csa_workspace_init")


# ------------------------------------------------------------------------------------------------
# Entry points (same names as the C-ABI, without the csa_ prefix)
# ------------------------------------------------------------------------------------------------
def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t


def kv_pack_fp4(layer, latent, idx_key, slot, swa_slot, ws, stream=None):
    n = int(slot.numel())
    lc = layer.c()
    _check(lib().csa_kv_pack_fp4(ctypes.byref(lc), _ptr(_bits(latent), "latent"),
                                 _ptr(_bits(idx_key), "idx_key"), _ptr(slot, "slot"),
                                 _ptr(swa_slot, "swa_slot"), n, _ptr(ws, "ws"), ws.numel(),
                                 _stream(stream)), "csa_kv_pack_fp4")


def kv_norm_rope_pack_fp4(layer, latent_prenorm, norm_weight, rope_cos_sin, idx_key, slot, swa_slot, ws,
                          stream=None):
    """Pack from the pre-norm latent: RMSNorm (norm_weight float32 [512]), RoPE on channels 448..511
    (rope_cos_sin float32 [n, 32, 2] of (cos, sin) pairs), bf16, then the FP4 / E4M3 / FP8 pack."""
    n = int(slot.numel())
    lc = layer.c()
    _check(lib().csa_kv_norm_rope_pack_fp4(ctypes.byref(lc), _ptr(_bits(latent_prenorm), "latent_prenorm"),
                                           _ptr(norm_weight, "norm_weight"), _ptr(rope_cos_sin, "rope_cos_sin"),
                                           _ptr(_bits(idx_key), "idx_key"), _ptr(slot, "slot"),
                                           _ptr(swa_slot, "swa_slot"), n, _ptr(ws, "ws"), ws.numel(),
                                           _stream(stream)), "csa_kv_norm_rope_pack_fp4")


def indexer_full(layer, batch, iq, iw, k, out_blocks, out_count, ws, stream=None):
    lc, bc = layer.c(), batch.c()
    _check(lib().csa_indexer_full(ctypes.byref(lc), ctypes.byref(bc), _ptr(_bits(iq), "iq"),
                                  _ptr(iw, "iw"), int(k), _ptr(out_blocks, "out_blocks"),
                                  _ptr(out_count, "out_count"), _ptr(ws, "ws"), ws.numel(),
                                  _stream(stream)), "csa_indexer_full")


def indexer_reindex(layer, batch, iq, iw, pool, pool_count, k_r, out_blocks, out_count, ws,
                    stream=None):
    lc, bc = layer.c(), batch.c()
    _check(lib().csa_indexer_reindex(ctypes.byref(lc), ctypes.byref(bc), _ptr(_bits(iq), "iq"),
                                     _ptr(iw, "iw"), _ptr(pool, "pool"),
                                     _ptr(pool_count, "pool_count"), int(pool.shape[1]), int(k_r),
                                     _ptr(out_blocks, "out_blocks"), _ptr(out_count, "out_count"),
                                     _ptr(ws, "ws"), ws.numel(), _stream(stream)),
           "csa_indexer_reindex")


def indexer_block_scores(layer, batch, iq, iw, scores, ws, pool=None, pool_count=None, stream=None):
    """Block scores into `scores` float32 [B, stride] (Full when pool is None, else Reindex)."""
    lc, bc = layer.c(), batch.c()
    _check(lib().csa_indexer_block_scores(ctypes.byref(lc), ctypes.byref(bc), _ptr(_bits(iq), "iq"),
                                          _ptr(iw, "iw"), _ptr(pool, "pool"),
                                          _ptr(pool_count, "pool_count"),
                                          int(pool.shape[1]) if pool is not None else 0,
                                          _ptr(scores, "scores"), int(scores.shape[1]), _ptr(ws, "ws"),
                                          ws.numel(), _stream(stream)), "csa_indexer_block_scores")


def indexer_screen_bounds(layer, batch, iq, iw, lower, upper, ws, stream=None):
    """Per-block bounds of the exact Full score from the tensor-core screen: float32 [B, stride] each,
    lower <= score <= upper in Top-K order (-NaN / +NaN where no bound could be formed)."""
    lc, bc = layer.c(), batch.c()
    if lower.shape != upper.shape:
        raise ValueError("lower and upper must have the same shape")
    _check(lib().csa_indexer_screen_bounds(ctypes.byref(lc), ctypes.byref(bc), _ptr(_bits(iq), "iq"),
                                           _ptr(iw, "iw"), _ptr(lower, "lower"), _ptr(upper, "upper"),
                                           int(lower.shape[1]), _ptr(ws, "ws"), ws.numel(), _stream(stream)),
           "csa_indexer_screen_bounds")


def topk_blocks(batch, scores, k, out_blocks, out_count, ws, pool=None, pool_count=None, stream=None):
    bc = batch.c()
    _check(lib().csa_topk_blocks(ctypes.byref(bc), _ptr(scores, "scores"), int(scores.shape[1]),
                                 _ptr(pool, "pool"), _ptr(pool_count, "pool_count"),
                                 int(pool.shape[1]) if pool is not None else 0, int(k),
                                 _ptr(out_blocks, "out_blocks"), _ptr(out_count, "out_count"),
                                 _ptr(ws, "ws"), ws.numel(), _stream(stream)), "csa_topk_blocks")


def index_reuse(prev_blocks, prev_count, out_blocks, out_count, ws, stream=None):
    _check(lib().csa_index_reuse(int(prev_blocks.shape[0]), _ptr(prev_blocks, "prev_blocks"),
                                 _ptr(prev_count, "prev_count"), int(prev_blocks.shape[1]),
                                 _ptr(out_blocks, "out_blocks"), _ptr(out_count, "out_count"),
                                 int(out_blocks.shape[1]), _ptr(ws, "ws"), ws.numel(),
                                 _stream(stream)), "csa_index_reuse")


def sparse_decode_attn(layer, batch, q, sm_scale, blocks, count, out, lse, ws, stream=None):
    lc, bc = layer.c(), batch.c()
    H = int(q.shape[1])
    _check(lib().csa_sparse_decode_attn(ctypes.byref(lc), ctypes.byref(bc), _ptr(_bits(q), "q"), H,
                                        float(sm_scale), _ptr(blocks, "blocks"),
                                        _ptr(count, "count"), int(blocks.shape[1]),
                                        _ptr(out, "out"), _ptr(lse, "lse"), _ptr(ws, "ws"),
                                        ws.numel(), _stream(stream)), "csa_sparse_decode_attn")


def decode_layer(mode, layer, batch, q, out, lse, blocks, count, ws, iq=None, iw=None, k=0,
                 prev_blocks=None, prev_count=None, sm_scale=None, stream=None):
    """One layer's decode step: Full (k), Reindex (pool = prev, k_r = k) or Reuse (prev)."""
    lc, bc = layer.c(), batch.c()
    step = LayerStepC(int(mode), _ptr(_bits(iq), "iq") if iq is not None else None,
                      _ptr(iw, "iw") if iw is not None else None, int(k),
                      _ptr(prev_blocks, "prev_blocks") if prev_blocks is not None else None,
                      _ptr(prev_count, "prev_count") if prev_count is not None else None,
                      int(prev_blocks.shape[1]) if prev_blocks is not None else 0,
                      _ptr(blocks, "blocks"), _ptr(count, "count"), int(blocks.shape[1]),
                      _ptr(_bits(q), "q"), int(q.shape[1]),
                      float(default_sm_scale() if sm_scale is None else sm_scale),
                      _ptr(out, "out"), _ptr(lse, "lse"))
    _check(lib().csa_decode_layer(ctypes.byref(lc), ctypes.byref(bc), ctypes.byref(step),
                                  _ptr(ws, "ws"), ws.numel(), _stream(stream)), "csa_decode_layer")


def indexer_full_noalloc(layer, batch, iq, iw, k, out_blocks, out_count, dev_status=None, stream=None):
    """csa_indexer_full without a workspace: the library's own fixed scratch array is used instead, so
    nothing is allocated.  For callers that cannot provide device memory; see include/csa.h for the
    size limit and the rule that calls overlapping on the GPU must not share a device."""
    lc, bc = layer.c(), batch.c()
    _check(lib().csa_indexer_full_noalloc(ctypes.byref(lc), ctypes.byref(bc), _ptr(_bits(iq), "iq"),
                                          _ptr(iw, "iw"), int(k), _ptr(out_blocks, "out_blocks"),
                                          _ptr(out_count, "out_count"), _ptr(dev_status, "dev_status"),
                                          _stream(stream)), "csa_indexer_full_noalloc")


def candidates_concat(ids, scores, counts, offsets, out_ids, out_scores, out_count, ws, stream=None):
    """ids int32 [R, B, cap] (local block ids), scores float32 [R, B, cap], counts / offsets int32
    [R, B] -> out_ids int32 [B, R * cap] (global ids), out_scores float32 [B, R * cap], out_count [B]."""
    R, B, cap = (int(x) for x in ids.shape)
    _check(lib().csa_candidates_concat(R, B, cap, _ptr(ids, "ids"), _ptr(scores, "scores"),
                                       _ptr(counts, "counts"), _ptr(offsets, "offsets"),
                                       _ptr(out_ids, "out_ids"), _ptr(out_scores, "out_scores"),
                                       _ptr(out_count, "out_count"), _ptr(ws, "ws"), ws.numel(),
                                       _stream(stream)), "csa_candidates_concat")


def shard_blocks(blocks, count, lo, hi, out_blocks, out_count, ws, stream=None):
    """Entries of blocks int32 [B, cap] (count [B]) in [lo[b], hi[b]) minus lo[b], in order."""
    B, cap = (int(x) for x in blocks.shape)
    _check(lib().csa_shard_blocks(B, _ptr(blocks, "blocks"), _ptr(count, "count"), cap, _ptr(lo, "lo"),
                                  _ptr(hi, "hi"), _ptr(out_blocks, "out_blocks"), _ptr(out_count, "out_count"),
                                  int(out_blocks.shape[1]), _ptr(ws, "ws"), ws.numel(), _stream(stream)),
           "csa_shard_blocks")


def attn_merge(out_parts, lse_parts, out, lse, stream=None):
    """out_parts float32 [R, B, H, 512], lse_parts float32 [R, B, H] -> out [B, H, 512], lse [B, H]."""
    R, B, H = (int(x) for x in lse_parts.shape)
    _check(lib().csa_attn_merge(R, B, H, _ptr(out_parts, "out_parts"), _ptr(lse_parts, "lse_parts"),
                                _ptr(out, "out"), _ptr(lse, "lse"), _stream(stream)), "csa_attn_merge")


def kv_record_bytes(n):
    """Bytes of the persistent record of an n-token sequence: 26,624 per 64-token page."""
    return int(lib().csa_kv_record_bytes(int(n)))


def _record_args(layer, block_table, n, buf, name):
    if buf.dtype != torch.uint8 or buf.numel() < kv_record_bytes(n):
        raise ValueError("%s must be a uint8 tensor of at least kv_record_bytes(n) bytes" % name)
    if block_table.dtype != torch.int32 or block_table.numel() < (int(n) + PAGE - 1) // PAGE:
        raise ValueError("block_table must be int32 with one entry per page of the sequence")
    return layer.c(), _ptr(block_table, "block_table"), _buf_ptr(buf, name)


def kv_export(layer, block_table, n, dst, ws, stream=None):
    """Copy the persistent record (FP4 codes, scales, indexer keys; no window) of the n-token sequence
    whose pages are block_table[0 .. ceil(n/64)) into dst (device, or pinned host)."""
    lc, bt, d = _record_args(layer, block_table, n, dst, "dst")
    _check(lib().csa_kv_export(ctypes.byref(lc), bt, int(n), d, _ptr(ws, "ws"), ws.numel(), _stream(stream)),
           "csa_kv_export")


def kv_import(layer, block_table, n, src, ws, stream=None):
    """Write a persistent record back into the pages block_table[0 .. ceil(n/64)).  The window is
    restored afterwards by replaying the last min(n, 128) tokens through kv_pack_fp4."""
    lc, bt, s = _record_args(layer, block_table, n, src, "src")
    _check(lib().csa_kv_import(ctypes.byref(lc), bt, int(n), s, _ptr(ws, "ws"), ws.numel(), _stream(stream)),
           "csa_kv_import")


def check_device_error(ws, stream=None):
    """Synchronise, read and clear the workspace status.  Returns (status, detail)."""
    d = ctypes.c_int64(0)
    s = lib().csa_check_device_error(_ptr(ws, "ws"), _stream(stream), ctypes.byref(d))
    return s, d.value
