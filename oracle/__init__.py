"""Plain, slow CPU oracle for the CSA2 FP4 compressed sparse-KV decode path.

TEST INFRASTRUCTURE ONLY.  Only the test suite, ``__graft_entry__.smoke()`` and the benchmark's
CPU-baseline leg may import this package.  The product library (the CUDA path behind the C-ABI)
never imports, links or executes anything here, and this package imports nothing from it.

The arithmetic lives in ``csa_oracle.c`` (compiled without FP contraction); this module only
marshals numpy arrays and does the plain paged-layout indexing that turns a block table into
per-position rows.

Sources, cited by page and section:
  [rebasdaily] rebasdaily.com article on DeepSeek-V4.1-Flash KV compression,
               section "同一份笔记，多层一起用" (CSA2 layer modes Full / Reindex / Reuse, the
               hierarchical indexer with its 2,048 x 8 = 16,384-position pool, FP4 main KV,
               FP8 SWA KV) and section "先让长输入少走一半路" (the sliding-window branch).
  [ailily]     ailily.cc article "每个 token 只占 890 字节", section 二 (mode table; one E4M3
               scale per 16 channels) and section 三 (the sqrt(512) and 448 x 6 range argument).

Parity pins: every function here is pinned by ``tests/test_oracle_*.py`` against library codecs,
closed forms, brute force or the pages' printed constants; none is marked "parity unpinned".
"""
import ctypes
import math

import numpy as np

from . import build as _build

PAGE = 64          # tokens per KV page
BLOCK = 8          # positions per indexer block ([rebasdaily] "每块 8 个位置")
WINDOW = 128       # sliding-window length
LATENT = 512       # latent channels (both key and value)
GROUP = 16         # channels per E4M3 scale ([ailily] 二)
IDX_HEADS = 8
IDX_DIM = 128

FULL, REINDEX, REUSE = 0, 1, 2

_lib = None


def lib():
    """Load (building first if needed) the compiled oracle."""
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        P = ctypes.c_void_p
        i64, i32, f64 = ctypes.c_int64, ctypes.c_int32, ctypes.c_double
        L.ora_e4m3_decode.restype = f64
        L.ora_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.ora_e2m1_decode.restype = f64
        L.ora_e2m1_decode.argtypes = [ctypes.c_uint8]
        L.ora_e4m3_encode.restype = ctypes.c_uint8
        L.ora_e4m3_encode.argtypes = [ctypes.c_float]
        L.ora_e2m1_encode.restype = ctypes.c_uint8
        L.ora_e2m1_encode.argtypes = [ctypes.c_float]
        for n in ("ora_e4m3_encode_n", "ora_e2m1_encode_n", "ora_e4m3_decode_n",
                  "ora_e2m1_decode_n"):
            getattr(L, n).restype = None
            getattr(L, n).argtypes = [i64, P, P]
        L.ora_pack_tokens.restype = None
        L.ora_pack_tokens.argtypes = [i64, P, P, P, P, P, P, P]
        L.ora_norm_rope.restype = None
        L.ora_norm_rope.argtypes = [i64, P, P, P, P]
        L.ora_index_score.restype = ctypes.c_float
        L.ora_index_score.argtypes = [P, P, P]
        L.ora_index_scores.restype = None
        L.ora_index_scores.argtypes = [i64, P, P, P, P]
        L.ora_block_scores.restype = None
        L.ora_block_scores.argtypes = [i64, P, P, P, P]
        L.ora_topk.restype = i32
        L.ora_topk.argtypes = [i64, P, P, i32, P]
        L.ora_attention.restype = ctypes.c_int
        L.ora_attention.argtypes = [i32, P, f64, i64, P, P, i64, P, P, P, P]
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ----------------------------------------------------------------------------------------------
# Codecs (OCP FP8 E4M3 "fn" and MX E2M1 definitions; the pages name the formats only)
# ----------------------------------------------------------------------------------------------
def e4m3_encode(x):
    """float32 array -> E4M3 codes (round-to-nearest-even, saturating to +-448, sign kept)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().ora_e4m3_encode_n(x.size, _p(x), _p(out))
    return out


def e2m1_encode(x):
    """float32 array -> E2M1 codes 0..15 (round-to-nearest-even, saturating to +-6, sign kept)."""
    x = _c(x, np.float32)
    out = np.empty(x.shape, np.uint8)
    lib().ora_e2m1_encode_n(x.size, _p(x), _p(out))
    return out


def e4m3_decode(c):
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().ora_e4m3_decode_n(c.size, _p(c), _p(out))
    return out


def e2m1_decode(c):
    c = _c(c, np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().ora_e2m1_decode_n(c.size, _p(c), _p(out))
    return out


# ----------------------------------------------------------------------------------------------
# Step 1: pack
# ----------------------------------------------------------------------------------------------
def pack_tokens(latent_bf16, key_bf16, with_swa=True):
    """Pack n tokens.  latent_bf16: uint16 [n,512] (bf16 bit patterns), key_bf16: uint16 [n,128].

    Returns dict with codes uint8 [n,256], scales uint8 [n,32], key8 uint8 [n,128] and, if
    with_swa, swa uint8 [n,512] and swa_scale float32 [n]."""
    lat = _c(latent_bf16, np.uint16).reshape(-1, LATENT)
    key = _c(key_bf16, np.uint16).reshape(-1, IDX_DIM)
    n = lat.shape[0]
    assert key.shape[0] == n
    out = dict(codes=np.zeros((n, 256), np.uint8), scales=np.zeros((n, 32), np.uint8),
               key8=np.zeros((n, IDX_DIM), np.uint8))
    swa = swa_scale = None
    if with_swa:
        out["swa"] = swa = np.zeros((n, LATENT), np.uint8)
        out["swa_scale"] = swa_scale = np.zeros((n,), np.float32)
    lib().ora_pack_tokens(n, _p(lat), _p(key), _p(out["codes"]), _p(out["scales"]),
                          _p(out["key8"]), _p(swa) if with_swa else None,
                          _p(swa_scale) if with_swa else None)
    return out


def norm_rope(latent_bf16, weight, cos_sin):
    """RMSNorm (weight [512], eps 1e-6) then RoPE on channels 448..511 of n pre-norm latents, in the
    binary32 order of ora_norm_rope.  latent_bf16 uint16 [n,512]; cos_sin float32 [n,32,2] (cos_i,
    sin_i of pair i = channels 448+2i, 449+2i).  Returns bf16 bit patterns uint16 [n,512]."""
    x = _c(latent_bf16, np.uint16).reshape(-1, LATENT)
    n = x.shape[0]
    w = _c(weight, np.float32).reshape(LATENT)
    cs = _c(cos_sin, np.float32).reshape(n, 32, 2)
    out = np.zeros((n, LATENT), np.uint16)
    lib().ora_norm_rope(n, _p(x), _p(w), _p(cs), _p(out))
    return out


def dequant_main(codes, scales):
    """FP4 entries -> float64 values [n,512]: e2m1(code) * e4m3(scale of its 16-channel group)."""
    codes = _c(codes, np.uint8).reshape(-1, 256)
    scales = _c(scales, np.uint8).reshape(-1, 32)
    lo = codes & 15
    hi = codes >> 4
    nib = np.stack([lo, hi], axis=-1).reshape(-1, LATENT)
    return e2m1_decode(nib) * np.repeat(e4m3_decode(scales), GROUP, axis=1)


def dequant_swa(swa, swa_scale):
    swa = _c(swa, np.uint8).reshape(-1, LATENT)
    return e4m3_decode(swa) * _c(swa_scale, np.float32).astype(np.float64)[:, None]


# ----------------------------------------------------------------------------------------------
# Steps 2-3: indexer score, block max, Top-K
# ----------------------------------------------------------------------------------------------
def index_scores(iq_bf16, iw, keys8):
    """Per-position scores (float32) of keys8 uint8 [n,128] under iq [8,128] bf16 and iw [8]."""
    iq = _c(iq_bf16, np.uint16).reshape(IDX_HEADS, IDX_DIM)
    iw = _c(iw, np.float32).reshape(IDX_HEADS)
    k = _c(keys8, np.uint8).reshape(-1, IDX_DIM)
    out = np.empty(k.shape[0], np.float32)
    lib().ora_index_scores(k.shape[0], _p(iq), _p(iw), _p(k), _p(out))
    return out


def block_scores(iq_bf16, iw, keys8):
    """Block scores float32 [ceil(L/8)] for keys8 [L,128]: max over each block's valid positions."""
    iq = _c(iq_bf16, np.uint16).reshape(IDX_HEADS, IDX_DIM)
    iw = _c(iw, np.float32).reshape(IDX_HEADS)
    k = _c(keys8, np.uint8).reshape(-1, IDX_DIM)
    L = k.shape[0]
    out = np.empty((L + BLOCK - 1) // BLOCK, np.float32)
    lib().ora_block_scores(L, _p(iq), _p(iw), _p(k), _p(out))
    return out


def topk(blocks, scores, k):
    """The min(k, n) best (larger score, then lower block id) of the candidates, ascending ids."""
    blocks = _c(blocks, np.int32)
    scores = _c(scores, np.float32)
    out = np.empty(max(min(k, blocks.size), 1), np.int32)
    cnt = lib().ora_topk(blocks.size, _p(blocks), _p(scores), int(k), _p(out))
    return out[:cnt].copy()


# ----------------------------------------------------------------------------------------------
# Step 4: attention
# ----------------------------------------------------------------------------------------------
def attention(q_bf16, tau, codes, scales, swa, swa_scale):
    """One sequence: q uint16 [H,512]; FP4 entries (codes [nE,256], scales [nE,32]); SWA entries
    (swa [nF,512], swa_scale [nF]).  Returns (out float64 [H,512], lse float64 [H])."""
    q = _c(q_bf16, np.uint16).reshape(-1, LATENT)
    H = q.shape[0]
    codes = _c(codes, np.uint8).reshape(-1, 256)
    scales = _c(scales, np.uint8).reshape(-1, 32)
    swa = _c(swa, np.uint8).reshape(-1, LATENT)
    swa_scale = _c(swa_scale, np.float32).reshape(-1)
    out = np.empty((H, LATENT), np.float64)
    lse = np.empty((H,), np.float64)
    rc = lib().ora_attention(H, _p(q), float(tau), codes.shape[0], _p(codes), _p(scales),
                             swa.shape[0], _p(swa), _p(swa_scale), _p(out), _p(lse))
    if rc != 0:
        raise MemoryError("oracle attention: allocation failed")
    return out, lse


# ----------------------------------------------------------------------------------------------
# Paged-layout helpers and one decode-layer step for one sequence
# ----------------------------------------------------------------------------------------------
def rows_of_positions(block_table_row, positions):
    """(page, offset-in-page) of each position under one sequence's block-table row."""
    positions = np.asarray(positions, np.int64)
    pages = np.asarray(block_table_row, np.int64)[positions // PAGE]
    return pages, positions % PAGE


def gather_keys(layer, block_table_row, L):
    pages, offs = rows_of_positions(block_table_row, np.arange(L))
    return layer["keys"][pages, offs]


def positions_of_blocks(blocks, L):
    blocks = np.asarray(blocks, np.int64)
    pos = (blocks[:, None] * BLOCK + np.arange(BLOCK)[None, :]).reshape(-1)
    return pos[pos < L]


def window_positions(L, W=WINDOW):
    return np.arange(max(0, L - W), L, dtype=np.int64)


def select_full(layer, block_table_row, L, iq, iw, k):
    """Full layer: score every block of the sequence and keep the Top-k ([rebasdaily] CSA2, Full)."""
    S = block_scores(iq, iw, gather_keys(layer, block_table_row, L))
    return topk(np.arange(S.size, dtype=np.int32), S, k)


def select_reindex(layer, block_table_row, L, iq, iw, pool, k_r):
    """Reindex layer: re-score only the pool's blocks with this layer's query, keep the Top-k_r
    ([rebasdaily] CSA2, Reindex: later layers search only inside the candidate pool)."""
    pool = np.asarray(pool, np.int32)
    keys = gather_keys(layer, block_table_row, L)
    S = block_scores(iq, iw, keys)
    return topk(pool, S[pool], k_r)


def select_reuse(prev):
    """Reuse layer: the previous layer's set, unchanged ([rebasdaily] CSA2, Reuse)."""
    return np.array(prev, np.int32, copy=True)


def attend(layer, block_table_row, swa_row, L, q, tau, blocks, W=WINDOW):
    """Sparse decode attention of one sequence over the FP4 entries of `blocks` (positions < L)
    and the FP8 window max(0, L-W) <= p < L of the sequence's SWA ring row."""
    pe = positions_of_blocks(blocks, L)
    pages, offs = rows_of_positions(block_table_row, pe)
    pw = window_positions(L, W)
    slots = pw % WINDOW
    return attention(q, tau, layer["codes"][pages, offs], layer["scales"][pages, offs],
                     layer["swa"][swa_row, slots], layer["swa_scale"][swa_row, slots])


def persistent_record(layer, block_table_row, n):
    """A sequence's persistent record: for each of its ceil(n/64) pages, in order, the page's codes
    [64][256], scales [64][32] and indexer keys [64][128] back to back; no window entry ([yomxxx] 三:
    the persistent KV tier in host memory or on SSD; [rebasdaily] 先让长输入少走一半路, SWA Bounded
    Replay: the window is restored by replaying the last tokens, not stored)."""
    pages = np.asarray(block_table_row, np.int64)[:(n + PAGE - 1) // PAGE]
    parts = []
    for p in pages:
        parts += [layer["codes"][p].reshape(-1), layer["scales"][p].reshape(-1), layer["keys"][p].reshape(-1)]
    return np.concatenate(parts) if parts else np.zeros((0,), np.uint8)


def default_tau():
    """Softmax temperature 1/sqrt(512) (the pages give none)."""
    return 1.0 / math.sqrt(LATENT)
