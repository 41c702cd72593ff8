"""Shared test helpers: oracle-side reconstruction of one sequence's caches from the seeded
generators, and the GPU-vs-oracle comparisons.  The oracle packs every token itself; nothing it
consumes comes from the CUDA path."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

ATTN_TOL = 2e-3     # max |gpu - oracle| <= ATTN_TOL * max |oracle| per sequence
LSE_TOL = 1e-3      # absolute


def gpu_available():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


needs_gpu = pytest.mark.skipif(not gpu_available(), reason="needs a CUDA device")


def oracle_layer_from_tokens(lat, key, L, with_swa=True):
    """Oracle caches of one sequence in its own identity page layout (pages 0..n-1, SWA row 0)."""
    p = oracle.pack_tokens(lat[:L], key[:L], with_swa=False)
    npages = (L + 63) // 64
    layer = dict(codes=np.zeros((npages, 64, 256), np.uint8), scales=np.zeros((npages, 64, 32), np.uint8),
                 keys=np.zeros((npages, 64, 128), np.uint8), swa=np.zeros((1, 128, 512), np.uint8),
                 swa_scale=np.zeros((1, 128), np.float32))
    pos = np.arange(L)
    layer["codes"][pos // 64, pos % 64] = p["codes"]
    layer["scales"][pos // 64, pos % 64] = p["scales"]
    layer["keys"][pos // 64, pos % 64] = p["key8"]
    if with_swa:
        w = oracle.window_positions(L)
        ps = oracle.pack_tokens(lat[w], key[w], with_swa=True)
        layer["swa"][0, w % 128] = ps["swa"]
        layer["swa_scale"][0, w % 128] = ps["swa_scale"]
    return layer, np.arange(npages), p


def assert_attention_close(out_gpu, lse_gpu, out_ref, lse_ref, what=""):
    out_gpu = np.asarray(out_gpu, np.float64)
    scale = np.abs(out_ref).max()
    err = np.abs(out_gpu - out_ref).max()
    assert err <= ATTN_TOL * scale, "%s: max err %.3e vs bound %.3e" % (what, err, ATTN_TOL * scale)
    lerr = np.abs(np.asarray(lse_gpu, np.float64) - lse_ref).max()
    assert lerr <= LSE_TOL, "%s: lse err %.3e" % (what, lerr)
    return err / scale


def _chunks(n, parts, align=1):
    step = max(align, ((n + parts - 1) // parts + align - 1) // align * align)
    return [(i, min(n, i + step)) for i in range(0, n, step)]


def pack_tokens_threaded(lat, key, with_swa=False, threads=8):
    """oracle.pack_tokens over token chunks in threads (the C oracle runs without the GIL)."""
    import concurrent.futures as cf
    n = lat.shape[0]
    parts = _chunks(n, threads)
    with cf.ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda ab: oracle.pack_tokens(lat[ab[0]:ab[1]], key[ab[0]:ab[1]], with_swa), parts))
    return {k: np.concatenate([r[k] for r in res]) for k in res[0]}


def block_scores_threaded(iq, iw, keys8, threads=8):
    import concurrent.futures as cf
    L = keys8.shape[0]
    parts = _chunks(L, threads, align=8)
    with cf.ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda ab: oracle.block_scores(iq, iw, keys8[ab[0]:ab[1]]), parts))
    return np.concatenate(res)


def attention_threaded(q, tau, codes, scales, swa, swa_scale, threads=8):
    import concurrent.futures as cf
    H = q.shape[0]
    parts = _chunks(H, threads)
    with cf.ThreadPoolExecutor(threads) as ex:
        res = list(ex.map(lambda ab: oracle.attention(q[ab[0]:ab[1]], tau, codes, scales, swa, swa_scale),
                          parts))
    return np.concatenate([r[0] for r in res]), np.concatenate([r[1] for r in res])


class OracleSeq:
    """One sequence's oracle-side caches (packed by the oracle from the seeded tokens) and the
    oracle's Full / Reindex / attention on them."""

    def __init__(self, lat, key, L):
        self.L = L
        p = pack_tokens_threaded(lat[:L], key[:L])
        self.codes, self.scales, self.key8 = p["codes"], p["scales"], p["key8"]
        w = oracle.window_positions(L)
        ps = oracle.pack_tokens(lat[w], key[w], with_swa=True)
        self.win_pos = w
        self.swa, self.swa_scale = ps["swa"], ps["swa_scale"]
        self._S = {}

    def block_scores(self, iq, iw):
        k = (iq.tobytes(), iw.tobytes())
        if k not in self._S:
            self._S[k] = block_scores_threaded(iq, iw, self.key8)
        return self._S[k]

    def full(self, iq, iw, k):
        S = self.block_scores(iq, iw)
        return oracle.topk(np.arange(S.size, dtype=np.int32), S, k)

    def reindex(self, iq, iw, pool, k_r):
        S = self.block_scores(iq, iw)
        return oracle.topk(np.asarray(pool, np.int32), S[np.asarray(pool)], k_r)

    def attend(self, q, tau, blocks):
        pe = oracle.positions_of_blocks(blocks, self.L)
        return attention_threaded(q, tau, self.codes[pe], self.scales[pe], self.swa, self.swa_scale)
