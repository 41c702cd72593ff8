"""Reindex on the GPU: csa_indexer_reindex against the oracle's select_reindex and against its two
public steps run one by one (csa_indexer_block_scores in pool mode, then csa_topk_blocks): pools of
100 to 6,000 blocks, every score tied, k_r at and above the pool size, and malformed pools reported."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

pytestmark = pytest.mark.gpu


def _dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is not None else t).cuda()


def _setup(lens, seed, same_key=False):
    """Keys of B sequences in scattered pages; returns the GPU layer, batch and the oracle layers."""
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    rng = np.random.default_rng(seed)
    bt, P = synth.block_tables(rng, lens, extra_pages=2)
    layer = csa.KVLayer(P, len(lens))
    keys = np.zeros((P, 64, 128), np.uint8)
    per_seq = []
    for b, L in enumerate(lens):
        k = synth.index_keys(rng, 1 if same_key else L)
        k8 = oracle.pack_tokens(np.zeros((k.shape[0], 512), np.uint16), k, with_swa=False)["key8"]
        if same_key:
            k8 = np.tile(k8, (L, 1))
        pos = np.arange(L)
        keys[bt[b][pos // 64], pos % 64] = k8
        per_seq.append(k8)
    layer.keys.copy_(torch.from_numpy(keys))
    batch = csa.Batch(_dev(np.array(lens, np.int32)), _dev(bt), _dev(np.zeros(len(lens), np.int32)), max(lens))
    return layer, batch, per_seq


def _pools(rng, lens, sizes, cap):
    pool = np.zeros((len(lens), cap), np.int32)
    cnt = np.zeros(len(lens), np.int32)
    for b, (L, n) in enumerate(zip(lens, sizes)):
        nb = (L + 7) // 8
        p = np.sort(rng.choice(nb, size=n, replace=False)).astype(np.int32)
        pool[b, :n] = p
        cnt[b] = n
    return pool, cnt


def _reindex(layer, batch, iq, iw, pool, cnt, k):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    B, cap = pool.shape
    ws = csa.workspace(B, 16, batch.max_seq_len, cap)
    out = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    oc = torch.zeros(B, dtype=torch.int32, device="cuda")
    csa.indexer_reindex(layer, batch, _dev(iq, torch.bfloat16), _dev(iw), _dev(pool), _dev(cnt), k, out, oc, ws)
    st = csa.check_device_error(ws)[0]
    c = oc.cpu().numpy()
    return [out[b, :c[b]].cpu().numpy() for b in range(B)], st


def _two_step(layer, batch, iq, iw, pool, cnt, k):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    B, cap = pool.shape
    ws = csa.workspace(B, 16, batch.max_seq_len, cap)
    sc = torch.zeros((B, cap), device="cuda")
    csa.indexer_block_scores(layer, batch, _dev(iq, torch.bfloat16), _dev(iw), sc, ws, pool=_dev(pool),
                             pool_count=_dev(cnt))
    out = torch.zeros((B, k), dtype=torch.int32, device="cuda")
    oc = torch.zeros(B, dtype=torch.int32, device="cuda")
    csa.topk_blocks(batch, sc, k, out, oc, ws, pool=_dev(pool), pool_count=_dev(cnt))
    assert csa.check_device_error(ws)[0] == 0
    c = oc.cpu().numpy()
    return [out[b, :c[b]].cpu().numpy() for b in range(B)]


@pytest.mark.parametrize("sizes,cap,k", [([256, 100, 256], 256, 40), ([2048, 2048, 1999, 2048], 2048, 512),
                                         ([4096, 3000], 4096, 512), ([6000, 5000], 6000, 700)])
def test_reindex_matches_oracle_and_two_step_path(sizes, cap, k):
    rng = np.random.default_rng([31, cap, k])
    lens = [int(8 * n + rng.integers(8, 4000)) for n in sizes]
    layer, batch, keys = _setup(lens, 32 + cap)
    iq, iw = synth.index_query(rng, len(lens))
    pool, cnt = _pools(rng, lens, sizes, cap)
    got, st = _reindex(layer, batch, iq, iw, pool, cnt, k)
    assert st == 0
    ref2 = _two_step(layer, batch, iq, iw, pool, cnt, k)
    for b, L in enumerate(lens):
        S = oracle.block_scores(iq[b], iw[b], keys[b])
        p = pool[b, :cnt[b]]
        ref = oracle.topk(p, S[p], k)
        assert got[b].tolist() == ref.tolist(), "seq %d" % b
        assert ref2[b].tolist() == ref.tolist()


def test_reindex_all_scores_tied_takes_the_lowest_blocks():
    rng = np.random.default_rng(33)
    lens = [20000, 30000]
    layer, batch, _ = _setup(lens, 34, same_key=True)
    iq, iw = synth.index_query(rng, 2)
    pool, cnt = _pools(rng, lens, [2048, 1500], 2048)
    got, st = _reindex(layer, batch, iq, iw, pool, cnt, 300)
    assert st == 0
    for b in range(2):
        assert got[b].tolist() == pool[b, :300].tolist()


def test_reindex_small_pool_is_returned_whole():
    rng = np.random.default_rng(35)
    lens = [9000]
    layer, batch, _ = _setup(lens, 36)
    iq, iw = synth.index_query(rng, 1)
    pool, cnt = _pools(rng, lens, [77], 128)
    got, st = _reindex(layer, batch, iq, iw, pool, cnt, 77)
    assert st == 0 and got[0].tolist() == pool[0, :77].tolist()


def test_reindex_malformed_pools_are_reported():
    """A block past the sequence, an unsorted pool, a count above the capacity: status 5, no fault."""
    rng = np.random.default_rng(37)
    lens = [9000, 9000, 9000]
    layer, batch, _ = _setup(lens, 38)
    iq, iw = synth.index_query(rng, 3)
    pool, cnt = _pools(rng, lens, [500, 500, 500], 512)
    pool[0, 499] = 100000          # block past the end of sequence 0
    pool[1, 10], pool[1, 11] = pool[1, 11], pool[1, 10]   # not ascending
    cnt[2] = 9999                  # above the capacity
    got, st = _reindex(layer, batch, iq, iw, pool, cnt, 100)
    assert st == 5
    assert len(got[2]) == 0
