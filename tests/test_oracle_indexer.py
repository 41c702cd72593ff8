"""Pins for the oracle's indexer score, block max and Top-K selection, and for the three layer
modes (rebasdaily article, section 同一份笔记，多层一起用: Full re-selects over the whole range,
Reindex searches only inside the pool, Reuse keeps the earlier layer's set)."""
import json
import os

import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def e4m3_codes_of(values):
    """E4M3 codes of values that E4M3 represents exactly (looked up in the decode table)."""
    table = {float(v): c for c, v in enumerate(oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8)))}
    table.update({-float(v): c | 0x80 for v, c in list(table.items()) if v != 0})
    return np.vectorize(lambda v: table[float(v)])(values).astype(np.uint8)


def exact_score(iq_bf16, iw, keys8):
    """sum_h w_h * max(0, q_h . k) evaluated exactly in float64 (used where every product and
    partial sum is exactly representable)."""
    q = synth.bf16_to_f32(iq_bf16).astype(np.float64).reshape(8, 128)
    k = oracle.e4m3_decode(keys8).reshape(-1, 128)
    d = k @ q.T
    return np.maximum(d, 0) @ np.asarray(iw, np.float64)


def test_score_exact_on_small_integers():
    rng = np.random.default_rng(31)
    q = rng.integers(-3, 4, (8, 128)).astype(np.float32)
    k = rng.integers(-4, 5, (500, 128)).astype(np.float64)
    w = rng.integers(0, 4, 8).astype(np.float32) / 2
    iq = synth.bf16_bits(q)
    k8 = e4m3_codes_of(k)
    got = oracle.index_scores(iq, w, k8).astype(np.float64)
    assert np.array_equal(got, exact_score(iq, w, k8))
    # ReLU really clips: some heads are negative on some keys
    assert ((k @ q.T.astype(np.float64)) < 0).any()


def test_score_within_float32_bound_of_exact():
    rng = np.random.default_rng(32)
    iq, iw = synth.index_query(rng, 1)
    keys = synth.index_keys(rng, 4000)
    k8 = oracle.pack_tokens(np.zeros((4000, 512), np.uint16), keys, with_swa=False)["key8"]
    got = oracle.index_scores(iq[0], iw[0], k8).astype(np.float64)
    q = synth.bf16_to_f32(iq[0]).astype(np.float64).reshape(8, 128)
    k = oracle.e4m3_decode(k8)
    d = k @ q.T
    ref = np.maximum(d, 0) @ iw[0].astype(np.float64)
    # each head: 16-term chains then a 3-level tree: |err| <= 19 u sum|q k|; then an 8-term chain
    u = 2.0 ** -24
    head_abs = np.abs(k) @ np.abs(q).T
    bound = (19 * u * head_abs) @ iw[0].astype(np.float64) * (1 + 9 * u) + 9 * u * np.abs(ref)
    assert (np.abs(got - ref) <= bound + 1e-30).all()
    assert (got >= 0).all()


def test_score_one_hot_key_and_weight():
    rng = np.random.default_rng(33)
    iq, _ = synth.index_query(rng, 1)
    q = synth.bf16_to_f32(iq[0]).reshape(8, 128)
    for h in range(8):
        w = np.zeros(8, np.float32)
        w[h] = 1
        for d in (0, 17, 64, 127):
            k = np.zeros((1, 128))
            k[0, d] = 1.0
            s = oracle.index_scores(iq[0], w, e4m3_codes_of(k))[0]
            assert s == max(q[h, d], 0.0)


def test_block_score_is_max_over_valid_positions():
    rng = np.random.default_rng(34)
    iq, iw = synth.index_query(rng, 1)
    keys = synth.index_keys(rng, 203)               # 25 full blocks + a 3-position tail
    k8 = oracle.pack_tokens(np.zeros((203, 512), np.uint16), keys, with_swa=False)["key8"]
    t = oracle.index_scores(iq[0], iw[0], k8)
    S = oracle.block_scores(iq[0], iw[0], k8)
    assert S.shape == (26,)
    for b in range(26):
        assert S[b] == t[8 * b:min(8 * b + 8, 203)].max()
    # permuting positions inside a block leaves block scores unchanged
    perm = np.concatenate([rng.permutation(8) + 8 * b for b in range(25)] + [np.arange(200, 203)])
    assert np.array_equal(oracle.block_scores(iq[0], iw[0], k8[perm]), S)


def brute_topk(scores, blocks, k):
    order = sorted(range(len(scores)), key=lambda i: (-float(scores[i]), int(blocks[i])))
    return sorted(int(blocks[i]) for i in order[:k])


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (100, 100), (100, 200), (1000, 64), (5000, 2048)])
def test_topk_matches_brute_force_with_ties(n, k):
    rng = np.random.default_rng(35 + n)
    scores = (rng.integers(0, 20, n) / 4).astype(np.float32)      # many exact ties
    blocks = np.arange(n, dtype=np.int32)
    got = oracle.topk(blocks, scores, k)
    assert got.tolist() == brute_topk(scores, blocks, k)
    assert got.size == min(k, n)
    assert (np.diff(got) > 0).all()


def test_topk_all_equal_scores_takes_lowest_ids():
    got = oracle.topk(np.arange(500, dtype=np.int32), np.zeros(500, np.float32), 64)
    assert got.tolist() == list(range(64))


def test_full_pool_holds_2048_blocks_of_8():
    L = 8 * 3000 + 5
    rng = np.random.default_rng(36)
    iq, iw = synth.index_query(rng, 1)
    k8 = oracle.pack_tokens(np.zeros((L, 512), np.uint16), synth.index_keys(rng, L),
                            with_swa=False)["key8"]
    S = oracle.block_scores(iq[0], iw[0], k8)
    pool = oracle.topk(np.arange(S.size, dtype=np.int32), S, GOLDEN["pool_blocks"]["value"])
    assert pool.size == GOLDEN["pool_blocks"]["value"]
    pos = oracle.positions_of_blocks(pool, L)
    assert pos.size == GOLDEN["pool_positions"]["value"] == pool.size * GOLDEN["block_positions"]["value"]
    # zero head weights: every block scores 0, so the lowest ids win
    z = oracle.block_scores(iq[0], np.zeros(8, np.float32), k8[:800])
    assert oracle.topk(np.arange(z.size, dtype=np.int32), z, 10).tolist() == list(range(10))


def make_layer(rng, L, num_extra_pages=3):
    bt, npages = synth.block_tables(rng, [L], extra_pages=num_extra_pages)
    keys = synth.index_keys(rng, L)
    lat = synth.latents(rng, np.arange(L))
    p = oracle.pack_tokens(lat, keys)
    layer = dict(codes=np.zeros((npages, 64, 256), np.uint8), scales=np.zeros((npages, 64, 32), np.uint8),
                 keys=np.zeros((npages, 64, 128), np.uint8), swa=np.zeros((1, 128, 512), np.uint8),
                 swa_scale=np.zeros((1, 128), np.float32))
    pages, offs = oracle.rows_of_positions(bt[0], np.arange(L))
    layer["codes"][pages, offs] = p["codes"]
    layer["scales"][pages, offs] = p["scales"]
    layer["keys"][pages, offs] = p["key8"]
    w = oracle.window_positions(L)
    layer["swa"][0, w % 128] = p["swa"][w]
    layer["swa_scale"][0, w % 128] = p["swa_scale"][w]
    return layer, bt[0], p


def test_reindex_searches_only_inside_the_pool():
    rng = np.random.default_rng(37)
    L = 8 * 700 + 3
    layer, bt, _ = make_layer(rng, L)
    iq, iw = synth.index_query(rng, 2)
    pool = oracle.select_full(layer, bt, L, iq[0], iw[0], 256)
    sub = oracle.select_reindex(layer, bt, L, iq[1], iw[1], pool, 64)
    assert sub.size == 64 and set(sub.tolist()) <= set(pool.tolist())
    assert (np.diff(sub) > 0).all()
    # k_r >= |pool| returns the pool itself
    assert np.array_equal(oracle.select_reindex(layer, bt, L, iq[1], iw[1], pool, 256), pool)
    assert np.array_equal(oracle.select_reindex(layer, bt, L, iq[1], iw[1], pool, 999), pool)
    # with the Full layer's own query, re-scoring inside its pool gives its own top-k_r
    assert np.array_equal(oracle.select_reindex(layer, bt, L, iq[0], iw[0], pool, 64),
                          oracle.select_full(layer, bt, L, iq[0], iw[0], 64))


def test_reuse_is_the_previous_set():
    prev = np.array([3, 9, 10, 400], np.int32)
    got = oracle.select_reuse(prev)
    assert got.tobytes() == prev.tobytes() and got is not prev
