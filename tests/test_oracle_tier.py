"""The oracle's persistent record pinned to what the pages fix: 416 bytes per token (FP4 512 channels
= 256 B, one E4M3 scale per 16 channels = 32 B, the 128-byte E4M3 indexer key), no window byte in
it, each token's bytes at the offsets the paged layout gives (checked against the per-token pack,
not against the record's own gather), and a restore (record into other pages, window replayed from
the last tokens) that attends exactly like the original caches."""
import numpy as np

import oracle
from fp4_compressed_sparse_kv_b200 import synth

REC = 64 * (256 + 32 + 128)


def _sequence(n, seed, extra_pages=3):
    rng = np.random.default_rng(seed)
    lat = synth.latents(rng, np.arange(n))
    key = synth.index_keys(rng, n)
    bt, P = synth.block_tables(rng, [n], extra_pages=extra_pages)
    p = oracle.pack_tokens(lat, key, with_swa=False)
    layer = dict(codes=rng.integers(0, 256, (P, 64, 256), dtype=np.uint8),
                 scales=rng.integers(0, 256, (P, 64, 32), dtype=np.uint8),
                 keys=rng.integers(0, 256, (P, 64, 128), dtype=np.uint8),
                 swa=np.zeros((2, 128, 512), np.uint8), swa_scale=np.zeros((2, 128), np.float32))
    pos = np.arange(n)
    pages, offs = bt[0][pos // 64], pos % 64
    layer["codes"][pages, offs] = p["codes"]
    layer["scales"][pages, offs] = p["scales"]
    layer["keys"][pages, offs] = p["key8"]
    w = oracle.window_positions(n)
    ps = oracle.pack_tokens(lat[w], key[w], with_swa=True)
    layer["swa"][1, w % 128] = ps["swa"]
    layer["swa_scale"][1, w % 128] = ps["swa_scale"]
    return lat, key, bt[0], layer, p


def test_record_size_is_416_bytes_per_token_of_whole_pages():
    assert REC == 26624
    for n in [1, 63, 64, 65, 700]:
        _, _, bt, layer, _ = _sequence(n, n)
        assert oracle.persistent_record(layer, bt, n).size == -(-n // 64) * REC
    assert oracle.persistent_record(layer, bt, 0).size == 0


def test_each_token_sits_at_its_layout_offset():
    n = 300
    _, _, bt, layer, p = _sequence(n, 11)
    rec = oracle.persistent_record(layer, bt, n)
    for t in range(n):
        base = (t // 64) * REC
        j = t % 64
        assert np.array_equal(rec[base + 256 * j: base + 256 * (j + 1)], p["codes"][t])
        assert np.array_equal(rec[base + 16384 + 32 * j: base + 16384 + 32 * (j + 1)], p["scales"][t])
        assert np.array_equal(rec[base + 18432 + 128 * j: base + 18432 + 128 * (j + 1)], p["key8"][t])


def test_window_is_not_stored():
    n = 200
    _, _, bt, layer, _ = _sequence(n, 12)
    a = oracle.persistent_record(layer, bt, n)
    layer["swa"][:] = 0x5A
    layer["swa_scale"][:] = 7.0
    assert np.array_equal(a, oracle.persistent_record(layer, bt, n))


def test_restore_with_replayed_window_attends_like_the_original():
    n = 777
    lat, key, bt, layer, _ = _sequence(n, 13)
    rec = oracle.persistent_record(layer, bt, n)
    # restore into a fresh layer with other page ids, by the layout's offsets
    P = len(bt) + 5
    new_bt = np.random.default_rng(3).permutation(P)[:len(bt)]
    fresh = dict(codes=np.zeros((P, 64, 256), np.uint8), scales=np.zeros((P, 64, 32), np.uint8),
                 keys=np.zeros((P, 64, 128), np.uint8), swa=np.zeros((1, 128, 512), np.uint8),
                 swa_scale=np.zeros((1, 128), np.float32))
    for i, pg in enumerate(new_bt):
        r = rec[i * REC:(i + 1) * REC]
        fresh["codes"][pg] = r[:16384].reshape(64, 256)
        fresh["scales"][pg] = r[16384:18432].reshape(64, 32)
        fresh["keys"][pg] = r[18432:].reshape(64, 128)
    w = oracle.window_positions(n)
    ps = oracle.pack_tokens(lat[w], key[w], with_swa=True)     # the replay
    fresh["swa"][0, w % 128] = ps["swa"]
    fresh["swa_scale"][0, w % 128] = ps["swa_scale"]
    rng = np.random.default_rng(4)
    q = synth.query(rng, 1, 16)[0]
    iq, iw = synth.index_query(rng, 1)
    k = 20
    s0 = oracle.select_full(layer, bt, n, iq[0], iw[0], k)
    s1 = oracle.select_full(fresh, new_bt, n, iq[0], iw[0], k)
    assert s0.tolist() == s1.tolist()
    o0, l0 = oracle.attend(layer, bt, 1, n, q, oracle.default_tau(), s0)
    o1, l1 = oracle.attend(fresh, new_bt, 0, n, q, oracle.default_tau(), s1)
    assert np.array_equal(o0, o1) and np.array_equal(l0, l1)
