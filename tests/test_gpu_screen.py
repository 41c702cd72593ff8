"""GPU checks of the Full indexer's tensor-core screen: its per-block bounds bracket the oracle's
exact binary32 block scores, on key and query distributions chosen to stress each term of the bound
(E4M3 subnormal keys, queries spanning many binades, zero heads, negative weights), on ragged
lengths that leave partial tiles, pages and blocks; and the screened Full selection equals the
oracle's Top-K, also when every score ties or the inputs are not finite."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

pytestmark = pytest.mark.gpu

E4M3_FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)


def keys_for(rng, kind, n):
    if kind == "gauss":
        return oracle.e4m3_encode(synth.bf16_to_f32(synth.index_keys(rng, n)))
    if kind == "codes":          # every finite E4M3 code equally likely: 8 decades, subnormals included
        return rng.choice(E4M3_FINITE, size=(n, 128))
    if kind == "subnormal":      # mostly subnormal and tiny codes, a few large ones
        k = rng.choice(np.array([c for c in E4M3_FINITE if (c & 0x78) <= 0x08], np.uint8), size=(n, 128))
        big = rng.random((n, 128)) < 0.01
        k[big] = rng.choice(E4M3_FINITE, size=int(big.sum()))
        return k
    raise KeyError(kind)


def query_for(rng, kind, B):
    iq, iw = synth.index_query(rng, B)
    if kind == "wide":           # magnitudes log-uniform over 2^-30 .. 2^12, random signs
        mag = np.exp2(rng.uniform(-30, 12, size=iq.shape)).astype(np.float32)
        iq = synth.bf16_bits(mag * rng.choice([-1.0, 1.0], size=iq.shape).astype(np.float32))
        iw = rng.standard_normal(iw.shape).astype(np.float32)
    elif kind == "zero_heads":   # some heads all zero, some weights zero or negative
        iq = iq.copy()
        iq[:, ::3, :] = 0
        iw = iw.copy()
        iw[:, 1] = 0.0
        iw[:, 2] = -iw[:, 2]
    elif kind == "tiny":         # every query value far below 1 (large power-of-two scales)
        f = synth.bf16_to_f32(iq) * np.float32(2.0 ** -100)
        iq = synth.bf16_bits(f)
    return iq, iw


def gpu_layer(keys_per_seq, seed):
    """Pages of every sequence placed at random distinct page ids; returns layer, batch, tables."""
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    rng = np.random.default_rng(seed)
    lens = [k.shape[0] for k in keys_per_seq]
    npg = [(L + 63) // 64 for L in lens]
    total = sum(npg) + 3
    perm = rng.permutation(total)
    layer = csa.KVLayer(total, 1)
    max_len = max(lens)
    maxp = (max_len + 63) // 64
    bt = np.zeros((len(lens), maxp), np.int32)
    keys = np.zeros((total, 64, 128), np.uint8)
    o = 0
    for b, k in enumerate(keys_per_seq):
        pages = perm[o:o + npg[b]]
        o += npg[b]
        bt[b, :npg[b]] = pages
        pos = np.arange(k.shape[0])
        keys[pages[pos // 64], pos % 64] = k
    layer.keys.copy_(torch.from_numpy(keys))
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    batch = csa.Batch(dev(np.array(lens, np.int32)), dev(bt), dev(np.zeros(len(lens), np.int32)), max_len)
    return layer, batch


def screen(layer, batch, iq, iw):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    B = iq.shape[0]
    nb = (batch.max_seq_len + 7) // 8
    lo = torch.full((B, nb), 12345.0, device="cuda")
    hi = torch.full((B, nb), 12345.0, device="cuda")
    ws = csa.workspace(B, 16, batch.max_seq_len, 1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    csa.indexer_screen_bounds(layer, batch, dev(iq), dev(iw), lo, hi, ws)
    assert csa.check_device_error(ws)[0] == 0
    return lo.cpu().numpy(), hi.cpu().numpy()


LENS = [1, 9, 64, 65, 127, 128, 129, 1000, 4999, 16387]


@pytest.mark.parametrize("kkind,qkind", [("gauss", "gauss"), ("codes", "gauss"), ("subnormal", "wide"),
                                         ("codes", "wide"), ("gauss", "zero_heads"), ("subnormal", "tiny")])
def test_bounds_bracket_exact_scores(kkind, qkind):
    rng = np.random.default_rng([11, len(kkind), len(qkind)])
    keys = [keys_for(rng, kkind, L) for L in LENS]
    iq, iw = query_for(rng, qkind, len(LENS))
    layer, batch = gpu_layer(keys, 5)
    lo, hi = screen(layer, batch, iq, iw)
    widths = []
    for b, L in enumerate(LENS):
        nb = (L + 7) // 8
        exact = oracle.block_scores(iq[b], iw[b], keys[b])
        l, h = lo[b, :nb], hi[b, :nb]
        assert np.isfinite(l).all() and np.isfinite(h).all(), "seq %d: bound not formed" % b
        bad = np.nonzero(~((l <= exact) & (exact <= h)))[0]
        assert bad.size == 0, "seq %d block %d: %r not in [%r, %r]" % (b, bad[0], exact[bad[0]], l[bad[0]], h[bad[0]])
        assert (lo[b, nb:] == 12345.0).all() and (hi[b, nb:] == 12345.0).all()   # untouched past the row
        nz = np.abs(exact) > 0
        widths.append(((h - l)[nz] / np.abs(exact[nz])))
    w = np.concatenate(widths)
    if qkind in ("gauss", "zero_heads") and kkind == "gauss":
        assert np.median(w) < 1e-2, "screen bound too loose: median relative width %.3e" % np.median(w)


def full_select(layer, batch, iq, iw, k):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    B = iq.shape[0]
    ws = csa.workspace(B, 16, batch.max_seq_len, k)
    out = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    csa.indexer_full(layer, batch, dev(iq), dev(iw), k, out, cnt, ws)
    assert csa.check_device_error(ws)[0] == 0
    c = cnt.cpu().numpy()
    o = out.cpu().numpy()
    return [o[b, :c[b]] for b in range(B)]


@pytest.mark.parametrize("case", ["ties", "zero_weights", "constant_row", "non_finite", "wide"])
def test_screened_full_selection_matches_oracle(case):
    rng = np.random.default_rng([12, len(case)])
    lens = [3000, 777, 40000, 64]   # 5,000 blocks in the third: the sampled classification path
    k = 100
    iq, iw = synth.index_query(rng, len(lens))
    if case == "ties":           # every key identical: all scores tie, lowest ids win
        keys = [np.tile(keys_for(rng, "gauss", 1), (L, 1)) for L in lens]
    elif case == "zero_weights":
        keys = [keys_for(rng, "gauss", L) for L in lens]
        iw = np.zeros_like(iw)
    elif case == "constant_row":  # a few distinct key rows: many exact ties at every level
        base = keys_for(rng, "gauss", 5)
        keys = [base[rng.integers(0, 5, L)] for L in lens]
    elif case == "non_finite":   # an infinite query value in one head of two sequences
        keys = [keys_for(rng, "gauss", L) for L in lens]
        iq = iq.copy()
        iq[0, 0, 3] = 0x7F80
        iq[2, 5, 100] = 0xFF80
    else:
        keys = [keys_for(rng, "codes", L) for L in lens]
        iq, iw = query_for(rng, "wide", len(lens))
    layer, batch = gpu_layer(keys, 6)
    got = full_select(layer, batch, iq, iw, k)
    for b, L in enumerate(lens):
        exact = oracle.block_scores(iq[b], iw[b], keys[b])
        ref = oracle.topk(np.arange(len(exact), dtype=np.int32), exact, k)
        assert got[b].tolist() == ref.tolist(), "sequence %d (L=%d)" % (b, L)


def test_screened_equals_exhaustive_exact_scan():
    """csa_indexer_full (screened) against csa_indexer_block_scores + csa_topk_blocks on the same GPU
    data, 8 sequences of 40,000 positions, several k; and the oracle on two of them."""
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    rng = np.random.default_rng(13)
    lens = [40000] * 6 + [39993, 20001]
    keys = [keys_for(rng, "gauss", L) for L in lens]
    iq, iw = synth.index_query(rng, len(lens))
    layer, batch = gpu_layer(keys, 7)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    nb = (max(lens) + 7) // 8
    for k in (1, 512, 2048):
        got = full_select(layer, batch, iq, iw, k)
        ws = csa.workspace(len(lens), 16, batch.max_seq_len, k)
        sc = torch.zeros((len(lens), nb), device="cuda")
        csa.indexer_block_scores(layer, batch, dev(iq), dev(iw), sc, ws)
        out = torch.zeros((len(lens), k), dtype=torch.int32, device="cuda")
        cnt = torch.zeros(len(lens), dtype=torch.int32, device="cuda")
        csa.topk_blocks(batch, sc, k, out, cnt, ws)
        assert csa.check_device_error(ws)[0] == 0
        for b in range(len(lens)):
            assert got[b].tolist() == out[b, :cnt[b]].cpu().tolist(), "k=%d seq %d" % (k, b)
    for b in (0, 7):
        exact = oracle.block_scores(iq[b], iw[b], keys[b])
        assert got[b].tolist() == oracle.topk(np.arange(len(exact), dtype=np.int32), exact, 2048).tolist()


@pytest.mark.parametrize("layout", ["sampled_high", "sampled_low"])
def test_large_k_over_interleaved_magnitudes(layout):
    """5,000 blocks, k = 3,000, large-score and small-score blocks interleaved on a fixed stride (4,096
    of the blocks on one side, the rest on the other): the threshold bins of the lower bounds fall in
    a crowded part of the distribution and thousands of blocks are sure; the selection still equals
    the oracle's."""
    rng = np.random.default_rng([14, len(layout)])
    n, m, k = 5000, 4096, 3000
    sampled = np.zeros(n, bool)
    sampled[(np.arange(m) * n) // m] = True
    big = sampled if layout == "sampled_high" else ~sampled
    scale = np.where(big, 4.0, 0.25).astype(np.float32)
    g = synth.bf16_to_f32(synth.index_keys(rng, 8 * n)).reshape(n, 8, 128)
    keys = [oracle.e4m3_encode((g * scale[:, None, None]).reshape(8 * n, 128))]
    iq, iw = synth.index_query(rng, 1)
    layer, batch = gpu_layer(keys, 8)
    got = full_select(layer, batch, iq, iw, k)
    exact = oracle.block_scores(iq[0], iw[0], keys[0])
    assert got[0].tolist() == oracle.topk(np.arange(n, dtype=np.int32), exact, k).tolist()


def cancelling_keys(rng, n, jr=(1, 17), M_choices=(448.0, 240.0, 96.0, 26.0)):
    """Every position, in each 32-channel slice (one K=32 tensor-core step): 15 channels +M, 15
    channels -M (M per position and slice), at random places, and two residue channels of magnitude
    M 2^-j, j uniform in jr, random signs.  With a query constant over the slice, the large
    products cancel exactly and leave a residue from 2^-1 down to 2^-17 of the largest product."""
    keys = np.zeros((n, 128), np.float32)
    for s in range(4):
        M = rng.choice(np.array(M_choices, np.float32), size=n)
        sl = np.zeros((n, 32), np.float32)
        sl[:, :15] = M[:, None]
        sl[:, 15:30] = -M[:, None]
        j = rng.uniform(jr[0], jr[1], size=(n, 2))
        sl[:, 30:] = (M[:, None] * np.exp2(-j) * rng.choice([-1.0, 1.0], size=(n, 2))).astype(np.float32)
        perm = np.argsort(rng.random((n, 32)), axis=1)
        keys[:, 32 * s:32 * (s + 1)] = np.take_along_axis(sl, perm, axis=1)
    return oracle.e4m3_encode(keys)


def test_bounds_bracket_exact_scores_under_slice_cancellation():
    """The accumulation constant of the bound (the tensor core's fp32 sum of one K=32 step errs by at
    most 2^-14 of the sum of its product magnitudes) under the worst case for it: in every slice the
    large products cancel exactly and only residues far below them remain.  Head h reads only slice
    h mod 4 (its query is a constant there, zero elsewhere), so its bound is about 2^-14 x 32 |c| M and
    the residues land on both sides of it; a tensor core that dropped or truncated the residues by more
    than the constant would push exact scores out of their brackets.  The screened Top-K must also
    equal the oracle's."""
    rng = np.random.default_rng(21)
    lens = [1, 100, 1000, 4099]
    jr = [(1, 17), (6, 12), (9, 17), (1, 17)]
    keys = [cancelling_keys(rng, L, j) for L, j in zip(lens, jr)]
    B = len(lens)
    c = synth.bf16_to_f32(synth.bf16_bits(rng.uniform(0.5, 3.0, size=(B, 8)).astype(np.float32)))
    c *= rng.choice([-1.0, 1.0], size=(B, 8)).astype(np.float32)
    q = np.zeros((B, 8, 128), np.float32)
    for h in range(8):
        s = h % 4
        q[:, h, 32 * s:32 * (s + 1)] = c[:, h, None]
    iq = synth.bf16_bits(q)
    iw = rng.random((B, 8)).astype(np.float32)
    layer, batch = gpu_layer(keys, 9)
    lo, hi = screen(layer, batch, iq, iw)
    below = above = 0
    for b, L in enumerate(lens):
        nb = (L + 7) // 8
        exact = oracle.block_scores(iq[b], iw[b], keys[b])
        l, h = lo[b, :nb], hi[b, :nb]
        bad = np.nonzero(~((l <= exact) & (exact <= h)))[0]
        assert bad.size == 0, "seq %d block %d: %r not in [%r, %r]" % (b, bad[0], exact[bad[0]], l[bad[0]], h[bad[0]])
        half = (h - l) / 2
        below += int((exact < half).sum())
        above += int((exact > 4 * half).sum())
    # the residues straddle the bound: some blocks score below the bracket's half-width, some far above
    assert below > 0 and above > 0, (below, above)
    k = 40
    got = full_select(layer, batch, iq, iw, k)
    for b, L in enumerate(lens):
        exact = oracle.block_scores(iq[b], iw[b], keys[b])
        assert got[b].tolist() == oracle.topk(np.arange(len(exact), dtype=np.int32), exact, k).tolist()


@pytest.mark.parametrize("rows", [1, 3])
def test_long_sequence_of_few_distinct_keys(rows):
    """200,003 positions (25,001 blocks) whose keys take only `rows` distinct values: every block is
    uncertain or tied, each CTA of the selection holds more uncertain blocks than its shared-memory
    list, and the k-th score is shared by thousands of blocks, of which the lowest-numbered must be
    taken.  The selection must equal the oracle's Top-K."""
    rng = np.random.default_rng([15, rows])
    L, k = 200003, 3000
    base = keys_for(rng, "gauss", rows)
    keys = [base[rng.integers(0, rows, L)] if rows > 1 else np.tile(base, (L, 1)), keys_for(rng, "gauss", 999)]
    iq, iw = synth.index_query(rng, 2)
    layer, batch = gpu_layer(keys, 10)
    got = full_select(layer, batch, iq, iw, k)
    for b in range(2):
        exact = oracle.block_scores(iq[b], iw[b], keys[b])
        assert got[b].tolist() == oracle.topk(np.arange(len(exact), dtype=np.int32), exact, k).tolist(), b
