"""CPU check of the Full indexer's screening bound (the formulas of the tensor-core screen in
csrc/screen.cu), independent of the GPU: the screen's approximate score is rebuilt in numpy under
the worst case the bound allows -- every tensor-core accumulator off by the full assumed relative
error 2^-14 of the sum of its product magnitudes, with the sign that hurts most -- and the oracle's
exact binary32 score must lie within the bound on every position.  Inputs: random E4M3 keys over all
finite codes (subnormals included), queries over many binades, mixed-sign weights, and keys built to
cancel against the query (q . k near 0, where ReLU switches).  The last test shows the check has
teeth: without its residual term the bound misses a crafted query."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

U = 2.0 ** -24
C_TC = 2.0 ** -14          # assumed tensor-core accumulation error, relative to sum |products|
ROUND_UP = 1.000001


def gamma(n):
    return n * U / (1 - n * U)


E4M3_FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)


def qterms(q):
    """Per head: power-of-two scale s, three E4M3 terms and the residual of q * 2^s (exact split)."""
    amax = np.abs(q).max(axis=1)
    s = np.zeros(8, np.int64)
    for h in range(8):
        if amax[h] > 0:
            _, e = np.frexp(np.float32(amax[h]))
            s[h] = 8 - e
    x = (q.astype(np.float64) * np.exp2(s)[:, None]).astype(np.float32)
    terms = []
    r = x.copy()
    for _ in range(3):
        c = oracle.e4m3_decode(oracle.e4m3_encode(r)).astype(np.float32)
        r = (r - c).astype(np.float32)          # exact (checked below)
        terms.append(c)
    assert np.array_equal(terms[0].astype(np.float64) + terms[1] + terms[2] + r, x.astype(np.float64))
    return s, terms, r


def screen_bounds(iq, iw, keys8, sign):
    """Approximate scores and bounds of every position, tensor-core error at its worst (sign +-1)."""
    q = synth.bf16_to_f32(iq).reshape(8, 128)
    w = np.asarray(iw, np.float32)
    s, terms, r = qterms(q)
    k = oracle.e4m3_decode(keys8).astype(np.float64)             # [n, 128]
    kmax = np.abs(k).max(axis=1)
    inv = np.exp2(-s.astype(np.float64))
    # screening constants (as the query-term kernel forms them)
    t1 = sum(np.abs(t.astype(np.float64)) for t in terms).sum(axis=1) * inv
    dl = np.abs(r.astype(np.float64)).sum(axis=1) * inv
    q1 = np.abs(q.astype(np.float64)).sum(axis=1)
    F = (C_TC + gamma(2) * (1 + C_TC)) * t1 + dl + gamma(19) * q1
    G = float(np.float32(np.sum(np.abs(w.astype(np.float64)) * F) * (1 + gamma(8)) * ROUND_UP))
    chain = float(np.float32(2 * gamma(8) * (1 + gamma(8)) * ROUND_UP))
    absl = float(np.float32(2.0 ** -100 * (1 + np.abs(w.astype(np.float64)).sum()) * 2))
    # per term: the exact dot product, then the worst accumulation error allowed, rounded to fp32
    D = []
    for t in terms:
        exact = k @ t.astype(np.float64).T                      # [n, 8]
        mag = np.abs(k) @ np.abs(t.astype(np.float64)).T
        D.append((exact + sign * C_TC * mag).astype(np.float32))
    n = keys8.shape[0]
    that = np.zeros(n, np.float32)
    wr = np.zeros(n, np.float64)
    for h in range(8):
        dh = ((D[0][:, h] + D[1][:, h]) + D[2][:, h]) * np.float32(inv[h])
        rh = np.maximum(dh, np.float32(0))
        that = (w[h].astype(np.float64) * rh + that).astype(np.float32)
        wr = wr + abs(float(w[h])) * rh.astype(np.float64)
    eps = kmax * G + chain * wr * ROUND_UP + absl
    return that.astype(np.float64), eps


def cancelling_keys(rng, iq, n):
    """Keys whose dot product with head 0 of the query nearly cancels: half the dims carry the
    query's signs, half the opposite, with E4M3 magnitudes near the query's."""
    q0 = synth.bf16_to_f32(iq).reshape(8, 128)[0]
    k = np.empty((n, 128), np.float32)
    for i in range(n):
        flip = rng.permutation(128) < 64
        k[i] = np.where(flip, -1.0, 1.0) * np.sign(q0) * np.abs(q0) * rng.uniform(0.9, 1.1, 128)
    return oracle.e4m3_encode(k)


@pytest.mark.parametrize("case", ["gauss", "codes", "wide", "cancel", "tiny"])
@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_exact_score_within_screen_bound(case, sign):
    rng = np.random.default_rng([21, len(case), int(sign > 0)])
    n = 3000
    iq, iw = synth.index_query(rng, 1)
    iq, iw = iq[0], iw[0]
    if case == "gauss":
        keys = oracle.e4m3_encode(synth.bf16_to_f32(synth.index_keys(rng, n)))
    elif case == "codes":
        keys = rng.choice(E4M3_FINITE, size=(n, 128))
    elif case == "wide":
        mag = np.exp2(rng.uniform(-30, 12, size=(8, 128))).astype(np.float32)
        iq = synth.bf16_bits(mag * rng.choice([-1.0, 1.0], size=(8, 128)).astype(np.float32))
        iw = rng.standard_normal(8).astype(np.float32)
        keys = rng.choice(E4M3_FINITE, size=(n, 128))
    elif case == "cancel":
        iw = np.array([1.0] + [0.0] * 7, np.float32)
        keys = cancelling_keys(rng, iq, n)
    else:
        iq = synth.bf16_bits(synth.bf16_to_f32(iq) * np.float32(2.0 ** -100))
        keys = oracle.e4m3_encode(synth.bf16_to_f32(synth.index_keys(rng, n)))
    exact = oracle.index_scores(iq, iw, keys).astype(np.float64)
    that, eps = screen_bounds(iq, iw, keys, sign)
    err = np.abs(exact - that)
    assert np.all(err <= eps), "max excess %.3e at %d" % ((err - eps).max(), int(np.argmax(err - eps)))


def test_bound_fails_without_the_residual_term():
    """The check above has teeth: dropping the residual term from the bound lets a query whose
    E4M3 split leaves a large residual (values far below the head's maximum) escape it."""
    rng = np.random.default_rng(22)
    q = np.full((8, 128), 9e-4, np.float32)  # below half the smallest E4M3 subnormal: every term is 0
    q[:, 0] = 200.0                          # one large value per head: the rest lands in the residual
    iq = synth.bf16_bits(q)
    iw = np.ones(8, np.float32)
    keys = oracle.e4m3_encode(np.abs(rng.standard_normal((2000, 128))).astype(np.float32))
    keys[:, 0] = 0                           # the large dim contributes nothing
    s, terms, r = qterms(synth.bf16_to_f32(iq).reshape(8, 128))
    exact = oracle.index_scores(iq, iw, keys).astype(np.float64)
    that, eps = screen_bounds(iq, iw, keys, 1.0)
    assert np.all(np.abs(exact - that) <= eps)
    k = oracle.e4m3_decode(keys).astype(np.float64)
    dl = (np.abs(r.astype(np.float64)).sum(axis=1) * np.exp2(-s.astype(np.float64)))
    without = eps - np.abs(k).max(axis=1) * np.sum(np.abs(iw) * dl) * (1 + gamma(8))
    assert np.any(np.abs(exact - that) > without)
