"""CPU check of the Full indexer's classification rule (the thresholds of the histogram passes in
csrc/screen.cu), on arbitrary valid bounds: T is the k-th largest lower-bound key with its low 8 bits
cleared, located through two 12-bit histogram levels; U is (that key with its low 8 bits set) plus
the widest interval, rounded up, or the largest key when some bound is not finite.  For every case,
with exact scores drawn anywhere inside their bounds, the blocks classed sure must all belong to the
exact Top-K (larger score first, lower id on ties), and every block of the exact Top-K must be sure
or uncertain.  Cases include massive ties, negative scores, intervals of wildly different widths,
bounds that differ only in low bits, and blocks without bounds (lower -NaN, upper +NaN)."""
import numpy as np
import pytest

import oracle


def order_key(f):
    u = np.asarray(f, np.float32).view(np.uint32).copy()
    u[u == 0x80000000] = 0
    neg = (u & 0x80000000) != 0
    return np.where(neg, ~u, u | 0x80000000).astype(np.uint32)


def key_to_float(k):
    k = np.uint32(k)
    u = (k & np.uint32(0x7FFFFFFF)) if (k & np.uint32(0x80000000)) else ~k
    return np.array([u], np.uint32).view(np.float32)[0]


def round_up_f32(x):
    """The smallest binary32 value >= the float64 x."""
    f = np.float32(x)
    if np.isfinite(x) and float(f) < x:
        f = np.nextafter(f, np.float32(np.inf))
    return np.float32(f)


def rank_bin(hist, rank):
    """Bin (of 4,096) holding the rank-th largest element and its rank inside the bin."""
    run = 0
    for b in range(4095, -1, -1):
        if run < rank <= run + hist[b]:
            return b, rank - run
        run += hist[b]
    return 0, 1


def classify(lo, hi, k):
    lk, hk = order_key(lo), order_key(hi)
    h1 = np.bincount(lk >> 20, minlength=4096)
    bin1, r1 = rank_bin(h1, k)
    in1 = (lk >> 20) == bin1
    h2 = np.bincount((lk[in1] >> 8) & 0xFFF, minlength=4096)
    bin2, _ = rank_bin(h2, r1)
    T = np.uint32((bin1 << 20) | (bin2 << 8))
    with np.errstate(invalid="ignore", over="ignore"):
        w = hi.astype(np.float64) - lo.astype(np.float64)   # exact for these inputs
    if not np.all(np.isfinite(w)):
        U = np.uint32(0xFFFFFFFF)                             # some bound is not finite: nothing is sure
    else:
        wmax = round_up_f32(float(w.max()))
        top = float(key_to_float(T | np.uint32(0xFF)))
        U = order_key(np.float32(round_up_f32(top + float(wmax))))[()]
    poss = hk >= T
    sure = poss & (lk > U)
    return sure, poss & ~sure


def check(lo, hi, scores, k):
    n = len(lo)
    sure, unc = classify(lo, hi, k)
    top = oracle.topk(np.arange(n, dtype=np.int32), scores.astype(np.float32), k)
    in_top = np.zeros(n, bool)
    in_top[top] = True
    assert not np.any(sure & ~in_top), "a sure block is outside the exact Top-K"
    assert not np.any(in_top & ~(sure | unc)), "an exact Top-K block was classed out"
    return sure.sum(), unc.sum()


def draw_inside(rng, lo, hi):
    t = rng.random(len(lo))
    s = lo.astype(np.float64) + t * (hi.astype(np.float64) - lo.astype(np.float64))
    s = np.clip(s.astype(np.float32), lo, hi)
    pick = rng.random(len(lo))
    s = np.where(pick < 0.1, lo, np.where(pick > 0.9, hi, s))   # endpoints too
    return s.astype(np.float32)


@pytest.mark.parametrize("seed", range(12))
def test_random_bounds(seed):
    rng = np.random.default_rng([41, seed])
    n = int(rng.integers(300, 6000))
    k = int(rng.integers(1, n))
    mid = (rng.standard_normal(n) * 10 ** rng.uniform(-3, 3)).astype(np.float32)
    width = np.abs(rng.standard_normal(n)).astype(np.float32) * np.float32(10 ** rng.uniform(-6, 0))
    if seed % 3 == 0:
        width[rng.random(n) < 0.01] *= 1000       # a few very wide intervals
    lo = (mid - width).astype(np.float32)
    hi = (mid + width).astype(np.float32)
    for _ in range(5):
        check(lo, hi, draw_inside(rng, lo, hi), k)


def test_massive_ties_and_low_bit_differences():
    rng = np.random.default_rng(42)
    n, k = 5000, 2048
    base = np.float32(3.0)
    lo = np.full(n, base, np.float32)
    hi = lo.copy()
    check(lo, hi, lo.copy(), k)                    # every score equal: lowest ids win
    u = base.view(np.uint32) + rng.integers(0, 300, n).astype(np.uint32)   # differ in the low 9 bits
    lo = u.view(np.float32)
    hi = (u + 3).astype(np.uint32).view(np.float32)
    for _ in range(5):
        check(lo, hi, draw_inside(rng, lo, hi), k)


def test_negative_scores_and_blocks_without_bounds():
    rng = np.random.default_rng(43)
    n, k = 3000, 500
    mid = -np.abs(rng.standard_normal(n)).astype(np.float32) * 5
    lo = (mid - 0.01).astype(np.float32)
    hi = (mid + 0.01).astype(np.float32)
    nob = rng.random(n) < 0.05
    lo_s, hi_s = lo.copy(), hi.copy()
    lo_s[nob] = np.array([0xFFFFFFFF], np.uint32).view(np.float32)[0]    # -NaN
    hi_s[nob] = np.array([0x7FFFFFFF], np.uint32).view(np.float32)[0]    # +NaN
    for _ in range(5):
        s = draw_inside(rng, lo, hi)
        s[nob] = rng.uniform(-20, 20, nob.sum()).astype(np.float32)     # anything at all
        check(lo_s, hi_s, s, k)


def test_tight_bounds_leave_few_uncertain():
    """The rule is also efficient when the bounds are tight: at the benchmark's shape (16,384 blocks,
    k = 2,048, relative widths near 1e-3) only a small band is uncertain."""
    rng = np.random.default_rng(44)
    n, k = 16384, 2048
    mid = np.abs(rng.standard_normal(n)).astype(np.float32) * 10 + 5
    lo = (mid * (1 - 1e-3)).astype(np.float32)
    hi = (mid * (1 + 1e-3)).astype(np.float32)
    n_sure, n_unc = check(lo, hi, draw_inside(rng, lo, hi), k)
    assert n_unc < 400 and n_sure > 1800
