"""Pins of the oracle's RMSNorm + RoPE step (before the pack): closed forms (a zero latent stays zero;
a constant latent normalises to a / sqrt(a^2 + 1e-6)), the exact effect of a quarter turn on every
rotated pair, agreement with a float64 evaluation of the formula within one bf16 rounding, with the
input generator's RMSNorm + RoPE within that bound too, and norm preservation.  A dropped epsilon, a
wrong mean divisor, a missing weight, a wrong rotation sign or a shifted pair index fails one of them."""
import numpy as np

import oracle
from fp4_compressed_sparse_kv_b200 import synth


def identity_cs(n):
    cs = np.zeros((n, 32, 2), np.float32)
    cs[..., 0] = 1.0
    return cs


def f64_reference(x_bf16, w, cs):
    v = synth.bf16_to_f32(x_bf16).astype(np.float64)
    r = 1.0 / np.sqrt(np.mean(v * v, axis=1, keepdims=True) + 1e-6)
    y = v * r * w.astype(np.float64)[None, :]
    a = y[:, 448::2].copy()
    b = y[:, 449::2].copy()
    c = cs[..., 0].astype(np.float64)
    s = cs[..., 1].astype(np.float64)
    y[:, 448::2] = a * c - b * s
    y[:, 449::2] = a * s + b * c
    return y


def bf16_ulp(v):
    """Spacing of bf16 numbers at |v| (for normal values)."""
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0 ** -126)))
    return np.exp2(e - 7)


def test_zero_latent_stays_zero():
    x = np.zeros((3, 512), np.uint16)
    out = oracle.norm_rope(x, np.ones(512, np.float32), identity_cs(3))
    assert (out == 0).all()


def test_constant_latent_closed_form():
    for a in (1.0, 0.25, 3.0, 1e-3):
        x = synth.bf16_bits(np.full((1, 512), a, np.float32))
        av = float(synth.bf16_to_f32(x)[0, 0])
        out = synth.bf16_to_f32(oracle.norm_rope(x, np.ones(512, np.float32), identity_cs(1)))[0]
        want = av / np.sqrt(av * av + 1e-6)
        assert np.all(np.abs(out - want) <= bf16_ulp(want)), (a, out[:3], want)


def test_quarter_turn_swaps_and_negates_each_pair():
    rng = np.random.default_rng(31)
    x = synth.bf16_bits(rng.standard_normal((4, 512)).astype(np.float32))
    w = rng.uniform(0.5, 1.5, 512).astype(np.float32)
    base = oracle.norm_rope(x, w, identity_cs(4))
    cs = np.zeros((4, 32, 2), np.float32)
    cs[..., 1] = 1.0                                   # cos 0, sin 1: (a, b) -> (-b, a)
    turned = oracle.norm_rope(x, w, cs)
    assert np.array_equal(turned[:, :448], base[:, :448])
    assert np.array_equal(turned[:, 448::2], base[:, 449::2] ^ np.uint16(0x8000))
    assert np.array_equal(turned[:, 449::2], base[:, 448::2])


def test_matches_float64_within_one_bf16_rounding():
    rng = np.random.default_rng(32)
    n = 64
    x = synth.bf16_bits((rng.standard_normal((n, 512)) * rng.uniform(0.01, 30, (n, 1))).astype(np.float32))
    w = rng.uniform(-2, 2, 512).astype(np.float32)
    ang = rng.uniform(-np.pi, np.pi, (n, 32))
    cs = np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32)
    got = synth.bf16_to_f32(oracle.norm_rope(x, w, cs)).astype(np.float64)
    ref = f64_reference(x, w, cs)
    # binary32 steps add a few 2^-24 relative errors, the bf16 rounding half an ulp: one ulp covers both
    assert np.all(np.abs(got - ref) <= bf16_ulp(ref) + 1e-30)


def test_agrees_with_the_input_generator():
    """The generator normalises with unit weight and rotates by pos * 10000^(-2i/64); given the same
    angles rounded to binary32, the oracle's step lands within one bf16 rounding of it."""
    rng = np.random.default_rng(33)
    n = 32
    pos = rng.integers(0, 200000, n)
    raw = synth.bf16_bits(rng.standard_normal((n, 512)).astype(np.float32))
    gen = synth.rope_last(synth.rms_norm(synth.bf16_to_f32(raw)), pos).astype(np.float64)
    i = np.arange(32, dtype=np.float64)
    ang = pos[:, None].astype(np.float64) * 10000.0 ** (-2.0 * i / 64)
    cs = np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32)
    got = synth.bf16_to_f32(oracle.norm_rope(raw, np.ones(512, np.float32), cs)).astype(np.float64)
    # one bf16 rounding, plus binary32-level differences (the generator divides, rounds its angles
    # differently and rotates in float64) that matter only where a rotated pair nearly cancels
    assert np.all(np.abs(got - gen) <= bf16_ulp(gen) + 1e-5)


def test_unit_weight_gives_unit_rms():
    rng = np.random.default_rng(34)
    x = synth.bf16_bits((rng.standard_normal((16, 512)) * 7).astype(np.float32))
    ang = rng.uniform(-3, 3, (16, 32))
    cs = np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32)
    out = synth.bf16_to_f32(oracle.norm_rope(x, np.ones(512, np.float32), cs)).astype(np.float64)
    rms = np.sqrt(np.mean(out * out, axis=1))
    assert np.all(np.abs(rms - 1.0) < 4e-3)
