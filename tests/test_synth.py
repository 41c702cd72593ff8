"""The input generators: determinism, shapes, and the pages' range argument (ailily.cc article
每个 token 只占 890 字节, section 三: unit-weight RMSNorm bounds the 512-channel latent's L2 norm by
sqrt(512) ~ 22.6 and RoPE keeps the norm, so every channel stays within 22.6)."""
import json
import math
import os

import numpy as np
import pytest

from fp4_compressed_sparse_kv_b200 import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


@pytest.mark.parametrize("heavy", [False, True])
def test_latent_range_bound(heavy):
    rng = np.random.default_rng(51)
    pos = rng.integers(0, 1 << 20, 20000)
    x = synth.bf16_to_f32(synth.latents(rng, pos, heavy_tail=heavy)).astype(np.float64)
    bound = math.sqrt(GOLDEN["latent_channels"]["value"])
    assert round(bound, 1) == GOLDEN["latent_abs_bound"]["value"]
    assert np.abs(x).max() <= bound * (1 + 2.0 ** -8)
    assert (np.linalg.norm(x, axis=1) <= bound * (1 + 2.0 ** -8)).all()
    # far below the largest FP4 x E4M3 magnitude
    assert np.abs(x).max() < GOLDEN["max_representable"]["value"] / 100


def test_rope_preserves_norm():
    rng = np.random.default_rng(52)
    x = synth.rms_norm(rng.standard_normal((100, 512), dtype=np.float32))
    y = synth.rope_last(x, np.arange(100) * 977)
    assert np.allclose(np.linalg.norm(x, axis=1), np.linalg.norm(y, axis=1), rtol=1e-6)
    assert np.array_equal(x[:, :448], y[:, :448])


def test_generators_are_deterministic():
    a = synth.latents(np.random.default_rng([1, 2]), np.arange(10))
    b = synth.latents(np.random.default_rng([1, 2]), np.arange(10))
    assert np.array_equal(a, b)
    w = synth.workload("mixed_serving")
    assert w.seq_lens == synth.workload("mixed_serving").seq_lens
    assert all(8192 <= L <= 262144 for L in w.seq_lens) and len(w.seq_lens) == 32


def test_bf16_rounding():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 3.0e38], np.float32)
    assert synth.bf16_to_f32(synth.bf16_bits(x)).tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5,
                                                               synth.bf16_to_f32(synth.bf16_bits(x))[4]]


def test_block_tables_are_a_partition():
    rng = np.random.default_rng(53)
    lens = [1, 64, 65, 1000]
    bt, n = synth.block_tables(rng, lens, extra_pages=2)
    used = np.concatenate([bt[b, :synth.pages_needed(L)] for b, L in enumerate(lens)])
    assert n == used.size + 2 and np.unique(used).size == used.size and used.max() < n
    assert (bt[0, 1:] == -1).all()
