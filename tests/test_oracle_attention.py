"""Pins for the oracle's sparse decode attention: when the Top-K covers every block it must equal
plain dense attention over all positions plus the window, computed here from library decoders
(ml_dtypes E2M1, torch E4M3) and scipy's softmax; closed forms for q = 0."""
import ml_dtypes
import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle
from fp4_compressed_sparse_kv_b200 import synth

from test_oracle_indexer import make_layer


def lib_dequant_main(codes, scales):
    nib = np.stack([codes & 15, codes >> 4], -1).reshape(codes.shape[0], 512).astype(np.uint8)
    v = nib.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = torch.from_numpy(np.ascontiguousarray(scales)).view(torch.float8_e4m3fn).double().numpy()
    return v * np.repeat(s, 16, axis=1)


def lib_dequant_swa(swa, swa_scale):
    u = torch.from_numpy(np.ascontiguousarray(swa)).view(torch.float8_e4m3fn).double().numpy()
    return u * swa_scale.astype(np.float64)[:, None]


def dense_reference(q_bf16, tau, vals):
    q = synth.bf16_to_f32(q_bf16).astype(np.float64).reshape(-1, 512)
    z = tau * (q @ vals.T)
    return softmax(z, axis=1) @ vals, logsumexp(z, axis=1)


@pytest.mark.parametrize("L,H", [(1, 4), (5, 2), (64, 16), (203, 8), (300, 4)])
def test_covering_topk_equals_dense_attention(L, H):
    rng = np.random.default_rng(41 + L)
    layer, bt, p = make_layer(rng, L)
    q = synth.query(rng, 1, H)[0]
    iq, iw = synth.index_query(rng, 1)
    nb = (L + 7) // 8
    blocks = oracle.select_full(layer, bt, L, iq[0], iw[0], nb + 5)
    assert blocks.tolist() == list(range(nb))
    tau = oracle.default_tau()
    out, lse = oracle.attend(layer, bt, 0, L, q, tau, blocks)
    w = oracle.window_positions(L)
    vals = np.concatenate([lib_dequant_main(p["codes"], p["scales"]),
                           lib_dequant_swa(p["swa"][w], p["swa_scale"][w])])
    ro, rl = dense_reference(q, tau, vals)
    assert np.allclose(out, ro, rtol=1e-11, atol=1e-12)
    assert np.allclose(lse, rl, rtol=1e-12, atol=1e-12)


def test_zero_query_gives_mean_of_all_values():
    rng = np.random.default_rng(42)
    L = 150
    layer, bt, p = make_layer(rng, L)
    blocks = np.array([0, 3, 7, 18], np.int32)   # block 18 holds positions 144..149 only
    q = np.zeros((3, 512), np.uint16)
    out, lse = oracle.attend(layer, bt, 0, L, q, 0.7, blocks)
    pe = oracle.positions_of_blocks(blocks, L)
    w = oracle.window_positions(L)
    vals = np.concatenate([lib_dequant_main(p["codes"][pe], p["scales"][pe]),
                           lib_dequant_swa(p["swa"][w], p["swa_scale"][w])])
    assert pe.size == 3 * 8 + 6 and vals.shape[0] == pe.size + 128
    assert np.allclose(out, vals.mean(axis=0)[None, :], rtol=1e-13, atol=1e-14)
    assert np.allclose(lse, np.log(vals.shape[0]), rtol=1e-14)


def test_single_position_counts_once_per_segment():
    rng = np.random.default_rng(43)
    layer, bt, p = make_layer(rng, 1)
    out, lse = oracle.attend(layer, bt, 0, 1, np.zeros((2, 512), np.uint16), 1.0,
                             np.array([0], np.int32))
    v0 = lib_dequant_main(p["codes"][:1], p["scales"][:1])[0]
    u0 = lib_dequant_swa(p["swa"][:1], p["swa_scale"][:1])[0]
    assert np.array_equal(out[0], (v0 + u0) / 2) or np.allclose(out[0], (v0 + u0) / 2, rtol=1e-15)
    assert np.allclose(lse, np.log(2.0))


def test_sharp_query_selects_one_entry():
    rng = np.random.default_rng(44)
    L = 200                       # position 9 lies outside the window 72..199
    layer, bt, p = make_layer(rng, L)
    v = lib_dequant_main(p["codes"], p["scales"])
    target = 9
    q = synth.bf16_bits((v[target] * 8).astype(np.float32)[None, :])
    out, _ = oracle.attend(layer, bt, 0, L, q, 1.0, np.array([1], np.int32))   # positions 8..15
    assert np.allclose(out[0], v[target], atol=1e-6 * np.abs(v[target]).max())
