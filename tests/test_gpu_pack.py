"""GPU parity of step 1 (kv_pack_fp4): every byte of the FP4 codes, E4M3 scales, E4M3 indexer keys,
FP8 window entries and window scales must equal the oracle's, including exhaustive sweeps of the
E2M1 and E4M3 conversions over every finite bf16 input."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

pytestmark = pytest.mark.gpu


def run_pack(lat, key, swa=True, seed=0):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    n = lat.shape[0]
    rng = np.random.default_rng(seed)
    npages = (n + 63) // 64 + 3
    rows = (n + 127) // 128 + 1
    layer = csa.KVLayer(npages, rows)
    slots = rng.permutation(npages * 64)[:n].astype(np.int64)
    sw = (rng.permutation(rows * 128)[:n].astype(np.int32) if swa else None)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dev = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).view(dt) if dt else
                              torch.from_numpy(np.ascontiguousarray(a))).cuda()
    csa.kv_pack_fp4(layer, dev(lat, torch.bfloat16), dev(key, torch.bfloat16), dev(slots),
                    dev(sw) if swa else None, ws)
    st, _ = csa.check_device_error(ws)
    assert st == 0
    codes = layer.codes.view(-1, 256).cpu().numpy()[slots]
    scales = layer.scales.view(-1, 32).cpu().numpy()[slots]
    keys = layer.keys.view(-1, 128).cpu().numpy()[slots]
    out = dict(codes=codes, scales=scales, key8=keys)
    if swa:
        out["swa"] = layer.swa.view(-1, 512).cpu().numpy()[sw]
        out["swa_scale"] = layer.swa_scale.view(-1).cpu().numpy()[sw]
    return out


def assert_same(got, ref, keys):
    for k in keys:
        a, b = got[k], ref[k]
        if k == "swa_scale":
            a, b = a.view(np.uint32), b.view(np.uint32)
        bad = np.nonzero((a != b).reshape(a.shape[0], -1).any(axis=1))[0]
        assert bad.size == 0, "%s differs in %d tokens, first %s" % (k, bad.size, bad[:5])


@pytest.mark.parametrize("heavy,n", [(False, 3001), (True, 3001), (False, 6003)])
def test_pack_bit_exact_generated(heavy, n):
    """3,001 tokens take one token per warp; 6,003 (a ragged last warp) four tokens per warp."""
    rng = np.random.default_rng(60 + heavy + n)
    lat = synth.latents(rng, rng.integers(0, 1 << 20, n), heavy_tail=heavy)
    key = synth.index_keys(rng, n)
    got = run_pack(lat, key)
    ref = oracle.pack_tokens(lat, key)
    assert_same(got, ref, ["codes", "scales", "key8", "swa", "swa_scale"])


def test_pack_edge_groups():
    rng = np.random.default_rng(62)
    n = 64
    x = rng.standard_normal((n, 512)).astype(np.float32)
    x[0] = 0.0
    x[1] = -0.0
    x[2, :16] = 1e-6                      # scale underflows E4M3 -> codes 0
    x[3, :16] = 3.0e38                    # scale saturates to 448, codes saturate to 6
    x[4, :16] = np.array([6, -6, 5, -5, 4, 3, 2.5, 1.75, 1.25, 0.75, 0.25, -0.1, 0, 1, 1.5, 2])
    x[5] *= 1e-30                         # subnormal-range values
    x[6] *= 1e30
    x[7, ::2] = -0.0
    lat = synth.bf16_bits(x)
    key = synth.bf16_bits(rng.standard_normal((n, 128)).astype(np.float32) * 100)
    key[0] = 0x8000                       # negative zero keys
    got = run_pack(lat, key)
    ref = oracle.pack_tokens(lat, key)
    assert_same(got, ref, ["codes", "scales", "key8", "swa", "swa_scale"])


def finite_bf16():
    u = np.arange(1 << 16, dtype=np.uint32)
    f = (u << 16).view(np.float32)
    return u[np.isfinite(f)].astype(np.uint16)


def test_e4m3_conversion_sweep_all_bf16():
    """Every finite bf16 pattern through the indexer-key cast (E4M3, RNE, saturating)."""
    vals = finite_bf16()
    n = (vals.size + 127) // 128
    key = np.resize(vals, n * 128).reshape(n, 128)
    lat = np.zeros((n, 512), np.uint16)
    got = run_pack(lat, key, swa=False)
    ref = oracle.pack_tokens(lat, key, with_swa=False)
    assert_same(got, ref, ["key8"])


def test_e2m1_conversion_sweep_all_bf16_in_range():
    """Every finite bf16 value in [-6, 6] through the FP4 encoder: each group holds 6.0 (so the
    scale decodes to exactly 1.0) followed by 15 swept values."""
    vals = finite_bf16()
    f = synth.bf16_to_f32(vals)
    vals = vals[np.abs(f) <= 6.0]
    per_tok = 32 * 15
    n = (vals.size + per_tok - 1) // per_tok
    sw = np.resize(vals, n * per_tok).reshape(n, 32, 15)
    lat = np.concatenate([np.full((n, 32, 1), synth.bf16_bits(np.float32(6.0)), np.uint16), sw],
                         axis=2).reshape(n, 512)
    key = np.zeros((n, 128), np.uint16)
    got = run_pack(lat, key, swa=False)
    ref = oracle.pack_tokens(lat, key, with_swa=False)
    assert (ref["scales"] == 0x38).all()
    assert_same(got, ref, ["codes", "scales"])


def test_pack_rejects_bad_slot():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    layer = csa.KVLayer(2, 1)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    lat = torch.zeros((2, 512), dtype=torch.bfloat16, device="cuda")
    key = torch.zeros((2, 128), dtype=torch.bfloat16, device="cuda")
    slot = torch.tensor([5, 128], dtype=torch.int64, device="cuda")   # 128 is past 2 pages
    csa.kv_pack_fp4(layer, lat, key, slot, None, ws)
    st, detail = csa.check_device_error(ws)
    assert st == 5 and detail == 1
    assert csa.check_device_error(ws)[0] == 0          # cleared by the read
