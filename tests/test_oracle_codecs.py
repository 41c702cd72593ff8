"""Pins for the oracle's element codecs and pack step, against what the pages and the public
format definitions fix.  The encoders are compared with two independent library codecs
(ml_dtypes for E2M1 and E4M3, torch for E4M3) and with closed-form error bounds."""
import json
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_sparse_kv_b200 import synth

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")))


def all_finite_bf16_as_f32():
    u = np.arange(1 << 16, dtype=np.uint32) << 16
    f = u.view(np.float32)
    return f[np.isfinite(f)]


def near_midpoints(points):
    """Each point and its float32 neighbours (1 and 2 ulps either side)."""
    p = np.asarray(points, np.float32)
    out = [p]
    for d in (1, 2):
        out.append(np.nextafter(p, np.float32(np.inf)))
        out.append(np.nextafter(p, np.float32(-np.inf)))
        p2 = p
        for _ in range(d):
            p2 = np.nextafter(p2, np.float32(np.inf))
        out.append(p2)
    x = np.concatenate(out)
    return np.concatenate([x, -x])


# ------------------------------------------------------------------------------------------------
# E2M1
# ------------------------------------------------------------------------------------------------
def test_e2m1_value_set():
    vals = oracle.e2m1_decode(np.arange(16, dtype=np.uint8))
    assert vals[:8].tolist() == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    assert (vals[8:] == -vals[:8]).all()
    assert np.signbit(vals[8])          # code 0x8 is negative zero
    assert vals.max() == GOLDEN["e2m1_max"]["value"]


def test_e2m1_decode_matches_ml_dtypes():
    codes = np.arange(16, dtype=np.uint8)
    ref = codes.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(oracle.e2m1_decode(codes), ref)


def test_e2m1_encode_matches_ml_dtypes():
    mids = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0]
    rng = np.random.default_rng(11)
    x = np.concatenate([all_finite_bf16_as_f32(), near_midpoints(mids),
                        rng.uniform(-8, 8, 200000).astype(np.float32),
                        np.array([0.0, -0.0, 1e-30, -1e-30, 1e30, -1e30], np.float32)])
    ref = x.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    got = oracle.e2m1_encode(x)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:8]], got[bad[:8]], ref[bad[:8]])


def test_e2m1_ties_round_to_even():
    x = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.25, -5.0], np.float32)
    assert oracle.e2m1_encode(x).tolist() == [0x0, 0x2, 0x2, 0x4, 0x4, 0x6, 0x6, 0x8, 0xE]


# ------------------------------------------------------------------------------------------------
# E4M3
# ------------------------------------------------------------------------------------------------
def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = oracle.e4m3_decode(codes)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan) and nan.sum() == 2
    assert np.array_equal(got[~nan], ref[~nan])
    assert np.nanmax(got) == GOLDEN["e4m3_max"]["value"]


def test_e4m3_encode_matches_torch_and_ml_dtypes_in_range():
    reps = oracle.e4m3_decode(np.arange(0x7F, dtype=np.uint8))
    mids = (reps[1:] + reps[:-1]) / 2
    rng = np.random.default_rng(12)
    x = np.concatenate([all_finite_bf16_as_f32(), near_midpoints(mids), near_midpoints(reps),
                        rng.uniform(-460, 460, 200000).astype(np.float32),
                        (rng.standard_normal(100000) * 1e-3).astype(np.float32)])
    x = x[np.abs(x) <= 464.0]          # beyond 464 torch and ml_dtypes overflow to NaN
    got = oracle.e4m3_encode(x)
    ref_t = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref_m = x.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ref_t, ref_m)
    bad = np.nonzero(got != ref_t)[0]
    assert bad.size == 0, (x[bad[:8]], got[bad[:8]], ref_t[bad[:8]])


def test_e4m3_saturates_to_finite_max():
    x = np.array([448.0, 449.0, 464.0, 465.0, 1e4, 1e38, -448.0, -500.0, -1e38], np.float32)
    assert oracle.e4m3_encode(x).tolist() == [0x7E] * 6 + [0xFE] * 3


def test_max_representable_magnitude_is_2688():
    top = oracle.e2m1_decode(np.array([0x7], np.uint8))[0] * oracle.e4m3_decode(
        np.array([0x7E], np.uint8))[0]
    assert top == GOLDEN["max_representable"]["value"] == 448 * 6
    # the largest value pack can produce: a group whose amax saturates the scale
    lat = np.zeros((1, 512), np.float32)
    lat[0, :16] = 3.0e38
    p = oracle.pack_tokens(synth.bf16_bits(lat), np.zeros((1, 128), np.uint16), with_swa=False)
    deq = oracle.dequant_main(p["codes"], p["scales"])
    assert deq.max() == 2688.0


# ------------------------------------------------------------------------------------------------
# Pack
# ------------------------------------------------------------------------------------------------
def pack_with_library_codecs(lat_bf16):
    """Independent restatement of the main-entry pack with ml_dtypes casts (valid while amax/6
    stays below 448, i.e. no scale saturation)."""
    x = synth.bf16_to_f32(lat_bf16).reshape(-1, 32, 16)
    a = np.abs(x).max(axis=-1)
    s = (a / np.float32(6.0)).astype(np.float32).astype(ml_dtypes.float8_e4m3fn)
    sd = s.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        y = (x / sd[..., None]).astype(np.float32)
    c = y.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    c = np.where(sd[..., None] == 0, 0, c).astype(np.uint8).reshape(-1, 256, 2)
    return (c[..., 0] | (c[..., 1] << 4)).astype(np.uint8), s.view(np.uint8)


@pytest.mark.parametrize("heavy", [False, True])
def test_pack_main_matches_library_restatement(heavy):
    rng = np.random.default_rng(21)
    lat = synth.latents(rng, np.arange(3000), heavy_tail=heavy)
    # add edge groups: all zero, negative zeros, tiny magnitudes that underflow the scale
    lat[0, :16] = 0
    lat[1, 16:32] = 0x8000
    lat[2, 32:48] = synth.bf16_bits(np.full(16, 1e-4, np.float32))
    lat[3, 48:64] = synth.bf16_bits(np.linspace(-6, 6, 16).astype(np.float32))
    p = oracle.pack_tokens(lat, np.zeros((lat.shape[0], 128), np.uint16), with_swa=False)
    codes, scales = pack_with_library_codecs(lat)
    assert np.array_equal(p["scales"], scales)
    assert np.array_equal(p["codes"], codes)


def e2m1_half_spacing(y):
    """Half the distance between neighbouring E2M1 magnitudes around |y| (|y| <= 6)."""
    a = np.abs(y)
    return np.where(a <= 2.0, 0.25, np.where(a <= 4.0, 0.5, 1.0))


def test_pack_roundtrip_error_bound():
    rng = np.random.default_rng(22)
    lat = synth.latents(rng, np.arange(4000), heavy_tail=True)
    p = oracle.pack_tokens(lat, np.zeros((lat.shape[0], 128), np.uint16), with_swa=False)
    x = synth.bf16_to_f32(lat).astype(np.float64).reshape(-1, 32, 16)
    xh = oracle.dequant_main(p["codes"], p["scales"]).reshape(-1, 32, 16)
    sd = oracle.e4m3_decode(p["scales"])[..., None]
    a = np.abs(x).max(axis=-1, keepdims=True)
    # the scale is E4M3(a/6): within E4M3's relative spacing (2^-4 either way) of a/6
    assert (np.abs(sd - a / 6) <= (a / 6) * 2.0 ** -4 + 2.0 ** -10).all()
    y = np.clip(np.abs(x) / np.where(sd == 0, 1, sd), 0, 6)
    bound = np.maximum(e2m1_half_spacing(y) * sd * (1 + 2.0 ** -20), np.abs(x) - 6 * sd)
    assert (np.abs(x - xh) <= bound + 1e-300).all()
    # the sign of every nonzero value survives
    nz = xh != 0
    assert (np.sign(xh[nz]) == np.sign(x[nz])).all()


def test_pack_special_groups():
    lat = np.zeros((2, 512), np.float32)
    lat[0, 16:32] = np.array([6, -6, 5, -5, 4, 3, 2.5, 1.75, 1.25, 0.75, 0.25, -0.1, 0, 1, 1.5, 2])
    lat[1, :] = -0.0
    p = oracle.pack_tokens(synth.bf16_bits(lat), np.zeros((2, 128), np.uint16))
    assert p["scales"][0, 0] == 0 and (p["codes"][0, :8] == 0).all()    # all-zero group
    assert p["scales"][0, 1] == 0x38                                       # 6/6 = 1.0
    nib = np.stack([p["codes"][0, 8:16] & 15, p["codes"][0, 8:16] >> 4], -1).reshape(-1)
    assert nib.tolist() == [0x7, 0xF, 0x6, 0xE, 0x6, 0x5, 0x4, 0x4, 0x2, 0x2, 0x0, 0x8, 0x0,
                            0x2, 0x3, 0x4]
    assert (p["scales"][1] == 0).all() and (p["codes"][1] == 0).all()      # scale 0 -> codes 0
    assert p["swa_scale"][1] == 0 and (p["swa"][1] == 0).all()


def test_swa_pack_bounds():
    rng = np.random.default_rng(23)
    lat = synth.latents(rng, np.arange(2000))
    p = oracle.pack_tokens(lat, np.zeros((lat.shape[0], 128), np.uint16))
    x = synth.bf16_to_f32(lat).astype(np.float64)
    a = np.abs(x).max(axis=1)
    assert np.array_equal(p["swa_scale"], (a.astype(np.float32) / np.float32(448)))
    u = oracle.dequant_swa(p["swa"], p["swa_scale"])
    s = p["swa_scale"].astype(np.float64)[:, None]
    # E4M3 keeps 3 mantissa bits: relative error <= 2^-4 for normals, absolute <= 2^-10 * s below
    err = np.abs(u - x)
    assert (err <= np.abs(x) * 2.0 ** -4 + s * 2.0 ** -10 + 1e-12).all()
    # the token's largest magnitude maps onto the top of E4M3's range
    top = np.abs(oracle.e4m3_decode(p["swa"])).max(axis=1)
    assert (np.abs(top - 448) <= 16).all()


def test_index_key_cast_matches_torch():
    rng = np.random.default_rng(24)
    key = synth.index_keys(rng, 3000)
    p = oracle.pack_tokens(np.zeros((3000, 512), np.uint16), key, with_swa=False)
    ref = torch.from_numpy(synth.bf16_to_f32(key)).to(torch.float8_e4m3fn).view(torch.uint8)
    assert np.array_equal(p["key8"], ref.numpy())
