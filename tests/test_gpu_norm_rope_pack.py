"""GPU parity of the pack from the pre-norm latent (csa_kv_norm_rope_pack_fp4): RMSNorm with the
caller's weight, RoPE on channels 448..511 with the caller's (cos, sin), bf16, then the FP4 / E4M3 /
FP8 pack.  Every byte of the codes, scales, keys, window entries and window scales must equal the
oracle's (its RMSNorm + RoPE step followed by its pack), on generated latents over six decades of
scale, all-zero tokens, negative weights, identity and quarter-turn rotations, and a ragged count."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

pytestmark = pytest.mark.gpu


def inputs(n, seed):
    rng = np.random.default_rng(seed)
    scale = np.exp(rng.uniform(np.log(1e-3), np.log(1e3), (n, 1)))
    raw = rng.standard_normal((n, 512)) * scale
    raw[:, rng.integers(0, 512, 3)] *= 40.0            # a few heavy channels
    raw[::97] = 0.0                                    # all-zero tokens
    lat = synth.bf16_bits(raw.astype(np.float32))
    w = rng.uniform(0.5, 1.5, 512).astype(np.float32)
    w[rng.integers(0, 512, 20)] *= -1.0
    ang = rng.uniform(-np.pi, np.pi, (n, 32))
    cs = np.stack([np.cos(ang), np.sin(ang)], -1).astype(np.float32)
    cs[1::11] = [1.0, 0.0]                             # identity
    cs[2::13] = [0.0, 1.0]                             # quarter turn
    key = synth.index_keys(rng, n)
    return lat, w, cs, key


def run(lat, w, cs, key, seed):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    n = lat.shape[0]
    rng = np.random.default_rng(seed)
    npages = (n + 63) // 64 + 3
    rows = (n + 127) // 128 + 1
    layer = csa.KVLayer(npages, rows)
    slots = rng.permutation(npages * 64)[:n].astype(np.int64)
    sw = rng.permutation(rows * 128)[:n].astype(np.int32)
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    dev = lambda a, dt=None: (torch.from_numpy(np.ascontiguousarray(a)).view(dt) if dt else
                              torch.from_numpy(np.ascontiguousarray(a))).cuda()
    csa.kv_norm_rope_pack_fp4(layer, dev(lat, torch.bfloat16), dev(w), dev(cs), dev(key, torch.bfloat16),
                              dev(slots), dev(sw), ws)
    assert csa.check_device_error(ws)[0] == 0
    return dict(codes=layer.codes.view(-1, 256).cpu().numpy()[slots],
                scales=layer.scales.view(-1, 32).cpu().numpy()[slots],
                key8=layer.keys.view(-1, 128).cpu().numpy()[slots],
                swa=layer.swa.view(-1, 512).cpu().numpy()[sw],
                swa_scale=layer.swa_scale.view(-1).cpu().numpy()[sw].view(np.uint32))


@pytest.mark.parametrize("n", [1, 3001])
def test_norm_rope_pack_bit_exact(n):
    lat, w, cs, key = inputs(n, 70 + n)
    got = run(lat, w, cs, key, 71 + n)
    normed = oracle.norm_rope(lat, w, cs)
    ref = oracle.pack_tokens(normed, key)
    ref["swa_scale"] = ref["swa_scale"].view(np.uint32)
    for k in ("codes", "scales", "key8", "swa", "swa_scale"):
        bad = np.nonzero((got[k] != ref[k]).reshape(n, -1).any(axis=1))[0]
        assert bad.size == 0, "%s differs in %d tokens, first %s" % (k, bad.size, bad[:5])
