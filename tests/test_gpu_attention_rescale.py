"""Attention parity when a head's running maximum jumps late: every head's query is a multiple of the
newest token's latent, so the window (the last entries the sequence's last split walks, after
selected blocks) holds scores far above the rest, and the O^T accumulated over the split's earlier
tiles must be rescaled.  The jump is ~11 log2 units (beyond the 2^8 growth the kernel tolerates
without rescaling, with the earlier entries still carrying weight) or ~33 (the newest token all but
alone).  Top-K 4,096 blocks over 148 splits gives each split three or four 64-entry tiles.  Against
the oracle: the Top-K set bit-exact, the attention within the same 2e-3 of max|out| as every
attention test."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

from helpers import assert_attention_close, oracle_layer_from_tokens

pytestmark = pytest.mark.gpu


def _dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is not None else t).cuda()


@pytest.mark.parametrize("n,c,H", [(70000, 0.35, 64), (70000, 1.0, 64), (70000, 0.35, 128)])
def test_late_maximum_forces_rescale(n, c, H):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    k = 4096
    rng = np.random.default_rng([n, H, int(c * 100)])
    lat = synth.latents(rng, np.arange(n))
    key = synth.index_keys(rng, n)
    layer_o, bt, _ = oracle_layer_from_tokens(lat, key, n)
    layer = csa.KVLayer(bt.shape[0], 1)
    ws = csa.workspace(1, H, n, k)
    pos = np.arange(n, dtype=np.int64)
    swa = np.where(pos >= n - 128, pos % 128, -1).astype(np.int32)
    csa.kv_pack_fp4(layer, _dev(lat, torch.bfloat16), _dev(key, torch.bfloat16), _dev(pos), _dev(swa), ws)
    newest = synth.bf16_to_f32(lat[n - 1])
    q = synth.bf16_bits(np.stack([c * newest + 0.05 * rng.standard_normal(512, dtype=np.float32)
                                  for _ in range(H)])[None])
    iq, iw = synth.index_query(rng, 1)
    batch = csa.Batch(_dev(np.array([n], np.int32)), _dev(bt[None].astype(np.int32)), _dev(np.array([0], np.int32)), n)
    blocks = torch.zeros((1, k), dtype=torch.int32, device="cuda")
    count = torch.zeros((1,), dtype=torch.int32, device="cuda")
    csa.indexer_full(layer, batch, _dev(iq, torch.bfloat16), _dev(iw), k, blocks, count, ws)
    out = torch.zeros((1, H, 512), dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, H), dtype=torch.float32, device="cuda")
    csa.sparse_decode_attn(layer, batch, _dev(q, torch.bfloat16), csa.default_sm_scale(), blocks, count, out, lse, ws)
    torch.cuda.synchronize()
    assert csa.check_device_error(ws)[0] == 0
    ref_set = oracle.select_full(layer_o, bt, n, iq[0], iw[0], k)
    assert blocks[0, :int(count[0])].cpu().numpy().tolist() == ref_set.tolist()
    o, l = oracle.attend(layer_o, bt, 0, n, q[0], oracle.default_tau(), ref_set)
    assert_attention_close(out[0].cpu().numpy(), lse[0].cpu().numpy(), o, l, "n=%d c=%.2f H=%d" % (n, c, H))
