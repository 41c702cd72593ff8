"""The persistent KV tier on the GPU: csa_kv_export's record equals the oracle's, byte for byte, into
device memory and into pinned host memory; csa_kv_import into other pages followed by the window
replay (csa_kv_pack_fp4 of the last tokens) restores caches whose bytes equal the oracle's and whose
decode result equals the oracle's; bad page ids, n = 0 and unpinned host pointers behave as the
header says."""
import ctypes

import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

from helpers import assert_attention_close

pytestmark = pytest.mark.gpu


def _dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is not None else t).cuda()


def _tokens(n, seed):
    rng = np.random.default_rng([seed, 77])
    return synth.latents(rng, np.arange(n), heavy_tail=True), synth.index_keys(rng, n)


def _oracle_layer(lat, key, bt, P, n, row, rows):
    p = oracle.pack_tokens(lat, key, with_swa=False)
    layer = dict(codes=np.zeros((P, 64, 256), np.uint8), scales=np.zeros((P, 64, 32), np.uint8),
                 keys=np.zeros((P, 64, 128), np.uint8), swa=np.zeros((rows, 128, 512), np.uint8),
                 swa_scale=np.zeros((rows, 128), np.float32))
    pos = np.arange(n)
    pages, offs = np.asarray(bt)[pos // 64], pos % 64
    layer["codes"][pages, offs] = p["codes"]
    layer["scales"][pages, offs] = p["scales"]
    layer["keys"][pages, offs] = p["key8"]
    w = oracle.window_positions(n)
    ps = oracle.pack_tokens(lat[w], key[w], with_swa=True)
    layer["swa"][row, w % 128] = ps["swa"]
    layer["swa_scale"][row, w % 128] = ps["swa_scale"]
    return layer


def _pack(layer, lat, key, bt, positions, row, ws):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    positions = np.asarray(positions, np.int64)
    slots = synth.slots_of(bt, positions)
    L = int(positions.max()) + 1 if positions.size else 0
    sw = np.where(positions >= L - 128, row * 128 + positions % 128, -1).astype(np.int32)
    csa.kv_pack_fp4(layer, _dev(lat[positions], torch.bfloat16), _dev(key[positions], torch.bfloat16),
                    _dev(slots), _dev(sw), ws)


@pytest.mark.parametrize("n", [1, 64, 777, 5000])
@pytest.mark.parametrize("where", ["device", "pinned"])
def test_export_is_the_oracle_record(n, where):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    lat, key = _tokens(n, n)
    rng = np.random.default_rng(n)
    bt, P = synth.block_tables(rng, [n], extra_pages=4)
    layer = csa.KVLayer(P, 2)
    ws = csa.workspace(1, 16, 64, 8)
    _pack(layer, lat, key, bt[0], np.arange(n), 1, ws)
    nbytes = csa.kv_record_bytes(n)
    assert nbytes == -(-n // 64) * 26624
    dst = (torch.full((nbytes,), 0xEE, dtype=torch.uint8, device="cuda") if where == "device"
           else torch.full((nbytes,), 0xEE, dtype=torch.uint8).pin_memory())
    csa.kv_export(layer, _dev(bt[0]), n, dst, ws)
    torch.cuda.synchronize()
    ref = oracle.persistent_record(_oracle_layer(lat, key, bt[0], P, n, 1, 2), bt[0], n)
    got = dst.cpu().numpy()
    # rows of the last page past n: the layer's zero-initialised bytes on both sides
    assert np.array_equal(got, ref)
    assert csa.check_device_error(ws)[0] == 0


@pytest.mark.parametrize("n,where", [(3000, "pinned"), (130, "device"), (100, "device")])
def test_import_and_window_replay_restore_the_caches(n, where):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    lat, key = _tokens(n, n + 1)
    rng = np.random.default_rng(n + 1)
    bt, P = synth.block_tables(rng, [n], extra_pages=2)
    src_layer = csa.KVLayer(P, 1)
    ws = csa.workspace(1, 16, n, 64)
    _pack(src_layer, lat, key, bt[0], np.arange(n), 0, ws)
    rec = (torch.empty((csa.kv_record_bytes(n),), dtype=torch.uint8, device="cuda") if where == "device"
           else torch.empty((csa.kv_record_bytes(n),), dtype=torch.uint8).pin_memory())
    csa.kv_export(src_layer, _dev(bt[0]), n, rec, ws)
    torch.cuda.synchronize()
    del src_layer
    # restore into a different layer: other page ids, another window row
    P2 = P + 7
    bt2 = np.random.default_rng(n + 2).permutation(P2)[:bt.shape[1]].astype(np.int32)
    dst_layer = csa.KVLayer(P2, 3)
    csa.kv_import(dst_layer, _dev(bt2), n, rec, ws)
    w = oracle.window_positions(n)
    _pack(dst_layer, lat, key, bt2, w, 2, ws)          # the bounded replay of the window
    torch.cuda.synchronize()
    ref = _oracle_layer(lat, key, bt2, P2, n, 2, 3)
    for f in ["codes", "scales", "keys"]:
        g = getattr(dst_layer, f).cpu().numpy()
        pos = np.arange(n)
        assert np.array_equal(g[bt2[pos // 64], pos % 64], ref[f][bt2[pos // 64], pos % 64]), f
    assert np.array_equal(dst_layer.swa[2].cpu().numpy()[w % 128], ref["swa"][2, w % 128])
    assert np.array_equal(dst_layer.swa_scale[2].cpu().numpy()[w % 128], ref["swa_scale"][2, w % 128])
    # one decode step on the restored caches equals the oracle's on its own
    H, k = 16, 40
    q = synth.query(rng, 1, H)
    iq, iw = synth.index_query(rng, 1)
    batch = csa.Batch(_dev(np.array([n], np.int32)), _dev(bt2[None]), _dev(np.array([2], np.int32)), n)
    blocks = torch.zeros((1, k), dtype=torch.int32, device="cuda")
    count = torch.zeros((1,), dtype=torch.int32, device="cuda")
    csa.indexer_full(dst_layer, batch, _dev(iq, torch.bfloat16), _dev(iw), k, blocks, count, ws)
    out = torch.zeros((1, H, 512), dtype=torch.float32, device="cuda")
    lse = torch.zeros((1, H), dtype=torch.float32, device="cuda")
    csa.sparse_decode_attn(dst_layer, batch, _dev(q, torch.bfloat16), csa.default_sm_scale(), blocks, count,
                           out, lse, ws)
    torch.cuda.synchronize()
    ref_set = oracle.select_full(ref, bt2, n, iq[0], iw[0], k)
    assert blocks[0, :int(count[0])].cpu().numpy().tolist() == ref_set.tolist()
    o, l = oracle.attend(ref, bt2, 2, n, q[0], oracle.default_tau(), ref_set)
    assert_attention_close(out[0].cpu().numpy(), lse[0].cpu().numpy(), o, l, "restored n=%d" % n)
    assert csa.check_device_error(ws)[0] == 0


def test_bad_page_is_reported_and_skipped():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    layer = csa.KVLayer(4, 1)
    layer.codes.fill_(3)
    ws = csa.workspace(1, 16, 64, 8)
    dst = torch.full((csa.kv_record_bytes(192),), 0x77, dtype=torch.uint8, device="cuda")
    csa.kv_export(layer, _dev(np.array([1, 9, 2], np.int32)), 192, dst, ws)
    st, detail = csa.check_device_error(ws)
    assert st == 5 and detail == 1
    d = dst.cpu().numpy().reshape(3, 26624)
    assert (d[1] == 0x77).all()            # the bad page's record untouched
    assert (d[0, :16384] == 3).all() and (d[2, :16384] == 3).all()


def test_zero_tokens_and_unpinned_host_memory():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    layer = csa.KVLayer(2, 1)
    ws = csa.workspace(1, 16, 64, 8)
    bt = _dev(np.array([0, 1], np.int32))
    dst = torch.zeros((16,), dtype=torch.uint8, device="cuda")
    csa.kv_export(layer, bt, 0, dst, ws)                 # a no-op
    assert csa.kv_record_bytes(0) == 0
    host = np.zeros(26624 + 16, np.uint8)
    addr = (host.ctypes.data + 15) // 16 * 16             # aligned, but pageable: refused before launch
    lc = layer.c()
    st = csa.lib().csa_kv_export(ctypes.byref(lc), bt.data_ptr(), 64, ctypes.c_void_p(addr), ws.data_ptr(),
                                 ws.numel(), None)
    assert st == 1
    with pytest.raises(ValueError):
        csa.kv_export(layer, bt, 64, torch.zeros((26624,), dtype=torch.uint8), ws)
    assert csa.check_device_error(ws)[0] == 0
