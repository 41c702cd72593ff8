"""GPU parity of steps 2-4 on small and ragged batches: Full and Reindex Top-K sets bit-exact,
Reuse bytewise, attention within 2e-3 of max|out| per sequence, against the oracle, which packs
every sequence itself from the same seeded generators."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

from helpers import assert_attention_close, oracle_layer_from_tokens

pytestmark = pytest.mark.gpu


def make_state(seq_lens, H, k, k_r=None, modes=(0,), heavy=False, seed=7):
    from fp4_compressed_sparse_kv_b200 import workloads
    w = synth.Workload("test", len(seq_lens), list(seq_lens), H, k, k_r or max(1, k // 4), list(modes),
                       heavy_tail=heavy, seed=[seed])
    return workloads.DecodeState(w)


def oracle_seq(st, b, kv_layer=0):
    from fp4_compressed_sparse_kv_b200 import workloads
    L = st.w.seq_lens[b]
    lat, key = workloads.seq_tokens(st.w, kv_layer, b)
    layer, bt, _ = oracle_layer_from_tokens(lat, key, L)
    return layer, bt, L


def gpu_set(st, l, b):
    n = int(st.count[l][b].item())
    return st.blocks[l][b, :n].cpu().numpy()


@pytest.mark.parametrize("seq_lens,H,k", [
    ([4096], 16, 64),                         # the tiny single-layer workload's shape
    ([1, 7, 64, 1000, 5003], 64, 64),         # ragged: k >= nb for the short ones, partial blocks
    ([20000, 333, 131], 32, 200),
    ([9000, 9001], 128, 500),
])
def test_full_layer_matches_oracle(seq_lens, H, k):
    import torch
    st = make_state(seq_lens, H, k)
    st.step()
    torch.cuda.synchronize()
    st.check()
    q, iq, iw = st.queries[0]
    tau = oracle.default_tau()
    for b, L in enumerate(seq_lens):
        layer, bt, _ = oracle_seq(st, b)
        ref_set = oracle.select_full(layer, bt, L, iq[b], iw[b], k)
        got = gpu_set(st, 0, b)
        assert got.tolist() == ref_set.tolist(), "sequence %d (L=%d)" % (b, L)
        out, lse = oracle.attend(layer, bt, 0, L, q[b], tau, ref_set)
        assert_attention_close(st.out[0][b].cpu().numpy(), st.lse[0][b].cpu().numpy(), out, lse,
                               "seq %d L=%d" % (b, L))


def test_stack_modes_match_oracle():
    """[Full, Reindex, Reuse, Reuse, Full, Reindex]: Reindex searches only the last Full layer's
    pool, Reuse copies the previous set, Reindex/Reuse attend over the most recent Full layer's KV."""
    import torch
    modes = [0, 1, 2, 2, 0, 1]
    st = make_state([3000, 12345], 64, 256, k_r=40, modes=modes, seed=8)
    st.step()
    torch.cuda.synchronize()
    st.check()
    tau = oracle.default_tau()
    for b, L in enumerate(st.w.seq_lens):
        caches = [oracle_seq(st, b, f) for f in range(2)]
        sets = []
        for l, m in enumerate(modes):
            q, iq, iw = st.queries[l]
            layer, bt, _ = caches[st.kv_of[l]]
            if m == 0:
                s = oracle.select_full(layer, bt, L, iq[b], iw[b], 256)
            elif m == 1:
                s = oracle.select_reindex(layer, bt, L, iq[b], iw[b], sets[st.full_of[l]], 40)
                assert set(s.tolist()) <= set(sets[st.full_of[l]].tolist())
            else:
                s = oracle.select_reuse(sets[l - 1])
            sets.append(s)
            got = gpu_set(st, l, b)
            assert got.tolist() == s.tolist(), "layer %d seq %d" % (l, b)
            out, lse = oracle.attend(layer, bt, 0, L, q[b], tau, s)
            assert_attention_close(st.out[l][b].cpu().numpy(), st.lse[l][b].cpu().numpy(), out, lse,
                                   "layer %d seq %d" % (l, b))


def test_reuse_is_bytewise_copy():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    prev = torch.randint(0, 1 << 20, (3, 48), dtype=torch.int32, device="cuda")
    cnt = torch.tensor([48, 0, 17], dtype=torch.int32, device="cuda")
    out = torch.full((3, 48), -7, dtype=torch.int32, device="cuda")
    oc = torch.zeros(3, dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    csa.index_reuse(prev, cnt, out, oc, ws)
    assert csa.check_device_error(ws)[0] == 0
    assert oc.tolist() == [48, 0, 17]
    assert torch.equal(out[0], prev[0]) and torch.equal(out[2, :17], prev[2, :17])
    assert (out[1] == -7).all() and (out[2, 17:] == -7).all()


def test_device_metadata_errors_are_reported():
    """A page id out of range and a selected block past the sequence are recorded, not faulted."""
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    st = make_state([700], 16, 16)
    bt_bad = st.batch.block_table.clone()
    bt_bad[0, 3] = 10 ** 6
    bad = csa.Batch(st.batch.seq_len, bt_bad, st.batch.swa_row, st.batch.max_seq_len)
    blocks = torch.zeros((1, 16), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(1, dtype=torch.int32, device="cuda")
    csa.indexer_full(st.layers[0], bad, st.iq[0], st.iw[0], 16, blocks, cnt, st.ws)
    assert csa.check_device_error(st.ws)[0] == 5
    blocks[0, 0] = 5000                     # block 5000 >= ceil(700/8)
    cnt[0] = 1
    out = torch.zeros((1, 16, 512), device="cuda")
    lse = torch.zeros((1, 16), device="cuda")
    csa.sparse_decode_attn(st.layers[0], st.batch, st.q[0], csa.default_sm_scale(), blocks, cnt,
                           out, lse, st.ws)
    assert csa.check_device_error(st.ws)[0] == 5
    assert torch.isfinite(out).all()


def test_host_argument_checks():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    st = make_state([100], 16, 8)
    out = torch.zeros((1, 16, 512), device="cuda")
    lse = torch.zeros((1, 16), device="cuda")
    with pytest.raises(csa.CsaError) as e:   # H = 24 is not supported
        csa.sparse_decode_attn(st.layers[0], st.batch, torch.zeros((1, 24, 512), dtype=torch.bfloat16,
                               device="cuda"), 0.1, st.blocks[0], st.count[0], out, lse, st.ws)
    assert e.value.status == 2
    with pytest.raises(csa.CsaError) as e:   # workspace too small
        csa.indexer_full(st.layers[0], st.batch, st.iq[0], st.iw[0], 8, st.blocks[0], st.count[0],
                         st.ws[:300])
    assert e.value.status == 3
    with pytest.raises(ValueError):
        csa.indexer_full(st.layers[0], st.batch, st.iq[0].cpu(), st.iw[0], 8, st.blocks[0],
                         st.count[0], st.ws)
