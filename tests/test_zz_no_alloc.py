"""The allocation-free Full indexer (csa_indexer_full_noalloc), for callers that cannot provide device
memory: called through the C-ABI twice in a row, it must return exactly the Top-K sets of the
workspace entry point csa_indexer_full and of the oracle (the selected sets are bit-for-bit defined),
report a clean status, and refuse sizes beyond its fixed scratch array.  This file is collected last
on purpose."""
import numpy as np
import pytest

from fp4_compressed_sparse_kv_b200 import synth

from helpers import OracleSeq

pytestmark = pytest.mark.gpu


def test_noalloc_indexer_matches_workspace_indexer_twice():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa, workloads
    w = synth.Workload("noalloc", 3, [20001, 777, 131072], 16, 256, seed=[77])
    st = workloads.DecodeState(w)
    k = 256
    ref_b = torch.full((3, k), -1, dtype=torch.int32, device="cuda")
    ref_c = torch.zeros(3, dtype=torch.int32, device="cuda")
    csa.indexer_full(st.layers[0], st.batch, st.iq[0], st.iw[0], k, ref_b, ref_c, st.ws)
    assert csa.check_device_error(st.ws)[0] == 0
    for call in range(2):
        got_b = torch.full((3, k), -1, dtype=torch.int32, device="cuda")
        got_c = torch.zeros(3, dtype=torch.int32, device="cuda")
        status = torch.full((4,), -5, dtype=torch.int32, device="cuda")
        csa.indexer_full_noalloc(st.layers[0], st.batch, st.iq[0], st.iw[0], k, got_b, got_c,
                                 dev_status=status)
        torch.cuda.synchronize()
        assert int(status[0]) == 0, "call %d" % call
        assert torch.equal(got_c, ref_c), "call %d" % call
        for b in range(3):
            n = int(ref_c[b])
            assert torch.equal(got_b[b, :n], ref_b[b, :n]), "call %d seq %d" % (call, b)


def test_noalloc_indexer_matches_oracle_on_ragged_batch():
    """Ragged lengths (a partial last block, a sequence with fewer blocks than k, one of 50,000
    tokens): the selected sets equal the oracle's exact Top-K, on two calls in a row."""
    import torch
    from fp4_compressed_sparse_kv_b200 import csa, workloads
    lens = [50001, 333, 4099]
    k = 300
    w = synth.Workload("noalloc-ragged", len(lens), lens, 16, k, seed=[78])
    st = workloads.DecodeState(w)
    _, iq, iw = st.queries[0]
    ref = []
    for b, L in enumerate(lens):
        lat, key = workloads.seq_tokens(w, 0, b)
        ref.append(OracleSeq(lat, key, L).full(iq[b], iw[b], k))
    for call in range(2):
        got_b = torch.full((len(lens), k), -1, dtype=torch.int32, device="cuda")
        got_c = torch.zeros(len(lens), dtype=torch.int32, device="cuda")
        status = torch.full((4,), -5, dtype=torch.int32, device="cuda")
        csa.indexer_full_noalloc(st.layers[0], st.batch, st.iq[0], st.iw[0], k, got_b, got_c,
                                 dev_status=status)
        torch.cuda.synchronize()
        assert int(status[0]) == 0, "call %d" % call
        for b in range(len(lens)):
            n = int(got_c[b])
            assert got_b[b, :n].cpu().numpy().tolist() == ref[b].tolist(), "call %d seq %d" % (call, b)


def test_noalloc_indexer_rejects_oversized_calls():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    B, L = 64, 200000        # 64 * 25,000 blocks * 4 B > 4 MiB of scratch
    layer = csa.KVLayer(1, 1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    batch = csa.Batch(dev(np.full(B, L, np.int32)), dev(np.zeros((B, (L + 63) // 64), np.int32)),
                      dev(np.zeros(B, np.int32)), L)
    iq = torch.zeros((B, 8, 128), dtype=torch.bfloat16, device="cuda")
    iw = torch.zeros((B, 8), dtype=torch.float32, device="cuda")
    out = torch.zeros((B, 64), dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    with pytest.raises(csa.CsaError) as e:
        csa.indexer_full_noalloc(layer, batch, iq, iw, 64, out, cnt)
    assert e.value.status == 3
