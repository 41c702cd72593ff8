"""GPU parity at the full workload sizes, in the launch configuration the benchmark times, checked
on sampled sequences that the oracle recomputes from the same seeds (its own packing, scoring,
Top-K and attention):

  decode_128k   B=8, L=131,072, H=64, Top-K 2,048 x 8
  stack20_256k  B=4, L=262,144, 20 layers [Full, Reindex, Reuse, Reuse] x 5, k_r = 512
  single_1m     B=1, L=1,048,576, Full + 3 Reindex, heavy-tailed latents
  mixed_serving 65,536-token prefill pack + B=32 ragged decode (L ~ U[8,192, 262,144])
"""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

from helpers import OracleSeq, assert_attention_close, pack_tokens_threaded

pytestmark = [pytest.mark.gpu, pytest.mark.slow]


def run_state(name):
    import torch
    from fp4_compressed_sparse_kv_b200 import workloads
    st = workloads.DecodeState(synth.workload(name))
    st.step()
    torch.cuda.synchronize()
    st.check()
    return st


def gpu_cache_rows(st, f, b):
    """The GPU's packed rows of sequence b of KV layer f, in position order."""
    L = st.w.seq_lens[b]
    slots = synth.slots_of(st.block_table_np[b], np.arange(L))
    lay = st.layers[f]
    return (lay.codes.view(-1, 256)[slots].cpu().numpy(), lay.scales.view(-1, 32)[slots].cpu().numpy(),
            lay.keys.view(-1, 128)[slots].cpu().numpy())


def check_sequence(st, b, layers, check_cache=True):
    from fp4_compressed_sparse_kv_b200 import workloads
    tau = oracle.default_tau()
    L = st.w.seq_lens[b]
    kvs = sorted({st.kv_of[l] for l in layers} | {st.kv_of[st.full_of[l]] for l in layers})
    seqs = {}
    for f in kvs:
        lat, key = workloads.seq_tokens(st.w, f, b)
        seqs[f] = OracleSeq(lat, key, L)
        if check_cache:
            c, s, k = gpu_cache_rows(st, f, b)
            assert np.array_equal(c, seqs[f].codes) and np.array_equal(s, seqs[f].scales)
            assert np.array_equal(k, seqs[f].key8)
    sets = {}
    worst = 0.0
    for l in sorted(layers):
        m = st.w.modes[l]
        q, iq, iw = st.queries[l]
        os_ = seqs[st.kv_of[l]]
        if m == 0:
            s = os_.full(iq[b], iw[b], st.layer_k[l])
        elif m == 1:
            fl = st.full_of[l]
            pool = sets[fl] if fl in sets else st.blocks[fl][b, :int(st.count[fl][b])].cpu().numpy()
            # the pool itself is checked where layer fl is sampled
            s = os_.reindex(iq[b], iw[b], pool, st.layer_k[l])
        else:
            s = sets[l - 1]
        sets[l] = s
        n = int(st.count[l][b].item())
        got = st.blocks[l][b, :n].cpu().numpy()
        assert got.tolist() == s.tolist(), "layer %d seq %d" % (l, b)
        out, lse = os_.attend(q[b], tau, s)
        worst = max(worst, assert_attention_close(st.out[l][b].cpu().numpy(), st.lse[l][b].cpu().numpy(),
                                                  out, lse, "layer %d seq %d" % (l, b)))
    return worst


def test_decode_128k():
    st = run_state("decode_128k")
    for b in (0, 5):
        check_sequence(st, b, [0])
    assert (st.count[0].cpu().numpy() == 2048).all()


def test_stack20_256k():
    st = run_state("stack20_256k")
    # layers 0-3 read KV layer 0; layers 16-19 read KV layer 4
    check_sequence(st, 2, [0, 1, 2, 3, 16, 17, 18, 19])


def test_single_1m():
    st = run_state("single_1m")
    check_sequence(st, 0, [0, 1, 2, 3])


def test_mixed_serving():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa, workloads
    w = synth.workload("mixed_serving")
    st = workloads.DecodeState(w)
    # (a) prefill chunk: 65,536 new tokens into the spare pages, its last 128 into the spare ring row
    rng = synth.rng_for(w, 0, 5000)
    n = w.prefill_tokens
    lat = synth.latents(rng, np.arange(n))
    key = synth.index_keys(rng, n)
    spare_row = int(np.setdiff1d(np.arange(st.num_rows), st.swa_row_np)[0])
    slots = (st.prefill_pages[np.arange(n) // 64].astype(np.int64) * 64 + np.arange(n) % 64)
    sw = np.where(np.arange(n) >= n - 128, spare_row * 128 + np.arange(n) % 128, -1).astype(np.int32)
    dev = lambda a, dt=None: (torch.from_numpy(a).view(dt) if dt else torch.from_numpy(a)).cuda()
    csa.kv_pack_fp4(st.layers[0], dev(lat, torch.bfloat16), dev(key, torch.bfloat16), dev(slots), dev(sw),
                    st.ws)
    # (b) ragged decode
    st.step()
    torch.cuda.synchronize()
    st.check()
    ref = pack_tokens_threaded(lat, key)
    lay = st.layers[0]
    assert np.array_equal(lay.codes.view(-1, 256)[slots].cpu().numpy(), ref["codes"])
    assert np.array_equal(lay.scales.view(-1, 32)[slots].cpu().numpy(), ref["scales"])
    assert np.array_equal(lay.keys.view(-1, 128)[slots].cpu().numpy(), ref["key8"])
    rs = oracle.pack_tokens(lat[-128:], key[-128:], with_swa=True)
    ring = sw[-128:]
    assert np.array_equal(lay.swa.view(-1, 512)[ring].cpu().numpy(), rs["swa"])
    # shortest and longest sequences
    lens = np.array(w.seq_lens)
    for b in (int(lens.argmin()), int(lens.argmax())):
        check_sequence(st, b, [0])
