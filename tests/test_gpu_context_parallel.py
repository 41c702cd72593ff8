"""Context-parallel decode on one GPU: the exchange kernels against their definitions, and a long
sequence split into page-aligned slices (each in its own caches, run in turn in one process) whose
Full-layer result must equal the oracle's unsharded one: the Top-k set bit for bit and the attention
within 2e-3 of max|out|."""
import numpy as np
import pytest

import oracle
from fp4_compressed_sparse_kv_b200 import synth

from helpers import OracleSeq, assert_attention_close

pytestmark = pytest.mark.gpu


def _dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    return (t.view(dtype) if dtype is not None else t).cuda()


def test_candidates_concat_and_shard_blocks():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    rng = np.random.default_rng(5)
    R, B, cap = 3, 2, 40
    counts = rng.integers(0, cap + 1, size=(R, B)).astype(np.int32)
    counts[1, 0] = 0
    ids = np.sort(rng.integers(0, 1000, size=(R, B, cap)), axis=2).astype(np.int32)
    scores = rng.standard_normal((R, B, cap)).astype(np.float32)
    offsets = (np.arange(R)[:, None] * 1000 + np.zeros((1, B), np.int64)).astype(np.int32)
    ws = csa.workspace(B, 16, 64, 8)
    out_ids = torch.zeros((B, R * cap), dtype=torch.int32, device="cuda")
    out_sc = torch.zeros((B, R * cap), dtype=torch.float32, device="cuda")
    out_n = torch.zeros((B,), dtype=torch.int32, device="cuda")
    csa.candidates_concat(_dev(ids), _dev(scores), _dev(counts), _dev(offsets), out_ids, out_sc, out_n, ws)
    for b in range(B):
        ref_i = np.concatenate([ids[r, b, :counts[r, b]] + offsets[r, b] for r in range(R)])
        ref_s = np.concatenate([scores[r, b, :counts[r, b]] for r in range(R)])
        n = int(out_n[b])
        assert n == ref_i.size
        assert out_ids[b, :n].cpu().numpy().tolist() == ref_i.tolist()
        assert np.array_equal(out_sc[b, :n].cpu().numpy(), ref_s)
    # the part of a set in [lo, hi), rebased
    blocks = np.sort(rng.choice(5000, size=(B, 64), replace=True), axis=1).astype(np.int32)
    count = np.array([64, 17], np.int32)
    lo, hi = np.array([1000, 0], np.int32), np.array([3000, 2500], np.int32)
    ob = torch.zeros((B, 64), dtype=torch.int32, device="cuda")
    oc = torch.zeros((B,), dtype=torch.int32, device="cuda")
    csa.shard_blocks(_dev(blocks), _dev(count), _dev(lo), _dev(hi), ob, oc, ws)
    for b in range(B):
        v = blocks[b, :count[b]]
        ref = v[(v >= lo[b]) & (v < hi[b])] - lo[b]
        assert int(oc[b]) == ref.size
        assert ob[b, :ref.size].cpu().numpy().tolist() == ref.tolist()
    assert csa.check_device_error(ws)[0] == 0


def test_attn_merge_is_the_log_sum_exp_merge():
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    rng = np.random.default_rng(6)
    R, B, H = 4, 3, 16
    out_p = rng.standard_normal((R, B, H, 512)).astype(np.float32)
    lse_p = (rng.standard_normal((R, B, H)) * 5).astype(np.float32)
    lse_p[2, 1, :] = -np.inf          # an empty part
    lse_p[:, 2, 3] = -np.inf          # every part empty for one head
    out = torch.zeros((B, H, 512), dtype=torch.float32, device="cuda")
    lse = torch.zeros((B, H), dtype=torch.float32, device="cuda")
    csa.attn_merge(_dev(out_p), _dev(lse_p), out, lse)
    lp = lse_p.astype(np.float64)
    M = np.max(lp, axis=0)
    with np.errstate(invalid="ignore", divide="ignore"):
        w = np.where(np.isfinite(lp), np.exp(lp - M), 0.0)
        den = w.sum(axis=0)
        ref = (w[..., None] * out_p).sum(axis=0) / den[..., None]
        ref_lse = M + np.log(den)
    ref[2, 3] = 0.0
    got = out.cpu().numpy()
    assert np.abs(got - ref).max() <= 1e-5 * np.abs(ref).max()
    g_lse = lse.cpu().numpy()
    assert g_lse[2, 3] == -np.inf
    mask = np.isfinite(ref_lse)
    assert np.abs(g_lse[mask] - ref_lse[mask]).max() <= 1e-5


def _pack_slice(lat, key, start, end, L):
    """One slice's own caches (identity pages), with the window in ring row 0 if it holds the end."""
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    n = end - start
    npages = (n + 63) // 64
    layer = csa.KVLayer(npages, 1)
    ws = csa.workspace(1, 16, 64, 8)
    for c0 in range(0, n, 1 << 16):
        c1 = min(n, c0 + (1 << 16))
        pos = np.arange(start + c0, start + c1)
        slots = (pos - start).astype(np.int64)
        sw = np.where(pos >= L - 128, pos % 128, -1).astype(np.int32) if end == L else np.full(pos.size, -1, np.int32)
        csa.kv_pack_fp4(layer, _dev(lat[pos], torch.bfloat16), _dev(key[pos], torch.bfloat16),
                        _dev(slots), _dev(sw), ws)
    return layer, torch.arange(npages, dtype=torch.int32)


@pytest.mark.slow
@pytest.mark.parametrize("R", [4])
def test_sharded_long_sequence_equals_the_oracle(R):
    """The 1,048,576-token single sequence (heavy-tailed latents, 64 heads, Top-K 2,048) in R slices."""
    import torch
    from fp4_compressed_sparse_kv_b200 import context_parallel as cp
    from fp4_compressed_sparse_kv_b200 import workloads
    w = synth.workload("single_1m")
    L, k = w.seq_lens[0], w.topk
    lat, key = workloads.seq_tokens(w, 0, 0)
    q, iq, iw = workloads.layer_queries(w, 0)
    shards = []
    for start, end in cp.page_aligned_slices(L, R):
        layer, bt = _pack_slice(lat, key, start, end, L)
        shards.append(cp.Shard(layer, start, end, L, bt, 0))
    ops = cp.CudaOps(w.heads, k)
    out, lse, gb, gc = cp.full_layer_all_slices(ops, shards, _dev(iq[:1], torch.bfloat16), _dev(iw[:1]),
                                                _dev(q[:1], torch.bfloat16))
    torch.cuda.synchronize()
    got = gb[0, :int(gc[0])].cpu().numpy()
    os_ = OracleSeq(lat, key, L)
    ref = os_.full(iq[0], iw[0], k)
    assert got.tolist() == ref.tolist()
    out_ref, lse_ref = os_.attend(q[0], oracle.default_tau(), ref)
    assert_attention_close(out[0].cpu().numpy(), lse[0].cpu().numpy(), out_ref, lse_ref, "sharded 1M, R=%d" % R)
    for ws in ops._ws.values():
        assert csa_ok(ws)


def csa_ok(ws):
    from fp4_compressed_sparse_kv_b200 import csa
    return csa.check_device_error(ws)[0] == 0
