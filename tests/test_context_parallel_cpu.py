"""Context-parallel decode of one sequence on CPU: two gloo ranks, each holding half of the positions,
run the library's host orchestration (context_parallel.full_layer: the candidate exchange, the global
Top-k of the concatenated candidates, the slice attention, the partial exchange and the merge) with
the compute steps done by the oracle.  Rank 0's result must equal the oracle's unsharded Full layer:
the same Top-k set, bit for bit, and the same attention within 1e-9 (both are float64 sums)."""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
from fp4_compressed_sparse_kv_b200 import context_parallel as cp
from fp4_compressed_sparse_kv_b200 import csa, synth, workloads

from helpers import oracle_layer_from_tokens

L, K, H = 20000, 300, 16


class OracleOps:
    """The compute steps of context_parallel on the oracle (host), with the CUDA ops' interface."""

    def __init__(self, slices_layer):
        self.layer = slices_layer   # shard -> oracle caches of its slice (identity pages, window row 0)

    def select_local(self, shard, iq, iw):
        lay = self.layer[shard.start]
        n = shard.end - shard.start
        keys = lay["keys"].reshape(-1, 128)[:n]
        S = oracle.block_scores(iq.numpy(), iw.numpy(), keys)
        blocks = oracle.topk(np.arange(S.size, dtype=np.int32), S, K)
        out_b = np.zeros((1, K), np.int32)
        out_s = np.zeros((1, K), np.float32)
        out_b[0, :blocks.size] = blocks
        out_s[0, :blocks.size] = S[blocks]
        return torch.from_numpy(out_b), torch.from_numpy(out_s), torch.tensor([blocks.size], dtype=torch.int32)

    def select_global(self, L_, ids, scores, counts, offsets):
        R = ids.shape[0]
        gid = np.concatenate([ids[r, 0, :int(counts[r, 0])].numpy() + int(offsets[r, 0]) for r in range(R)])
        gsc = np.concatenate([scores[r, 0, :int(counts[r, 0])].numpy() for r in range(R)])
        chosen = oracle.topk(gid.astype(np.int32), gsc.astype(np.float32), K)
        out = np.zeros((1, K), np.int32)
        out[0, :chosen.size] = chosen
        return torch.from_numpy(out), torch.tensor([chosen.size], dtype=torch.int32)

    def attend_local(self, shard, q, blocks, count, sm_scale):
        g = blocks[0, :int(count[0])].numpy()
        mine = g[(g >= shard.block_lo) & (g < shard.block_hi)] - shard.block_lo
        n = shard.end - shard.start
        lay = self.layer[shard.start]
        pe = oracle.positions_of_blocks(mine.astype(np.int32), n)
        codes = lay["codes"].reshape(-1, 256)[pe]
        scales = lay["scales"].reshape(-1, 32)[pe]
        if shard.holds_last:
            w = oracle.window_positions(shard.L) - shard.start
            swa, swa_scale = lay["swa"][0, (w + shard.start) % 128], lay["swa_scale"][0, (w + shard.start) % 128]
        else:
            swa, swa_scale = np.zeros((0, 512), np.uint8), np.zeros((0,), np.float32)
        if codes.shape[0] + swa.shape[0] == 0:
            return torch.zeros((1, H, 512), dtype=torch.float64), torch.full((1, H), -np.inf, dtype=torch.float64)
        out, lse = oracle.attention(q.numpy(), sm_scale, codes, scales, swa, swa_scale)
        return torch.from_numpy(out[None]), torch.from_numpy(lse[None])

    def merge(self, out_parts, lse_parts):
        lp = lse_parts.numpy()
        M = lp.max(axis=0)
        w = np.where(np.isfinite(lp), np.exp(lp - M), 0.0)
        den = w.sum(axis=0)
        out = (w[..., None] * out_parts.numpy()).sum(axis=0) / den[..., None]
        return torch.from_numpy(out), torch.from_numpy(M + np.log(den))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _problem():
    w = synth.Workload("cp-cpu", 1, [L], H, K, seed=[91])
    lat, key = workloads.seq_tokens(w, 0, 0)
    q, iq, iw = workloads.layer_queries(w, 0)
    return lat, key, q[0], iq[0], iw[0]


def _rank(rank, world, port, result_path):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lat, key, q, iq, iw = _problem()
        start, end = cp.page_aligned_slices(L, world)[rank]
        layer, _, _ = oracle_layer_from_tokens(lat[start:end], key[start:end], end - start, with_swa=False)
        if end == L:   # the window, from the whole sequence's last positions, in this slice's row 0
            wp = oracle.window_positions(L)
            ps = oracle.pack_tokens(lat[wp], key[wp], with_swa=True)
            layer["swa"][0, wp % 128] = ps["swa"]
            layer["swa_scale"][0, wp % 128] = ps["swa_scale"]
        npages = (end - start + 63) // 64
        shard = cp.Shard(None, start, end, L, torch.arange(npages, dtype=torch.int32), 0, device="cpu")
        ops = OracleOps({start: layer})
        out, lse, gb, gc = cp.full_layer(ops, cp.DistComm(), shard, torch.from_numpy(iq), torch.from_numpy(iw),
                                         torch.from_numpy(q), oracle.default_tau())
        if rank == 0:
            np.savez(result_path, out=out.numpy(), lse=lse.numpy(), blocks=gb[0, :int(gc[0])].numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_context_parallel_full_layer_equals_the_unsharded_oracle(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    res = str(tmp_path / "cp.npz")
    mp.start_processes(_rank, args=(2, port, res), nprocs=2, join=True, start_method="spawn")
    got = np.load(res)
    lat, key, q, iq, iw = _problem()
    layer, bt, _ = oracle_layer_from_tokens(lat, key, L)
    ref_set = oracle.select_full(layer, bt, L, iq, iw, K)
    assert got["blocks"].tolist() == ref_set.tolist()
    out, lse = oracle.attend(layer, bt, 0, L, q, oracle.default_tau(), ref_set)
    assert np.abs(got["out"][0] - out).max() <= 1e-9 * np.abs(out).max()
    assert np.abs(got["lse"][0] - lse).max() <= 1e-9


def test_page_aligned_slices_cover_the_sequence():
    for L_, R in [(20000, 2), (1 << 20, 4), (131, 2), (64 * 7 + 5, 3)]:
        sl = cp.page_aligned_slices(L_, R)
        assert sl[0][0] == 0 and sl[-1][1] == L_
        assert all(a < b for a, b in sl)
        assert all(sl[i][1] == sl[i + 1][0] for i in range(R - 1))
        assert all(a % 64 == 0 for a, _ in sl)
    with pytest.raises(ValueError):
        cp.page_aligned_slices(100, 3)
