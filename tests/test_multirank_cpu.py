"""Multi-rank host logic of the benchmark on CPU with the gloo backend (world size 2): the job's step
time is the maximum over ranks, and every rank runs its own batch of the same shape (data-parallel
replicas; the decode path itself has no collective)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, q):
    import sys
    import torch.distributed as dist
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        m = bench.max_over_ranks(1.5 + rank, "cpu")
        w = bench.rank_workload("decode_128k", rank)
        q.put((rank, m, w.seed, w.batch, w.seq_lens[0], w.heads))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(2):
        r, m, seed, B, L, H = q.get(timeout=120)
        out[r] = (m, seed, B, L, H)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert out[0][0] == out[1][0] == 2.5                 # max over ranks
    assert out[0][1] != out[1][1]                         # distinct batches
    assert out[0][2:] == out[1][2:] == (8, 131072, 64)    # same shape on every rank
