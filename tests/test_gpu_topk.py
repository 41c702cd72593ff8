"""GPU parity of step 3 alone (csa_topk_blocks) on crafted block scores: exact Top-K sets against the
oracle's sort, with heavy ties (lower block id wins), all-equal scores, negative scores and -0, both
the shared-memory path (<= 16,384 candidates) and the streaming path (more), Full and Reindex (pool)
modes."""
import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.gpu


def run_topk(scores_rows, k, pool_rows=None):
    import torch
    from fp4_compressed_sparse_kv_b200 import csa
    B = len(scores_rows)
    if pool_rows is None:
        n = [len(r) for r in scores_rows]
        lens = [8 * x for x in n]
        stride = max(n)
    else:
        n = [len(p) for p in pool_rows]
        lens = [8 * (int(p.max()) + 1) if len(p) else 8 for p in pool_rows]
        stride = max(max(n), 1)
    max_len = max(lens)
    sc = np.full((B, stride), -1.0, np.float32)
    for b, r in enumerate(scores_rows):
        sc[b, :len(r)] = r
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    bt = dev(np.zeros((B, (max_len + 63) // 64), np.int32))
    batch = csa.Batch(dev(np.array(lens, np.int32)), bt, dev(np.zeros(B, np.int32)), max_len)
    out = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    cnt = torch.zeros(B, dtype=torch.int32, device="cuda")
    ws = torch.zeros(256, dtype=torch.uint8, device="cuda")
    pool = pc = None
    if pool_rows is not None:
        pa = np.full((B, stride), -1, np.int32)
        for b, p in enumerate(pool_rows):
            pa[b, :len(p)] = p
        pool, pc = dev(pa), dev(np.array(n, np.int32))
    csa.topk_blocks(batch, dev(sc), k, out, cnt, ws, pool=pool, pool_count=pc)
    assert csa.check_device_error(ws)[0] == 0
    c = cnt.cpu().numpy()
    o = out.cpu().numpy()
    return [o[b, :c[b]] for b in range(B)]


@pytest.mark.parametrize("n,k,levels", [(100, 10, 5), (16384, 2048, 40), (16385, 2048, 40),
                                        (131072, 2048, 1000), (5000, 4999, 3), (3000, 2048, 0)])
def test_topk_full_mode(n, k, levels):
    rng = np.random.default_rng(n + k)
    rows = []
    for b in range(3):
        if levels:
            r = (rng.integers(0, levels, n) / 7).astype(np.float32)
        else:
            r = rng.standard_normal(n).astype(np.float32) * 30
        rows.append(r)
    rows[1][: n // 3] = 0.0          # a run of exact ties at zero
    rows[2][::5] = -0.0              # -0 ties with +0
    got = run_topk(rows, k)
    for b, r in enumerate(rows):
        ref = oracle.topk(np.arange(n, dtype=np.int32), r, k)
        assert got[b].tolist() == ref.tolist(), "row %d" % b


def test_topk_all_equal_and_negative():
    n, k = 20000, 777
    rows = [np.full(n, 3.5, np.float32), -np.abs(np.random.default_rng(1).standard_normal(n)).astype(np.float32)]
    got = run_topk(rows, k)
    assert got[0].tolist() == list(range(k))
    assert got[1].tolist() == oracle.topk(np.arange(n, dtype=np.int32), rows[1], k).tolist()


def test_topk_pool_mode():
    rng = np.random.default_rng(9)
    pools, rows = [], []
    for m in (2048, 300, 2048):
        p = np.sort(rng.choice(50000, m, replace=False)).astype(np.int32)
        pools.append(p)
        rows.append((rng.integers(0, 50, m) / 3).astype(np.float32))
    got = run_topk(rows, 512, pool_rows=pools)
    for b in range(3):
        assert got[b].tolist() == oracle.topk(pools[b], rows[b], 512).tolist()
