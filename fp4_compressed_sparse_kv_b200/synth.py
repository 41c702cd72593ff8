"""Seeded synthetic inputs for the CSA2 FP4 sparse-KV decode path.

This module holds input generation only: random draws, the RMSNorm + RoPE that produce a
post-norm latent (the pages' range argument starts from such a latent: ailily.cc article
"每个 token 只占 890 字节", section 三), bf16 rounding, and paged-layout bookkeeping.  It contains
none of the path's arithmetic (no FP4/FP8 encoding, no scoring, no attention).  Both the CUDA
path's tests/benchmark and the CPU oracle receive the arrays it returns.

bf16 tensors are numpy uint16 arrays holding bf16 bit patterns.
"""
from dataclasses import dataclass, field
from typing import List

import numpy as np

PAGE = 64
LATENT = 512
ROPE_DIMS = 64
IDX_HEADS = 8
IDX_DIM = 128
WINDOW = 128


def bf16_bits(x):
    """float32 array -> bf16 bit patterns (uint16), round-to-nearest-even."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    r = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + r) >> 16).astype(np.uint16)


def bf16_to_f32(b):
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32)


def rms_norm(x, eps=1e-6):
    """RMSNorm with unit weight, in float32."""
    x = np.asarray(x, np.float32)
    ms = np.mean(x * x, axis=-1, keepdims=True, dtype=np.float32)
    return (x / np.sqrt(ms + np.float32(eps))).astype(np.float32)


def rope_last(x, positions, dims=ROPE_DIMS, base=10000.0):
    """Rotary embedding on the last `dims` channels, interleaved pairs (c, c+1), angle pos*theta_i
    with theta_i = base^(-2i/dims), evaluated in float64 and rounded to float32."""
    x = np.array(x, np.float32, copy=True)
    pos = np.asarray(positions, np.float64).reshape(-1, 1)
    i = np.arange(dims // 2, dtype=np.float64)
    ang = pos * base ** (-2.0 * i / dims)
    c, s = np.cos(ang), np.sin(ang)
    lo = x.shape[-1] - dims
    a = x[:, lo::2].astype(np.float64)
    b = x[:, lo + 1::2].astype(np.float64)
    x[:, lo::2] = (a * c - b * s).astype(np.float32)
    x[:, lo + 1::2] = (a * s + b * c).astype(np.float32)
    return x


def latents(rng, positions, heavy_tail=False):
    """bf16 [n,512] post-RMSNorm/RoPE latents for the given positions.  Pre-norm channels are
    N(0,1); with heavy_tail each channel is N(0,9) (std 3) with probability 1% instead."""
    positions = np.asarray(positions)
    n = positions.size
    x = rng.standard_normal((n, LATENT), dtype=np.float32)
    if heavy_tail:
        wide = rng.random((n, LATENT), dtype=np.float32) < np.float32(0.01)
        x = np.where(wide, x * np.float32(3.0), x)
    return bf16_bits(rope_last(rms_norm(x), positions))


def index_keys(rng, n):
    """bf16 [n,128] indexer keys, N(0,1)."""
    return bf16_bits(rng.standard_normal((n, IDX_DIM), dtype=np.float32))


def index_query(rng, B):
    """Indexer query bf16 [B,8,128] ~ N(0,1) and head weights float32 [B,8] ~ U(0,1)."""
    iq = bf16_bits(rng.standard_normal((B, IDX_HEADS, IDX_DIM), dtype=np.float32))
    iw = rng.random((B, IDX_HEADS), dtype=np.float32)
    return iq, iw


def query(rng, B, H):
    """Attention query bf16 [B,H,512] ~ N(0,1) over the shared latent."""
    return bf16_bits(rng.standard_normal((B, H, LATENT), dtype=np.float32))


def pages_needed(L):
    return (int(L) + PAGE - 1) // PAGE


def block_tables(rng, seq_lens, extra_pages=0):
    """Seeded paged layout: every sequence's pages are distinct ids from a random permutation of
    all pages, so neighbouring positions of a sequence live in scattered pages.  Unused table
    entries are -1.  Returns (block_table int32 [B, max_pages], num_pages)."""
    need = [pages_needed(L) for L in seq_lens]
    total = int(sum(need)) + int(extra_pages)
    perm = rng.permutation(total).astype(np.int32)
    mp = max(need)
    bt = np.full((len(seq_lens), mp), -1, np.int32)
    o = 0
    for b, n in enumerate(need):
        bt[b, :n] = perm[o:o + n]
        o += n
    return bt, total


def slots_of(block_table_row, positions):
    """Global slot ids page*64 + offset of one sequence's positions."""
    positions = np.asarray(positions, np.int64)
    return np.asarray(block_table_row, np.int64)[positions // PAGE] * PAGE + positions % PAGE


# ------------------------------------------------------------------------------------------------
# The five workloads, by their sizes
# ------------------------------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    batch: int
    seq_lens: List[int]
    heads: int
    topk: int                 # Full-layer Top-K in blocks of 8 positions
    reindex_topk: int = 512   # Reindex Top-K in blocks (pool is the last Full layer's set)
    modes: List[int] = field(default_factory=lambda: [0])   # 0 Full, 1 Reindex, 2 Reuse
    heavy_tail: bool = False
    seed: object = 0
    prefill_tokens: int = 0   # mixed serving step: tokens packed in the same step


def workload(name):
    """Return one of: tiny_4k, decode_128k, stack20_256k, single_1m, mixed_serving."""
    if name == "tiny_4k":
        return Workload(name, 1, [4096], 16, 64, seed=0)
    if name == "decode_128k":
        return Workload(name, 8, [131072] * 8, 64, 2048, seed=[2])
    if name == "stack20_256k":
        return Workload(name, 4, [262144] * 4, 64, 2048, 512, [0, 1, 2, 2] * 5, seed=[3])
    if name == "single_1m":
        return Workload(name, 1, [1048576], 64, 2048, 512, [0, 1, 1, 1], heavy_tail=True,
                        seed=[4])
    if name == "mixed_serving":
        rng = np.random.default_rng([5, 999])
        lens = rng.integers(8192, 262144, endpoint=True, size=32).tolist()
        return Workload(name, 32, lens, 64, 2048, seed=[5], prefill_tokens=65536)
    raise KeyError(name)


WORKLOADS = ["tiny_4k", "decode_128k", "stack20_256k", "single_1m", "mixed_serving"]


def rng_for(w, layer, stream):
    """Independent stream per (workload, layer, purpose)."""
    seed = w.seed if isinstance(w.seed, list) else [w.seed]
    return np.random.default_rng(list(seed) + [layer, stream])
