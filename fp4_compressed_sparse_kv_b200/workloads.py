"""Build a synthetic decode workload on the GPU: generate each sequence's latents and indexer keys
with the seeded generators in `synth`, pack them into paged caches with the library's own pack
kernel, and hold per-layer queries.  Used by the benchmark and the GPU tests.

Seeds: the latents of KV layer f and sequence b come from rng_for(w, f, 1000 + b), its indexer keys
from rng_for(w, f, 2000 + b); layer l's attention query from rng_for(w, l, 3000) and its indexer
query and weights from rng_for(w, l, 4000); the page permutation from rng_for(w, 0, 100).
"""
import concurrent.futures as cf

import numpy as np
import torch

from . import csa, synth

FULL, REINDEX, REUSE = csa.FULL, csa.REINDEX, csa.REUSE


def seq_tokens(w, kv_layer, b):
    """Host bf16 latents [L,512] and indexer keys [L,128] of sequence b of KV layer kv_layer."""
    L = w.seq_lens[b]
    lat = synth.latents(synth.rng_for(w, kv_layer, 1000 + b), np.arange(L), heavy_tail=w.heavy_tail)
    key = synth.index_keys(synth.rng_for(w, kv_layer, 2000 + b), L)
    return lat, key


def layer_queries(w, layer):
    """q bf16 [B,H,512], iq bf16 [B,8,128], iw float32 [B,8] of decoder layer `layer`."""
    q = synth.query(synth.rng_for(w, layer, 3000), w.batch, w.heads)
    iq, iw = synth.index_query(synth.rng_for(w, layer, 4000), w.batch)
    return q, iq, iw


def kv_layer_of(modes):
    """Index of the KV layer (the most recent Full layer) each decoder layer reads."""
    out, f = [], -1
    for m in modes:
        if m == FULL:
            f += 1
        if f < 0:
            raise ValueError("the first layer must be Full")
        out.append(f)
    return out


def swa_slots(swa_row, positions):
    return (int(swa_row) * synth.WINDOW + np.asarray(positions, np.int64) % synth.WINDOW).astype(np.int32)


def to_dev(a, device, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.to(device, non_blocking=False)


class DecodeState:
    """Device-resident caches, metadata and per-layer inputs of one workload."""

    def __init__(self, w, device="cuda", threads=8, prefill_rows=1):
        self.w = w
        self.device = device
        B = w.batch
        rng = synth.rng_for(w, 0, 100)
        extra = (w.prefill_tokens + synth.PAGE - 1) // synth.PAGE
        self.block_table_np, self.num_pages = synth.block_tables(rng, w.seq_lens, extra_pages=extra)
        self.swa_row_np = rng.permutation(B + prefill_rows).astype(np.int32)[:B]
        self.num_rows = B + prefill_rows
        self.prefill_pages = np.setdiff1d(np.arange(self.num_pages),
                                          self.block_table_np[self.block_table_np >= 0])
        self.kv_of = kv_layer_of(w.modes)
        self.full_of = [max(i for i in range(l + 1) if w.modes[i] == FULL) for l in range(len(w.modes))]
        self.n_kv = max(self.kv_of) + 1
        self.max_seq_len = max(w.seq_lens)
        self.batch = csa.Batch(to_dev(np.array(w.seq_lens, np.int32), device),
                               to_dev(self.block_table_np, device),
                               to_dev(self.swa_row_np, device), self.max_seq_len)
        self.layers = [csa.KVLayer(self.num_pages, self.num_rows, device) for _ in range(self.n_kv)]
        self.cap = max(w.topk, w.reindex_topk)
        self.ws = csa.workspace(B, w.heads, self.max_seq_len, self.cap, device)
        self._fill(threads)
        self.queries = [layer_queries(w, l) for l in range(len(w.modes))]
        self.q = [to_dev(q, device, torch.bfloat16) for q, _, _ in self.queries]
        self.iq = [to_dev(iq, device, torch.bfloat16) for _, iq, _ in self.queries]
        self.iw = [to_dev(iw, device) for _, _, iw in self.queries]
        ks = [w.topk if m == FULL else w.reindex_topk for m in w.modes]
        for i, m in enumerate(w.modes):       # a Reuse layer keeps the capacity of what it copies
            if m == REUSE:
                ks[i] = ks[i - 1]
        self.layer_k = ks
        self.blocks = [torch.zeros((B, k), dtype=torch.int32, device=device) for k in ks]
        self.count = [torch.zeros((B,), dtype=torch.int32, device=device) for _ in ks]
        self.out = [torch.zeros((B, w.heads, synth.LATENT), dtype=torch.float32, device=device)
                    for _ in ks]
        self.lse = [torch.zeros((B, w.heads), dtype=torch.float32, device=device) for _ in ks]
        # the new token of each sequence (position L-1), re-packed every decode step
        self.new_tokens = []
        for f in range(self.n_kv):
            lat = np.stack([self._last[f][b][0] for b in range(B)])
            key = np.stack([self._last[f][b][1] for b in range(B)])
            self.new_tokens.append((to_dev(lat, device, torch.bfloat16), to_dev(key, device, torch.bfloat16)))
        slots = np.array([synth.slots_of(self.block_table_np[b], [w.seq_lens[b] - 1])[0]
                          for b in range(B)], np.int64)
        sw = np.array([swa_slots(self.swa_row_np[b], [w.seq_lens[b] - 1])[0] for b in range(B)],
                      np.int32)
        self.new_slot = to_dev(slots, device)
        self.new_swa_slot = to_dev(sw, device)
        del self._last

    def _fill(self, threads):
        """Generate every sequence's tokens (threads) and pack them on the GPU."""
        w = self.w
        self._last = [[None] * w.batch for _ in range(self.n_kv)]
        jobs = [(f, b) for f in range(self.n_kv) for b in range(w.batch)]

        def gen(fb):
            f, b = fb
            return f, b, seq_tokens(w, f, b)

        def chunks():
            with cf.ThreadPoolExecutor(max_workers=threads) as ex:
                for i in range(0, len(jobs), threads):       # bounded host memory
                    yield from ex.map(gen, jobs[i:i + threads])

        if True:
            for f, b, (lat, key) in chunks():
                L = w.seq_lens[b]
                slots = synth.slots_of(self.block_table_np[b], np.arange(L))
                pos = np.arange(L)
                sw = np.where(pos >= L - synth.WINDOW, swa_slots(self.swa_row_np[b], pos), -1)
                csa.kv_pack_fp4(self.layers[f], to_dev(lat, self.device, torch.bfloat16),
                                to_dev(key, self.device, torch.bfloat16),
                                to_dev(slots, self.device), to_dev(sw.astype(np.int32), self.device),
                                self.ws)
                self._last[f][b] = (lat[-1:].copy(), key[-1:].copy())
        torch.cuda.synchronize()

    # --------------------------------------------------------------------------------------------
    def pack_new_tokens(self, f, stream=None):
        lat, key = self.new_tokens[f]
        csa.kv_pack_fp4(self.layers[f], lat.view(-1, synth.LATENT), key.view(-1, synth.IDX_DIM),
                        self.new_slot, self.new_swa_slot, self.ws, stream)

    def decode_layer(self, l, stream=None):
        m = self.w.modes[l]
        f = self.kv_of[l]
        # Reindex searches the pool of the most recent Full layer; Reuse copies the previous set
        src = self.full_of[l] if m == REINDEX else l - 1
        prev_b = self.blocks[src] if l > 0 else None
        prev_c = self.count[src] if l > 0 else None
        csa.decode_layer(m, self.layers[f], self.batch, self.q[l], self.out[l], self.lse[l],
                         self.blocks[l], self.count[l], self.ws, iq=self.iq[l], iw=self.iw[l],
                         k=self.layer_k[l], prev_blocks=prev_b, prev_count=prev_c, stream=stream)

    def step(self, stream=None):
        """One decode step over every layer: pack the new token of each KV layer, then
        indexer + attention per layer."""
        for l, m in enumerate(self.w.modes):
            if m == FULL:
                self.pack_new_tokens(self.kv_of[l], stream)
            self.decode_layer(l, stream)

    def check(self):
        s, d = csa.check_device_error(self.ws)
        if s != 0:
            raise csa.CsaError(s, "device status (detail %d)" % d)
