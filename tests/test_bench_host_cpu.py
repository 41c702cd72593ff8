"""Host logic of bench.py on CPU: the algorithmic bytes and FLOPs of a decode_128k step (the figures the
roofline divides by), the gate that reports committed DRAM traffic only while the kernels' sources
still hash to what the capture was taken on, and the label that says whether the peak is measured."""
import os
import types

import numpy as np
import torch

import bench
from fp4_compressed_sparse_kv_b200 import synth


def _decode_128k_state():
    """A stand-in for a finished decode_128k step: every sequence selected 2,048 full blocks."""
    w = synth.workload("decode_128k")
    B, k = w.batch, 2048
    blocks = torch.arange(k, dtype=torch.int32).repeat(B, 1) * 3        # in range: 3 * 2047 < 16,384
    count = torch.full((B,), k, dtype=torch.int32)
    return types.SimpleNamespace(w=w, layer_k=[k], blocks=[blocks], count=[count])


def test_decode_128k_algorithmic_bytes_and_flops():
    st = _decode_128k_state()
    by = bench.algorithmic_bytes(st)
    # keys of every position once, the queries and weights, the selected ids
    assert by["indexer_full"] == 8 * 131072 * 128 + 8 * (2048 + 32) + 8 * 2048 * 4 == 134_299_904
    # 16,384 FP4 entries of 288 B and 128 window entries of 516 B per sequence, q in, out and lse out
    assert by["sparse_decode_attn"] == 8 * 16384 * 288 + 8 * 128 * 516 + 8 * 64 * (1024 + 2048 + 4) == 39_852_032
    assert by["kv_pack_fp4"] == 8 * (1024 + 256 + 256 + 32 + 128 + 512 + 4 + 12)
    assert bench.attn_flops(st) == 8 * (16384 + 128) * 4 * 64 * 512


def test_positions_past_the_end_are_not_counted():
    st = _decode_128k_state()
    st.w.seq_lens[0] = 131072 - 5                   # the last block of sequence 0 is partial
    st.blocks[0][0, -1] = (131072 - 5) // 8         # and selected
    by = bench.algorithmic_bytes(st)
    full = 8 * 16384 * 288 + 8 * 128 * 516 + 8 * 64 * (1024 + 2048 + 4)
    assert by["sparse_decode_attn"] == full - 5 * 288


def test_traffic_is_reported_only_on_the_captured_source(tmp_path, monkeypatch):
    csrc = tmp_path / "fp4_compressed_sparse_kv_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in set(sum(bench.KERNEL_SOURCES.values(), [])):
        (csrc / n).write_text("// " + n + "\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.source_sha(bench.KERNEL_SOURCES["sparse_decode_attn"])
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.txt").write_text(
        "# call workload bytes_per_call source_sha\nsparse_decode_attn decode_128k 57991680 %s\n" % sha)
    assert bench.traffic_from_profiles("sparse_decode_attn", "decode_128k") == 57991680.0
    assert bench.traffic_from_profiles("sparse_decode_attn", "tiny_4k") is None
    assert bench.traffic_from_profiles("indexer_full", "decode_128k") is None
    (csrc / "attention_tc.cu").write_text("// changed\n")
    assert bench.traffic_from_profiles("sparse_decode_attn", "decode_128k") is None


def test_peak_labels(tmp_path, monkeypatch):
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    p = bench.measured_peaks()
    assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0
    assert bench.peak_label(p, "hbm_gbs").startswith("fallback (no MEASURED_PEAKS.json")
    (tmp_path / "MEASURED_PEAKS.json").write_text('{"hbm_gbs": 6527.8, "bf16_tflops": 1642.8}')
    p = bench.measured_peaks()
    assert p["source"] == "measured" and p["hbm_gbs"] == 6527.8 and p["bf16_tflops_sustained"] == 1642.8
    assert bench.peak_label(p, "bf16_tflops", ", burst") == "measured (MEASURED_PEAKS.json bf16_tflops, burst)"
