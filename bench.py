#!/usr/bin/env python
"""Decode-step benchmark of the CSA2 FP4 sparse-KV path.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one decode step of the whole path over one batch: pack the new token of every sequence
(FP4 + E4M3 key + FP8 window entry), score every block (Full) or the pool (Reindex), exact Top-K,
sparse attention over the selected FP4 entries plus the FP8 window, and the split combine.  The
default workload is B=8 sequences of 131,072 tokens, 64 heads, Top-K 2,048 blocks x 8.  Inputs are
seeded synthetic data resident in HBM; L2 is flushed (a 256 MB write, then a 256 MB read) before every
timed step.

Multi-GPU: one process per GPU (torchrun); every rank runs its own batch (data-parallel replicas,
no collective on the path); the step time is the max over ranks.  Rank 0 prints one JSON line.

--impl reference times the CPU oracle (test infrastructure, plain C, threads over blocks and heads)
on one sequence per step of the same workload.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode tokens/s at 128K ctx; sparse FP4-KV attn achieved HBM GB/s vs roofline"
UNIT = "tokens/s"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decode_128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="time eager launches only")
    ap.add_argument("--no-tier", action="store_true", help="skip the persistent-tier copy measurement")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="CPU baseline sample budget")
    return ap.parse_args()


def env_rank():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    # an earlier B200 measurement (STREAM-style copy; cuBLAS bf16 GEMM burst and sustained), used only
    # when no measured-peaks file is present
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def peak_label(peaks, key, note=""):
    if peaks["source"] == "measured":
        return "measured (MEASURED_PEAKS.json %s%s)" % (key, note)
    return "fallback (no MEASURED_PEAKS.json; earlier B200 measurement of %s%s)" % (key, note)


# ------------------------------------------------------------------------------------------------
# nvidia-smi clock sampling during the timed region
# ------------------------------------------------------------------------------------------------
class Clocks:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.3)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = [r.split(",") for r in open(self.path).read().strip().splitlines() if r.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 9:
                continue
            try:
                sm.append(float(r[1]))
                mx = max(mx, float(r[2]))
            except ValueError:
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return None
        loaded = [x for x in sm if x > 0.5 * max(sm)] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------------------------------------
# Our arm
# ------------------------------------------------------------------------------------------------
def source_sha(names):
    h = hashlib.sha1()
    for n in names:
        h.update(open(os.path.join(ROOT, "fp4_compressed_sparse_kv_b200", "csrc", n), "rb").read())
    return h.hexdigest()[:12]


KERNEL_SOURCES = {"indexer_full": ["screen.cu", "select.cu", "score.cuh", "radix.cuh", "common.cuh", "convert.cuh",
                                   "pipeline.cuh", "tcgen05.cuh"],
                  "indexer_reindex": ["indexer.cu", "score.cuh", "radix.cuh", "common.cuh", "convert.cuh",
                                      "pipeline.cuh"],
                  "sparse_decode_attn": ["attention_cc.cu", "attention_tc.cu", "attention_common.cuh", "tcgen05.cuh",
                                         "common.cuh", "convert.cuh", "pipeline.cuh"],
                  "kv_pack_fp4": ["pack.cu", "common.cuh", "convert.cuh", "pipeline.cuh"],
                  "kv_pack_fp4_prefill": ["pack.cu", "common.cuh", "convert.cuh", "pipeline.cuh"]}


def traffic_from_profiles(call, workload):
    """DRAM bytes per launch from the committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    sha = source_sha(KERNEL_SOURCES[call])
    for line in open(p):
        f = line.split()
        if len(f) >= 4 and not line.startswith("#") and f[0] == call and f[1] == workload and f[3] == sha:
            return float(f[2])
    return None


def max_over_ranks(value, device):
    """The largest value over all ranks (the job's step time is its slowest rank's)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_workload(name, rank):
    """Rank r's batch: the named workload's shape with its own seed (rank 0 keeps the base seed)."""
    from fp4_compressed_sparse_kv_b200 import synth
    w = synth.workload(name)
    if rank > 0:
        w.seed = (w.seed if isinstance(w.seed, list) else [w.seed]) + [rank]
    return w


class Prefill:
    """The mixed serving step's prefill chunk: w.prefill_tokens new tokens of one sequence, packed into
    the spare pages, its last 128 tokens into the spare window row (device inputs plus pinned copies)."""

    def __init__(self, st, dev):
        import numpy as np
        import torch

        from fp4_compressed_sparse_kv_b200 import synth
        w = st.w
        n = w.prefill_tokens
        rng = synth.rng_for(w, 0, 5000)
        lat = synth.latents(rng, np.arange(n))
        key = synth.index_keys(rng, n)
        spare_row = int(np.setdiff1d(np.arange(st.num_rows), st.swa_row_np)[0])
        slots = st.prefill_pages[np.arange(n) // 64].astype(np.int64) * 64 + np.arange(n) % 64
        sw = np.where(np.arange(n) >= n - 128, spare_row * 128 + np.arange(n) % 128, -1).astype(np.int32)
        self.n = n
        self.h_lat = torch.from_numpy(lat).view(torch.bfloat16).pin_memory()
        self.h_key = torch.from_numpy(key).view(torch.bfloat16).pin_memory()
        self.lat = self.h_lat.to(dev)
        self.key = self.h_key.to(dev)
        self.slots = torch.from_numpy(slots).to(dev)
        self.sw = torch.from_numpy(sw).to(dev)


def make_plan(st, prefill=None):
    """The step as a list of (call name, kernels launched, fn): the library's public calls."""
    from fp4_compressed_sparse_kv_b200 import csa
    w = st.w
    plan = []
    if prefill is not None:
        plan.append(("kv_pack_fp4_prefill", 1,
                     lambda: csa.kv_pack_fp4(st.layers[0], prefill.lat, prefill.key, prefill.slots, prefill.sw,
                                             st.ws)))
    for l, m in enumerate(w.modes):
        f = st.kv_of[l]
        lay = st.layers[f]
        if m == csa.FULL:
            plan.append(("kv_pack_fp4", 1, lambda f=f: st.pack_new_tokens(f)))
            # query terms, screen, selection (one launch when every block is selected)
            n_full = 1 if (st.max_seq_len + 7) // 8 <= st.layer_k[l] else 3
            plan.append(("indexer_full", n_full,
                         lambda l=l, lay=lay: csa.indexer_full(lay, st.batch, st.iq[l], st.iw[l], st.layer_k[l],
                                                               st.blocks[l], st.count[l], st.ws)))
        elif m == csa.REINDEX:
            fl = st.full_of[l]
            plan.append(("indexer_reindex", 2,
                         lambda l=l, lay=lay, fl=fl: csa.indexer_reindex(
                             lay, st.batch, st.iq[l], st.iw[l], st.blocks[fl], st.count[fl], st.layer_k[l],
                             st.blocks[l], st.count[l], st.ws)))
        else:
            plan.append(("index_reuse", 1,
                         lambda l=l: csa.index_reuse(st.blocks[l - 1], st.count[l - 1], st.blocks[l],
                                                     st.count[l], st.ws)))
        plan.append(("sparse_decode_attn", 2,
                     lambda l=l, lay=lay: csa.sparse_decode_attn(lay, st.batch, st.q[l], csa.default_sm_scale(),
                                                                 st.blocks[l], st.count[l], st.out[l], st.lse[l],
                                                                 st.ws)))
    return plan


def algorithmic_bytes(st, prefill=None):
    """Bytes each call must move per step, from the sizes and the selected sets (after a step)."""
    import numpy as np
    w = st.w
    B, H = w.batch, w.heads
    lens = np.array(w.seq_lens, np.int64)
    nF = np.minimum(lens, 128)
    out = {}

    def add(k, v):
        out[k] = out.get(k, 0.0) + float(v)

    if prefill is not None:   # bf16 latent and key in; codes, scales, keys out; 128 window entries
        add("kv_pack_fp4_prefill", prefill.n * (1024 + 256 + 256 + 32 + 128 + 8 + 4) + 128 * 516)
    for l, m in enumerate(w.modes):
        if m == 0:
            add("kv_pack_fp4", B * (1024 + 256 + 256 + 32 + 128 + 512 + 4 + 12))
            # every key once, the queries and weights, the selected ids
            add("indexer_full", (lens * 128).sum() + B * (2048 + 32) + B * st.layer_k[l] * 4)
        elif m == 1:
            pc = st.count[st.full_of[l]].cpu().numpy().astype(np.int64)
            # the pool's keys, the pool ids, the queries and weights, the selected ids
            add("indexer_reindex", (pc * 8 * 128).sum() + pc.sum() * 4 + B * (2048 + 32) + B * st.layer_k[l] * 4)
        else:
            add("index_reuse", st.count[l - 1].cpu().numpy().sum() * 8)
        blocks = st.blocks[l].cpu().numpy()
        cnt = st.count[l].cpu().numpy()
        n_fp4 = 0
        for b in range(B):
            pos = blocks[b, :cnt[b]].astype(np.int64)[:, None] * 8 + np.arange(8)[None, :]
            n_fp4 += int((pos < lens[b]).sum())
        add("sparse_decode_attn", n_fp4 * 288 + nF.sum() * 516 + B * H * (1024 + 2048 + 4))
    return out


def attn_flops(st):
    """Dense-equivalent FLOPs of the attention: QK and PV over every attended entry."""
    import numpy as np
    total = 0
    lens = np.array(st.w.seq_lens, np.int64)
    for l in range(len(st.w.modes)):
        cnt = st.count[l].cpu().numpy().astype(np.int64)
        n = np.minimum(cnt * 8, lens) + np.minimum(lens, 128)
        total += int(n.sum()) * 4 * st.w.heads * 512
    return total


def measure_kv_tier(st, dev, flush_l2, hbm_gbs, reps=3):
    """Export and import of every sequence's persistent record (FP4 codes, scales, indexer keys) of
    the first KV layer, to and from HBM and pinned host memory: one csa_kv_export / csa_kv_import per
    sequence, timed with CUDA events over the whole batch after an L2 flush."""
    import torch

    from fp4_compressed_sparse_kv_b200 import csa
    w, lay = st.w, st.layers[0]
    lens = [int(x) for x in w.seq_lens]
    sizes = [csa.kv_record_bytes(n) for n in lens]
    offs = [sum(sizes[:b]) for b in range(len(sizes))]
    total = sum(sizes)
    bufs = {"hbm": torch.empty((total,), dtype=torch.uint8, device=dev),
            "host": torch.empty((total,), dtype=torch.uint8).pin_memory()}
    rows = [st.batch.block_table[b].clone() for b in range(len(lens))]   # 16-byte aligned rows
    ws = csa.workspace(1, 16, 64, 8, device=dev)
    stream = torch.cuda.current_stream()
    out = {"record_bytes": total, "sequences": len(lens), "bytes_per_token": 416}

    def run(kind, where):
        fn = csa.kv_export if kind == "export" else csa.kv_import
        buf = bufs[where]
        for b, n in enumerate(lens):
            fn(lay, rows[b], n, buf[offs[b]:offs[b] + sizes[b]], ws)

    for kind in ("export", "import"):
        for where in ("hbm", "host"):
            run(kind, where)
            torch.cuda.synchronize()
            ms = []
            for _ in range(reps):
                flush_l2()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                run(kind, where)
                b_.record(stream)
                b_.synchronize()
                ms.append(a.elapsed_time(b_))
            t = sum(ms) / reps
            # HBM to HBM moves every byte twice through DRAM (read + write); to or from the host each
            # byte crosses the host link once and DRAM once
            moved = 2 * total if where == "hbm" else total
            rec = {"ms": round(t, 4), "gbs": round(moved / (t * 1e-3) / 1e9, 1)}
            if where == "hbm":
                rec["hbm_frac"] = round(moved / (t * 1e-3) / 1e9 / hbm_gbs, 4)
            out["%s_%s" % (kind, where)] = rec
    st.check()
    if csa.check_device_error(ws)[0] != 0:
        raise RuntimeError("persistent-tier copy reported a device-data error")
    return out


def run_ours(args, rank, world, local):
    import numpy as np
    import torch
    import torch.distributed as dist

    from fp4_compressed_sparse_kv_b200 import build as cuda_build
    from fp4_compressed_sparse_kv_b200 import csa, synth, workloads

    if rank == 0:
        cuda_build.build()
    if world > 1:
        dist.barrier()
    torch.cuda.set_device(local)
    dev = "cuda:%d" % local
    w = rank_workload(args.workload, rank)   # every rank processes its own batch of the same shape
    t0 = time.time()
    st = workloads.DecodeState(w, device=dev)
    setup_s = time.time() - t0
    prefill = Prefill(st, dev) if w.prefill_tokens else None
    plan = make_plan(st, prefill)
    # L2 flush before every timed step: write 256 MB, then read another 256 MB, so that no input is
    # served from L2 and the L2 holds no dirty lines whose write-back would share DRAM with the step
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.zeros(256 << 20, dtype=torch.uint8, device=dev)

    def flush_l2():
        flush_w.zero_()
        flush_r.sum(dtype=torch.int64)

    stream = torch.cuda.current_stream()

    def step():
        for _, _, fn in plan:
            fn()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st.check()
    bytes_per_call = algorithmic_bytes(st, prefill)
    flops_attn = attn_flops(st)

    K = args.steps
    names = [n for n, _, _ in plan]
    # The step replayed as one CUDA graph (how a decode step runs in serving: no per-launch host
    # overhead); fall back to eager launches if capture is not possible here.
    graph = None
    if not args.no_graph:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                step()
            for _ in range(args.warmup):
                graph.replay()
            torch.cuda.synchronize()
            st.check()
        except Exception as exc:  # noqa: BLE001 - report and continue eagerly
            print("graph capture unavailable (%s); timing eager launches" % exc, file=sys.stderr)
            graph = None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(plan) + 1)] for _ in range(K)]
    gev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    clocks = Clocks(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    wall0 = time.time()
    if graph is not None:
        for i in range(K):
            flush_l2()
            gev[i][0].record(stream)
            graph.replay()
            gev[i][1].record(stream)
    # per-call breakdown: the same step with eager launches and an event around every call
    for i in range(K):
        flush_l2()
        for j, (_, _, fn) in enumerate(plan):
            ev[i][j].record(stream)
            fn()
        ev[i][len(plan)].record(stream)
    torch.cuda.synchronize()
    # and replayed as a graph with the events captured between the calls (timestamps taken on the
    # device; an event node orders the calls around it, so this graph is timed apart from the headline)
    graph_calls = None
    if graph is not None:
        try:
            cev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(plan) + 1)]
            g3 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g3):
                for j, (_, _, fn) in enumerate(plan):
                    cev[j].record()
                    fn()
                cev[len(plan)].record()
            g3.replay()
            torch.cuda.synchronize()
            graph_calls = []
            for i in range(K):
                flush_l2()
                g3.replay()
                torch.cuda.synchronize()
                graph_calls.append([cev[j].elapsed_time(cev[j + 1]) for j in range(len(plan))])
            del g3
        except Exception as exc:  # noqa: BLE001 - report and keep the eager breakdown
            print("per-call graph timing unavailable (%s)" % exc, file=sys.stderr)
            graph_calls = None
    if world > 1:
        dist.barrier()
    wall = time.time() - wall0
    clk = clocks.stop()
    st.check()

    per_call = {}
    step_ms = []
    for i in range(K):
        step_ms.append(ev[i][0].elapsed_time(ev[i][len(plan)]))
        for j, n in enumerate(names):
            per_call.setdefault(n, []).append(
                graph_calls[i][j] if graph_calls is not None else ev[i][j].elapsed_time(ev[i][j + 1]))
    call_ms = {n: sum(v) / K for n, v in per_call.items()}     # per step, summed over layers
    calls_per_step = {n: names.count(n) for n in set(names)}
    eager_ms = sum(step_ms) / K
    mean_ms = sum(gev[i][0].elapsed_time(gev[i][1]) for i in range(K)) / K if graph is not None else eager_ms
    max_ms = max_over_ranks(mean_ms, dev)

    # ---- end to end through the public API: pinned host inputs in, results out, every step
    B, H = w.batch, w.heads
    n_kv = st.n_kv
    h_lat = [st.new_tokens[f][0].cpu().pin_memory() for f in range(n_kv)]
    h_key = [st.new_tokens[f][1].cpu().pin_memory() for f in range(n_kv)]
    h_q = [x.cpu().pin_memory() for x in st.q]
    h_iq = [x.cpu().pin_memory() for x in st.iq]
    h_iw = [x.cpu().pin_memory() for x in st.iw]
    h_out = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in st.out]
    h_lse = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in st.lse]
    h_pre = [prefill.h_lat, prefill.h_key] if prefill is not None else []
    h2d = sum(x.numel() * x.element_size() for x in h_lat + h_key + h_q + h_iq + h_iw + h_pre)
    d2h = sum(x.numel() * x.element_size() for x in h_out + h_lse)

    def e2e_step():
        if prefill is not None:
            prefill.lat.copy_(prefill.h_lat, non_blocking=True)
            prefill.key.copy_(prefill.h_key, non_blocking=True)
        for f in range(n_kv):
            st.new_tokens[f][0].copy_(h_lat[f], non_blocking=True)
            st.new_tokens[f][1].copy_(h_key[f], non_blocking=True)
        for l in range(len(w.modes)):
            st.q[l].copy_(h_q[l], non_blocking=True)
            st.iq[l].copy_(h_iq[l], non_blocking=True)
            st.iw[l].copy_(h_iw[l], non_blocking=True)
        step()
        for l in range(len(w.modes)):
            h_out[l].copy_(st.out[l], non_blocking=True)
            h_lse[l].copy_(st.lse[l], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    e_ms = []
    for i in range(K):
        flush_l2()
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        e2e_step()
        b_.record(stream)
        b_.synchronize()
        e_ms.append(a.elapsed_time(b_))
    e2e_eager_ms = max_over_ranks(sum(e_ms) / K, dev)
    # the same step (copies in, the public calls, copies out) captured once and replayed, as a serving
    # loop runs its decode step; the host waits for each step's results before the next
    e2e_ms, e2e_graph = e2e_eager_ms, False
    if graph is not None:
        try:
            g2 = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g2):
                e2e_step()
            g2.replay()
            torch.cuda.synchronize()
            g_ms = []
            for i in range(K):
                flush_l2()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                g2.replay()
                b_.record(stream)
                b_.synchronize()
                g_ms.append(a.elapsed_time(b_))
            e2e_ms, e2e_graph = max_over_ranks(sum(g_ms) / K, dev), True
        except Exception as exc:  # noqa: BLE001 - report and keep the eager number
            print("e2e graph capture unavailable (%s)" % exc, file=sys.stderr)

    if rank != 0:
        return None

    peaks = measured_peaks()
    tier = None if args.no_tier else measure_kv_tier(st, dev, flush_l2, peaks["hbm_gbs"])
    dominant = max(call_ms, key=call_ms.get)
    kernels = {}
    for n in call_ms:
        gbs = bytes_per_call.get(n, 0.0) / (call_ms[n] * 1e-3) / 1e9
        kernels[n] = {"ms_per_step": round(call_ms[n], 5), "calls_per_step": calls_per_step[n],
                      "bytes_per_step": bytes_per_call.get(n, 0.0), "gbs": round(gbs, 1),
                      "hbm_frac": round(gbs / peaks["hbm_gbs"], 4)}
    per_launch_ms = call_ms[dominant] / calls_per_step[dominant]
    per_launch_bytes = bytes_per_call[dominant] / calls_per_step[dominant]
    per_launch_flops = (flops_attn if dominant == "sparse_decode_attn" else 0.0) / calls_per_step[dominant]
    traffic = traffic_from_profiles(dominant, args.workload)
    # the bound is whichever floor is higher: bytes at the measured copy bandwidth or FLOPs at the
    # measured dense tensor rate (f16 operands run at the bf16 rate)
    if per_launch_flops / (peaks["bf16_tflops"] * 1e12) > per_launch_bytes / (peaks["hbm_gbs"] * 1e9):
        achieved = per_launch_flops / (per_launch_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "kernel": dominant, "achieved": round(achieved, 1), "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": round(achieved / peaks["bf16_tflops"], 4), "traffic": traffic,
                "peak_source": peak_label(peaks, "bf16_tflops", ", burst; f16 same rate"),
                "bytes_frac": round(per_launch_bytes / (per_launch_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)}
    else:
        achieved = per_launch_bytes / (per_launch_ms * 1e-3) / 1e9
        roof = {"bound": "hbm", "kernel": dominant, "achieved": round(achieved, 1), "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "traffic": traffic, "peak_source": peak_label(peaks, "hbm_gbs")}
    step_bytes = sum(bytes_per_call.values())
    attn_ms = call_ms.get("sparse_decode_attn", 0.0)
    line = {
        "metric": METRIC, "value": round(world * B / (max_ms * 1e-3), 2), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(max_ms, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "fp4-e2m1/e4m3 KV, f32 indexer, f16 x f16 -> f32 attn",
        "data": "synthetic (seeded; RMSNorm+RoPE latents, N(0,1) keys and queries)",
        "config": {"workload": args.workload, "batch_per_gpu": B, "seq_len": max(w.seq_lens),
                   "heads": H, "topk_blocks": w.topk, "modes": w.modes, "l2": "flushed before each step (256 MB write, then 256 MB read: no input in L2, no dirty lines)",
                   "parallelism": "dp%d replicas" % world},
        "roofline": roof,
        "step_roofline": {"bytes": step_bytes, "achieved_gbs": round(step_bytes / (max_ms * 1e-3) / 1e9, 1),
                          "frac": round(step_bytes / (max_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4)},
        "attention": {"ms": round(attn_ms, 5), "tflops": round(flops_attn / (attn_ms * 1e-3) / 1e12, 2) if attn_ms else None,
                      "hbm_frac": kernels.get("sparse_decode_attn", {}).get("hbm_frac")},
        "kernels": kernels,
        "e2e": {"value": round(world * B / (e2e_ms * 1e-3), 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e_ms, 5),
                "timing": ("CUDA-graph replay of copies in + public calls + copies out, host synchronised each step"
                           if e2e_graph else "eager public calls with the copies, host synchronised each step"),
                "eager": {"value": round(world * B / (e2e_eager_ms * 1e-3), 2), "ms_per_step": round(e2e_eager_ms, 5)}},
        "kv_tier": tier,
        "gpu_launches": (1 + (graph is not None) + (graph_calls is not None)) * K * sum(k for _, k, _ in plan),
        "timing": ("CUDA-graph replay of the step (headline); per-call figures from a replay of the same "
                   "graph with events captured between the calls; eager step %.5f ms" % eager_ms)
                  if graph_calls is not None else
                  ("CUDA-graph replay of the step (headline); per-call figures from eager launches with an "
                   "event around every call, eager step %.5f ms" % eager_ms) if graph is not None
                  else "eager launches with an event around every call",
        "clocks": clk,
        "wall_s_timed": round(wall, 3),
        "setup_s": round(setup_s, 1),
    }
    return line, st


# ------------------------------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and the reference arm)
# ------------------------------------------------------------------------------------------------
def oracle_sample_setup(w, b):
    """Oracle caches of sequence b, packed by the oracle itself (threads; not timed)."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from helpers import OracleSeq
    from fp4_compressed_sparse_kv_b200 import workloads
    lat, key = workloads.seq_tokens(w, 0, b)
    return OracleSeq(lat, key, w.seq_lens[b]), lat[-1:], key[-1:]


def oracle_step(os_, lat_new, key_new, q, iq, iw, k):
    """One decode step of one sequence on the CPU oracle, single thread."""
    import oracle
    oracle.pack_tokens(lat_new, key_new, with_swa=True)
    S = oracle.block_scores(iq, iw, os_.key8)
    blocks = oracle.topk(__import__("numpy").arange(S.size, dtype="int32"), S, k)
    pe = oracle.positions_of_blocks(blocks, os_.L)
    oracle.attention(q, oracle.default_tau(), os_.codes[pe], os_.scales[pe], os_.swa, os_.swa_scale)


def oracle_step_threaded(os_, lat_new, key_new, q, iq, iw, k, threads):
    """The same decode step on the CPU oracle with its block scores and attention heads spread over
    threads (the C oracle runs without the GIL)."""
    import numpy as np
    import oracle
    from helpers import attention_threaded, block_scores_threaded
    oracle.pack_tokens(lat_new, key_new, with_swa=True)
    S = block_scores_threaded(iq, iw, os_.key8, threads=threads)
    blocks = oracle.topk(np.arange(S.size, dtype="int32"), S, k)
    pe = oracle.positions_of_blocks(blocks, os_.L)
    attention_threaded(q, oracle.default_tau(), os_.codes[pe], os_.scales[pe], os_.swa, os_.swa_scale,
                       threads=threads)


def cpu_cores_info():
    model = ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return model, os.cpu_count()


def run_oracle_sample(w, budget_s, max_steps=None, warmup=0, threads=1, prepared=None):
    from fp4_compressed_sparse_kv_b200 import workloads
    os_, lat, key = prepared if prepared is not None else oracle_sample_setup(w, 0)
    q, iq, iw = workloads.layer_queries(w, 0)

    def one():
        if threads == 1:
            oracle_step(os_, lat, key, q[0], iq[0], iw[0], w.topk)
        else:
            oracle_step_threaded(os_, lat, key, q[0], iq[0], iw[0], w.topk, threads)

    for _ in range(warmup):
        one()
    times = []
    t_start = time.time()
    while True:
        t0 = time.time()
        one()
        times.append(time.time() - t0)
        if max_steps is not None and len(times) >= max_steps:
            break
        if max_steps is None and time.time() - t_start >= budget_s:
            break
    return times


def run_reference(args, rank, world):
    if rank != 0:
        return
    from fp4_compressed_sparse_kv_b200 import synth
    w = synth.workload(args.workload)
    model, ncpu = cpu_cores_info()
    times = run_oracle_sample(w, 0, max_steps=args.steps, warmup=args.warmup, threads=ncpu)
    s = sum(times)
    value = len(times) / s
    sample = ("oracle decode step of sequence 0 of %d (context %d, %d heads, Top-K %d): pack of the new "
              "token, block scores over the whole context, Top-K, attention; block scores and heads over "
              "%d threads" % (w.batch, w.seq_lens[0], w.heads, w.topk, ncpu))
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 5), "unit": UNIT, "n_gpus": world,
            "steps": len(times), "warmup": args.warmup, "ms_per_step": round(1e3 * s / len(times), 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 attention, f32 indexer",
            "data": "synthetic (seeded)",
            # the workload of the other arm; each timed step is the bounded sample named in cpu_baseline
            "config": {"workload": args.workload, "batch_per_gpu": w.batch, "seq_len": max(w.seq_lens),
                       "heads": w.heads, "topk_blocks": w.topk, "modes": w.modes,
                       "l2": "not applicable (host)", "parallelism": "dp%d replicas" % world},
            "cpu_baseline": {"value": round(value, 5), "unit": UNIT, "cores": ncpu, "kind": "oracle",
                             "sample": sample, "cpu": model, "host_cpus": ncpu},
            "e2e": {"value": round(value, 5), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    rank, world, local = env_rank()
    if world != args.gpus and world == 1 and args.gpus > 1:
        print(json.dumps({"error": "--gpus %d needs torchrun with %d processes" % (args.gpus, args.gpus)}))
        return 2
    if args.impl == "reference":
        run_reference(args, rank, world)
        return 0
    import torch.distributed as dist
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    try:
        res = run_ours(args, rank, world, local)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank == 0 and res is not None:
        line, st = res
        if world == 1 and not args.no_cpu_baseline:
            model, ncpu = cpu_cores_info()
            prepared = oracle_sample_setup(st.w, 0)
            t1 = run_oracle_sample(st.w, args.cpu_seconds / 2, prepared=prepared)
            tn = run_oracle_sample(st.w, args.cpu_seconds / 2, threads=ncpu, prepared=prepared)
            line["cpu_baseline"] = {
                "value": round(len(tn) / sum(tn), 5), "unit": UNIT, "cores": ncpu, "kind": "oracle",
                "sample": "%d oracle decode steps of sequence 0 (context %d, %d heads, Top-K %d) with block scores "
                          "and attention heads over %d threads; %d more on one thread"
                          % (len(tn), st.w.seq_lens[0], st.w.heads, st.w.topk, ncpu, len(t1)),
                "one_thread": {"value": round(len(t1) / sum(t1), 5), "cores": 1},
                "cpu": model, "host_cpus": ncpu}
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
