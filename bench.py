"""Benchmark of the CSA2 decode step over an FP4 global KV cache.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one decode token through the decoder's 20-layer CSA2 schedule (first group
Full + 3 Reuse, the Full layer building the 2048 x 8 candidate pool; then 4 groups of
Reindex + 3 Reuse), preceded by the append of the token's own compressed entry.  The
default workload is that step at a context of 131,072 entries (64 heads x 512, indexer
16 x 128, Top-512, window 128, 1% outlier rows); ``--workload decoder_step_1m`` runs it at
1,048,576.  The metric is decode layer-steps/s (20 per step) over the whole job.

Timing: W untimed warm-up steps, then K steps, each replayed from CUDA graphs and timed
with CUDA events on the launching stream; L2 is flushed (a 256 MB write) between steps,
outside the timed events.  Multi-GPU: one independent replica per rank (the decode step of
one sequence does not shard), max time over ranks.  rank 0 prints one JSON line.

The same line carries, under "workloads", the other sizes the metric and the pages' workloads
name, each timed the same way in the same run: the decoder step at 1,048,576 entries (the
metric's second context, also summarised as "value_1m"), the 64-sequence ragged decode
batch (append + Full Top-512 + attention) and the 4,096-query encoder chunk (Full index with
causal visibility + 6 attention layers), each with the roofline of its index and attention.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "CSA2 decode layer-steps/s at 128K and 1M ctx; achieved HBM GB/s vs roofline"
UNIT = "layer-steps/s"
L2_FLUSH_BYTES = 256 << 20
# Algorithmic bytes of one decode query's attention: the selected FP4 rows (288 B each at
# D = 512), the window rows and Q (bf16) and the output, counted at 2 bytes per element as in
# the roofline plan; the fp32 output this library writes adds H * D * 2 more bytes, reported
# separately.


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, "fallback"


# ----------------------------------------------------------------------------------------
# clocks sampled during the timed region
# ----------------------------------------------------------------------------------------
class ClockSampler:
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"csa2_clocks_{os.getpid()}.csv")

    def start(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=self.f, stderr=subprocess.DEVNULL)
            # make sure sampling has started before the timed region begins
            t0 = time.time()
            while time.time() - t0 < 3.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.02)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        os.unlink(self.path)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None, "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of the same workload
# ----------------------------------------------------------------------------------------
def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [d.get("num_threads", 1) for d in threadpool_info()]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


def oracle_sample(W, budget_s: float):
    """Run the oracle over the decoder schedule for the workload's query, step after step,
    until ``budget_s`` seconds of oracle work.  The stored FP4 cache is the oracle's own
    quantisation of the seeded rows, filled on first touch outside the timed spans (the GPU's
    cache is likewise filled before timing); each timed step quantises the appended row,
    scores, selects, builds the pool, re-scores the pool, dequantises the selected rows and
    attends.  Returns (layer_steps, seconds, description)."""
    from fp4_kv_cache_03_b200 import synth
    from oracle import csa2_ref as R
    n = W.lengths[0]
    kI = synth.bf16_bits_to_f32(synth.index_k_rows(W.seed, 0, n, W.d_I)).astype(np.float64)
    kv = synth.kv_rows(W.seed, 0, n, W.D, W.outlier_frac)
    x_new = synth.append_rows(W.seed, 0, 1, W.D)
    kv[n - 1] = x_new[0]
    kI[n - 1] = synth.bf16_bits_to_f32(synth.append_index_k(W.seed, 0, 1, W.d_I))[0]
    stored = {}                                    # row -> (codes, scales): the FP4 cache

    def fill(pos):
        need = [int(p) for p in pos if int(p) not in stored]
        if need:
            c, sc = R.quantize_rows(kv[need])
            for i, p in enumerate(need):
                stored[p] = (c[i], sc[i])

    t_q = int(W.q_pos()[0])
    layers = []
    for li, mode in enumerate(W.modes):
        q = synth.bf16_bits_to_f32(synth.queries(W.seed, li, 1, W.H, W.D))[0]
        qI = synth.bf16_bits_to_f32(synth.index_queries(W.seed, li, 1, W.H_I, W.d_I))[0]
        w = synth.index_weights(W.seed, li, 1, W.H_I)[0]
        pos = R.window_positions(t_q, W.window)
        swa = synth.bf16_bits_to_f32(synth.swa_rows(W.seed, li, 0, int(pos[0]), len(pos), W.D))
        layers.append((mode, q, qI, w, swa))
    done, t_total, steps = 0, 0.0, 0
    while True:
        t0 = time.perf_counter()
        untimed = 0.0
        R.quantize_rows(x_new)                                   # a1 append
        latest = pool = None
        for mode, q, qI, w, swa in layers:
            if mode == "full":
                sc = R.index_scores(qI, w, kI)
                latest = R.topk_ascending(sc, W.topk)
                if W.pool_blocks and pool is None:
                    pool = R.build_pool(sc, W.pool_blocks, W.block)
            elif mode == "reindex":
                latest = R.reindex(qI, w, kI, pool, W.block, n, W.topk)
            sel = latest[latest >= 0]
            t1 = time.perf_counter()
            fill(sel)
            untimed += time.perf_counter() - t1
            rows = R.dequantize_rows(np.stack([stored[int(p)][0] for p in sel]),
                                     np.stack([stored[int(p)][1] for p in sel]))
            R.sparse_attention(q, rows, swa, 1.0 / math.sqrt(W.D))
            done += 1
        t_total += time.perf_counter() - t0 - untimed
        steps += 1
        if t_total >= budget_s:
            break
    return done, t_total, (f"{steps} decoder step(s) x {len(W.modes)} layers, 1 query, "
                           f"{n} entries; cache quantised outside the timed spans")


# ----------------------------------------------------------------------------------------
# the job across ranks: every rank runs an independent replica; the job's time is the
# slowest rank's, and the job's throughput counts the units of every rank
# ----------------------------------------------------------------------------------------
def schedule_of(modes) -> str:
    """'full, 3 reuse, reindex, 3 reuse, ...': the layer modes, runs of Reuse counted."""
    out, i = [], 0
    while i < len(modes):
        j = i
        while j < len(modes) and modes[j] == modes[i]:
            j += 1
        out.append(modes[i] if j - i == 1 else f"{j - i} {modes[i]}")
        i = j
    return ", ".join(out)


def max_over_ranks(x: float, device="cpu") -> float:
    """Largest x over all ranks of the default process group (x itself without one)."""
    import torch
    dist = torch.distributed
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    dev = "cpu" if dist.get_backend() == "gloo" else device
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(steps_per_rank: int, world: int, layers: int, t_max: float) -> float:
    """Layer-steps/s of the whole job: every rank's steps over the slowest rank's time."""
    return steps_per_rank * world * layers / t_max


# ----------------------------------------------------------------------------------------
def run_reference(args, rank):
    """The oracle arm: the same metric, on the host cores, bounded."""
    if rank != 0:
        return
    from fp4_kv_cache_03_b200 import synth
    W = synth.workload(args.workload)
    ls, t, what = oracle_sample(W, max(10.0, 2.0 * args.steps))
    v = ls / t
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t * len(W.modes) / ls,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": W.name, "context_entries": W.lengths[0],
                                            "layers": len(W.modes), "batch": W.num_q},
            "cpu_baseline": {"value": v, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                             "sample": what},
            "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def attn_alg_bytes(W) -> int:
    """Algorithmic bytes of one attention call over all its queries."""
    per_q = W.topk * (W.D // 2 + W.D // 16) + W.window * W.D * 2 + 2 * W.H * W.D * 2
    return W.num_q * per_q


def attn_flops(W) -> int:
    """Tensor-core FLOPs of one attention call: S and O over Top-K + window keys, all heads."""
    return W.num_q * 2 * 2 * W.H * (W.topk + W.window) * W.D


def index_bytes(W, esize=2) -> int:
    """Indexer-K bytes a Full index call streams: d_I elements (bf16: 2 bytes, E4M3: 1) per
    visible entry of every query."""
    return int(np.sum(W.q_visible())) * W.d_I * esize


def index_flops(W) -> int:
    return int(np.sum(W.q_visible())) * W.H_I * W.d_I * 2


def captured_attn_traffic(workload_name: str, root: str | None = None):
    """DRAM bytes per launch of the attention kernel from the committed ncu capture
    (profiles/attn_tc_traffic.json under ``root``, the repository by default), or None when
    that capture is of another workload or the kernel's sources have changed since it was
    taken (their SHA-256 differs)."""
    here = root or os.path.dirname(os.path.abspath(__file__))
    try:
        with open(os.path.join(here, "profiles", "attn_tc_traffic.json")) as f:
            rec = json.load(f)
        h = hashlib.sha256()
        for rel in rec["source_files"]:
            with open(os.path.join(here, rel), "rb") as f:
                h.update(f.read())
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("workload") != workload_name or h.hexdigest() != rec.get("source_sha256"):
        return None
    return int(rec["dram_bytes_per_launch"])


def attn_launches(W, sms: int) -> int:
    """Launches of one attention call: the kernel, plus the merge when a query is split
    (the split rule of the library: SMs per query, at most the tiles and 16)."""
    n_tiles = -(-W.topk // 128) + -(-W.window // 128)
    nsplit = 1 if n_tiles <= 1 else max(1, min(n_tiles, 16, sms // max(1, W.num_q)))
    return 1 + (1 if nsplit > 1 else 0)


def coalesce_io(dw):
    """Lays out the step's per-layer inputs and outputs as slices of a few contiguous device
    tensors, as a caller that feeds whole steps would hold them: all layers' Q, indexer Q and
    weights, window rows and outputs each in one tensor.  The end-to-end copies are then one
    transfer per kind instead of one per layer.  Runs before any graph capture (graphs keep
    the pointers); returns the tensors by name."""
    import torch
    Ls = dw.layers
    io = {"q": torch.stack([L.q for L in Ls]), "swa": torch.stack([L.swa for L in Ls]),
          "out": torch.stack(dw.out)}
    ix = [L for L in Ls if L.qI is not None]
    if ix:
        io["qI"] = torch.stack([L.qI for L in ix])
        io["w"] = torch.stack([L.w for L in ix])
    for i, L in enumerate(Ls):
        L.q, L.swa = io["q"][i], io["swa"][i]
    for j, L in enumerate(ix):
        L.qI, L.w = io["qI"][j], io["w"][j]
    dw.out = [io["out"][i] for i in range(len(Ls))]
    return io


class Timed:
    """A workload on the device with its step captured as CUDA graphs: the append, then the
    whole layer schedule, each layer one csa2_layer_step call (index by its mode, then
    attention).  Two more graphs hold the Full index call alone and the attention calls
    alone, for their rooflines."""

    def __init__(self, W, dev, stream, indexer_e4m3=False):
        import torch
        from fp4_kv_cache_03_b200 import csa2, synth
        from fp4_kv_cache_03_b200.workload import DeviceWorkload
        self.W, self.stream = W, stream
        self.dw = dw = DeviceWorkload(W, device=dev, indexer_e4m3=indexer_e4m3)
        self.io = coalesce_io(dw)
        self.full_li = W.modes.index(synth.FULL)
        build_pool = W.pool_blocks > 0

        def part_append():
            dw.append(stream=stream)

        def part_schedule():                       # (the append has its own graph)
            dw.run_step(stream=stream, attention=True, via_layer_step=True, append=False)

        def part_full():
            L = dw.layers[self.full_li]
            csa2.index_full(L.qI, L.w, dw.idx_k, dw.seqs, W.topk, dw.indices[0], dw.ws_full,
                            dw.max_visible, q_visible=dw.q_visible,
                            pool_blocks=W.pool_blocks if build_pool else 0, block=W.block,
                            pool=dw.pool if build_pool else None, stream=stream)

        def part_attention():
            latest, n_idx = dw.indices[0], 1
            for li, L in enumerate(dw.layers):
                if L.mode == synth.REINDEX:
                    latest = dw.indices[n_idx]
                    n_idx += 1
                dw.attend(li, latest, stream=stream)

        self.parts = (part_append, part_schedule) if W.append else (part_schedule,)
        self.graphs = []
        with torch.cuda.stream(stream):
            for fn in self.parts:                      # eager once before capture
                fn()
            stream.synchronize()
            for fn in self.parts:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    fn()
                self.graphs.append(g)
            self.g_attn = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_attn, stream=stream):
                part_attention()
            self.g_full = torch.cuda.CUDAGraph()
            with torch.cuda.graph(self.g_full, stream=stream):
                part_full()
        stream.synchronize()
        st = dw.status()
        if st != csa2.OK:
            raise csa2.CSA2Error(st, f"{W.name}: warm-up step")

    def release(self):
        self.graphs = []
        self.g_attn = self.g_full = None

    def replay_step(self):
        for g in self.graphs:
            g.replay()

    def time_steps(self, steps, warmup, flush):
        """Per-step device times (ms), L2 flushed between steps."""
        import torch
        evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        with torch.cuda.stream(self.stream):
            for k in range(-warmup, steps):
                flush.zero_()
                if k >= 0: evs[k][0].record(self.stream)
                self.replay_step()
                if k >= 0: evs[k][1].record(self.stream)
        self.stream.synchronize()
        return [a.elapsed_time(b) for a, b in evs]

    def time_graph(self, g, reps, flush):
        """Mean device time (s) of one replay of graph g, L2 flushed between replays."""
        import torch
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(reps)]
        with torch.cuda.stream(self.stream):
            for k in range(-3, reps):
                flush.zero_()
                if k >= 0: ev[k][0].record(self.stream)
                g.replay()
                if k >= 0: ev[k][1].record(self.stream)
        self.stream.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / 1e3 / reps


def workload_summary(Ts, steps, warmup, flush, hbm, tflops, sms, name=None):
    """Throughput and rooflines of a workload made of one or more groups (each a Timed),
    from their graphs; a step runs every group's step in turn."""
    import torch
    from fp4_kv_cache_03_b200 import csa2, synth
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    stream = Ts[0].stream
    with torch.cuda.stream(stream):
        for k in range(-warmup, steps):
            flush.zero_()
            if k >= 0: evs[k][0].record(stream)
            for T in Ts:
                T.replay_step()
            if k >= 0: evs[k][1].record(stream)
    stream.synchronize()
    t_step = statistics.mean(a.elapsed_time(b) for a, b in evs) / 1e3
    units = sum(T.W.num_q * len(T.W.modes) for T in Ts)
    T = Ts[0]
    W = T.W
    n_layers = len(W.modes)
    t_full = T.time_graph(T.g_full, max(3, min(steps, 50)), flush)
    t_attn = T.time_graph(T.g_attn, max(3, min(steps, 50)), flush) / n_layers
    for Tg in Ts:
        st = Tg.dw.status()
        if st != csa2.OK:
            raise csa2.CSA2Error(st, f"{Tg.W.name}: timed steps")
    ib, ab = index_bytes(W, 1 if T.dw.indexer_e4m3 else 2), attn_alg_bytes(W)
    n_index = sum(1 for m in W.modes if m != synth.REUSE)
    per_group = (1 if W.append else 0) + 3 * n_index + n_layers * attn_launches(W, sms)
    return {
        "workload": name or W.name, "value": units / t_step, "unit": UNIT,
        "ms_per_step": t_step * 1e3, "layer_steps_per_step": units, "steps": steps,
        "groups": len(Ts), "indexer_k": "e4m3" if T.dw.indexer_e4m3 else "bf16",
        "index_full": {"ms_per_call": t_full * 1e3, "alg_bytes": ib, "achieved_gbs": ib / t_full / 1e9,
                       "frac_hbm": ib / t_full / 1e9 / hbm,
                       "tflops": index_flops(W) / t_full / 1e12},
        "attention": {"ms_per_call": t_attn * 1e3, "queries": W.num_q, "alg_bytes": ab,
                      "achieved_gbs": ab / t_attn / 1e9, "frac_hbm": ab / t_attn / 1e9 / hbm,
                      "tflops": attn_flops(W) / t_attn / 1e12,
                      "frac_bf16_peak": attn_flops(W) / t_attn / 1e12 / tflops},
        "gpu_launches_per_step": per_group * len(Ts),
    }


def compressor_summary(dev, stream, flush, hbm, tflops, steps):
    """The encoder's sequence compressor fused with the append (csa2_compress_append) at the
    encoder chunk's size: 65,536 tokens of 512 at ratio 2 -> 32,768 FP4 entries of 512."""
    import torch
    from fp4_kv_cache_03_b200 import csa2, synth
    n, m, D_in, D = 32768, 2, 512, 512
    bf = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(torch.bfloat16)
    x = bf(synth.compressor_tokens(11, n * m, D_in))
    w_t = bf(synth.compressor_map(11, D, m * D_in))
    dst = torch.arange(n, dtype=torch.int64, device=dev)
    codes = torch.zeros(n, D // 2, dtype=torch.uint8, device=dev)
    scales = torch.zeros(n, D // 16, dtype=torch.uint8, device=dev)
    ws = csa2.workspace(csa2.quant_append_workspace(), dev)
    with torch.cuda.stream(stream):
        csa2.compress_append(x, m, w_t, dst, codes, scales, ws, stream=stream)
        stream.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            csa2.compress_append(x, m, w_t, dst, codes, scales, ws, stream=stream)
    stream.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    with torch.cuda.stream(stream):
        for k in range(-3, steps):
            flush.zero_()
            if k >= 0: ev[k][0].record(stream)
            g.replay()
            if k >= 0: ev[k][1].record(stream)
    stream.synchronize()
    if csa2.status_fetch(ws) != csa2.OK:
        raise csa2.CSA2Error(csa2.status_fetch(ws), "compress_append")
    t = sum(a.elapsed_time(b) for a, b in ev) / 1e3 / steps
    flops = 2.0 * n * m * D_in * D
    nbytes = n * m * D_in * 2 + D * m * D_in * 2 + n * (D // 2 + D // 16) + n * 8
    return {"workload": "compress_append (65,536 tokens x 512 -> 32,768 FP4 entries, ratio 2)",
            "ms_per_call": t * 1e3, "steps": steps, "gpu_launches_per_step": 1,
            "tflops": flops / t / 1e12, "frac_bf16_peak": flops / t / 1e12 / tflops,
            "alg_bytes": nbytes, "achieved_gbs": nbytes / t / 1e9, "frac_hbm": nbytes / t / 1e9 / hbm}


def run_ours(args, rank, world, local_rank):
    import torch
    from fp4_kv_cache_03_b200 import csa2, synth

    torch.cuda.set_device(local_rank)
    dev = f"cuda:{local_rank}"
    W = synth.workload(args.workload)
    stream = torch.cuda.Stream(device=dev)
    sms = csa2.device_sms()
    hbm, tflops, src = peaks()
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    T = Timed(W, dev, stream)
    dw = T.dw
    n_layers = len(W.modes)

    # --- the timed steps of the headline workload ---
    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            flush.zero_()
            T.replay_step()
    stream.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    props = torch.cuda.get_device_properties(local_rank)
    uuid = getattr(props, "uuid", None)
    clocks = ClockSampler(f"GPU-{uuid}" if uuid is not None else local_rank)
    clocks.start()
    step_ms = T.time_steps(args.steps, 0, flush)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    t_total = max_over_ranks(sum(step_ms) / 1e3, dev)
    st = dw.status()
    if st != csa2.OK:
        raise csa2.CSA2Error(st, "timed steps")

    # --- e2e through the API with host buffers: inputs H2D each step, results D2H ---
    pin = lambda t: t.detach().cpu().pin_memory()
    # (the step's inputs and outputs are held as a few contiguous tensors: coalesce_io)
    io = T.io
    h_in = []
    if W.append:
        h_in += [(pin(dw.append_x), dw.append_x), (pin(dw.append_k), dw.append_k)]
    h_in.append((pin(io["q"]), io["q"]))
    new_rows = io["swa"][:, -1]                        # every layer's new window row
    h_in.append((pin(new_rows), new_rows))
    if "qI" in io:
        h_in += [(pin(io["qI"]), io["qI"]), (pin(io["w"]), io["w"])]
    h_out = [(torch.empty_like(io["out"], device="cpu").pin_memory(), io["out"])]
    h2d = sum(h.numel() * h.element_size() for h, _ in h_in)
    d2h = sum(h.numel() * h.element_size() for h, _ in h_out)
    e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    with torch.cuda.stream(stream):
        for k in range(args.steps):
            flush.zero_()
            e2e_ev[k][0].record(stream)
            for h, d in h_in:
                d.copy_(h, non_blocking=True)
            T.replay_step()
            for h, d in h_out:
                h.copy_(d, non_blocking=True)
            e2e_ev[k][1].record(stream)
    stream.synchronize()
    e2e_t = max_over_ranks(sum(e[0].elapsed_time(e[1]) for e in e2e_ev) / 1e3, dev)

    # --- the dominant op, sparse attention, and the Full index: their own graphs ---
    t_attn = T.time_graph(T.g_attn, max(3, min(args.steps, 200)), flush) / n_layers
    t_full = T.time_graph(T.g_full, max(3, min(args.steps, 200)), flush)
    ab = attn_alg_bytes(W)
    attn_achieved = ab / t_attn / 1e9
    ib = index_bytes(W)
    achieved = ib / t_full / 1e9
    value = job_throughput(args.steps, world, n_layers * W.num_q, t_total)
    n_index = sum(1 for m in W.modes if m != synth.REUSE)
    launches_per_step = (1 if W.append else 0) + 3 * n_index + n_layers * attn_launches(W, sms)
    peak_source = f"{src} (MEASURED_PEAKS.json hbm_gbs)" if src == "measured" else src
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16/fp4->fp32",
        "data": "synthetic (seeded; shapes of the pages' decoder, no weights)",
        "config": {"workload": W.name,
                   "context_entries": W.lengths[0] if W.num_seqs == 1 else
                   f"{W.num_seqs} sequences, {int(np.sum(W.lengths))} in all",
                   "layers": n_layers, "schedule": schedule_of(W.modes), "batch": W.num_q,
                   "D": W.D, "H": W.H, "indexer": f"{W.H_I}x{W.d_I}", "topk": W.topk,
                   "window": W.window,
                   "pool": f"{W.pool_blocks}x{W.block}" if W.pool_blocks else "none",
                   "l2": "flushed between timed steps (256 MB write)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"kernel": "csa2_sparse_attn (attn_tc_kernel + merge), one layer call",
                     "bound": "hbm", "achieved": attn_achieved, "peak": hbm, "unit": "GB/s",
                     "frac": attn_achieved / hbm, "traffic": captured_attn_traffic(W.name),
                     "traffic_note": "attn_tc_kernel's dram__bytes_read.sum + dram__bytes_write.sum per launch "
                                     "from the committed ncu capture of these sources (null when they changed)",
                     "peak_source": peak_source,
                     "alg_bytes_per_launch": ab, "alg_bytes_note": "per query: 512 FP4 rows x 288 B + 128 window rows + Q + out, bf16",
                     "fp32_out_extra_bytes": W.num_q * W.H * W.D * 2,
                     "ms_per_launch": t_attn * 1e3,
                     "note": "one decode query: a latency-bound chain; the batched workloads below show the throughput regime"},
        "roofline_index_full": {"kernel": "csa2_index_full (clear + score scan + Top-K + pool select)",
                                "bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                                "frac": achieved / hbm, "alg_bytes_per_launch": ib,
                                "ms_per_launch": t_full * 1e3},
        "e2e": {"value": job_throughput(args.steps, world, n_layers * W.num_q, e2e_t), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    T.release()
    del T, dw
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()

    # --- the other workloads, same run, same timing rules (fewer steps) ---
    if not args.no_extras and world == 1:
        extras = {}
        k = max(3, min(args.steps, 20))
        # name: (member workloads, E4M3 indexer K)
        groups = {"decoder_step_1m": (("decoder_step_1m",), False),
                  "decoder_step_128k_e4m3_indexer": (("decoder_step_128k",), True),
                  "decoder_step_1m_e4m3_indexer": (("decoder_step_1m",), True),
                  "ragged_decode": (("ragged_decode",), False),
                  "encoder_stack": (synth.ENCODER_STACK, False)}
        for name, (members, e4m3) in groups.items():
            if name == W.name:
                continue
            Ts = [Timed(synth.workload(m), dev, stream, indexer_e4m3=e4m3) for m in members]
            extras[name] = workload_summary(Ts, k, 3, flush, hbm, tflops, sms, name=name)
            for Tg in Ts:
                Tg.release()
            del Ts
            torch.cuda.synchronize(dev)
            torch.cuda.empty_cache()
        extras["compress_append"] = compressor_summary(dev, stream, flush, hbm, tflops, k)
        line["workloads"] = extras
        if "decoder_step_1m" in extras:
            x = extras["decoder_step_1m"]
            line["value_1m"] = x["value"]
            line["roofline_index_full_1m"] = {"achieved": x["index_full"]["achieved_gbs"], "peak": hbm,
                                              "unit": "GB/s", "frac": x["index_full"]["frac_hbm"],
                                              "alg_bytes_per_launch": x["index_full"]["alg_bytes"],
                                              "ms_per_launch": x["index_full"]["ms_per_call"]}
        line["gpu_launches"] += sum(x["gpu_launches_per_step"] * x["steps"] for x in extras.values())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        ls, t, what = oracle_sample(W, args.cpu_seconds)
        line["cpu_baseline"] = {"value": ls / t, "unit": UNIT, "cores": cpu_threads(),
                                "kind": "oracle", "sample": what}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="decoder_step_128k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="time only --workload (skip the 1M, ragged and encoder workloads)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    if world > 1:
        import datetime

        import torch
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
