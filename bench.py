#!/usr/bin/env python
"""Benchmark of the MSA decode step: tokens/s at 32K context x 32 streams on
one B200 (or N replicas, one per GPU, for --gpus N), and the achieved HBM
bandwidth of the step and of its dominant kernel.

A step is one pass of the whole hot path over one batch of decode queries:
append the new token's indexer key and K/V rows, fused block scores
(score + causal mask + maxpool + local bias), top-16 selection and the
block-sparse attention, all through the C ABI.  Every step re-appends the
token at the last slot and queries there, so each step is the same work.
Inputs (2.1 GB of F32 indexer keys + 2.1 GB of bf16 K/V per GPU) are larger
than the 126 MB L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  Multi-GPU runs (torchrun) shard independent
streams: each rank holds its own 32 streams (weak scaling, no collective on
the data path; one all-reduce of the timing at the end).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "MSA decode tokens/s @32K ctx x32 streams; achieved HBM GB/s vs peak"
WORKLOAD = W.DECODE_32K_X32

# DRAM traffic of one block-scores launch on the 32-stream workload, per key
# type, from the ncu captures summarised in
# profiles/block_scores_gemv_decode_8x32k.md: bytes read + written on 8
# streams, scaled by 4 to 32 streams (the reads grow in proportion to the
# keys scanned).  Valid only for the kernel source it was taken on (sha256
# prefix of msa_scores_gemv.cuh); any other source reports null.
SCORES_TRAFFIC = {"source_sha": "b9bc1ca3c5d4d5a4",
                  "bytes_per_launch": {"f32": 4 * (536_911_872 + 3_886_848), "f16": 4 * (268_474_112 + 2_967_040)}}

# The same for the token-score kernel of the token-level variant, from the
# 16-stream capture summarised in profiles/dsa_token_scores_decode_16x32k.md,
# scaled by 2 to 32 streams (sha256 prefix of msa_dsa_scores.cuh).
DSA_SCORES_TRAFFIC = {"source_sha": "6c6fa9e892144930", "bytes_per_launch": 2 * (134_557_696 + 5_160_960)}


def variant_metric(metric: str, args) -> str:
    """The metric name, marked with the cache variant a run uses."""
    tags = ((["F16 indexer cache"] if args.idx_f16 else []) + (["paged caches"] if args.paged else [])
            + (["one fused kernel"] if getattr(args, "fused", False) else []))
    return metric.replace("x32 streams", "x32 streams, " + ", ".join(tags)) if tags else metric


def scores_source_sha(name: str = "msa_scores_gemv.cuh") -> str:
    p = os.path.join(ROOT, "block_sparse_attention_maxpool_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "src": "fallback"}


# ---------------------------------------------------------------------------
# algorithmic bytes
# ---------------------------------------------------------------------------
def scores_bytes(w, key_bytes: int = 4) -> int:
    """Bytes the block-score kernel must move per launch: every visible
    indexer key once (512 B per key per group; 256 B with the F16 cache),
    the indexer queries, and the block-score output."""
    G, Di = w.n_kv_heads, w.idx_dim
    n_q = w.n_queries
    keys = n_q * G * w.l_total * Di * key_bytes   # decode: each query sees l_total keys
    return keys + n_q * G * Di * 4 + n_q * G * (w.capacity // w.block) * 4


def dsa_scores_bytes(w, n_index_heads: int = 64) -> int:
    """Bytes the token-score kernel must move per launch: every visible fp16
    indexer key once (256 B), each query's fp16 head vectors and weights,
    and the float32 score row it writes."""
    Di = w.idx_dim
    per_q = w.l_total * Di * 2 + n_index_heads * Di * 2 + n_index_heads * 4 + w.capacity * 4
    return per_q * w.n_queries


def dsa_step_bytes(w, top_k: int = 2048, n_index_heads: int = 64) -> int:
    """Bytes one token-level decode step must move: the token scores (keys
    in, scores out), the score row read back by the top-k, the kept tokens'
    K/V rows of every group, the selection, query and output."""
    G, D = w.n_kv_heads, w.head_dim
    kept = min(top_k, w.l_total)
    per_q = (w.capacity * 4 + kept * G * D * 2 * 2 + 2048 * 4 * 2 + w.n_q_heads * D * 2 * 2)
    return dsa_scores_bytes(w, n_index_heads) + per_q * w.n_queries


def step_bytes(w, key_bytes: int = 4) -> int:
    """Bytes one decode step must move: visible indexer keys, the 16 selected
    K/V blocks per group, the query and the output (the plan's per-stream
    count: 67,108,864 + 4,194,304 + 34,816 at 32K context)."""
    G, D = w.n_kv_heads, w.head_dim
    idx = w.l_total * G * w.idx_dim * key_bytes
    kv = min(w.top_k, w.l_total // w.block + 1) * w.block * G * D * 2 * 2
    qo = w.n_q_heads * D * 2 * 2 + G * w.idx_dim * 4
    return (idx + kv + qo) * w.n_streams


# ---------------------------------------------------------------------------
# multi-GPU: replicas over disjoint streams, timing reduced by max
# ---------------------------------------------------------------------------
def shard_streams(streams_per_rank: int, rank: int) -> range:
    """Global ids of the decode streams rank `rank` owns: each rank holds its
    own contiguous run of independent streams (no data crosses GPUs)."""
    return range(rank * streams_per_rank, (rank + 1) * streams_per_rank)


def max_over_ranks(values, device=None) -> list[float]:
    """Element-wise maximum of per-rank timings (slowest rank decides)."""
    import torch.distributed as dist
    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(streams_per_rank: int, world: int, ms_per_step: float) -> float:
    """Whole-job decode throughput: one token per stream per step on every rank."""
    return streams_per_rank * world / (ms_per_step * 1e-3)


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    """Samples SM clock and throttle reasons with nvidia-smi every 200 ms."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device: int):
        self.rows = []
        self.proc = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def mark(self):
        return len(self.rows)

    def stop(self, since: int = 0) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = [r for r in self.rows[since:] if len(r) >= 8] or [r for r in self.rows if len(r) >= 8]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def run_ours(args, rank, world, dev):
    import block_sparse_attention_maxpool_b200 as msa
    from block_sparse_attention_maxpool_b200 import build as msa_build

    if rank == 0:
        msa_build.build()
    if world > 1:
        torch.distributed.barrier(device_ids=[dev])
    w = W.WORKLOADS[args.workload]
    if args.streams is not None and args.streams != w.n_streams:    # smaller case for profiler captures
        w = W.Workload(f"{w.name}_{args.streams}streams", args.streams, w.l_existing, w.l_total, w.queries,
                       quantize_idx=w.quantize_idx)
    prefill = w.queries == "new"
    shape = msa.Shape(n_streams=w.n_streams, capacity=w.capacity)
    if args.dsa:                                # token-level variant: lightning-indexer inputs
        dinp = W.make_dsa_inputs(w, streams=shard_streams(w.n_streams, rank))
        inp = dinp.base
        names = ("k_cache", "v_cache", "tok_stream", "tok_pos", "k_new", "v_new", "q_stream", "q_pos", "q")
    else:
        inp = W.make_inputs(w, streams=shard_streams(w.n_streams, rank))   # this rank's own streams
        names = ("idx_k_cache", "k_cache", "v_cache", "tok_stream", "tok_pos", "idx_k_new", "k_new", "v_new",
                 "q_stream", "q_pos", "idx_q", "q")
    d = {n: getattr(inp, n).to(dev) for n in names}
    if args.dsa:
        d["k_idx_cache"] = dinp.k_idx_cache.half().to(dev)
        d["k_idx_new"] = dinp.k_idx_new.to(dev)
        d["q_idx"] = dinp.q_idx.to(dev)
        d["weights"] = dinp.weights.to(dev)
        del dinp
    pages = None
    if args.paged:
        # the same caches as shuffled page pools behind a block table
        lay = W.page_layout(inp, seed=rank)
        d["idx_k_cache"], d["k_cache"], d["v_cache"] = (lay.idx_pool.to(dev), lay.k_pool.to(dev),
                                                      lay.v_pool.to(dev))
        pages = msa.Pages(lay.block_table.to(dev), lay.n_pages)
        del lay
    del inp
    if args.idx_f16:
        d["idx_k_cache"] = d["idx_k_cache"].half()         # F16 indexer-key cache variant
    key_bytes = 2 if args.idx_f16 else 4
    n_q = w.n_queries
    G = w.n_kv_heads
    dshape = msa.DsaShape(n_streams=w.n_streams, capacity=w.capacity)
    bufs = {
        "block_scores": torch.empty((n_q, G, shape.n_blocks), dtype=torch.float32, device=dev),
        "sel": torch.empty((n_q, G, shape.top_k), dtype=torch.int32, device=dev),
        "n_sel": torch.empty((n_q, G), dtype=torch.int32, device=dev),
        "scores": torch.empty((n_q, w.capacity) if args.dsa else (1,), dtype=torch.float32, device=dev),
        "tok_sel": torch.empty((n_q, msa.DSA_SEL_WIDTH) if args.dsa else (1,), dtype=torch.int32, device=dev),
        "tok_n": torch.empty((n_q,), dtype=torch.int32, device=dev),
        "out": torch.empty((n_q, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=dev),
    }
    mode = msa.MODE_PREFILL if prefill else msa.MODE_DECODE
    ws = msa.msa_workspace_bytes(shape, n_q, mode)
    bufs["workspace"] = torch.empty((max(ws, 16),), dtype=torch.uint8, device=dev)
    # kernels per step: 2 appends, block scores (1 streaming kernel, or 6 on the
    # tensor-core tile path of prefill batches), select, attention (+ combine in decode)
    tiles = n_q >= 256 and n_q >= 64 * w.n_streams
    launches_per_step = 2 + (6 if tiles else 1) + 1 + (1 if prefill else 2)
    if args.dsa:
        launches_per_step = 2 + 1 + 1 + 2        # appends, token scores, top-k, attention + combine
    stream = torch.cuda.current_stream(dev)
    scale = 1.0 / math.sqrt(shape.head_dim)

    def dsa_append(st):
        msa.msa_dsa_indexer_append(dshape, d["k_idx_cache"], d["k_idx_new"], d["tok_stream"], d["tok_pos"], st)
        msa.msa_kv_append(shape, d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d["tok_stream"],
                          d["tok_pos"], st)

    def dsa_scores(st):
        msa.msa_dsa_token_scores(dshape, d["q_idx"], d["weights"], d["k_idx_cache"], d["q_stream"], d["q_pos"],
                                 bufs["scores"], st)

    def dsa_select(st):
        msa.msa_dsa_select_topk(dshape, bufs["scores"], d["q_pos"], bufs["tok_sel"], bufs["tok_n"], st)

    def dsa_attend(st):
        msa.msa_dsa_sparse_attn_decode(shape, d["q"], d["k_cache"], d["v_cache"], bufs["tok_sel"], d["q_stream"],
                                       d["q_pos"], scale, bufs["out"], bufs["workspace"], st)

    def part_append(st):
        append = msa.msa_indexer_append_f16 if args.idx_f16 else msa.msa_indexer_append
        append(shape, d["idx_k_cache"], d["idx_k_new"], d["tok_stream"], d["tok_pos"], st, pages)
        msa.msa_kv_append(shape, d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d["tok_stream"],
                          d["tok_pos"], st, pages)

    def part_scores(st):
        msa.msa_block_scores(shape, d["idx_q"], d["idx_k_cache"], d["q_stream"], d["q_pos"],
                             bufs["block_scores"], st, bufs["workspace"], pages)

    def part_select(st):
        msa.msa_select_topk(shape, bufs["block_scores"], d["q_pos"], bufs["sel"], bufs["n_sel"], st)

    def part_attend(st):
        attn = msa.msa_sparse_attn_prefill if prefill else msa.msa_sparse_attn_decode
        attn(shape, d["q"], d["k_cache"], d["v_cache"], bufs["sel"], d["q_stream"], d["q_pos"], scale,
             bufs["out"], bufs["workspace"], st, pages)

    if args.dsa:
        part_append, part_scores, part_select, part_attend = dsa_append, dsa_scores, dsa_select, dsa_attend
    if args.fused:                                   # the whole step as one persistent kernel
        bufs["workspace_fused"] = torch.empty((msa.msa_decode_step_fused_workspace_bytes(shape, n_q),),
                                              dtype=torch.uint8, device=dev)
        launches_per_step = 1

        def part_append(st):                         # noqa: F811
            pass

        def part_scores(st):                         # noqa: F811
            msa.decode_step_fused(shape, {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}, d, bufs, st)

        def part_select(st):                         # noqa: F811
            pass

        def part_attend(st):                         # noqa: F811
            pass

    # the kernel the roofline line describes: attention in prefill batches
    # (most of the step), the score kernel otherwise
    parts = [part_append, part_scores, part_select, part_attend]
    timed = 3 if (prefill and not args.dsa and not args.fused) else 1

    def step(ev=None):
        for i, part in enumerate(parts):
            if ev is not None and i == timed:
                ev[0].record(stream)
            part(stream)
            if ev is not None and i == timed:
                ev[1].record(stream)

    clocks = ClockSampler(dev) if rank == 0 else None
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if msa.msa_get_device_error(stream) != 0:
        raise RuntimeError("device error during warm-up")
    graphs = None
    if not args.no_graph:
        # The step's launches captured once and replayed: the same kernels on
        # the same buffers, without per-launch host work.  One graph per part,
        # so events between them still time the roofline kernel on its own.
        graphs = [torch.cuda.CUDAGraph() for _ in range(4)]
        for i, (g, part) in enumerate(zip(graphs, parts)):
            if args.fused and i != 1:                        # the fused step is one kernel: one graph
                graphs[i] = None
                continue
            with torch.cuda.graph(g):
                part(None)
        torch.cuda.synchronize(dev)

        def step(ev=None):                                   # noqa: F811  (graph replay)
            for i, g in enumerate(graphs):
                if ev is not None and i == timed:
                    ev[0].record(stream)
                if g is not None:
                    g.replay()
                if ev is not None and i == timed:
                    ev[1].record(stream)
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)

    # ---- device-resident timing -------------------------------------------
    kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier(device_ids=[dev])
    torch.cuda.synchronize(dev)
    mark = clocks.mark() if clocks else 0
    t0.record(stream)
    for i in range(args.steps):
        step(kev[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if world > 1:
        torch.distributed.barrier(device_ids=[dev])
    ms = t0.elapsed_time(t1) / args.steps
    k_ms = statistics.mean(a.elapsed_time(b) for a, b in kev)

    # ---- end to end: host inputs in, host output out, every step ------------
    host_names = ("tok_stream", "tok_pos", "idx_k_new", "k_new", "v_new", "q_stream", "q_pos", "idx_q", "q")
    if args.dsa:
        host_names = ("tok_stream", "tok_pos", "k_idx_new", "k_new", "v_new", "q_stream", "q_pos", "q_idx",
                      "weights", "q")
    host = {n: d[n].cpu().pin_memory() for n in host_names}
    h_out = torch.empty(bufs["out"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = max(3, min(args.steps, 200 if not prefill else 20))

    def api_step():
        for part in parts:
            part(stream)

    e2e_launch = "direct"
    pipe = None
    if not args.no_graph:
        if not (args.dsa or args.fused):
            # the public pipelined replay: two captures of the step alternate,
            # each step's packed inputs go in on one copy stream and its output
            # comes back on another while the neighbouring steps run
            pipe = msa.StepPipeline(shape, {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}, d,
                                    prefill, pages)
            packed = pipe.pack(host, pipe.host_buffer())
            host_names = ()                                     # the packed buffer carries every input
            h2d = packed.numel()

            def api_step():                                     # noqa: F811
                pipe.step(packed)                               # inputs in, replay, output out
        else:
            g_api = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_api):
                for part in parts:
                    part(None)
            api_step = g_api.replay                             # noqa: F811
        e2e_launch = "cuda graphs, transfers overlapped with the neighbouring steps" if pipe else "cuda graph"

    for _ in range(3):
        for n in host_names:
            d[n].copy_(host[n], non_blocking=True)
        api_step()
        if pipe is None:
            h_out.copy_(bufs["out"], non_blocking=True)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        for n in host_names:
            d[n].copy_(host[n], non_blocking=True)
        api_step()
        if pipe is None:
            h_out.copy_(bufs["out"], non_blocking=True)
    if pipe is not None:
        pipe.wait_all()                                         # the last outputs are on the host
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if msa.msa_get_device_error(stream) != 0:
        raise RuntimeError("device error during timing")
    clk = clocks.stop(mark) if clocks else None

    ms, e2e_ms, k_ms = max_over_ranks([ms, e2e_ms, k_ms], device=dev)
    if rank != 0:
        return None

    peaks = load_peaks()
    if args.dsa:
        line = dsa_line(args, w, world, ms, k_ms, e2e_ms, e2e_steps, h2d, d2h, launches_per_step, clk, peaks,
                        graphs)
        line["e2e"]["launch"] = e2e_launch
        return line
    if prefill:
        line = prefill_line(args, w, world, ms, k_ms, e2e_ms, e2e_steps, h2d, d2h, launches_per_step, clk, peaks,
                            graphs)
        line["e2e"]["launch"] = e2e_launch
        return line
    sbytes = scores_bytes(w, key_bytes) if not args.fused else step_bytes(w, key_bytes)
    achieved = sbytes / (k_ms * 1e-3) / 1e9
    traffic = None
    if SCORES_TRAFFIC["source_sha"] == scores_source_sha() and w == WORKLOAD and not args.paged and not args.fused:
        traffic = SCORES_TRAFFIC["bytes_per_launch"]["f16" if args.idx_f16 else "f32"]   # this workload only
    step_gbs = step_bytes(w, key_bytes) / (ms * 1e-3) / 1e9
    line = {
        "metric": variant_metric(METRIC, args),
        "value": job_tokens_per_s(w.n_streams, world, ms),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": ("f16" if args.idx_f16 else "f32") + " indexer / bf16 attention (f32 accumulate)",
        "data": "synthetic (seeded N(0,1) K/V/Q bf16, indexer N(0,1)/sqrt(128) f32)",
        "config": {"workload": w.name, "streams_per_gpu": w.n_streams, "context": w.l_total,
                   "launch": "cuda graphs" if graphs is not None else "direct",
                   "caches": "paged (shuffled pages + block table)" if args.paged else "contiguous",
                   "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                   "block": w.block, "top_k": w.top_k, "parallelism": f"replicas{world}",
                   "l2": f"inputs {2 * w.n_streams * w.capacity * w.n_kv_heads * 512 / 1e9:.1f} GB per GPU > 126 MB L2, no flush"},
        "step_hbm": {"achieved_gbs": step_gbs, "peak_gbs": peaks["hbm_gbs"],
                     "frac": step_gbs / peaks["hbm_gbs"], "bytes_per_step": step_bytes(w, key_bytes)},
        "roofline": {"kernel": "decode_step_fused" if args.fused else "block_scores_gemv", "bound": "hbm",
                     "achieved": achieved,
                     "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic, "algorithmic_bytes": sbytes, "ms_per_launch": k_ms,
                     "peak_src": peaks["src"]},
        "e2e": {"value": job_tokens_per_s(w.n_streams, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps,
                "launch": e2e_launch},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }
    return line


DSA_METRIC = ("MSA token-level variant (lightning indexer, 64 heads, top-2048 tokens) decode tokens/s "
              "@32K ctx x32 streams; achieved HBM GB/s vs peak")


def dsa_line(args, w, world, ms, k_ms, e2e_ms, e2e_steps, h2d, d2h, launches_per_step, clk, peaks, graphs):
    sbytes = dsa_scores_bytes(w)
    traffic = None
    if DSA_SCORES_TRAFFIC["source_sha"] == scores_source_sha("msa_dsa_scores.cuh") and w == WORKLOAD:
        traffic = DSA_SCORES_TRAFFIC["bytes_per_launch"]
    achieved = sbytes / (k_ms * 1e-3) / 1e9
    step_gbs = dsa_step_bytes(w) / (ms * 1e-3) / 1e9
    return {
        "metric": DSA_METRIC if w == WORKLOAD else DSA_METRIC.replace("@32K ctx x32 streams", f"({w.name})"),
        "value": job_tokens_per_s(w.n_streams, world, ms), "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None,
        "dtype": "f16 indexer (f32 accumulate) / bf16 attention (f32 accumulate)",
        "data": "synthetic (seeded N(0,1) K/V/Q bf16; indexer keys and heads N(0,1)/sqrt(128) fp16, "
                "weights N(0,1)/8 f32)",
        "config": {"workload": w.name, "variant": "token-level (lightning indexer)", "streams_per_gpu": w.n_streams,
                   "context": w.l_total, "index_heads": 64, "top_k_tokens": 2048, "relu": True,
                   "launch": "cuda graphs" if graphs is not None else "direct",
                   "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
                   "parallelism": f"replicas{world}",
                   "l2": f"inputs {w.n_streams * w.capacity * (256 + w.n_kv_heads * 512) / 1e9:.1f} GB per GPU "
                         "> 126 MB L2, no flush"},
        "step_hbm": {"achieved_gbs": step_gbs, "peak_gbs": peaks["hbm_gbs"], "frac": step_gbs / peaks["hbm_gbs"],
                     "bytes_per_step": dsa_step_bytes(w)},
        "roofline": {"kernel": "dsa_scores", "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                     "algorithmic_bytes": sbytes, "ms_per_launch": k_ms, "peak_src": peaks["src"]},
        "e2e": {"value": job_tokens_per_s(w.n_streams, world, e2e_ms), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }


def prefill_flops(w) -> tuple[int, int]:
    """Algorithmic FLOPs of one prefill step: the indexer contraction over
    each query's visible keys (2 * Di per key per group) and the attention
    over each query's attended rows (QK and PV: 4 * D per row per head)."""
    ind = att = 0
    for p in range(w.l_existing, w.l_total):
        nvis = p // w.block + 1
        rows = p + 1 if nvis <= w.top_k else (w.top_k - 1) * w.block + p % w.block + 1
        ind += 2 * w.idx_dim * w.n_kv_heads * (p + 1)
        att += 4 * w.head_dim * w.n_q_heads * rows
    return ind * w.n_streams, att * w.n_streams


def prefill_line(args, w, world, ms, k_ms, e2e_ms, e2e_steps, h2d, d2h, launches_per_step, clk, peaks,
                 graphs=None):
    ind, att = prefill_flops(w)
    tokens = w.n_queries * world
    tf = (ind + att) / (ms * 1e-3) / 1e12
    ktf = att / (k_ms * 1e-3) / 1e12                 # the attention kernel: its algorithmic FLOPs
    kernel = "sparse_attn_prefill_union"
    return {
        "metric": f"MSA prefill tokens/s ({w.name}); achieved TFLOP/s vs bf16 peak",
        "value": tokens / (ms * 1e-3), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 indexer / bf16 attention (f32 accumulate)", "data": "synthetic",
        "config": {"workload": w.name, "streams_per_gpu": w.n_streams, "new_tokens": w.n_new,
                   "context": w.l_total, "parallelism": f"replicas{world}",
                   "caches": "paged (shuffled pages + block table)" if args.paged else "contiguous",
                   "launch": "cuda graphs" if graphs is not None else "direct"},
        "step_tensor": {"achieved_tflops": tf, "peak_tflops": peaks["bf16_tflops"],
                        "frac": tf / peaks["bf16_tflops"], "indexer_flops": ind, "attention_flops": att},
        "roofline": {"kernel": kernel, "bound": "tensor", "achieved": ktf, "peak": peaks["bf16_tflops"],
                     "unit": "TFLOP/s", "frac": ktf / peaks["bf16_tflops"], "traffic": None,
                     "ms_per_launch": k_ms, "peak_src": peaks["src"]},
        "e2e": {"value": tokens / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "steps": e2e_steps},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clk,
    }


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(n_streams: int, seed: int = 0):
    import oracle
    w = WORKLOAD
    inp = W.make_inputs(w, seed=seed, streams=range(n_streams))
    caches = [oracle.indexer_append(c, n, inp.tok_stream, inp.tok_pos)
              for c, n in ((inp.idx_k_cache, inp.idx_k_new), (inp.k_cache, inp.k_new), (inp.v_cache, inp.v_new))]

    def run():
        oracle.msa_step(caches[0], caches[1], caches[2], inp.idx_q, inp.q, inp.q_stream, inp.q_pos,
                        w.block, w.top_k)
    return run


def cpu_baseline(budget_s: float = 10.0, n_streams: int = 8) -> dict:
    run = oracle_sample(n_streams)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": reps * n_streams / el, "unit": "tokens/s", "cores": torch.get_num_threads(),
            "kind": "oracle",
            "sample": f"{n_streams} of the 32 streams of {WORKLOAD.name}, all steps (append, FP64 block "
                      f"scores, selection, attention), repeated {reps}x over {el:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    run = oracle_sample(1)
    for _ in range(args.warmup):
        run()
    budget = 120.0
    times = []
    for _ in range(args.steps):
        t = time.perf_counter()
        run()
        times.append(time.perf_counter() - t)
        if sum(times) > budget:
            break
    ms = 1e3 * sum(times) / len(times)
    value = 1.0 / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": len(times), "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD.name, "streams_per_step": 1},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": torch.get_num_threads(), "kind": "oracle",
                         "sample": f"1 of 32 streams of {WORKLOAD.name} per step (FP64 CPU oracle)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--idx-f16", action="store_true",
                    help="decode with the F16 indexer-key cache variant instead of the F32 cache")
    ap.add_argument("--dsa", action="store_true",
                    help="time the token-level variant (lightning indexer, top-2048 tokens) on the same workload")
    ap.add_argument("--fused", action="store_true",
                    help="run the whole decode step as one persistent kernel (msa_decode_step_fused)")
    ap.add_argument("--paged", action="store_true",
                    help="run the paged calls on the same caches laid out as shuffled page pools")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every kernel from Python in the timed loop instead of replaying CUDA graphs")
    ap.add_argument("--workload", choices=sorted(W.WORKLOADS), default=WORKLOAD.name,
                    help="workload to time (default: the 32-stream 32K decode benchmark)")
    ap.add_argument("--streams", type=int, default=None,
                    help="override the workload's stream count (smaller cases for profiler captures)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    if args.dsa and (args.paged or args.idx_f16 or W.WORKLOADS[args.workload].queries != "last"):
        ap.error("--dsa times decode workloads with contiguous caches")
    if args.fused and (args.paged or args.idx_f16 or args.dsa or W.WORKLOADS[args.workload].queries != "last"):
        ap.error("--fused times decode workloads with contiguous F32 caches")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))

    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        line = run_ours(args, rank, world, local)
        if line is not None:
            if (world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD.name and not args.idx_f16
                    and not args.paged and not args.dsa and not args.fused):
                line["cpu_baseline"] = cpu_baseline()
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
