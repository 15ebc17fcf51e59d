#!/usr/bin/env python
"""Benchmark of the MSA decode step: tokens/s at 32K context x 32 streams on
one B200 (or N replicas, one per GPU, for --gpus N), and the achieved HBM
bandwidth of the step and of its dominant kernel.

A step is one pass of the whole hot path over one batch of queries: append
the new tokens' indexer keys and K/V rows, fused block scores (score + causal
mask + maxpool + local bias), top-16 selection and the block-sparse
attention, all through the C ABI.  Every decode step re-appends the token at
the last slot and queries there, so each step is the same work; two input
sets (different new tokens and queries for the same caches, so different
block selections) alternate from step to step, so that the K/V blocks one
step reads are not the ones the step before left in L2.  Decode inputs (2.1
GB of F32 indexer keys + 2.1 GB of bf16 K/V per GPU) are larger than the 126
MB L2; workloads whose inputs are not have L2 flushed (a 256 MB write)
between timed steps, outside the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` times the step replayed as one
CUDA graph per input set; the dominant kernel's time comes from a second
pass that replays the step's parts as separate graphs with events between
them.  At N = 1 the line also carries the other four workloads
(``workloads``: step time, roofline fraction of their dominant kernels, the
oracle timed on a sample on the host cores, and a sampled oracle check of
the selection with its near-tie count) and the shared-layer step
(``shared_layer``: append + attention reusing a previous layer's selection).
Multi-GPU runs (torchrun) shard independent streams: each rank holds its own
32 streams (weak scaling, no collective on the data path; one all-reduce of
the timing at the end).
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
N_SETS = 2                     # decode input sets alternated between steps
L2_BYTES = 126 * 1024 * 1024
NOMINAL_HBM_GBS = 7700.0       # B200 HBM3e, HGX figure (context beside the measured copy peak)

# DRAM traffic of one block-scores launch on the 32-stream workload, per key
# type: dram__bytes_read.sum + dram__bytes_write.sum of one ncu capture of
# the 8-stream case (one launch), scaled by 4 to 32 streams (the reads grow
# in proportion to the keys scanned).  Each figure is valid only for the
# kernel source it was taken on (sha256 prefix of msa_scores_gemv.cuh); any
# other source reports null.
SCORES_TRAFFIC = {"f32": {"source_sha": "fbcb00edc6a2593a", "bytes_per_launch": 4 * (536_912_896 + 3_008_000)},
                  "f16": {"source_sha": "b9bc1ca3c5d4d5a4", "bytes_per_launch": 4 * (268_474_112 + 2_967_040)}}

# The same for the token-score kernel of the token-level variant, from a
# capture of the 16-stream case, scaled by 2 to 32 streams (sha256 prefix
# of msa_dsa_scores.cuh).
DSA_SCORES_TRAFFIC = {"source_sha": "1f3f0fc92a3f7ca2", "bytes_per_launch": 2 * (134_548_480 + 3_636_992)}


def variant_metric(metric: str, args) -> str:
    """The metric name, marked with the cache variant a run uses."""
    tags = ((["F16 indexer cache"] if args.idx_f16 else []) + (["paged caches"] if args.paged else [])
            + (["one fused kernel"] if getattr(args, "fused", False) else [])
            + (["shared layer: append + attention on a previous layer's selection"]
               if getattr(args, "shared_layer", False) else []))
    return metric.replace("x32 streams", "x32 streams, " + ", ".join(tags)) if tags else metric


def scores_source_sha(name: str = "msa_scores_gemv.cuh") -> str:
    p = os.path.join(ROOT, "block_sparse_attention_maxpool_b200", "csrc", name)
    return hashlib.sha256(open(p, "rb").read()).hexdigest()[:16]


def load_peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


def host_cores() -> int:
    """Host cores this process may run on (the oracle's threads)."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


# ---------------------------------------------------------------------------
# algorithmic bytes and flops
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


def kv_bytes_per_stream(w) -> int:
    """The selected K/V blocks of one decode query, every group."""
    return min(w.top_k, w.l_total // w.block + 1) * w.block * w.n_kv_heads * w.head_dim * 2 * 2


def step_bytes(w, key_bytes: int = 4) -> int:
    """Bytes one decode step must move: visible indexer keys, the 16 selected
    K/V blocks per group, the query and the output (per stream 67,108,864 +
    4,194,304 + 34,816 at 32K context)."""
    G, D = w.n_kv_heads, w.head_dim
    idx = w.l_total * G * w.idx_dim * key_bytes
    qo = w.n_q_heads * D * 2 * 2 + G * w.idx_dim * 4
    return (idx + kv_bytes_per_stream(w) + qo) * w.n_streams


def shared_layer_bytes(w) -> int:
    """Bytes one shared-layer decode step must move: the new K/V rows, the
    selected K/V blocks of every group, the selection, query and output (no
    indexer keys: the selection is the previous layer's)."""
    G, D = w.n_kv_heads, w.head_dim
    per = G * D * 2 * 2 + kv_bytes_per_stream(w) + G * w.top_k * 4 + w.n_q_heads * D * 2 * 2
    return per * w.n_streams


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


def input_bytes(w) -> int:
    """Bytes of the caches and per-step inputs one step reads."""
    cache = w.n_streams * w.capacity * w.n_kv_heads * (w.idx_dim * 4 + w.head_dim * 2 * 2)
    q = w.n_queries * (w.n_kv_heads * w.idx_dim * 4 + w.n_q_heads * w.head_dim * 2)
    return cache + q


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

    def summary(self, since: int = 0, until: int | None = None) -> dict | None:
        rows = [r for r in self.rows[since:until] if len(r) >= 8] or [r for r in self.rows if len(r) >= 8]
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}

    def stop(self, since: int = 0) -> dict | None:
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        return self.summary(since)


# ---------------------------------------------------------------------------
# one workload's step on the device
# ---------------------------------------------------------------------------
STEP_NAMES = ("tok_stream", "tok_pos", "idx_k_new", "k_new", "v_new", "q_stream", "q_pos", "idx_q", "q")


class Step:
    """The inputs, buffers and parts of one workload's step on the device.

    ``parts`` are the step's calls through the C ABI (appends, block scores,
    selection, attention; one call for the fused variant; appends and
    attention for the shared-layer step), each ``part(stream, set_index)``.
    Decode workloads hold ``N_SETS`` input sets for the same caches."""

    def __init__(self, msa, args, w, rank, dev, variant="full", n_sets=N_SETS):
        self.msa, self.w, self.dev, self.variant = msa, w, dev, variant
        self.dsa, self.fused = args.dsa, args.fused
        self.prefill = w.queries == "new"
        self.shape = msa.Shape(n_streams=w.n_streams, capacity=w.capacity, n_q_heads=w.n_q_heads,
                               n_kv_heads=w.n_kv_heads)
        streams = shard_streams(w.n_streams, rank)
        if self.dsa:                                # token-level variant: lightning-indexer inputs
            dinp = W.make_dsa_inputs(w, streams=streams)
            inp = dinp.base
        else:
            inp = W.make_inputs(w, streams=streams)  # this rank's own streams
        self.inp_host = inp
        d = {n: getattr(inp, n).to(dev) for n in ("idx_k_cache", "k_cache", "v_cache") + STEP_NAMES}
        if self.dsa:
            d["k_idx_cache"] = dinp.k_idx_cache.half().to(dev)
            d["k_idx_new"] = dinp.k_idx_new.to(dev)
            d["q_idx"] = dinp.q_idx.to(dev)
            d["weights"] = dinp.weights.to(dev)
            del dinp
        self.pages = None
        if args.paged:
            lay = W.page_layout(inp, seed=rank)          # the same caches as shuffled page pools
            d["idx_k_cache"], d["k_cache"], d["v_cache"] = (lay.idx_pool.to(dev), lay.k_pool.to(dev),
                                                          lay.v_pool.to(dev))
            self.pages = msa.Pages(lay.block_table.to(dev), lay.n_pages)
            del lay
        if args.idx_f16:
            d["idx_k_cache"] = d["idx_k_cache"].half()     # F16 indexer-key cache variant
        self.idx_f16 = args.idx_f16
        self.caches = {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
        # input sets: set 0 is the workload's draw, the others redraw the
        # new tokens and queries (decode, not for the token-level variant)
        self.sets = [d]
        if not self.prefill and not self.dsa and n_sets > 1:
            for k in range(1, n_sets):
                extra = W.make_step_set(w, seed=1000 + k, streams=streams)
                dk = dict(d)
                for n, t in extra.items():
                    dk[n] = t.to(dev)
                self.sets.append(dk)
        n_q, G = w.n_queries, w.n_kv_heads
        sh = self.shape
        self.bufs = {
            "block_scores": torch.empty((n_q, G, sh.n_blocks), dtype=torch.float32, device=dev),
            "sel": torch.empty((n_q, G, sh.top_k), dtype=torch.int32, device=dev),
            "n_sel": torch.empty((n_q, G), dtype=torch.int32, device=dev),
            "scores": torch.empty((n_q, w.capacity) if self.dsa else (1,), dtype=torch.float32, device=dev),
            "tok_sel": torch.empty((n_q, msa.DSA_SEL_WIDTH) if self.dsa else (1,), dtype=torch.int32, device=dev),
            "tok_n": torch.empty((n_q,), dtype=torch.int32, device=dev),
            "out": torch.empty((n_q, sh.n_q_heads, sh.head_dim), dtype=torch.bfloat16, device=dev),
        }
        mode = msa.MODE_PREFILL if self.prefill else msa.MODE_DECODE
        self.bufs["workspace"] = torch.empty((max(msa.msa_workspace_bytes(sh, n_q, mode), 16),), dtype=torch.uint8,
                                             device=dev)
        if self.fused:
            self.bufs["workspace_fused"] = torch.empty((msa.msa_decode_step_fused_workspace_bytes(sh, n_q),),
                                                       dtype=torch.uint8, device=dev)
        # the shared-layer step reads each set's selection from a previous full step
        self.set_sel = [torch.empty_like(self.bufs["sel"]) for _ in self.sets] if variant == "shared" else None
        self.dshape = msa.DsaShape(n_streams=w.n_streams, capacity=w.capacity)
        self.scale = 1.0 / math.sqrt(sh.head_dim)
        tiles = n_q >= 256 and n_q >= 64 * w.n_streams
        if self.dsa:
            self.launches = 2 + 1 + 1 + 1        # appends, token scores, top-k, attention
        elif self.fused:
            self.launches = 1
        elif variant == "shared":
            self.launches = 1 + 1                # K/V append, attention
        else:
            appends = 2 if args.idx_f16 else 1
            # decode: selection and merges inside the attention kernel; prefill: top-k, plan, attention
            self.launches = appends + (6 if tiles else 1) + (3 if self.prefill else 1)
        self.parts = self._parts()

    def switch(self, variant: str):
        """Re-use the inputs, caches and buffers for another variant of the
        step ("full" or "shared"); graphs are captured again."""
        self.variant = variant
        self.set_sel = [torch.empty_like(self.bufs["sel"]) for _ in self.sets] if variant == "shared" else None
        self.launches = 1 + 1 if variant == "shared" else self.launches
        self.whole, self.split = [], []
        self.parts = self._parts()

    # ---- the parts of a step ------------------------------------------------
    def _parts(self):
        msa, sh, b, pages = self.msa, self.shape, self.bufs, self.pages

        def append(st, i):
            d = self.sets[i]
            if self.idx_f16:
                msa.msa_indexer_append_f16(sh, d["idx_k_cache"], d["idx_k_new"], d["tok_stream"], d["tok_pos"], st,
                                           pages)
                msa.msa_kv_append(sh, d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d["tok_stream"],
                                  d["tok_pos"], st, pages)
            else:                                   # one launch for the three caches
                msa.msa_step_append(sh, d["idx_k_cache"], d["k_cache"], d["v_cache"], d["idx_k_new"], d["k_new"],
                                    d["v_new"], d["tok_stream"], d["tok_pos"], st, pages)

        def scores(st, i):
            d = self.sets[i]
            msa.msa_block_scores(sh, d["idx_q"], d["idx_k_cache"], d["q_stream"], d["q_pos"], b["block_scores"],
                                 st, b["workspace"], pages)

        def select(st, i):
            msa.msa_select_topk(sh, b["block_scores"], self.sets[i]["q_pos"], b["sel"], b["n_sel"], st)

        def attend(st, i):
            d = self.sets[i]
            fn = msa.msa_sparse_attn_prefill if self.prefill else msa.msa_sparse_attn_decode
            fn(sh, d["q"], d["k_cache"], d["v_cache"], b["sel"], d["q_stream"], d["q_pos"], self.scale,
               b["out"], b["workspace"], st, pages)

        if self.dsa:
            ds = self.dshape

            def append(st, i):                          # noqa: F811
                d = self.sets[i]
                msa.msa_dsa_indexer_append(ds, d["k_idx_cache"], d["k_idx_new"], d["tok_stream"], d["tok_pos"], st)
                msa.msa_kv_append(sh, d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d["tok_stream"],
                                  d["tok_pos"], st)

            def scores(st, i):                          # noqa: F811
                d = self.sets[i]
                msa.msa_dsa_token_scores(ds, d["q_idx"], d["weights"], d["k_idx_cache"], d["q_stream"],
                                         d["q_pos"], b["scores"], st)

            def select(st, i):                          # noqa: F811
                msa.msa_dsa_select_topk(ds, b["scores"], self.sets[i]["q_pos"], b["tok_sel"], b["tok_n"], st)

            def attend(st, i):                          # noqa: F811
                d = self.sets[i]
                msa.msa_dsa_sparse_attn_decode(sh, d["q"], d["k_cache"], d["v_cache"], b["tok_sel"],
                                               d["q_stream"], d["q_pos"], self.scale, b["out"], b["workspace"], st)
            return [append, scores, select, attend]
        if self.fused:
            def fused(st, i):
                msa.decode_step_fused(sh, self.caches, self.sets[i], b, st)
            return [fused]
        if not self.prefill and self.variant == "full":
            def select_attend(st, i):               # the top-16 inside the attention kernel
                d = self.sets[i]
                msa.msa_select_attn_decode(sh, b["block_scores"], d["q"], d["k_cache"], d["v_cache"],
                                           d["q_stream"], d["q_pos"], self.scale, b["sel"], b["n_sel"], b["out"],
                                           b["workspace"], st, pages)
            return [append, scores, select_attend]
        if self.variant == "shared":
            def kv_append(st, i):
                d = self.sets[i]
                msa.msa_kv_append(sh, d["k_cache"], d["v_cache"], d["k_new"], d["v_new"], d["tok_stream"],
                                  d["tok_pos"], st, pages)

            def attend_shared(st, i):
                d = self.sets[i]
                msa.msa_sparse_attn_decode(sh, d["q"], d["k_cache"], d["v_cache"], self.set_sel[i], d["q_stream"],
                                           d["q_pos"], self.scale, b["out"], b["workspace"], st, pages)
            return [kv_append, attend_shared]
        return [append, scores, select, attend]

    def full_step(self, st, i):
        """A whole step (appends, scores, selection, attention) on set i."""
        if self.variant == "shared" or self.fused:
            msa = self.msa
            d = self.sets[i]
            msa.decode_step(self.shape, self.caches, d, self.bufs, st, self.prefill, self.pages)
            return
        for part in self.parts:
            part(st, i)

    def prepare(self, stream):
        """One-time set-up: the shared-layer step's selections come from one
        full step per set (the previous layer's selection)."""
        if self.variant == "shared":
            for i in range(len(self.sets)):
                self.full_step(stream, i)
                self.set_sel[i].copy_(self.bufs["sel"])

    # ---- graphs --------------------------------------------------------------
    def capture(self):
        """Per input set: one graph of the whole step, and one graph per part."""
        self.whole, self.split = [], []
        for i in range(len(self.sets)):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for part in self.parts:
                    part(None, i)
            self.whole.append(g)
            gs = []
            for part in self.parts:
                gp = torch.cuda.CUDAGraph()
                with torch.cuda.graph(gp):
                    part(None, i)
                gs.append(gp)
            self.split.append(gs)
        torch.cuda.synchronize(self.dev)

    def release(self):
        self.whole, self.split = [], []
        self.sets = []
        self.caches = {}
        self.bufs = {}


class L2Flush:
    """Writes a 256 MB buffer (twice the 126 MB L2) between timed steps."""

    def __init__(self, dev):
        self.buf = torch.empty((2 * L2_BYTES,), dtype=torch.uint8, device=dev)
        self.n = 0

    def __call__(self):
        self.n += 1
        self.buf.fill_(self.n & 255)


def time_whole(step: Step, steps: int, stream, use_graph: bool, flush=None) -> float:
    """Milliseconds per step, the whole step replayed (one graph per input
    set, sets alternating); with ``flush`` each step is timed on its own
    with L2 flushed before it, outside the timed span."""
    n = len(step.sets)

    def run(i):
        if use_graph:
            step.whole[i % n].replay()
        else:
            for part in step.parts:
                part(stream, i % n)
    if flush is None:
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        for i in range(steps):
            run(i)
        t1.record(stream)
        torch.cuda.synchronize(step.dev)
        return t0.elapsed_time(t1) / steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for i in range(steps):
        flush()
        ev[i][0].record(stream)
        run(i)
        ev[i][1].record(stream)
    torch.cuda.synchronize(step.dev)
    return sum(a.elapsed_time(b) for a, b in ev) / steps


def time_parts(step: Step, steps: int, stream, timed: list[int], use_graph: bool, flush=None) -> list[float]:
    """Mean milliseconds of each part in ``timed``: the parts replayed as
    separate graphs (or launched directly), events around the timed ones."""
    n = len(step.sets)
    ev = {j: [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
          for j in timed}
    for i in range(steps):
        if flush is not None:
            flush()
        for j, part in enumerate(step.parts):
            if j in ev:
                ev[j][i][0].record(stream)
            if use_graph:
                step.split[i % n][j].replay()
            else:
                part(stream, i % n)
            if j in ev:
                ev[j][i][1].record(stream)
    torch.cuda.synchronize(step.dev)
    return [statistics.mean(a.elapsed_time(b) for a, b in ev[j]) for j in timed]


# ---------------------------------------------------------------------------
# sampled oracle check of the GPU selection (near-ties counted)
# ---------------------------------------------------------------------------
def selection_check(w, sel_gpu: torch.Tensor, queries: list[int], rel: float = 1e-5) -> dict:
    """Compare the GPU's selection of ``queries`` (indices into the step's
    queries, set 0) with the oracle's.  An id mismatch is a near-tie when the
    oracle's ranks top_k and top_k + 1 differ (not exactly equal) by less than
    ``rel`` of their magnitude and every differing block scores within that
    band; anything else is a mismatch."""
    import oracle
    per = 1 if w.queries == "last" else w.n_new
    rows_by_stream = {}
    for j, q in enumerate(queries):
        rows_by_stream.setdefault(q // per, []).append((j, q))
    bs = torch.empty((len(queries), w.n_kv_heads, w.capacity // w.block), dtype=torch.float64)
    qp = torch.empty((len(queries),), dtype=torch.int32)
    for s_id, pairs in rows_by_stream.items():          # one stream's draw at a time
        inp = W.make_inputs(w, streams=range(s_id, s_id + 1))
        idx = oracle.indexer_append(inp.idx_k_cache, inp.idx_k_new, inp.tok_stream, inp.tok_pos)
        local = torch.tensor([q - s_id * per for _, q in pairs], dtype=torch.long)
        js = torch.tensor([j for j, _ in pairs], dtype=torch.long)
        bs[js] = oracle.block_scores(inp.idx_q[local], idx, inp.q_stream[local], inp.q_pos[local], w.block)
        qp[js] = inp.q_pos[local]
        del inp, idx
    sel_o, _ = oracle.select_blocks(bs, qp, w.block, w.top_k)
    got = sel_gpu[torch.tensor(queries, dtype=torch.long)]
    exact = near = bad = 0
    for i in range(len(queries)):
        for g in range(w.n_kv_heads):
            if torch.equal(got[i, g], sel_o[i, g]):
                exact += 1
                continue
            bnd = oracle.boundary_scores(bs[i, g], int(qp[i]), w.block, w.top_k)
            diff = set(x for x in got[i, g].tolist() if x >= 0) ^ set(x for x in sel_o[i, g].tolist() if x >= 0)
            ok = False
            if bnd is not None and bnd[0] != bnd[1]:
                band = rel * max(abs(bnd[0]), abs(bnd[1]))
                ok = abs(bnd[0] - bnd[1]) < band and all(abs(float(bs[i, g, b]) - bnd[0]) <= band for b in diff)
            near += ok
            bad += not ok
    return {"queries": len(queries), "pairs": len(queries) * w.n_kv_heads, "exact": exact, "near_ties": near,
            "mismatches": bad}


def sample_queries(w) -> list[int]:
    """Queries of the sampled oracle check: four spread streams of decode
    workloads (every stream when there are at most four), 256 spread queries
    of prefill workloads."""
    if w.queries == "last":
        n = w.n_queries
        return list(range(n)) if n <= 4 else sorted({0, n // 3, (2 * n) // 3, n - 1})
    n = w.n_queries
    return sorted(set(range(0, n, max(1, n // 256))) | {n - 1})


# ---------------------------------------------------------------------------
# CPU oracle timing (baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample(w, seed: int = 0):
    """A bounded sample of workload ``w`` for the oracle: decode workloads
    run whole streams (as many as hold 256 MB of FP64 indexer keys, at least
    one); prefill workloads run 64 queries spread over the batch (scores,
    selection and attention; the caches hold every token)."""
    import oracle
    if w.queries == "last":
        n_streams = max(1, min(w.n_streams, (1 << 28) // (w.l_total * w.n_kv_heads * w.idx_dim * 8)))
        inp = W.make_inputs(w, seed=seed, streams=range(n_streams))
        caches = [oracle.indexer_append(c, n, inp.tok_stream, inp.tok_pos)
                  for c, n in ((inp.idx_k_cache, inp.idx_k_new), (inp.k_cache, inp.k_new), (inp.v_cache, inp.v_new))]

        def run():
            oracle.msa_step(caches[0], caches[1], caches[2], inp.idx_q, inp.q, inp.q_stream, inp.q_pos,
                            w.block, w.top_k)
        what = (f"{n_streams} of the {w.n_streams} streams of {w.name}, whole steps (append done once; FP64 "
                f"block scores, selection, attention)")
        return run, n_streams, what
    per_stream = max(1, 64 // w.n_streams)
    inp = W.make_inputs(w, seed=seed)
    caches = [oracle.indexer_append(c, n, inp.tok_stream, inp.tok_pos)
              for c, n in ((inp.idx_k_cache, inp.idx_k_new), (inp.k_cache, inp.k_new), (inp.v_cache, inp.v_new))]
    pick = []
    for s in range(w.n_streams):
        idx = (inp.q_stream == s).nonzero().flatten()
        pick += idx[torch.linspace(0, idx.numel() - 1, per_stream).round().long()].tolist()
    pick = torch.tensor(sorted(set(pick)), dtype=torch.long)
    sub = [inp.idx_q[pick], inp.q[pick], inp.q_stream[pick], inp.q_pos[pick]]

    def run():
        oracle.msa_step(caches[0], caches[1], caches[2], sub[0], sub[1], sub[2], sub[3], w.block, w.top_k)
    what = (f"{pick.numel()} of the {w.n_queries} queries of {w.name}, spread evenly over each stream "
            f"(FP64 block scores, selection, attention; the append of the new tokens done once)")
    return run, int(pick.numel()), what


def cpu_baseline(w=WORKLOAD, budget_s: float = 10.0) -> dict:
    cores = host_cores()
    torch.set_num_threads(cores)
    run, units, what = oracle_sample(w)
    reps, t0 = 0, time.perf_counter()
    while True:
        run()
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return {"value": reps * units / el, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{what}, repeated {reps}x over {el:.1f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    cores = host_cores()
    torch.set_num_threads(cores)
    run, units, what = oracle_sample(WORKLOAD)
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
    value = units / (ms * 1e-3)
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": len(times), "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD.name, "streams_per_step": units},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": f"{what} per step (FP64 CPU oracle)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------
def warm(step: Step, stream, warmup: int, use_graph: bool):
    for i in range(warmup):
        for part in step.parts:
            part(stream, i % len(step.sets))
    torch.cuda.synchronize(step.dev)
    if use_graph:
        step.capture()
        for i in range(warmup):
            step.whole[i % len(step.sets)].replay()
        torch.cuda.synchronize(step.dev)


def roofline_decode(w, step: Step, k_ms: float, peaks: dict, key_bytes: int) -> dict:
    """Roofline of the decode block-score kernel (or the fused step)."""
    if step.fused:
        sbytes, kernel = step_bytes(w, key_bytes), "decode_step_fused"
    elif step.dsa:
        sbytes, kernel = dsa_scores_bytes(w), "dsa_scores"
    else:
        sbytes, kernel = scores_bytes(w, key_bytes), "block_scores_gemv"
    achieved = sbytes / (k_ms * 1e-3) / 1e9
    traffic = None
    cap = SCORES_TRAFFIC["f16" if key_bytes == 2 else "f32"]
    if not step.fused and not step.dsa and cap["source_sha"] == scores_source_sha() \
            and w == WORKLOAD and step.pages is None:
        traffic = cap["bytes_per_launch"]
    if step.dsa and DSA_SCORES_TRAFFIC["source_sha"] == scores_source_sha("msa_dsa_scores.cuh") and w == WORKLOAD:
        traffic = DSA_SCORES_TRAFFIC["bytes_per_launch"]
    return {"kernel": kernel, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": traffic, "algorithmic_bytes": sbytes,
            "ms_per_launch": k_ms, "peak_src": peaks["src"] + " (stream copy, read+write bytes; a read-only "
                                                            "stream can exceed it)",
            "nominal_frac": achieved / NOMINAL_HBM_GBS, "nominal_gbs": NOMINAL_HBM_GBS}


def measure_extra(msa, args, w, rank, dev, stream, peaks) -> dict:
    """Step time, roofline and sampled checks of one of the other workloads."""
    prefill = w.queries == "new"
    step = Step(msa, args, w, rank, dev)
    flush = L2Flush(dev) if (prefill or input_bytes(w) < 4 * L2_BYTES) else None
    steps = min(args.steps, 20 if prefill else 500)
    warm(step, stream, max(3, min(args.warmup, 5)), True)
    ms = time_whole(step, steps, stream, True, flush)
    out = {"ms_per_step": ms, "steps": steps, "input_sets": len(step.sets),
           "l2": "flushed between timed steps (256 MB write, outside the timed span)" if flush else
                 f"inputs {input_bytes(w) / 1e9:.1f} GB > 126 MB L2, no flush",
           "gpu_launches_per_step": step.launches}
    if prefill:
        ind, att = prefill_flops(w)
        s_ms, a_ms = time_parts(step, steps, stream, [1, 3], True, flush)
        tf = (ind + att) / (ms * 1e-3) / 1e12
        out.update({
            "value": w.n_queries / (ms * 1e-3), "unit": "tokens/s",
            "step_tensor": {"achieved_tflops": tf, "peak_tflops": peaks["bf16_tflops"],
                            "frac": tf / peaks["bf16_tflops"], "indexer_flops": ind, "attention_flops": att},
            "roofline": {"kernel": "sparse_attn_prefill_union", "bound": "tensor",
                         "achieved": att / (a_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": att / (a_ms * 1e-3) / 1e12 / peaks["bf16_tflops"], "traffic": None,
                         "ms_per_launch": a_ms, "peak_src": peaks["src"] + " (cuBLAS bf16 burst)"},
            "indexer_roofline": {"kernel": "block_scores_tc (with its split pre-passes)", "bound": "tensor",
                                 "achieved": ind / (s_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                                 "unit": "TFLOP/s", "frac": ind / (s_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                 "ms_per_call": s_ms},
        })
    else:
        (k_ms,) = time_parts(step, steps, stream, [1], True, flush)
        gbs = step_bytes(w) / (ms * 1e-3) / 1e9
        out.update({
            "value": w.n_streams / (ms * 1e-3), "unit": "tokens/s",
            "step_hbm": {"achieved_gbs": gbs, "peak_gbs": peaks["hbm_gbs"], "frac": gbs / peaks["hbm_gbs"],
                         "bytes_per_step": step_bytes(w)},
            "roofline": roofline_decode(w, step, k_ms, peaks, 4),
        })
    step.full_step(stream, 0)
    torch.cuda.synchronize(dev)
    if msa.msa_get_device_error(stream) != 0:
        raise RuntimeError(f"device error in {w.name}")
    sel = step.bufs["sel"].cpu()
    step.release()
    del step
    torch.cuda.empty_cache()
    out["selection_check"] = selection_check(w, sel, sample_queries(w))
    out["cpu_baseline"] = cpu_baseline(w, budget_s=5.0)
    return out


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
    use_graph = not args.no_graph
    stream = torch.cuda.current_stream(dev)
    variant = "shared" if args.shared_layer else "full"
    step = Step(msa, args, w, rank, dev, variant)
    key_bytes = 2 if args.idx_f16 else 4
    step.prepare(stream)
    flush = L2Flush(dev) if (prefill or input_bytes(w) < 4 * L2_BYTES) else None
    clocks = ClockSampler(dev) if rank == 0 else None
    warm(step, stream, args.warmup, use_graph)
    if msa.msa_get_device_error(stream) != 0:
        raise RuntimeError("device error during warm-up")

    # ---- device-resident timing: the whole step, one graph per input set -----
    if world > 1:
        torch.distributed.barrier(device_ids=[dev])
    torch.cuda.synchronize(dev)
    mark = clocks.mark() if clocks else 0
    ms = time_whole(step, args.steps, stream, use_graph, flush)
    if world > 1:
        torch.distributed.barrier(device_ids=[dev])
    mark_end = clocks.mark() if clocks else 0
    # ---- the dominant kernel, timed in a second pass ---------------------------
    if step.fused:
        timed = [0]
    elif variant == "shared":
        timed = [1]
    else:
        timed = [3, 1] if prefill else [1]
    k_times = time_parts(step, args.steps, stream, timed, use_graph, flush)
    k_ms = k_times[0]

    # ---- end to end: host inputs in, host output out, every step ------------
    d0 = step.sets[0]
    host_names = ("tok_stream", "tok_pos", "idx_k_new", "k_new", "v_new", "q_stream", "q_pos", "idx_q", "q")
    if step.dsa:
        host_names = ("tok_stream", "tok_pos", "k_idx_new", "k_new", "v_new", "q_stream", "q_pos", "q_idx",
                      "weights", "q")
    hosts = [{n: s[n].cpu().pin_memory() for n in host_names} for s in step.sets]
    h_out = torch.empty(step.bufs["out"].shape, dtype=torch.bfloat16).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hosts[0].values())
    d2h = h_out.numel() * h_out.element_size()
    e2e_steps = max(3, min(args.steps, 200 if not prefill else 20))
    n_sets = len(step.sets)
    pipe = None
    if use_graph and variant == "full" and not (step.dsa or step.fused):
        # the public pipelined replay: two captures of the step alternate,
        # each step's packed inputs go in on one copy stream and its output
        # comes back on another while the neighbouring steps run
        pipe = msa.StepPipeline(step.shape, step.caches, d0, prefill, step.pages)
        packed = [pipe.pack(h, pipe.host_buffer()) for h in hosts]
        h2d = packed[0].numel()

        def api_step(i):
            pipe.step(packed[i % n_sets])                   # inputs in, replay, output out
        e2e_launch = "cuda graphs, transfers overlapped with the neighbouring steps"
    else:
        def api_step(i):                                    # noqa: F811
            dset = step.sets[i % n_sets]
            for n in host_names:
                dset[n].copy_(hosts[i % n_sets][n], non_blocking=True)
            if use_graph:
                step.whole[i % n_sets].replay()
            else:
                for part in step.parts:
                    part(stream, i % n_sets)
            h_out.copy_(step.bufs["out"], non_blocking=True)
        e2e_launch = "cuda graph" if use_graph else "direct"
    for i in range(3):
        api_step(i)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(e2e_steps):
        api_step(i)
    if pipe is not None:
        pipe.wait_all()                                     # the last outputs are on the host
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    if msa.msa_get_device_error(stream) != 0:
        raise RuntimeError("device error during timing")
    clk = clocks.summary(mark, mark_end) if clocks else None

    ms, e2e_ms, k_ms = max_over_ranks([ms, e2e_ms, k_ms], device=dev)
    sel_host = None
    if rank == 0 and world == 1 and not step.dsa and variant == "full":
        step.full_step(stream, 0)
        torch.cuda.synchronize(dev)
        sel_host = step.bufs["sel"].cpu()
    launches = step.launches
    del pipe
    if rank != 0:
        step.release()
        if clocks:
            clocks.stop()
        return None

    peaks = load_peaks()
    cfg = {"workload": w.name, "streams_per_gpu": w.n_streams, "context": w.l_total,
           "launch": "cuda graphs (whole step, one graph per input set)" if use_graph else "direct",
           "caches": "paged (shuffled pages + block table)" if args.paged else "contiguous",
           "q_heads": w.n_q_heads, "kv_heads": w.n_kv_heads, "head_dim": w.head_dim,
           "block": w.block, "top_k": w.top_k, "parallelism": f"replicas{world}", "input_sets": n_sets,
           "l2": "flushed between timed steps (256 MB write, outside the timed span)" if flush else
                 f"inputs {input_bytes(w) / 1e9:.1f} GB per GPU > 126 MB L2, no flush; "
                 f"{n_sets} input sets alternate"}
    line = {
        "metric": variant_metric(METRIC, args) if w == WORKLOAD or not prefill else
        f"MSA prefill tokens/s ({w.name}); achieved TFLOP/s vs bf16 peak",
        "value": job_tokens_per_s(w.n_streams, world, ms) if not prefill else w.n_queries * world / (ms * 1e-3),
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("f16" if args.idx_f16 else "f32") + " indexer / bf16 attention (f32 accumulate)",
        "data": "synthetic (seeded N(0,1) K/V/Q bf16, indexer N(0,1)/sqrt(128) f32)",
        "config": cfg,
    }
    if step_is_dsa(args):
        line["metric"] = DSA_METRIC if w == WORKLOAD else DSA_METRIC.replace("@32K ctx x32 streams", f"({w.name})")
        line["dtype"] = "f16 indexer (f32 accumulate) / bf16 attention (f32 accumulate)"
        line["data"] = ("synthetic (seeded N(0,1) K/V/Q bf16; indexer keys and heads N(0,1)/sqrt(128) fp16, "
                        "weights N(0,1)/8 f32)")
        cfg.update({"variant": "token-level (lightning indexer)", "index_heads": 64, "top_k_tokens": 2048,
                    "relu": True})
        sb = dsa_step_bytes(w)
        line["step_hbm"] = {"achieved_gbs": sb / (ms * 1e-3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
                            "frac": sb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "bytes_per_step": sb}
        line["roofline"] = roofline_decode(w, _Kind(dsa=True), k_ms, peaks, 2)
    elif prefill:
        ind, att = prefill_flops(w)
        tf = (ind + att) / (ms * 1e-3) / 1e12
        line["step_tensor"] = {"achieved_tflops": tf, "peak_tflops": peaks["bf16_tflops"],
                               "frac": tf / peaks["bf16_tflops"], "indexer_flops": ind, "attention_flops": att}
        ktf = att / (k_ms * 1e-3) / 1e12
        line["roofline"] = {"kernel": "sparse_attn_prefill_union", "bound": "tensor", "achieved": ktf,
                            "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": ktf / peaks["bf16_tflops"],
                            "traffic": None, "ms_per_launch": k_ms, "peak_src": peaks["src"]}
        s_ms = k_times[1]
        line["indexer_roofline"] = {"kernel": "block_scores_tc (with its split pre-passes)", "bound": "tensor",
                                    "achieved": ind / (s_ms * 1e-3) / 1e12, "peak": peaks["bf16_tflops"],
                                    "unit": "TFLOP/s", "frac": ind / (s_ms * 1e-3) / 1e12 / peaks["bf16_tflops"],
                                    "ms_per_call": s_ms}
    elif variant == "shared":
        sb = shared_layer_bytes(w)
        line["step_hbm"] = {"achieved_gbs": sb / (ms * 1e-3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
                            "frac": sb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "bytes_per_step": sb}
        a = kv_bytes_per_stream(w) * w.n_streams / (k_ms * 1e-3) / 1e9
        line["roofline"] = {"kernel": "sparse_attn_decode_sk", "bound": "hbm", "achieved": a,
                            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": a / peaks["hbm_gbs"], "traffic": None,
                            "algorithmic_bytes": kv_bytes_per_stream(w) * w.n_streams, "ms_per_launch": k_ms,
                            "peak_src": peaks["src"]}
    else:
        sb = step_bytes(w, key_bytes)
        line["step_hbm"] = {"achieved_gbs": sb / (ms * 1e-3) / 1e9, "peak_gbs": peaks["hbm_gbs"],
                            "frac": sb / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "bytes_per_step": sb}
        line["roofline"] = roofline_decode(w, _Kind(fused=args.fused, paged=args.paged), k_ms, peaks, key_bytes)
    e2e_value = (job_tokens_per_s(w.n_streams, world, e2e_ms) if not prefill
                 else w.n_queries * world / (e2e_ms * 1e-3))
    line["e2e"] = {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                   "ms_per_step": e2e_ms, "steps": e2e_steps, "launch": e2e_launch}
    line["gpu_launches"] = launches * args.steps
    line["clocks"] = clk
    if sel_host is not None:
        line["selection_check"] = selection_check(w, sel_host, sample_queries(w))

    default_run = (world == 1 and w == WORKLOAD and not (args.idx_f16 or args.paged or args.dsa or args.fused
                                                        or args.shared_layer or args.no_graph))
    if default_run and not args.no_extras:
        # the shared-layer step on the same workload, then the other four workloads
        sh_step = step
        sh_step.switch("shared")
        sh_step.prepare(stream)
        warm(sh_step, stream, max(3, min(args.warmup, 5)), True)
        sh_ms = time_whole(sh_step, min(args.steps, 2000), stream, True)
        (sh_k,) = time_parts(sh_step, min(args.steps, 2000), stream, [1], True)
        if msa.msa_get_device_error(stream) != 0:
            raise RuntimeError("device error in the shared-layer step")
        sb = shared_layer_bytes(w)
        line["shared_layer"] = {
            "what": "append of the new K/V rows + attention over the selection a previous layer made (no block "
                    "scores, no selection): the step of a layer that reuses another layer's top-k",
            "ms_per_step": sh_ms, "value": w.n_streams / (sh_ms * 1e-3), "unit": "tokens/s",
            "bytes_per_step": sb, "achieved_gbs": sb / (sh_ms * 1e-3) / 1e9,
            "frac": sb / (sh_ms * 1e-3) / 1e9 / peaks["hbm_gbs"], "attention_ms": sh_k,
            "gpu_launches_per_step": sh_step.launches, "full_step_ms": ms}
        sh_step.release()
        del sh_step, step
        torch.cuda.empty_cache()
        line["workloads"] = {}
        for other in (W.DECODE_4K, W.DECODE_128K_X8, W.PREFILL_16K, W.CHUNKED_PREFILL_TIES):
            line["workloads"][other.name] = measure_extra(msa, args, other, rank, dev, stream, peaks)
    else:
        step.release()
        del step
        torch.cuda.empty_cache()
    if clocks:
        clocks.stop()
    return line


class _Kind:
    """Which kernel a decode roofline line describes."""

    def __init__(self, dsa=False, fused=False, paged=False):
        self.dsa, self.fused = dsa, fused
        self.pages = True if paged else None


def step_is_dsa(args) -> bool:
    return bool(args.dsa)


DSA_METRIC = ("MSA token-level variant (lightning indexer, 64 heads, top-2048 tokens) decode tokens/s "
              "@32K ctx x32 streams; achieved HBM GB/s vs peak")


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="only the headline workload (no shared-layer step, no other workloads)")
    ap.add_argument("--idx-f16", action="store_true",
                    help="decode with the F16 indexer-key cache variant instead of the F32 cache")
    ap.add_argument("--dsa", action="store_true",
                    help="time the token-level variant (lightning indexer, top-2048 tokens) on the same workload")
    ap.add_argument("--fused", action="store_true",
                    help="run the whole decode step as one persistent kernel (msa_decode_step_fused)")
    ap.add_argument("--shared-layer", action="store_true",
                    help="time the step of a layer that reuses a previous layer's selection "
                         "(K/V append + attention only)")
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
    decode_wl = W.WORKLOADS[args.workload].queries == "last"
    if args.dsa and (args.paged or args.idx_f16 or not decode_wl):
        ap.error("--dsa times decode workloads with contiguous caches")
    if args.fused and (args.paged or args.idx_f16 or args.dsa or not decode_wl):
        ap.error("--fused times decode workloads with contiguous F32 caches")
    if args.shared_layer and (args.dsa or args.fused or not decode_wl):
        ap.error("--shared-layer times decode workloads (block selection)")
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
                    and not args.paged and not args.dsa and not args.fused and not args.shared_layer):
                line["cpu_baseline"] = cpu_baseline()
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
