"""Seeded synthetic inputs for MiniMax Sparse Attention (MSA) workloads.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic.  Both the CPU oracle (tests, CPU baseline) and the CUDA
path (tests, bench) take their inputs from here, so both sides always see the
same bytes.

Geometry follows the head layout stated in the llama.cpp pull request "Add
MiniMax-M3 (MSA: MiniMax Sparse Attention) support" (review comment with the
random-init test model): head_dim 128, 4 KV heads = 4 indexer groups, indexer
dim 128, block 128, top-k 16; 64 query heads (16 per group).

Recipe (identical for every workload):
  * torch CPU ``Generator`` seeded with ``seed`` (default 0);
  * draw order: indexer keys, K, V (each stream in turn, shape [G][L][dim]),
    then indexer queries, then Q;
  * indexer values are float32 N(0,1)/sqrt(idx_dim); with ``quantize_idx`` they
    are rounded to the nearest multiple of 1/8 (torch.round, half to even) so
    that equal block scores occur;
  * K, V and Q are float32 N(0,1) draws rounded to bfloat16 (round to nearest
    even).
Positions [0, L_existing) are in the cache before the step; positions
[L_existing, L_total) are the step's new tokens (appended by the step);
capacity is L_total rounded up to a multiple of the block size, and slots past
L_total are zero.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

N_Q_HEADS = 64
N_KV_HEADS = 4
HEAD_DIM = 128
IDX_DIM = 128
BLOCK = 128
TOP_K = 16


@dataclass(frozen=True)
class Workload:
    """Shape of one synthetic MSA step.

    ``queries`` selects which positions issue a query: "last" (one decode
    query per stream at L_total-1) or "new" (every appended token queries,
    as in prefill).
    """
    name: str
    n_streams: int
    l_existing: int
    l_total: int
    queries: str = "last"
    quantize_idx: bool = False
    n_q_heads: int = N_Q_HEADS
    n_kv_heads: int = N_KV_HEADS
    head_dim: int = HEAD_DIM
    idx_dim: int = IDX_DIM
    block: int = BLOCK
    top_k: int = TOP_K
    description: str = ""

    @property
    def capacity(self) -> int:
        return -(-self.l_total // self.block) * self.block

    @property
    def n_new(self) -> int:
        return self.l_total - self.l_existing

    @property
    def n_queries(self) -> int:
        per = 1 if self.queries == "last" else self.n_new
        return self.n_streams * per


# The five workloads of the benchmark plan (names say what they are).
DECODE_4K = Workload("decode_1x4k", 1, 4095, 4096, "last",
                     description="1 stream, 4096-token context, one query at 4095")
DECODE_32K_X32 = Workload("decode_32x32k", 32, 32767, 32768, "last",
                          description="32 streams x 32768-token context, one query each at 32767")
PREFILL_16K = Workload("prefill_1x16k", 1, 0, 16384, "new",
                       description="16384 tokens appended to an empty cache, every token queries")
DECODE_128K_X8 = Workload("decode_8x128k", 8, 131071, 131072, "last",
                          description="8 streams x 131072-token context, one query each")
CHUNKED_PREFILL_TIES = Workload("chunked_prefill_4x2k_on_64k_ties", 4, 65536, 67584, "new",
                                quantize_idx=True,
                                description="4 streams append 2048 tokens to a 65536-token cache; "
                                            "indexer values quantised to 1/8")
WORKLOADS = {w.name: w for w in (DECODE_4K, DECODE_32K_X32, PREFILL_16K, DECODE_128K_X8,
                                 CHUNKED_PREFILL_TIES)}


@dataclass
class Inputs:
    """All tensors of one step, on the CPU, in the library's layouts.

    idx_k_cache [S][G][cap][Di] f32, k_cache/v_cache [S][G][cap][D] bf16 hold
    the existing tokens only (new slots are zero).  The new tokens are
    idx_k_new [n_tok][G][Di] f32, k_new/v_new [n_tok][G][D] bf16 with
    tok_stream/tok_pos [n_tok] int32.  Queries: q_stream/q_pos [n_q] int32,
    idx_q [n_q][G][Di] f32, q [n_q][Hq][D] bf16.
    """
    w: Workload
    idx_k_cache: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    tok_stream: torch.Tensor
    tok_pos: torch.Tensor
    idx_k_new: torch.Tensor
    k_new: torch.Tensor
    v_new: torch.Tensor
    q_stream: torch.Tensor
    q_pos: torch.Tensor
    idx_q: torch.Tensor
    q: torch.Tensor
    extra: dict = field(default_factory=dict)


def _idx_draw(g: torch.Generator, shape, idx_dim: int, quantize: bool) -> torch.Tensor:
    x = torch.randn(shape, generator=g, dtype=torch.float32) / math.sqrt(idx_dim)
    if quantize:
        x = torch.round(x * 8.0) / 8.0
    return x


def _bf16_draw(g: torch.Generator, shape) -> torch.Tensor:
    return torch.randn(shape, generator=g, dtype=torch.float32).to(torch.bfloat16)


def make_inputs(w: Workload, seed: int = 0, streams: range | None = None) -> Inputs:
    """Draw the inputs of workload ``w``.

    ``streams`` restricts the draw to a sub-range of streams (a bounded sample
    for CPU timing); the generator is seeded per stream block so that a
    sampled stream gets the same values it has in the full draw.
    """
    S = w.n_streams
    streams = range(S) if streams is None else streams
    G, Di, D, Hq = w.n_kv_heads, w.idx_dim, w.head_dim, w.n_q_heads
    cap, L, L0 = w.capacity, w.l_total, w.l_existing
    ns = len(streams)

    idx_full = torch.zeros((ns, G, cap, Di), dtype=torch.float32)
    k_full = torch.zeros((ns, G, cap, D), dtype=torch.bfloat16)
    v_full = torch.zeros((ns, G, cap, D), dtype=torch.bfloat16)
    nq_per = 1 if w.queries == "last" else w.n_new
    idx_q = torch.empty((ns * nq_per, G, Di), dtype=torch.float32)
    q = torch.empty((ns * nq_per, Hq, D), dtype=torch.bfloat16)

    for i, s in enumerate(streams):
        # one independent generator per stream: a stream's values do not
        # depend on which other streams are drawn
        g = torch.Generator().manual_seed(seed * 1_000_003 + s)
        idx_full[i, :, :L] = _idx_draw(g, (G, L, Di), Di, w.quantize_idx)
        k_full[i, :, :L] = _bf16_draw(g, (G, L, D))
        v_full[i, :, :L] = _bf16_draw(g, (G, L, D))
        idx_q[i * nq_per:(i + 1) * nq_per] = _idx_draw(g, (nq_per, G, Di), Di, w.quantize_idx)
        q[i * nq_per:(i + 1) * nq_per] = _bf16_draw(g, (nq_per, Hq, D))

    # split into existing cache + new tokens
    new_pos = torch.arange(L0, L, dtype=torch.int32)
    tok_stream = torch.repeat_interleave(torch.arange(ns, dtype=torch.int32), len(new_pos))
    tok_pos = new_pos.repeat(ns)
    idx_k_new = idx_full[:, :, L0:L].permute(0, 2, 1, 3).reshape(-1, G, Di).contiguous()
    k_new = k_full[:, :, L0:L].permute(0, 2, 1, 3).reshape(-1, G, D).contiguous()
    v_new = v_full[:, :, L0:L].permute(0, 2, 1, 3).reshape(-1, G, D).contiguous()
    idx_full[:, :, L0:L] = 0
    k_full[:, :, L0:L] = 0
    v_full[:, :, L0:L] = 0

    if w.queries == "last":
        q_stream = torch.arange(ns, dtype=torch.int32)
        q_pos = torch.full((ns,), L - 1, dtype=torch.int32)
    else:
        q_stream = tok_stream.clone()
        q_pos = tok_pos.clone()
    return Inputs(w, idx_full, k_full, v_full, tok_stream, tok_pos, idx_k_new, k_new, v_new,
                  q_stream, q_pos, idx_q, q)


def make_step_set(w: Workload, seed: int, streams: range | None = None) -> dict:
    """Another draw of a decode step's new tokens and queries for the same
    caches: idx_k_new, k_new, v_new [ns][G][dim] (one token per stream, at
    its last slot), idx_q [ns][G][Di] and q [ns][Hq][D], from per-stream
    generators seeded seed * 1000003 + stream + 9000000007.  Steps that
    alternate between such sets append and query different values at the same
    slot, so their block selections (and the K/V blocks they read) differ."""
    if w.queries != "last" or w.n_new != 1:
        raise ValueError("step sets are drawn for one-token decode steps")
    S = w.n_streams
    streams = range(S) if streams is None else streams
    G, Di, D, Hq = w.n_kv_heads, w.idx_dim, w.head_dim, w.n_q_heads
    ns = len(streams)
    out = {"idx_k_new": torch.empty((ns, G, Di)), "k_new": torch.empty((ns, G, D), dtype=torch.bfloat16),
           "v_new": torch.empty((ns, G, D), dtype=torch.bfloat16), "idx_q": torch.empty((ns, G, Di)),
           "q": torch.empty((ns, Hq, D), dtype=torch.bfloat16)}
    for i, s in enumerate(streams):
        g = torch.Generator().manual_seed(seed * 1_000_003 + s + 9_000_000_007)
        out["idx_k_new"][i] = _idx_draw(g, (G, Di), Di, w.quantize_idx)
        out["k_new"][i] = _bf16_draw(g, (G, D))
        out["v_new"][i] = _bf16_draw(g, (G, D))
        out["idx_q"][i] = _idx_draw(g, (G, Di), Di, w.quantize_idx)
        out["q"][i] = _bf16_draw(g, (Hq, D))
    return out


def make_custom(n_streams: int, capacity: int, lengths, q_positions, *, seed: int = 0,
                n_q_heads: int = N_Q_HEADS, n_kv_heads: int = N_KV_HEADS,
                head_dim: int = HEAD_DIM, idx_dim: int = IDX_DIM, quantize_idx: bool = False,
                kv_dtype=torch.bfloat16):
    """Caches already holding ``lengths[s]`` tokens per stream and an explicit
    list of (stream, position) queries.  Used for ragged / edge-case tests.

    Returns (idx_k_cache, k_cache, v_cache, q_stream, q_pos, idx_q, q).
    """
    g = torch.Generator().manual_seed(seed)
    G = n_kv_heads
    idx = torch.zeros((n_streams, G, capacity, idx_dim), dtype=torch.float32)
    k = torch.zeros((n_streams, G, capacity, head_dim), dtype=kv_dtype)
    v = torch.zeros((n_streams, G, capacity, head_dim), dtype=kv_dtype)
    for s in range(n_streams):
        L = lengths[s]
        idx[s, :, :L] = _idx_draw(g, (G, L, idx_dim), idx_dim, quantize_idx)
        k[s, :, :L] = torch.randn((G, L, head_dim), generator=g).to(kv_dtype)
        v[s, :, :L] = torch.randn((G, L, head_dim), generator=g).to(kv_dtype)
    q_stream = torch.tensor([sp[0] for sp in q_positions], dtype=torch.int32)
    q_pos = torch.tensor([sp[1] for sp in q_positions], dtype=torch.int32)
    n_q = len(q_positions)
    idx_q = _idx_draw(g, (n_q, G, idx_dim), idx_dim, quantize_idx)
    q = torch.randn((n_q, n_q_heads, head_dim), generator=g).to(kv_dtype)
    return idx, k, v, q_stream, q_pos, idx_q, q


# ---------------------------------------------------------------------------
# paged layout of a step's caches
# ---------------------------------------------------------------------------
POISON = 64.0   # value of every row in a page no stream maps (reading one shows)


@dataclass
class PagedCaches:
    """The step's caches laid out as page pools [n_pages][G][block][row] plus
    the block table [S][capacity / block] (int32) naming each logical block's
    page.  Spare pages and the pages of unmapped blocks hold POISON."""
    block_table: torch.Tensor
    n_pages: int
    idx_pool: torch.Tensor
    k_pool: torch.Tensor
    v_pool: torch.Tensor


def page_layout(inp: Inputs, seed: int = 0, spare_pages: int = 3, shared_prefix_blocks: int = 0,
                unmapped_from: int | None = None) -> PagedCaches:
    """Scatter the contiguous caches of ``inp`` into shuffled pages.

    Every (stream, block) gets its own page at a random pool slot, except
    that streams 1.. map their first ``shared_prefix_blocks`` blocks to
    stream 0's pages (a shared prefix: their logical rows there become stream
    0's rows; keep those blocks below the existing length so no step appends
    into a shared page).  Blocks from ``unmapped_from`` on get table entry -1.
    """
    S, G, cap, Di = inp.idx_k_cache.shape
    D = inp.k_cache.shape[3]
    B = inp.w.block
    nb = cap // B
    last = nb if unmapped_from is None else min(nb, unmapped_from)
    own = [(s, b) for s in range(S) for b in range(last) if s == 0 or b >= shared_prefix_blocks]
    n_pages = len(own) + spare_pages
    g = torch.Generator().manual_seed(seed * 7919 + 101)
    slot = torch.randperm(n_pages, generator=g)
    table = torch.full((S, nb), -1, dtype=torch.int32)
    for i, (s, b) in enumerate(own):
        table[s, b] = int(slot[i])
    for s in range(1, S):
        for b in range(min(shared_prefix_blocks, last)):
            table[s, b] = table[0, b]
    idx_pool = torch.full((n_pages, G, B, Di), POISON, dtype=inp.idx_k_cache.dtype)
    k_pool = torch.full((n_pages, G, B, D), POISON, dtype=inp.k_cache.dtype)
    v_pool = torch.full((n_pages, G, B, D), POISON, dtype=inp.v_cache.dtype)
    for s, b in own:
        pg = int(table[s, b])
        idx_pool[pg] = inp.idx_k_cache[s, :, b * B:(b + 1) * B]
        k_pool[pg] = inp.k_cache[s, :, b * B:(b + 1) * B]
        v_pool[pg] = inp.v_cache[s, :, b * B:(b + 1) * B]
    return PagedCaches(table, n_pages, idx_pool, k_pool, v_pool)


# ---------------------------------------------------------------------------
# token-level variant (lightning indexer) inputs
# ---------------------------------------------------------------------------
DSA_INDEX_HEADS = 64


@dataclass
class DsaInputs:
    """A step of the token-level variant: the MSA step's K/V caches, tokens
    and queries (``base``; its indexer fields are unused) plus the lightning
    indexer's inputs: k_idx_cache [S][cap][Di] f32 holding the existing
    tokens' keys (new slots zero; the cache itself is fp16, rounded by the
    append or by the caller), k_idx_new [n_tok][Di] f32, q_idx
    [n_q][H_I][Di] fp16 and weights [n_q][H_I] f32."""
    base: Inputs
    k_idx_cache: torch.Tensor
    k_idx_new: torch.Tensor
    q_idx: torch.Tensor
    weights: torch.Tensor


def make_dsa_inputs(w: Workload, seed: int = 0, streams: range | None = None,
                    n_index_heads: int = DSA_INDEX_HEADS, quantize: bool = False) -> DsaInputs:
    """Draw a token-level step.  K/V/Q come from ``make_inputs``; the indexer
    draws use their own per-stream generators (seed * 1000003 + stream +
    7000000019), in the order keys [L][Di], query heads [n_q][H_I][Di],
    weights [n_q][H_I].  Keys and query heads are N(0,1)/sqrt(Di), weights
    N(0,1)/sqrt(H_I).  With ``quantize`` keys and query heads are multiples of
    1/8 and weights multiples of 1/4, so every score is exact in float32 and
    equal scores occur."""
    base = make_inputs(w, seed, streams)
    S = w.n_streams
    streams = range(S) if streams is None else streams
    Di, cap, L, L0 = w.idx_dim, w.capacity, w.l_total, w.l_existing
    ns = len(streams)
    nq_per = 1 if w.queries == "last" else w.n_new
    keys = torch.zeros((ns, cap, Di), dtype=torch.float32)
    q_idx = torch.empty((ns * nq_per, n_index_heads, Di), dtype=torch.float32)
    weights = torch.empty((ns * nq_per, n_index_heads), dtype=torch.float32)
    for i, s in enumerate(streams):
        g = torch.Generator().manual_seed(seed * 1_000_003 + s + 7_000_000_019)
        keys[i, :L] = torch.randn((L, Di), generator=g) / math.sqrt(Di)
        q_idx[i * nq_per:(i + 1) * nq_per] = torch.randn((nq_per, n_index_heads, Di), generator=g) / math.sqrt(Di)
        weights[i * nq_per:(i + 1) * nq_per] = torch.randn((nq_per, n_index_heads), generator=g) / math.sqrt(n_index_heads)
    if quantize:
        keys = torch.round(keys * 8.0) / 8.0
        q_idx = torch.round(q_idx * 8.0) / 8.0
        weights = torch.round(weights * 4.0) / 4.0
    k_new = keys[:, L0:L].reshape(-1, Di).contiguous()
    keys[:, L0:L] = 0
    return DsaInputs(base, keys, k_new, q_idx.to(torch.float16), weights)
