"""Plain FP64 CPU oracle of MiniMax Sparse Attention (MSA).

TEST INFRASTRUCTURE ONLY.  Nothing in the library imports this module; only
the tests, the smoke check and the benchmark's CPU-baseline / reference arm
may call it.  It shares no code with the CUDA path.

What it computes, and where each step is stated (page titles as cited):

* "Add MiniMax-M3 (MSA: MiniMax Sparse Attention) support" (llama.cpp pull
  request), section "Overview": a per-GQA-group indexer scores the visible
  causal context, the scores are max-pooled into 128-token key blocks, the
  top-16 blocks are kept with the query's local block always included, and
  attention runs over the selected blocks only.
* same page, section "Implementation": block scores
  bs = maxpool_128(idx_q * idx_k^T + causal mask) plus a large positive bias
  on the query's local block, ranked together for top-k; selection is per GQA
  group (one indexer head per group, shared by the group's query heads).
* same page, review comment measuring on Vulkan (RADV): the number selected is
  k = min(indexer_top_k, n_blocks); below top_k*block tokens every block is
  taken and MSA equals dense attention.
* same page, review comment on --kv-unified: blocks are anchored to absolute
  slots (the flat slot index is pooled every 128 slots); the local block is
  position/128.
* same page, issue thread on unified KV caches: with streams interleaved in
  one buffer, scoring and gathering must map a stream's logical position to
  the physical slot holding it through a page indirection
  (``logical_cache``, ``paged_append``);
* "mtmd: Add Vision Support for Minimax-M3" commit message (squash of the MSA
  branch): indexer scores are accumulated in F32 (the oracle uses FP64, which
  is at least that exact) and the KV length is a multiple of 128.

Readings where the pages are silent (each also listed in the design notes):
* the local-force bias is the constant LOCAL_BIAS = 2**100 (any bias larger
  than twice the largest |score| gives the same selection);
* equal block scores rank the lower block index first;
* selected ids are reported in ascending order, padded with -1;
* query head h belongs to group h // (n_q_heads / n_kv_heads);
* the query at position p attends to the rows j <= p of its selected blocks
  (only the local block can hold rows past p);
* scores are plain dot products (no scale, activation or weights).

Every floating-point step runs in float64 on the CPU.  Tensors may be any
float dtype; they are converted exactly (bf16/f32 -> f64) before use.
"""
from __future__ import annotations

import math

import torch

F64 = torch.float64
NEG_INF = float("-inf")
LOCAL_BIAS = 2.0 ** 100


def _cpu64(x: torch.Tensor) -> torch.Tensor:
    if x.device.type != "cpu":
        raise ValueError("the oracle runs on CPU tensors only")
    return x.to(F64)


def n_visible_blocks(pos: int, block: int) -> int:
    """Blocks holding at least one token j <= pos (slot-anchored blocks)."""
    return pos // block + 1


def local_block(pos: int, block: int) -> int:
    """The query's own block, position / block (kv-unified review comment)."""
    return pos // block


# ---------------------------------------------------------------------------
# indexer-key cache append
# ---------------------------------------------------------------------------
def indexer_append(idx_k_cache: torch.Tensor, idx_k_new: torch.Tensor,
                   tok_stream: torch.Tensor, tok_pos: torch.Tensor) -> torch.Tensor:
    """Return a copy of the cache with row ``idx_k_new[t]`` written at
    (stream tok_stream[t], slot tok_pos[t]) for every group.

    The indexer keeps its own per-layer F32 key cache beside K/V ("Add
    MiniMax-M3 ..." pull request, section "Implementation").  The same rule
    writes new K/V rows into the bf16 K/V caches.
    """
    out = idx_k_cache.clone()
    for t in range(tok_stream.numel()):
        s, p = int(tok_stream[t]), int(tok_pos[t])
        out[s, :, p, :] = idx_k_new[t]
    return out


# ---------------------------------------------------------------------------
# block scores
# ---------------------------------------------------------------------------
def token_scores(idx_q_vec: torch.Tensor, idx_k_rows: torch.Tensor) -> torch.Tensor:
    """s_j = idx_q . idx_k[j] for the given key rows, in float64."""
    return _cpu64(idx_k_rows) @ _cpu64(idx_q_vec)


def pooled_scores(idx_q_vec: torch.Tensor, idx_k_sg: torch.Tensor, pos: int, block: int,
                  n_blocks: int) -> torch.Tensor:
    """maxpool_block over the causally visible scores of one (query, group).

    ``idx_k_sg`` is the [capacity][idx_dim] cache of the query's stream and
    group.  Entry b is max_{j in [b*block, (b+1)*block), j <= pos} s_j; blocks
    with no visible token are -inf (the causal mask sets s_j = -inf for
    j > pos before pooling).
    """
    s = token_scores(idx_q_vec, idx_k_sg[: pos + 1])          # visible tokens only
    out = torch.full((n_blocks,), NEG_INF, dtype=F64)
    for b in range(n_visible_blocks(pos, block)):
        out[b] = s[b * block: min((b + 1) * block, pos + 1)].max()
    return out


def block_scores(idx_q: torch.Tensor, idx_k_cache: torch.Tensor, q_stream: torch.Tensor,
                 q_pos: torch.Tensor, block: int, local_bias: float = LOCAL_BIAS) -> torch.Tensor:
    """bs[n_q][G][capacity/block]: pooled scores plus the local-force bias.

    idx_q [n_q][G][Di], idx_k_cache [S][G][capacity][Di].
    """
    n_q, G = idx_q.shape[0], idx_q.shape[1]
    n_blocks = idx_k_cache.shape[2] // block
    bs = torch.empty((n_q, G, n_blocks), dtype=F64)
    for i in range(n_q):
        s, p = int(q_stream[i]), int(q_pos[i])
        for g in range(G):
            row = pooled_scores(idx_q[i, g], idx_k_cache[s, g], p, block, n_blocks)
            row[local_block(p, block)] += local_bias
            bs[i, g] = row
    return bs


# ---------------------------------------------------------------------------
# top-k block selection
# ---------------------------------------------------------------------------
def ranked_blocks(bs_row: torch.Tensor, pos: int, block: int) -> list[int]:
    """Visible blocks ordered best first: higher score, then lower index."""
    nvis = n_visible_blocks(pos, block)
    vals = [float(bs_row[b]) for b in range(nvis)]
    return sorted(range(nvis), key=lambda b: (-vals[b], b))


def select_one(bs_row: torch.Tensor, pos: int, block: int, top_k: int) -> list[int]:
    """The min(top_k, visible blocks) best blocks, ids ascending."""
    ranked = ranked_blocks(bs_row, pos, block)
    return sorted(ranked[:top_k])


def select_blocks(bs: torch.Tensor, q_pos: torch.Tensor, block: int, top_k: int):
    """sel[n_q][G][top_k] int32 (ascending, -1 padded) and n_sel[n_q][G]."""
    n_q, G = bs.shape[0], bs.shape[1]
    sel = torch.full((n_q, G, top_k), -1, dtype=torch.int32)
    n_sel = torch.zeros((n_q, G), dtype=torch.int32)
    for i in range(n_q):
        p = int(q_pos[i])
        for g in range(G):
            ids = select_one(bs[i, g], p, block, top_k)
            sel[i, g, : len(ids)] = torch.tensor(ids, dtype=torch.int32)
            n_sel[i, g] = len(ids)
    return sel, n_sel


def boundary_scores(bs_row: torch.Tensor, pos: int, block: int, top_k: int):
    """(score of the last selected block, score of the best unselected block)
    in ranking order, or None when every visible block is selected.  Used for
    the near-tie rule of the parity tests."""
    ranked = ranked_blocks(bs_row, pos, block)
    if len(ranked) <= top_k:
        return None
    return float(bs_row[ranked[top_k - 1]]), float(bs_row[ranked[top_k]])


# ---------------------------------------------------------------------------
# block-sparse attention
# ---------------------------------------------------------------------------
def attended_rows(sel_ids, pos: int, block: int) -> list[int]:
    """Token rows a query attends to: rows of its selected blocks with j <= pos."""
    rows = []
    for b in sel_ids:
        b = int(b)
        if b < 0:
            continue
        rows.extend(range(b * block, min((b + 1) * block, pos + 1)))
    return rows


def sparse_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                     sel: torch.Tensor, q_stream: torch.Tensor, q_pos: torch.Tensor, block: int,
                     scale: float | None = None, queries=None) -> torch.Tensor:
    """out[n_q][Hq][D] float64: per query head h (group g = h // (Hq/G)),
    softmax(scale * q_h . K_rows^T) . V_rows over the attended rows of the
    group's selection.

    q [n_q][Hq][D], k_cache/v_cache [S][G][capacity][D], sel [n_q][G][top_k].
    ``queries`` limits the work to a subset of query indices (other rows of
    the result are NaN).
    """
    n_q, Hq, D = q.shape
    G = k_cache.shape[1]
    heads_per_group = Hq // G
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = torch.full((n_q, Hq, D), float("nan"), dtype=F64)
    for i in (range(n_q) if queries is None else queries):
        s, p = int(q_stream[i]), int(q_pos[i])
        for g in range(G):
            rows = attended_rows(sel[i, g].tolist(), p, block)
            if not rows:
                out[i, g * heads_per_group:(g + 1) * heads_per_group] = 0.0
                continue
            idx = torch.tensor(rows, dtype=torch.long)
            K = _cpu64(k_cache[s, g].index_select(0, idx))      # [R][D]
            V = _cpu64(v_cache[s, g].index_select(0, idx))      # [R][D]
            for h in range(g * heads_per_group, (g + 1) * heads_per_group):
                logits = (K @ _cpu64(q[i, h])) * scale         # [R]
                w = torch.exp(logits - logits.max())
                w = w / w.sum()
                out[i, h] = w @ V
    return out


# ---------------------------------------------------------------------------
# paged caches: a sequence-relative page indirection
# ---------------------------------------------------------------------------
def logical_cache(pool: torch.Tensor, block_table: torch.Tensor, block: int) -> torch.Tensor:
    """The per-stream cache that a page pool holds: slot j of stream s (group
    g) is slot j % block of page block_table[s][j // block].

    "Add MiniMax-M3 ..." pull request, issue thread on --kv-unified: block
    scoring and gathering index absolute slots of one flat buffer, which is
    only right while each stream owns a fixed range; a unified cache needs a
    map from a stream's logical position to the physical slot holding it,
    consulted by the scoring and gather steps (the page index of the
    reference MSA kernel).  pool is [n_pages][G][block][row]; block_table is
    [S][n_blocks].  Blocks whose entry names no page are NaN, so reading one
    poisons the result.
    """
    S, n_blocks = block_table.shape
    n_pages, G, B, row = pool.shape
    if B != block:
        raise ValueError("a page holds one block")
    out = torch.full((S, G, n_blocks * block, row), float("nan"), dtype=pool.dtype)
    for s in range(S):
        for b in range(n_blocks):
            page = int(block_table[s, b])
            if 0 <= page < n_pages:
                out[s, :, b * block:(b + 1) * block, :] = pool[page]
    return out


def paged_append(pool: torch.Tensor, new_rows: torch.Tensor, tok_stream: torch.Tensor,
                 tok_pos: torch.Tensor, block_table: torch.Tensor, block: int) -> torch.Tensor:
    """Return a copy of the pool with row new_rows[t] (every group) written at
    slot tok_pos[t] % block of the page that holds block tok_pos[t] // block
    of stream tok_stream[t]: the append of ``indexer_append`` through the
    page indirection of ``logical_cache``."""
    out = pool.clone()
    for t in range(tok_stream.numel()):
        s, p = int(tok_stream[t]), int(tok_pos[t])
        page = int(block_table[s, p // block])
        out[page, :, p % block, :] = new_rows[t].to(pool.dtype)
    return out


def msa_step(inp_idx_k_cache, k_cache, v_cache, idx_q, q, q_stream, q_pos, block: int,
             top_k: int, scale: float | None = None, queries=None):
    """Block scores, selection and sparse attention for a batch of queries."""
    bs = block_scores(idx_q, inp_idx_k_cache, q_stream, q_pos, block)
    sel, n_sel = select_blocks(bs, q_pos, block, top_k)
    out = sparse_attention(q, k_cache, v_cache, sel, q_stream, q_pos, block, scale, queries)
    return bs, sel, n_sel, out
