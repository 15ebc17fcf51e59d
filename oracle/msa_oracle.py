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

* "deepseek2 : GLM-DSA sparse attention (lightning indexer)" (ik_llama.cpp
  pull request), section "What this does" and its review thread: the
  token-level variant (``dsa_*`` functions): per-head indexer products times
  per-head weights, summed over the indexer heads, top-k tokens kept.

Readings where the pages are silent (each also listed in the design notes):
* the local-force bias is the constant LOCAL_BIAS = 2**100 (any bias larger
  than twice the largest |score| gives the same selection);
* equal block scores rank the lower block index first;
* selected ids are reported in ascending order, padded with -1;
* query head h belongs to group h // (n_q_heads / n_kv_heads);
* the query at position p attends to the rows j <= p of its selected blocks
  (only the local block can hold rows past p);
* scores are plain dot products (no scale, activation or weights);
* a NaN block score ranks as -inf (inputs never hold one; the rule only fixes
  what the selection does if one appears).

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
    """s_j = idx_q . idx_k[j] for the given key rows, in float64.  With a
    [Di][n] matrix of n query vectors the result is s[j][i]."""
    return _cpu64(idx_k_rows) @ _cpu64(idx_q_vec)


def pool_visible(s: torch.Tensor, positions, block: int, n_blocks: int) -> torch.Tensor:
    """maxpool_block over the causally masked token scores of n queries.

    ``s`` [n][L] holds query i's scores over slots 0..L-1, and query i sees
    the slots j <= positions[i] ("idx_q*idx_k^T + causal mask": every later
    slot scores -inf).  Entry [i][b] is the largest masked score in slots
    [b*block, (b+1)*block), so a block with no visible slot is -inf.
    """
    n, L = s.shape
    pos = torch.as_tensor(positions, dtype=torch.long).reshape(n, 1)
    masked = _cpu64(s).masked_fill(torch.arange(L).reshape(1, L) > pos, NEG_INF)   # causal mask
    width = n_blocks * block
    padded = torch.full((n, width), NEG_INF, dtype=F64)
    padded[:, :min(L, width)] = masked[:, :width]
    return padded.reshape(n, n_blocks, block).amax(dim=2)                          # maxpool_block


def pooled_scores(idx_q_vec: torch.Tensor, idx_k_sg: torch.Tensor, pos: int, block: int,
                  n_blocks: int) -> torch.Tensor:
    """maxpool_block over the causally visible scores of one (query, group).

    ``idx_k_sg`` is the [capacity][idx_dim] cache of the query's stream and
    group.  Entry b is max_{j in [b*block, (b+1)*block), j <= pos} s_j; blocks
    with no visible token are -inf.
    """
    s = token_scores(idx_q_vec, idx_k_sg)                     # every slot of the cache
    return pool_visible(s.reshape(1, -1), [pos], block, n_blocks)[0]


def block_scores(idx_q: torch.Tensor, idx_k_cache: torch.Tensor, q_stream: torch.Tensor,
                 q_pos: torch.Tensor, block: int, local_bias: float = LOCAL_BIAS,
                 chunk: int = 256) -> torch.Tensor:
    """bs[n_q][G][capacity/block]: pooled scores plus the local-force bias.

    idx_q [n_q][G][Di], idx_k_cache [S][G][capacity][Di].  The queries of one
    stream are scored ``chunk`` at a time as one matrix product against the
    keys up to the chunk's last position (the same dot products as one query
    at a time; only the number of queries per product differs).
    """
    n_q, G = idx_q.shape[0], idx_q.shape[1]
    n_blocks = idx_k_cache.shape[2] // block
    bs = torch.empty((n_q, G, n_blocks), dtype=F64)
    streams = q_stream.to(torch.long)
    positions = q_pos.to(torch.long)
    for s in sorted(set(streams.tolist())):
        mine = (streams == s).nonzero().flatten()
        for g in range(G):
            keys = _cpu64(idx_k_cache[s, g])
            for c0 in range(0, mine.numel(), chunk):
                ii = mine[c0:c0 + chunk]
                L = int(positions[ii].max()) + 1
                sc = token_scores(idx_q[ii, g].T, keys[:L]).T                # [n][L]
                bs[ii, g] = pool_visible(sc, positions[ii], block, n_blocks)
    for i in range(n_q):
        bs[i, :, local_block(int(positions[i]), block)] += local_bias
    return bs


# ---------------------------------------------------------------------------
# top-k block selection
# ---------------------------------------------------------------------------
def ranked_blocks(bs_row: torch.Tensor, pos: int, block: int) -> list[int]:
    """Visible blocks ordered best first: higher score, then lower index.  A
    NaN score ranks as -inf (below every finite score, tied with -inf and
    ordered by index), and -0 equals +0."""
    nvis = n_visible_blocks(pos, block)
    vals = bs_row[:nvis].tolist()

    def rank_key(b):
        v = vals[b]
        return (math.inf if v != v else -v, b)
    return sorted(range(nvis), key=rank_key)


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


# ---------------------------------------------------------------------------
# token-level variant: the lightning indexer (DSA)
# ---------------------------------------------------------------------------
# "deepseek2 : GLM-DSA sparse attention (lightning indexer)" (ik_llama.cpp
# pull request), section "What this does": the indexer scores each query
# against the indexer keys, keeps the top-k highest-scoring keys per query
# (tokens, not blocks; GLM-5.2's indexer top_k is 2048) and masks the rest out
# of attention.  The indexer-key cache holds one F16 key per token
# ([head_size, kv_size]).  The review thread describes the score as the
# per-indexer-head products q_h . k "element-wise multiplied with another
# matrix" (per-head weights) and then reduced over the indexer heads.  The
# keys' Hadamard rotation is applied by the caller before the keys reach the
# cache (an orthogonal rotation of both sides leaves q . k unchanged).
# Readings where the page is silent: each head's product passes through a
# ReLU when ``relu`` is true (the published lightning-indexer definition the
# page names; the page itself does not print the formula); equal scores keep
# the lower token index; with at most top_k visible tokens every visible token
# is kept (the page's "no-op-exact" check: the sparse mask then equals the
# causal mask).
def dsa_token_scores(q_idx: torch.Tensor, weights: torch.Tensor, k_idx_cache: torch.Tensor,
                     q_stream: torch.Tensor, q_pos: torch.Tensor, relu: bool = True) -> torch.Tensor:
    """I[t][s] = sum_h weights[t][h] * act(q_idx[t][h] . k_idx_cache[stream][s])
    for the visible tokens s <= q_pos[t], -inf for s > q_pos[t].

    q_idx [n_q][H][Di], weights [n_q][H], k_idx_cache [S][cap][Di]."""
    n_q, H, Di = q_idx.shape
    cap = k_idx_cache.shape[1]
    out = torch.full((n_q, cap), NEG_INF, dtype=F64)
    for t in range(n_q):
        s, p = int(q_stream[t]), int(q_pos[t])
        keys = _cpu64(k_idx_cache[s, :p + 1])                  # [p+1][Di]
        per_head = keys @ _cpu64(q_idx[t]).T                   # [p+1][H]
        if relu:
            per_head = per_head.clamp_min(0.0)
        out[t, :p + 1] = per_head @ _cpu64(weights[t])
    return out


def dsa_ranked_tokens(scores_row: torch.Tensor, pos: int) -> list[int]:
    """Visible tokens ordered by (score descending, index ascending); a NaN
    score ranks as -inf (the variant's stated rule)."""
    def rank_key(s):
        v = float(scores_row[s])
        return (math.inf if v != v else -v, s)
    return sorted(range(pos + 1), key=rank_key)


def dsa_select_one(scores_row: torch.Tensor, pos: int, top_k: int) -> list[int]:
    """Kept tokens of one query, ascending: every visible token when there
    are at most top_k of them, else the first top_k of the ranking."""
    if pos + 1 <= top_k:
        return list(range(pos + 1))
    return sorted(dsa_ranked_tokens(scores_row, pos)[:top_k])


def dsa_select_tokens(scores: torch.Tensor, q_pos: torch.Tensor, top_k: int, width: int):
    """sel [n_q][width] int32 (ascending token ids, -1 padded) and n_sel [n_q]."""
    n_q = scores.shape[0]
    sel = torch.full((n_q, width), -1, dtype=torch.int32)
    n_sel = torch.zeros((n_q,), dtype=torch.int32)
    for t in range(n_q):
        ids = dsa_select_one(scores[t], int(q_pos[t]), top_k)
        sel[t, :len(ids)] = torch.tensor(ids, dtype=torch.int32)
        n_sel[t] = len(ids)
    return sel, n_sel


def dsa_boundary_scores(scores_row: torch.Tensor, pos: int, top_k: int):
    """(score of rank top_k, score of rank top_k + 1), or None when every
    visible token is kept."""
    if pos + 1 <= top_k:
        return None
    ranked = dsa_ranked_tokens(scores_row, pos)
    return float(scores_row[ranked[top_k - 1]]), float(scores_row[ranked[top_k]])


def dsa_sparse_attention(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
                         sel_tok: torch.Tensor, q_stream: torch.Tensor, q_pos: torch.Tensor,
                         scale: float | None = None) -> torch.Tensor:
    """out[n_q][Hq][D] float64: every head h (group g = h // (Hq/G)) attends to
    the kept tokens of its query (one token set shared by all groups) in its
    group's K/V rows: softmax(scale * q_h . K_rows^T) . V_rows."""
    n_q, Hq, D = q.shape
    G = k_cache.shape[1]
    heads_per_group = Hq // G
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = torch.zeros((n_q, Hq, D), dtype=F64)
    for t in range(n_q):
        s, p = int(q_stream[t]), int(q_pos[t])
        rows = [int(j) for j in sel_tok[t].tolist() if 0 <= int(j) <= p]
        if not rows:
            continue
        for g in range(G):
            K = _cpu64(k_cache[s, g, rows])
            V = _cpu64(v_cache[s, g, rows])
            for h in range(g * heads_per_group, (g + 1) * heads_per_group):
                logits = (K @ _cpu64(q[t, h])) * scale
                w = torch.exp(logits - logits.max())
                out[t, h] = (w / w.sum()) @ V
    return out
