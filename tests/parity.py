"""Helpers shared by the GPU parity tests: run MSA steps through the C ABI on
seeded inputs and compare them with the CPU oracle.

Comparison rules
  * cache append, selection from identical float32 scores: bit-exact;
  * block scores (float32 on the GPU vs float64 in the oracle).  Streaming
    kernel: the float32 dot product of 128 terms, formed as 4-term FMA chains
    summed over a 32-lane tree, rounds each term at most ~9 times, so
    |err| <= 9 u sum_d |q_d k_d| (u = 2^-24).  Tensor-core tile kernel: each
    factor is split exactly as 2^-e (hi + lo) in fp16, so hi + lo differs
    from it by at most 2^-23 of the row scale, the dropped lo.lo product is
    at most 2^-22 |q_d k_d|, and the float32 accumulation of 24 partial
    products adds at most 24 u of the running sum: together below 56 u sum_d
    |q_d k_d|.  The test allows 64 u times the largest such sum in the block,
    plus exact agreement of -inf and of the local bias;
  * end-to-end selection: ids bit-exact, except (q, g) pairs whose oracle
    ranks top_k and top_k+1 are within 1e-5 relative (and not exactly equal);
    those are counted and the attention is checked with the GPU's selection;
  * attention (bf16 out vs float64): elementwise |got - want| <= 4e-3 plus
    half a bf16 ulp of want (the rounding of a correctly rounded bf16 output
    is at most half an ulp, so only the output's own rounding is excused on
    top of the 4e-3 bound), and mean |got - want| <= 5e-4.
"""
from __future__ import annotations

import dataclasses
import math

import torch

import block_sparse_attention_maxpool_b200 as msa
import oracle
import workloads as W
from tests.oracle_pins import near_tie_excused

U32 = 2.0 ** -24
ATTN_MAX_ABS = 4e-3
ATTN_MEAN_ABS = 5e-4


def shape_of(w) -> msa.Shape:
    return msa.Shape(n_streams=w.n_streams, capacity=w.capacity, n_q_heads=w.n_q_heads,
                     n_kv_heads=w.n_kv_heads, head_dim=w.head_dim, idx_dim=w.idx_dim,
                     block=w.block, top_k=w.top_k)


def to_dev(inp, dev="cuda", idx_f16=False):
    names = ["idx_k_cache", "k_cache", "v_cache", "tok_stream", "tok_pos", "idx_k_new", "k_new",
             "v_new", "q_stream", "q_pos", "idx_q", "q"]
    d = {n: getattr(inp, n).to(dev).contiguous() for n in names}
    if idx_f16:
        d["idx_k_cache"] = d["idx_k_cache"].half()
    return d


def run_step(shape, d, prefill=False, pages=None):
    caches = {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    out, sel, n_sel, bs = msa.decode_step(shape, caches, d, prefill=prefill, pages=pages)
    err = msa.msa_get_device_error()
    return out, sel, n_sel, bs, err


def oracle_caches(inp, idx_f16=False):
    """The caches after the step's append.  With the F16 indexer-cache variant
    the keys are the F32 keys rounded to fp16 by torch (nearest even)."""
    if idx_f16:
        idx = oracle.indexer_append(inp.idx_k_cache.half(), inp.idx_k_new.half(), inp.tok_stream, inp.tok_pos)
    else:
        idx = oracle.indexer_append(inp.idx_k_cache, inp.idx_k_new, inp.tok_stream, inp.tok_pos)
    k = oracle.indexer_append(inp.k_cache, inp.k_new, inp.tok_stream, inp.tok_pos)
    v = oracle.indexer_append(inp.v_cache, inp.v_new, inp.tok_stream, inp.tok_pos)
    return idx, k, v


def score_bounds(idx_q, idx_k_cache, q_stream, q_pos, block, chunk=256):
    """Per (query, group, block): 64 u max_j sum_d |q_d k_jd| over visible j
    (the queries of one stream in chunks, as one product of absolute values)."""
    n_q, G = idx_q.shape[0], idx_q.shape[1]
    nblk = idx_k_cache.shape[2] // block
    out = torch.zeros((n_q, G, nblk), dtype=torch.float64)
    streams, positions = q_stream.long(), q_pos.long()
    for s in sorted(set(streams.tolist())):
        mine = (streams == s).nonzero().flatten()
        for g in range(G):
            keys = idx_k_cache[s, g].double().abs()
            for c0 in range(0, mine.numel(), chunk):
                ii = mine[c0:c0 + chunk]
                L = int(positions[ii].max()) + 1
                a = idx_q[ii, g].double().abs() @ keys[:L].T                     # [n][L]
                a = a.masked_fill(torch.arange(L).view(1, L) > positions[ii].view(-1, 1), 0.0)
                pad = torch.zeros((ii.numel(), nblk * block), dtype=torch.float64)
                pad[:, :L] = a
                out[ii, g] = 64 * U32 * pad.view(-1, nblk, block).amax(dim=2)
    return out


def check_scores(bs_gpu, bs_orc, bounds):
    g = bs_gpu.double()
    inf_g, inf_o = torch.isinf(g) & (g < 0), torch.isinf(bs_orc) & (bs_orc < 0)
    assert torch.equal(inf_g, inf_o), "-inf pattern differs"
    fin = ~inf_o
    big = bs_orc >= oracle.LOCAL_BIAS / 2
    assert torch.equal(g[big], bs_orc[big]), "local bias differs"
    small = fin & ~big
    err = (g[small] - bs_orc[small]).abs()
    ok = err <= bounds[small] + 1e-30
    assert bool(ok.all()), f"block score error {err.max():.3e} above bound"
    return float(err.max()) if err.numel() else 0.0


def check_selection(sel_gpu, nsel_gpu, bs_orc, q_pos, block, top_k):
    """Returns (merged sel for the attention check, number of excused near-ties)."""
    sel_o, nsel_o = oracle.select_blocks(bs_orc, q_pos, block, top_k)
    merged = sel_o.clone()
    excused = 0
    n_q, G = sel_o.shape[0], sel_o.shape[1]
    mism = (sel_gpu != sel_o).any(dim=2) | (nsel_gpu != nsel_o)
    for i, g in mism.nonzero().tolist():
        p = int(q_pos[i])
        got = [b for b in sel_gpu[i, g].tolist() if b >= 0]
        want = [b for b in sel_o[i, g].tolist() if b >= 0]
        bnd = oracle.boundary_scores(bs_orc[i, g], p, block, top_k)
        assert near_tie_excused(bnd, bs_orc[i, g], got, want), \
            f"selection differs at query {i} group {g}: gpu {got} oracle {want} boundary {bnd}"
        assert len(got) == len(want) and got == sorted(got)
        merged[i, g] = sel_gpu[i, g]
        excused += 1
    return merged, excused


def bf16_ulp(x: torch.Tensor) -> torch.Tensor:
    """The spacing of bf16 numbers at |x| (8 significant bits): 2^(e-8) for
    |x| in [2^(e-1), 2^e)."""
    _, e = torch.frexp(x.abs().clamp_min(2.0 ** -126))
    return torch.ldexp(torch.ones_like(x), e - 8)


def check_attention(out_gpu, out_orc, rows=None):
    """|got - want| <= 4e-3 + half a bf16 ulp of want for every element,
    mean |got - want| <= 5e-4 (want: the float64 oracle).  Returns (max abs
    error, mean abs error, the largest fraction of its element's tolerance
    an error uses)."""
    g = out_gpu.double()
    w = out_orc
    if rows is not None:
        g, w = g[rows], w[rows]
    ulp = bf16_ulp(w)
    tol = ATTN_MAX_ABS + 0.5 * ulp
    d = (g - w).abs()
    bad = d > tol
    assert not bool(bad.any()), (f"attention max err {d.max():.3e} (tol {tol[bad].min():.3e}) "
                                 f"at {bad.nonzero()[0].tolist()}")
    mean = float(d.mean())
    assert mean <= ATTN_MEAN_ABS, f"attention mean abs err {mean:.3e}"
    return float(d.max()), mean, float((d / tol).max())


def full_parity(inp, queries=None, prefill=False, dev="cuda", idx_f16=False, paged=None, attn_queries=None):
    """Run one step on the GPU and compare every part with the oracle on the
    query indices ``queries`` (all when None); the attention on
    ``attn_queries`` only, when given (a subset of ``queries``).  With ``paged`` (keyword
    arguments of workloads.page_layout) the GPU runs the paged calls on
    shuffled page pools and the oracle reads the same pools through its own
    logical view.  Returns a small report."""
    w = inp.w
    shape = shape_of(w)
    d = to_dev(inp, dev, idx_f16)
    pages = None
    if paged is not None:
        lay = W.page_layout(inp, **paged)
        d["idx_k_cache"] = lay.idx_pool.to(dev)
        if idx_f16:
            d["idx_k_cache"] = d["idx_k_cache"].half()
        d["k_cache"], d["v_cache"] = lay.k_pool.to(dev), lay.v_pool.to(dev)
        pages = msa.Pages(lay.block_table.to(dev), lay.n_pages)
        # the oracle's inputs: the pools seen through its logical view
        inp = dataclasses.replace(
            inp, idx_k_cache=oracle.logical_cache(lay.idx_pool, lay.block_table, w.block),
            k_cache=oracle.logical_cache(lay.k_pool, lay.block_table, w.block),
            v_cache=oracle.logical_cache(lay.v_pool, lay.block_table, w.block))
    out, sel, n_sel, bs, err = run_step(shape, d, prefill, pages)
    assert err == 0, f"device error word {err:#x}"
    idx_o, k_o, v_o = oracle_caches(inp, idx_f16)
    if paged is None:
        assert torch.equal(d["idx_k_cache"].cpu(), idx_o), "indexer cache after append"
        assert torch.equal(d["k_cache"].cpu(), k_o) and torch.equal(d["v_cache"].cpu(), v_o), "K/V append"
    else:
        bt = lay.block_table
        ipool = lay.idx_pool.half() if idx_f16 else lay.idx_pool
        new_idx = inp.idx_k_new.half() if idx_f16 else inp.idx_k_new
        want_i = oracle.paged_append(ipool, new_idx, inp.tok_stream, inp.tok_pos, bt, w.block)
        want_k = oracle.paged_append(lay.k_pool, inp.k_new, inp.tok_stream, inp.tok_pos, bt, w.block)
        want_v = oracle.paged_append(lay.v_pool, inp.v_new, inp.tok_stream, inp.tok_pos, bt, w.block)
        assert torch.equal(d["idx_k_cache"].cpu(), want_i), "indexer pool after append"
        assert torch.equal(d["k_cache"].cpu(), want_k) and torch.equal(d["v_cache"].cpu(), want_v), "K/V pools"
    n_q = inp.q_pos.numel()
    qsub = torch.arange(n_q) if queries is None else torch.as_tensor(queries, dtype=torch.long)
    qs, qp = inp.q_stream[qsub], inp.q_pos[qsub]
    bs_o = oracle.block_scores(inp.idx_q[qsub], idx_o, qs, qp, w.block)
    bounds = score_bounds(inp.idx_q[qsub], idx_o, qs, qp, w.block)
    bs_g, sel_g, nsel_g, out_g = bs.cpu()[qsub], sel.cpu()[qsub], n_sel.cpu()[qsub], out.cpu()[qsub]
    max_score_err = check_scores(bs_g, bs_o, bounds)
    merged, excused = check_selection(sel_g, nsel_g, bs_o, qp, w.block, w.top_k)
    if attn_queries is not None:
        pick = {int(x): j for j, x in enumerate(qsub.tolist())}
        rows = torch.tensor([pick[int(x)] for x in attn_queries], dtype=torch.long)
    else:
        rows = torch.arange(qsub.numel())
    out_o = oracle.sparse_attention(inp.q[qsub[rows]], k_o, v_o, merged[rows], qs[rows], qp[rows], w.block,
                                    1.0 / math.sqrt(w.head_dim))
    max_err, mean_err, used = check_attention(out_g[rows], out_o)
    return dict(queries=len(qsub), attn_queries=int(rows.numel()), near_ties=excused,
                max_score_err=max_score_err, attn_max_abs=max_err, attn_mean_abs=mean_err, attn_tol_used=used)
