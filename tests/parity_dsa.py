"""Parity helpers of the token-level (lightning-indexer) variant: run a step
through the C ABI on seeded inputs and compare it with the CPU oracle.

Comparison rules
  * key-cache append (fp16, nearest even) and K/V append: bit-exact;
  * top-k from identical float32 scores: bit-exact;
  * token scores (float32 on the GPU vs float64): each head's dot product of
    fp16 vectors has exact products and float32 accumulation of 128 terms
    (error at most 128 u sum_d |q_d k_d|, u = 2^-24); the ReLU adds none, the
    weight product 1 u, and the float32 sum over 64 heads at most 64 u of
    sum_h |w_h x_h|.  The test allows 256 u sum_h |w_h| sum_d |q_hd k_d|, and
    exact agreement of -inf;
  * end-to-end selection: ids bit-exact, except swaps at the top-k boundary
    between tokens whose oracle scores lie within the sum of their score
    bounds of the oracle's k-th score (never an exact tie); those are counted
    and the attention is checked with the GPU's selection;
  * attention: as for the block-sparse path (|got - bf16(want)| <=
    max(4e-3, 1 bf16 ulp), mean |got - want| <= 5e-4).
"""
from __future__ import annotations

import math

import torch

import block_sparse_attention_maxpool_b200 as msa
import oracle
from tests import parity as PT

U32 = 2.0 ** -24


def dsa_shape_of(w, top_k=2048, relu=True) -> msa.DsaShape:
    return msa.DsaShape(n_streams=w.n_streams, capacity=w.capacity, top_k=top_k, relu=relu)


def score_bounds(q_idx, weights, keys, q_stream, q_pos):
    """256 u sum_h |w_h| sum_d |q_hd k_sd| per (query, visible token)."""
    n_q = q_idx.shape[0]
    cap = keys.shape[1]
    out = torch.zeros((n_q, cap), dtype=torch.float64)
    for t in range(n_q):
        s, p = int(q_stream[t]), int(q_pos[t])
        a = keys[s, :p + 1].double().abs() @ q_idx[t].double().abs().T     # [p+1][H]
        out[t, :p + 1] = 256 * U32 * (a @ weights[t].double().abs())
    return out


def check_scores(sc_gpu, sc_orc, bounds):
    g = sc_gpu.double()
    inf_g, inf_o = torch.isneginf(g), torch.isneginf(sc_orc)
    assert torch.equal(inf_g, inf_o), "-inf pattern differs"
    fin = ~inf_o
    err = (g[fin] - sc_orc[fin]).abs()
    assert bool((err <= bounds[fin] + 1e-30).all()), f"token score error {err.max():.3e} above bound"
    return float(err.max()) if err.numel() else 0.0


def check_selection(sel_gpu, nsel_gpu, sc_orc, bounds, q_pos, top_k):
    """Returns (selection for the attention check, number of excused swaps)."""
    sel_o, nsel_o = oracle.dsa_select_tokens(sc_orc, q_pos, top_k, msa.DSA_SEL_WIDTH)
    merged = sel_o.clone()
    excused = 0
    for t in range(sel_o.shape[0]):
        if torch.equal(sel_gpu[t], sel_o[t]) and int(nsel_gpu[t]) == int(nsel_o[t]):
            continue
        p = int(q_pos[t])
        got = set(x for x in sel_gpu[t].tolist() if x >= 0)
        want = set(x for x in sel_o[t].tolist() if x >= 0)
        assert len(got) == len(want) == int(nsel_gpu[t]), f"query {t}: kept counts differ"
        assert sel_gpu[t, :len(got)].tolist() == sorted(got), f"query {t}: ids not ascending"
        bnd = oracle.dsa_boundary_scores(sc_orc[t], p, top_k)
        assert bnd is not None and bnd[0] != bnd[1], f"query {t}: selection differs with no boundary swap"
        sk = bnd[0]
        k_tok = [x for x in want if float(sc_orc[t, x]) == sk]
        for x in got ^ want:
            slack = float(bounds[t, x]) + max(float(bounds[t, y]) for y in k_tok)
            assert abs(float(sc_orc[t, x]) - sk) <= slack, \
                f"query {t}: token {x} (score {float(sc_orc[t, x])}) swapped far from the boundary {sk}"
        merged[t] = sel_gpu[t]
        excused += 1
    return merged, excused


def to_dev(dinp, dev="cuda"):
    d = PT.to_dev(dinp.base, dev)
    d["k_idx_cache"] = dinp.k_idx_cache.half().to(dev)
    d["k_idx_new"] = dinp.k_idx_new.to(dev)
    d["q_idx"] = dinp.q_idx.to(dev)
    d["weights"] = dinp.weights.to(dev)
    return d


def full_parity(dinp, top_k=2048, relu=True, queries=None, dev="cuda"):
    """One token-level step on the GPU against the oracle on the query
    indices ``queries`` (all when None).  Returns a small report."""
    inp = dinp.base
    w = inp.w
    shape = PT.shape_of(w)
    dshape = dsa_shape_of(w, top_k, relu)
    d = to_dev(dinp, dev)
    caches = {k: d[k] for k in ("k_idx_cache", "k_cache", "v_cache")}
    out, sel, n_sel, sc = msa.dsa_decode_step(shape, dshape, caches, d)
    err = msa.msa_get_device_error()
    assert err == 0, f"device error word {err:#x}"
    # caches after the append
    keys = oracle.indexer_append(dinp.k_idx_cache.half().unsqueeze(1), dinp.k_idx_new.half().unsqueeze(1),
                                 inp.tok_stream, inp.tok_pos)[:, 0]
    assert torch.equal(d["k_idx_cache"].cpu(), keys), "indexer key cache after append"
    _, k_o, v_o = PT.oracle_caches(inp)
    assert torch.equal(d["k_cache"].cpu(), k_o) and torch.equal(d["v_cache"].cpu(), v_o), "K/V append"
    n_q = inp.q_pos.numel()
    qsub = torch.arange(n_q) if queries is None else torch.as_tensor(queries, dtype=torch.long)
    qs, qp = inp.q_stream[qsub], inp.q_pos[qsub]
    sc_o = oracle.dsa_token_scores(dinp.q_idx[qsub], dinp.weights[qsub], keys, qs, qp, relu)
    bounds = score_bounds(dinp.q_idx[qsub], dinp.weights[qsub], keys, qs, qp)
    max_score_err = check_scores(sc.cpu()[qsub], sc_o, bounds)
    merged, excused = check_selection(sel.cpu()[qsub], n_sel.cpu()[qsub], sc_o, bounds, qp, top_k)
    out_o = oracle.dsa_sparse_attention(inp.q[qsub], k_o, v_o, merged, qs, qp, 1.0 / math.sqrt(w.head_dim))
    max_err, mean_err, _ = PT.check_attention(out.cpu()[qsub], out_o)
    return dict(queries=len(qsub), boundary_swaps=excused, max_score_err=max_score_err,
                attn_max_abs=max_err, attn_mean_abs=mean_err)
