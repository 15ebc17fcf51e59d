"""Pins of the CPU oracle against facts fixed outside the oracle itself.

Each ``pin_*`` takes an oracle module (the real one, or a copy with a planted
mistake) and raises AssertionError when the oracle disagrees with:
  * hand-worked examples under tests/golden/ (each cites the rule it follows);
  * library routines for special cases (torch.amax for pooling with a basis
    query, scaled_dot_product_attention in float64 for attention);
  * brute force over all candidate block subsets on tiny inputs;
  * closed forms (uniform attention, single token) and invariants (local
    block forced, count = min(top_k, visible), permutation of unselected
    blocks, positive rescaling of the query).
"""
from __future__ import annotations

import glob
import itertools
import json
import math
import os

import torch
import torch.nn.functional as F

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
F64 = torch.float64


def _t(x, dtype=F64):
    return torch.tensor(x, dtype=dtype)


def golden_cases():
    out = []
    for path in sorted(glob.glob(os.path.join(GOLDEN, "*.json"))):
        with open(path) as fh:
            out.append((os.path.basename(path), json.load(fh)))
    return out


# ---------------------------------------------------------------------------
# hand-worked examples
# ---------------------------------------------------------------------------
def pin_golden(o):
    for name, c in golden_cases():
        exp = c["expected"]
        if "tok_stream" in c:                                    # append example
            got = o.indexer_append(_t(c["idx_k_cache"]), _t(c["idx_k_new"]),
                                   _t(c["tok_stream"], torch.int32), _t(c["tok_pos"], torch.int32))
            assert torch.equal(got, _t(exp["idx_k_cache"])), name
            continue
        block, top_k = c["block"], c["top_k"]
        idx_q, idx_k = _t(c["idx_q"]), _t(c["idx_k_cache"])
        q_stream, q_pos = _t(c["q_stream"], torch.int32), _t(c["q_pos"], torch.int32)
        n_blocks = idx_k.shape[2] // block
        G = idx_q.shape[1]
        if "pooled" in exp:
            for i in range(idx_q.shape[0]):
                for g in range(G):
                    got = o.pooled_scores(idx_q[i, g], idx_k[int(q_stream[i]), g], int(q_pos[i]),
                                          block, n_blocks)
                    assert torch.equal(got, _t(exp["pooled"][i][g])), (name, i, g, got)
        if "local" in exp:
            for i in range(idx_q.shape[0]):
                assert o.local_block(int(q_pos[i]), block) == exp["local"][i], name
        bs = o.block_scores(idx_q, idx_k, q_stream, q_pos, block)
        for i in range(idx_q.shape[0]):
            loc = int(q_pos[i]) // block
            for g in range(G):
                assert float(bs[i, g, loc]) >= o.LOCAL_BIAS / 2, (name, "local bias")
        sel, n_sel = o.select_blocks(bs, q_pos, block, top_k)
        assert sel.tolist() == exp["sel"], (name, sel.tolist())
        assert n_sel.tolist() == exp["n_sel"], (name, n_sel.tolist())
        if "boundary" in exp:
            for i in range(idx_q.shape[0]):
                for g in range(G):
                    b = o.boundary_scores(bs[i, g], int(q_pos[i]), block, top_k)
                    e = exp["boundary"][i][g]
                    assert (b is None) == (e is None), name
                    if b is not None:
                        assert list(b) == e, (name, b)
        if "out" in exp:
            out = o.sparse_attention(_t(c["q"]), _t(c["k_cache"]), _t(c["v_cache"]), sel,
                                     q_stream, q_pos, block)
            assert torch.allclose(out, _t(exp["out"]), rtol=0, atol=c["tolerance"]), (name, out)


# ---------------------------------------------------------------------------
# scores: basis queries against torch.amax, bilinearity
# ---------------------------------------------------------------------------
def pin_basis_query_pooling(o, seed=1):
    """With idx_q = c * e_d (c > 0) the pooled score of block b is c times
    the largest d-th coordinate among the block's visible keys; with c < 0 it
    is c times the smallest.  Checked with torch.amax/amin on the raw cache."""
    g = torch.Generator().manual_seed(seed)
    block, Di, cap = 4, 3, 24
    keys = torch.randn((cap, Di), generator=g, dtype=F64)
    n_blocks = cap // block
    for pos in (0, 1, 3, 4, 5, 10, 11, 12, 23):
        for d in range(Di):
            for c in (1.0, 2.5, -1.0):
                q = torch.zeros(Di, dtype=F64)
                q[d] = c
                got = o.pooled_scores(q, keys, pos, block, n_blocks)
                for b in range(n_blocks):
                    lo, hi = b * block, min((b + 1) * block, pos + 1)
                    if lo > pos:
                        assert got[b] == float("-inf"), (pos, b)
                        continue
                    col = keys[lo:hi, d]
                    want = c * (torch.amax(col) if c > 0 else torch.amin(col))
                    assert torch.isclose(got[b], want, rtol=0, atol=1e-14), (pos, d, c, b)


def pin_scores_bilinear(o, seed=2):
    """token_scores is linear in the query and equals the key column on a
    basis vector, so it is the dot product over every dimension."""
    g = torch.Generator().manual_seed(seed)
    Di, R = 5, 9
    keys = torch.randn((R, Di), generator=g, dtype=F64)
    q1 = torch.randn(Di, generator=g, dtype=F64)
    q2 = torch.randn(Di, generator=g, dtype=F64)
    s = o.token_scores(q1 * 3.0 - q2, keys)
    assert torch.allclose(s, 3.0 * o.token_scores(q1, keys) - o.token_scores(q2, keys), atol=1e-12)
    for d in range(Di):
        e = torch.zeros(Di, dtype=F64)
        e[d] = 1.0
        assert torch.equal(o.token_scores(e, keys), keys[:, d])


# ---------------------------------------------------------------------------
# selection: brute force over subsets, ties, invariants
# ---------------------------------------------------------------------------
def _bruteforce_select(pooled, pos, block, top_k):
    """All subsets of min(top_k, visible) visible blocks that contain the local
    block; keep those with the largest sum of the other blocks' pooled scores
    and, among them, the lexicographically smallest sorted id list."""
    nvis = pos // block + 1
    local = pos // block
    k = min(top_k, nvis)
    others = [b for b in range(nvis) if b != local]
    best, best_ids = None, None
    for comb in itertools.combinations(others, k - 1):
        total = sum(pooled[b] for b in comb)
        ids = sorted(comb + (local,))
        if best is None or total > best or (total == best and ids < best_ids):
            best, best_ids = total, ids
    return best_ids


def pin_selection_bruteforce(o, seed=3):
    g = torch.Generator().manual_seed(seed)
    block, top_k, Di = 4, 3, 3
    cap = 36
    for trial in range(60):
        quant = trial % 2 == 1                      # odd trials: many exact ties
        keys = torch.randn((cap, Di), generator=g, dtype=F64)
        q = torch.randn((Di,), generator=g, dtype=F64)
        if quant:
            keys = torch.round(keys * 2) / 2
            q = torch.round(q * 2) / 2
        pos = int(torch.randint(0, cap, (1,), generator=g))
        n_blocks = cap // block
        pooled = o.pooled_scores(q, keys, pos, block, n_blocks)
        bs = pooled.clone()
        bs[pos // block] += o.LOCAL_BIAS
        got = o.select_one(bs, pos, block, top_k)
        want = _bruteforce_select(pooled.tolist(), pos, block, top_k)
        assert got == want, (trial, pos, got, want)


def pin_selection_nan_rule(o):
    """A NaN block score ranks as -inf: below every finite score and tied
    with -inf, ties going to the lower index; -0 equals +0.  The expected
    orders are written out by hand from that rule."""
    nan, inf = float("nan"), float("inf")
    row = torch.tensor([nan, 0.5, -inf, -3.0, nan, 2.0, -0.0, 0.0], dtype=F64)
    assert o.ranked_blocks(row, 7 * 4, 4) == [5, 1, 6, 7, 3, 0, 2, 4]
    assert o.select_one(row, 7 * 4, 4, 6) == [0, 1, 3, 5, 6, 7]
    row2 = torch.tensor([-inf, nan, nan, 1.0, -inf], dtype=F64)
    assert o.ranked_blocks(row2, 4 * 4 + 2, 4) == [3, 0, 1, 2, 4]
    sel, n_sel = o.select_blocks(row2.reshape(1, 1, 5), torch.tensor([4 * 4 + 2], dtype=torch.int32), 4, 3)
    assert sel.tolist() == [[[0, 1, 3]]] and n_sel.tolist() == [[3]]


def pin_selection_invariants(o, seed=4):
    g = torch.Generator().manual_seed(seed)
    block, top_k, Di, cap = 4, 3, 4, 48
    n_blocks = cap // block
    for trial in range(40):
        keys = torch.randn((1, 1, cap, Di), generator=g, dtype=F64)
        q = torch.randn((1, 1, Di), generator=g, dtype=F64)
        pos = int(torch.randint(0, cap, (1,), generator=g))
        qs, qp = torch.zeros(1, dtype=torch.int32), torch.tensor([pos], dtype=torch.int32)
        bs = o.block_scores(q, keys, qs, qp, block)
        sel, n_sel = o.select_blocks(bs, qp, block, top_k)
        ids = [b for b in sel[0, 0].tolist() if b >= 0]
        nvis = pos // block + 1
        assert len(ids) == int(n_sel[0, 0]) == min(top_k, nvis)
        assert pos // block in ids
        assert ids == sorted(set(ids)) and all(0 <= b < nvis for b in ids)
        assert sel[0, 0, len(ids):].eq(-1).all()
        # a positive rescale of the query ranks blocks the same way
        bs2 = o.block_scores(q * 7.5, keys, qs, qp, block)
        assert o.select_blocks(bs2, qp, block, top_k)[0].tolist() == sel.tolist()
        # permuting the contents of unselected full blocks (away from the
        # local block) leaves the selection unchanged
        loc = pos // block
        uns = [b for b in range(nvis) if b not in ids and b != loc]
        if len(uns) >= 2:
            perm = uns[1:] + uns[:1]
            k2 = keys.clone()
            for src, dst in zip(uns, perm):
                k2[0, 0, dst * block:(dst + 1) * block] = keys[0, 0, src * block:(src + 1) * block]
            bs3 = o.block_scores(q, k2, qs, qp, block)
            assert o.select_blocks(bs3, qp, block, top_k)[0].tolist() == sel.tolist()


def pin_local_forced(o):
    """The local block is taken even when its own score is the lowest."""
    block, top_k, Di, cap = 4, 2, 1, 20
    keys = torch.full((1, 1, cap, Di), 5.0, dtype=F64)
    pos = 17                                         # local block 4 = rows 16..19
    keys[0, 0, 16:20] = -50.0
    q = torch.ones((1, 1, Di), dtype=F64)
    qp = torch.tensor([pos], dtype=torch.int32)
    bs = o.block_scores(q, keys, torch.zeros(1, dtype=torch.int32), qp, block)
    sel, _ = o.select_blocks(bs, qp, block, top_k)
    assert sel[0, 0].tolist() == [0, 4]              # tie among 0..3 at 5 -> block 0


# ---------------------------------------------------------------------------
# attention: SDPA in float64, closed forms
# ---------------------------------------------------------------------------
def _sdpa_reference(q, k_cache, v_cache, q_stream, q_pos, mask_rows_fn, scale=None):
    """torch scaled_dot_product_attention (float64, CPU, GQA enabled) with a
    per-query boolean mask over key rows."""
    n_q, Hq, D = q.shape
    G, cap = k_cache.shape[1], k_cache.shape[2]
    out = torch.empty((n_q, Hq, D), dtype=F64)
    for i in range(n_q):
        s, p = int(q_stream[i]), int(q_pos[i])
        mask = torch.zeros((G, 1, cap), dtype=torch.bool)
        for g in range(G):
            mask[g, 0, mask_rows_fn(i, g, p)] = True
        mask = mask.repeat_interleave(Hq // G, dim=0)            # [Hq][1][cap]
        o1 = F.scaled_dot_product_attention(
            q[i].to(F64).unsqueeze(1), k_cache[s].to(F64), v_cache[s].to(F64),
            attn_mask=mask, scale=scale, enable_gqa=True)
        out[i] = o1[:, 0]
    return out


def _attn_case(seed, S, cap, G, Hq, D, lengths, queries):
    g = torch.Generator().manual_seed(seed)
    k = torch.zeros((S, G, cap, D), dtype=F64)
    v = torch.zeros((S, G, cap, D), dtype=F64)
    idx = torch.zeros((S, G, cap, 3), dtype=F64)
    for s in range(S):
        L = lengths[s]
        k[s, :, :L] = torch.randn((G, L, D), generator=g, dtype=F64)
        v[s, :, :L] = torch.randn((G, L, D), generator=g, dtype=F64)
        idx[s, :, :L] = torch.randn((G, L, 3), generator=g, dtype=F64)
    qs = torch.tensor([a for a, _ in queries], dtype=torch.int32)
    qp = torch.tensor([b for _, b in queries], dtype=torch.int32)
    q = torch.randn((len(queries), Hq, D), generator=g, dtype=F64)
    iq = torch.randn((len(queries), G, 3), generator=g, dtype=F64)
    return k, v, idx, qs, qp, q, iq


def pin_dense_equivalence(o, seed=5):
    """With no more visible blocks than top_k, MSA is dense causal attention
    (RADV review comment: byte-identical MSA/dense below top_k*block)."""
    block, top_k, G, Hq, D, cap = 4, 4, 2, 6, 8, 16
    k, v, idx, qs, qp, q, iq = _attn_case(seed, 2, cap, G, Hq, D, [16, 13],
                                          [(0, 0), (0, 3), (0, 4), (1, 9), (1, 12), (0, 15)])
    bs = o.block_scores(iq, idx, qs, qp, block)
    sel, _ = o.select_blocks(bs, qp, block, top_k)
    got = o.sparse_attention(q, k, v, sel, qs, qp, block)
    want = _sdpa_reference(q, k, v, qs, qp, lambda i, g, p: torch.arange(p + 1))
    assert torch.allclose(got, want, rtol=0, atol=1e-12), (got - want).abs().max()


def pin_block_mask_equivalence(o, seed=6):
    """With more visible blocks than top_k, MSA is attention under the mask
    'row in a selected block and row <= position'."""
    block, top_k, G, Hq, D, cap = 4, 2, 2, 4, 8, 40
    k, v, idx, qs, qp, q, iq = _attn_case(seed, 2, cap, G, Hq, D, [40, 33],
                                          [(0, 39), (0, 21), (1, 32), (1, 17), (0, 8)])
    bs = o.block_scores(iq, idx, qs, qp, block)
    sel, _ = o.select_blocks(bs, qp, block, top_k)

    def rows(i, g, p):
        r = torch.arange(cap)
        keep = torch.zeros(cap, dtype=torch.bool)
        for b in sel[i, g].tolist():
            if b >= 0:
                keep |= (r // block) == b
        return keep & (r <= p)

    got = o.sparse_attention(q, k, v, sel, qs, qp, block)
    want = _sdpa_reference(q, k, v, qs, qp, rows)
    assert torch.allclose(got, want, rtol=0, atol=1e-12), (got - want).abs().max()


def pin_attention_closed_forms(o, seed=7):
    """Equal keys give uniform weights (mean of the attended V rows); a
    query at position 0 returns its own V row."""
    g = torch.Generator().manual_seed(seed)
    block, G, Hq, D, cap = 4, 2, 4, 3, 32
    k = torch.zeros((1, G, cap, D), dtype=F64)
    k[:] = torch.randn((D,), generator=g, dtype=F64)             # all rows equal
    v = torch.randn((1, G, cap, D), generator=g, dtype=F64)
    q = torch.randn((1, Hq, D), generator=g, dtype=F64)
    for pos, sel_ids in ((25, [1, 3, 6]), (0, [0]), (30, [7]), (13, [0, 2, 3])):
        sel = torch.full((1, G, 3), -1, dtype=torch.int32)
        sel[0, :, :len(sel_ids)] = torch.tensor(sel_ids, dtype=torch.int32)
        out = o.sparse_attention(q, k, v, sel, torch.zeros(1, dtype=torch.int32),
                                 torch.tensor([pos], dtype=torch.int32), block)
        rows = [j for b in sel_ids for j in range(b * block, b * block + block) if j <= pos]
        for h in range(Hq):
            gg = h // (Hq // G)
            want = v[0, gg, rows].mean(dim=0)
            assert torch.allclose(out[0, h], want, atol=1e-12), (pos, h)


def pin_append_random(o, seed=8):
    g = torch.Generator().manual_seed(seed)
    cache = torch.randn((3, 2, 8, 4), generator=g)
    new = torch.randn((5, 2, 4), generator=g)
    ts = torch.tensor([2, 0, 2, 1, 0], dtype=torch.int32)
    tp = torch.tensor([7, 0, 3, 5, 6], dtype=torch.int32)
    out = o.indexer_append(cache, new, ts, tp)
    touched = set()
    for t in range(5):
        assert torch.equal(out[int(ts[t]), :, int(tp[t])], new[t])
        touched.add((int(ts[t]), int(tp[t])))
    for s in range(3):
        for p in range(8):
            if (s, p) not in touched:
                assert torch.equal(out[s, :, p], cache[s, :, p])


def _pool_from_contiguous(cache, block):
    """Closed form of the identity paging: page s * n_blocks + b holds block b
    of stream s, i.e. the [S][G][cap][row] cache with its block axis moved in
    front of the group axis."""
    S, G, cap, row = cache.shape
    nb = cap // block
    return cache.reshape(S, G, nb, block, row).permute(0, 2, 1, 3, 4).reshape(S * nb, G, block, row)


def pin_paged_identity_layout(o, seed=9):
    """Identity block table over a reshaped contiguous cache: the logical view
    must return the cache exactly (a transposed table, a slot reordered inside
    a page or a wrong page index all break it)."""
    g = torch.Generator().manual_seed(seed)
    cache = torch.randn((3, 2, 12, 5), generator=g, dtype=torch.float64)
    pool = _pool_from_contiguous(cache, 4)
    table = torch.arange(9, dtype=torch.int32).view(3, 3)
    assert torch.equal(o.logical_cache(pool, table, 4), cache)


def pin_paged_permutation_and_sharing(o, seed=10):
    """Moving pages to other pool slots (spare pages holding garbage) and
    renaming the table entries the same way leaves the logical view unchanged;
    a block mapped to another stream's page shows that page's rows; a block
    with no page reads as NaN."""
    g = torch.Generator().manual_seed(seed)
    cache = torch.randn((3, 2, 12, 5), generator=g, dtype=torch.float64)
    pool = _pool_from_contiguous(cache, 4)
    table = torch.arange(9, dtype=torch.int32).view(3, 3)
    perm = torch.randperm(11, generator=g)              # old page i -> new slot perm[i]
    moved = torch.full((11, 2, 4, 5), 1.0e6, dtype=torch.float64)
    moved[perm[:9]] = pool
    table2 = perm[table.long()].to(torch.int32)
    assert torch.equal(o.logical_cache(moved, table2, 4), cache)
    table3 = table2.clone()
    table3[2, 0] = table2[0, 0]                          # stream 2 shares stream 0's first page
    table3[1, 2] = -1                                    # stream 1's last block unmapped
    view = o.logical_cache(moved, table3, 4)
    assert torch.equal(view[2, :, :4], cache[0, :, :4]) and torch.equal(view[2, :, 4:], cache[2, :, 4:])
    assert bool(torch.isnan(view[1, :, 8:]).all()) and torch.equal(view[1, :, :8], cache[1, :, :8])


def pin_paged_append_commutes(o, seed=11):
    """Appending through the page table and then taking the logical view equals
    taking the view and appending to it (the contiguous append is pinned by
    pin_append_random); pages no token maps to are left untouched."""
    g = torch.Generator().manual_seed(seed)
    cache = torch.randn((3, 2, 12, 5), generator=g, dtype=torch.float64)
    pool = torch.cat([_pool_from_contiguous(cache, 4), torch.randn((2, 2, 4, 5), generator=g, dtype=torch.float64)])
    perm = torch.randperm(11, generator=g)
    moved = torch.empty_like(pool)
    moved[perm] = pool
    table = perm[torch.arange(9).view(3, 3)].to(torch.int32)
    new = torch.randn((6, 2, 5), generator=g, dtype=torch.float64)
    ts = torch.tensor([2, 0, 2, 1, 0, 1], dtype=torch.int32)
    tp = torch.tensor([11, 0, 3, 5, 6, 8], dtype=torch.int32)
    after = o.paged_append(moved, new, ts, tp, table, 4)
    assert torch.equal(o.logical_cache(after, table, 4), o.indexer_append(cache, new, ts, tp))
    spare = perm[9:]
    assert torch.equal(after[spare], moved[spare])


def _dsa_case(seed, S=2, cap=12, H=3, Di=4, n_q=3):
    g = torch.Generator().manual_seed(seed)
    keys = torch.randn((S, cap, Di), generator=g, dtype=F64)
    q = torch.randn((n_q, H, Di), generator=g, dtype=F64)
    w = torch.randn((n_q, H), generator=g, dtype=F64)
    qs = torch.tensor([i % S for i in range(n_q)], dtype=torch.int32)
    qp = torch.tensor([cap - 1 - 3 * i for i in range(n_q)], dtype=torch.int32)
    return keys, q, w, qs, qp


def pin_dsa_scores_identities(o, seed=12):
    """Lightning-indexer score identities: a basis query on one head with unit
    weight reads one key coordinate (through the ReLU when enabled); the score
    is linear in the weights; relu(x) - relu(-x) = x turns the ReLU scores of
    q and -q into the plain weighted dot products; tokens past the query are
    -inf."""
    keys, q, w, qs, qp = _dsa_case(seed)
    n_q, H, Di = q.shape
    # basis query: head 1 = e_2, weight e_1 -> score[s] = act(key[s][2])
    qb = torch.zeros_like(q)
    qb[:, 1, 2] = 1.0
    wb = torch.zeros_like(w)
    wb[:, 1] = 1.0
    for relu in (False, True):
        sc = o.dsa_token_scores(qb, wb, keys, qs, qp, relu=relu)
        for t in range(n_q):
            p = int(qp[t])
            col = keys[int(qs[t]), :p + 1, 2]
            want = col.clamp_min(0.0) if relu else col
            assert torch.equal(sc[t, :p + 1], want)
            assert bool(torch.isneginf(sc[t, p + 1:]).all())
    # linear in the weights
    w2 = torch.randn(w.shape, generator=torch.Generator().manual_seed(seed + 1), dtype=F64)
    for relu in (False, True):
        a = o.dsa_token_scores(q, w + 2.0 * w2, keys, qs, qp, relu)
        b = o.dsa_token_scores(q, w, keys, qs, qp, relu) + 2.0 * o.dsa_token_scores(q, w2, keys, qs, qp, relu)
        fin = torch.isfinite(a)
        assert torch.equal(fin, torch.isfinite(b))
        assert torch.allclose(a[fin], b[fin], rtol=0, atol=1e-12)
    # relu(x) - relu(-x) = x
    plus = o.dsa_token_scores(q, w, keys, qs, qp, True)
    minus = o.dsa_token_scores(-q, w, keys, qs, qp, True)
    plain = o.dsa_token_scores(q, w, keys, qs, qp, False)
    fin = torch.isfinite(plain)
    assert torch.allclose((plus - minus)[fin], plain[fin], rtol=0, atol=1e-12)
    # a ReLU score with nonnegative weights is nonnegative
    assert bool((o.dsa_token_scores(q, w.abs(), keys, qs, qp, True)[fin] >= 0).all())


def _bruteforce_tokens(row, pos, top_k):
    """The k-subset of visible tokens whose (score, -index) pairs, sorted
    descending, are lexicographically largest."""
    nvis = pos + 1
    k = min(top_k, nvis)
    best, best_ids = None, None
    for comb in itertools.combinations(range(nvis), k):
        key = sorted(((float(row[s]), -s) for s in comb), reverse=True)
        if best is None or key > best:
            best, best_ids = key, sorted(comb)
    return best_ids


def pin_dsa_selection_bruteforce(o, seed=13):
    """Token top-k against brute force over every subset, on small integer
    scores with many ties, for every visible length and several k."""
    g = torch.Generator().manual_seed(seed)
    for trial in range(40):
        n = 9
        row = torch.randint(-2, 3, (n,), generator=g).to(F64)
        pos = int(torch.randint(0, n, (1,), generator=g))
        for top_k in (1, 2, 3, 5, 9):
            assert o.dsa_select_one(row, pos, top_k) == _bruteforce_tokens(row, pos, top_k), (row, pos, top_k)
    sel, n_sel = o.dsa_select_tokens(torch.tensor([[3.0, 1.0, 3.0, 2.0, float("-inf")]], dtype=F64),
                                     torch.tensor([3], dtype=torch.int32), 2, 4)
    assert sel.tolist() == [[0, 2, -1, -1]] and n_sel.tolist() == [2]
    assert o.dsa_boundary_scores(torch.tensor([3.0, 1.0, 3.0, 2.0], dtype=F64), 3, 2) == (3.0, 2.0)
    assert o.dsa_boundary_scores(torch.tensor([3.0, 1.0], dtype=F64), 1, 2) is None
    # a NaN score ranks as -inf: below every finite score, ties with -inf by index
    nan_row = torch.tensor([float("nan"), 0.5, float("-inf"), -3.0, float("nan")], dtype=F64)
    assert o.dsa_ranked_tokens(nan_row, 4) == [1, 3, 0, 2, 4]


def _dsa_attn_case(seed, cap=12, G=2, Hq=4, D=6):
    g = torch.Generator().manual_seed(seed)
    k = torch.randn((2, G, cap, D), generator=g, dtype=F64)
    v = torch.randn((2, G, cap, D), generator=g, dtype=F64)
    q = torch.randn((3, Hq, D), generator=g, dtype=F64)
    qs = torch.tensor([0, 1, 1], dtype=torch.int32)
    qp = torch.tensor([11, 7, 4], dtype=torch.int32)
    return k, v, q, qs, qp


def pin_dsa_noop_exact(o, seed=14):
    """With at most top_k visible tokens every token is kept and the attention
    is dense causal attention (the DSA page's "no-op-exact" check), against
    scaled_dot_product_attention in float64."""
    k, v, q, qs, qp = _dsa_attn_case(seed)
    scores = torch.randn((3, 12), generator=torch.Generator().manual_seed(seed), dtype=F64)
    sel, n_sel = o.dsa_select_tokens(scores, qp, 16, 16)
    assert n_sel.tolist() == [12, 8, 5]
    got = o.dsa_sparse_attention(q, k, v, sel, qs, qp)
    want = _sdpa_reference(q, k, v, qs, qp, lambda i, g, p: list(range(p + 1)))
    assert torch.allclose(got, want, rtol=0, atol=1e-12), (got - want).abs().max()


def pin_dsa_mask_equivalence(o, seed=15):
    """With more visible tokens than top_k the attention equals
    scaled_dot_product_attention under a boolean mask of the kept tokens, the
    same set for every group."""
    k, v, q, qs, qp = _dsa_attn_case(seed)
    scores = torch.randn((3, 12), generator=torch.Generator().manual_seed(seed), dtype=F64)
    top_k = 3
    sel, n_sel = o.dsa_select_tokens(scores, qp, top_k, 4)
    assert n_sel.tolist() == [3, 3, 3]
    kept = [_bruteforce_tokens(scores[i], int(qp[i]), top_k) for i in range(3)]
    got = o.dsa_sparse_attention(q, k, v, sel, qs, qp)
    want = _sdpa_reference(q, k, v, qs, qp, lambda i, g, p: kept[i])
    assert torch.allclose(got, want, rtol=0, atol=1e-12), (got - want).abs().max()


ALL_PINS = [pin_golden, pin_basis_query_pooling, pin_scores_bilinear, pin_selection_bruteforce,
            pin_selection_nan_rule, pin_selection_invariants, pin_local_forced, pin_dense_equivalence,
            pin_block_mask_equivalence, pin_attention_closed_forms, pin_append_random,
            pin_paged_identity_layout, pin_paged_permutation_and_sharing, pin_paged_append_commutes,
            pin_dsa_scores_identities, pin_dsa_selection_bruteforce, pin_dsa_noop_exact, pin_dsa_mask_equivalence]


def run_all(o):
    for pin in ALL_PINS:
        pin(o)


def near_tie_excused(boundary, oracle_bs_row, got_ids, want_ids, rel=1e-5):
    """Near-tie rule for comparing a GPU selection with the oracle's: a set
    mismatch is excused only when the oracle's last-selected and first-
    unselected scores differ (no exact tie) by less than rel of their
    magnitude and every block in the symmetric difference scores within that
    band of the last-selected score."""
    if boundary is None:
        return False
    s16, s17 = boundary
    if s16 == s17:
        return False
    band = rel * max(abs(s16), abs(s17))
    if abs(s16 - s17) >= band:
        return False
    diff = set(got_ids) ^ set(want_ids)
    return all(abs(float(oracle_bs_row[b]) - s16) <= band for b in diff)


def max_abs_tolerances():
    """bf16 output tolerances against the FP64 oracle."""
    return 4e-3, 5e-4
