"""Plant plausible mistakes in a private copy of the CPU oracle and check that
at least one pin fails for each.  Shows the pins are strong enough to catch
a dropped term, a wrong sign or index, a transposed operand, a reversed tie
rule, a missing bias or mask, or a wrong head-to-group mapping.  CPU only;
the real oracle module is never modified."""
import importlib.util
import math
import os

import pytest
import torch

from tests import oracle_pins as P

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "msa_oracle.py")


def fresh_oracle(tag):
    spec = importlib.util.spec_from_file_location(f"_oracle_copy_{tag}", ORACLE_SRC)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_causal_off_by_one(o):
    orig = o.pool_visible

    def pool_visible(s, positions, block, n_blocks):
        pos = torch.as_tensor(positions, dtype=torch.long).clamp_min(1) - 1
        return orig(s, pos, block, n_blocks)
    o.pool_visible = pool_visible


def _mut_no_causal_mask(o):
    orig = o.pool_visible

    def pool_visible(s, positions, block, n_blocks):
        # pools every slot of a visible block, including the ones past the query
        pos = torch.as_tensor(positions, dtype=torch.long).reshape(-1)
        out = orig(s, torch.full_like(pos, s.shape[1] - 1), block, n_blocks)
        for i in range(out.shape[0]):
            out[i, int(pos[i]) // block + 1:] = float("-inf")
        return out
    o.pool_visible = pool_visible


def _mut_tie_higher_index(o):
    def ranked_blocks(row, pos, block):
        nvis = o.n_visible_blocks(pos, block)
        return sorted(range(nvis), key=lambda b: (-float(row[b]), -b))
    o.ranked_blocks = ranked_blocks


def _mut_no_bias(o):
    o.LOCAL_BIAS = 0.0

    orig = o.block_scores

    def block_scores(idx_q, idx_k, qs, qp, block, local_bias=0.0):
        return orig(idx_q, idx_k, qs, qp, block, 0.0)
    o.block_scores = block_scores


def _mut_gqa_modulo(o):
    def sparse_attention(q, k_cache, v_cache, sel, q_stream, q_pos, block, scale=None, queries=None):
        n_q, Hq, D = q.shape
        G = k_cache.shape[1]
        scale = 1.0 / math.sqrt(D) if scale is None else scale
        out = torch.empty((n_q, Hq, D), dtype=torch.float64)
        for i in range(n_q):
            s, p = int(q_stream[i]), int(q_pos[i])
            for h in range(Hq):
                g = h % G
                rows = torch.tensor(o.attended_rows(sel[i, g].tolist(), p, block))
                K = k_cache[s, g, rows].double()
                V = v_cache[s, g, rows].double()
                w = torch.softmax(K @ q[i, h].double() * scale, 0)
                out[i, h] = w @ V
        return out
    o.sparse_attention = sparse_attention


def _mut_no_scale(o):
    orig = o.sparse_attention

    def sparse_attention(q, k, v, sel, qs, qp, block, scale=None, queries=None):
        return orig(q, k, v, sel, qs, qp, block, 1.0, queries)
    o.sparse_attention = sparse_attention


def _mut_nvis_off_by_one(o):
    o.n_visible_blocks = lambda pos, block: max(pos // block, 1)


def _mut_transposed_scores(o):
    def token_scores(q, rows):
        rows = rows.double()
        # uses the key's coordinates in reverse order
        return rows.flip(-1) @ q.double()
    o.token_scores = token_scores


def _mut_dropped_term(o):
    def token_scores(q, rows):
        return rows.double()[:, :-1] @ q.double()[:-1]
    o.token_scores = token_scores


def _mut_future_rows(o):
    def attended_rows(sel_ids, pos, block):
        rows = []
        for b in sel_ids:
            if int(b) >= 0:
                rows.extend(range(int(b) * block, (int(b) + 1) * block))
        return rows
    o.attended_rows = attended_rows


def _mut_sign(o):
    orig = o.sparse_attention

    def sparse_attention(q, k, v, sel, qs, qp, block, scale=None, queries=None):
        D = q.shape[-1]
        return orig(q, k, v, sel, qs, qp, block, -1.0 / math.sqrt(D), queries)
    o.sparse_attention = sparse_attention


def _mut_k_minus_one(o):
    def select_one(row, pos, block, top_k):
        return sorted(o.ranked_blocks(row, pos, block)[:max(top_k - 1, 1)])
    o.select_one = select_one


def _mut_unsorted_ids(o):
    def select_one(row, pos, block, top_k):
        return o.ranked_blocks(row, pos, block)[:top_k]
    o.select_one = select_one


def _mut_lowest_scores(o):
    def ranked_blocks(row, pos, block):
        nvis = o.n_visible_blocks(pos, block)
        loc = pos // block
        rest = sorted((b for b in range(nvis) if b != loc), key=lambda b: (float(row[b]), b))
        return [loc] + rest
    o.ranked_blocks = ranked_blocks


def _mut_nan_unordered(o):
    def ranked_blocks(row, pos, block):
        nvis = o.n_visible_blocks(pos, block)
        vals = [float(row[b]) for b in range(nvis)]
        return sorted(range(nvis), key=lambda b: (-vals[b], b))     # NaN left as NaN
    o.ranked_blocks = ranked_blocks


def _mut_append_swapped(o):
    def indexer_append(cache, new, ts, tp):
        out = cache.clone()
        for t in range(ts.numel()):
            out[int(ts[t]), :, int(tp[t])] = new[ts.numel() - 1 - t]
        return out
    o.indexer_append = indexer_append


def _mut_paged_table_transposed(o):
    def logical_cache(pool, table, block):
        S, nb = table.shape
        out = torch.full((S, pool.shape[1], nb * block, pool.shape[3]), float("nan"), dtype=pool.dtype)
        for s in range(S):
            for b in range(nb):
                page = int(table[b % S, s % nb])
                out[s, :, b * block:(b + 1) * block] = pool[page]
        return out
    o.logical_cache = logical_cache


def _mut_paged_slots_reversed(o):
    orig = o.logical_cache

    def logical_cache(pool, table, block):
        return orig(pool.flip(2), table, block)
    o.logical_cache = logical_cache


def _mut_paged_append_next_slot(o):
    def paged_append(pool, new, ts, tp, table, block):
        out = pool.clone()
        for t in range(ts.numel()):
            s, p = int(ts[t]), int(tp[t])
            out[int(table[s, p // block]), :, (p + 1) % block] = new[t]
        return out
    o.paged_append = paged_append


def _mut_dsa_no_relu(o):
    orig = o.dsa_token_scores

    def dsa_token_scores(q, w, k, qs, qp, relu=True):
        return orig(q, w, k, qs, qp, False)
    o.dsa_token_scores = dsa_token_scores


def _mut_dsa_unweighted(o):
    orig = o.dsa_token_scores

    def dsa_token_scores(q, w, k, qs, qp, relu=True):
        return orig(q, torch.ones_like(w), k, qs, qp, relu)
    o.dsa_token_scores = dsa_token_scores


def _mut_dsa_future_tokens(o):
    orig = o.dsa_token_scores

    def dsa_token_scores(q, w, k, qs, qp, relu=True):
        full = torch.full_like(qp, k.shape[1] - 1)
        return orig(q, w, k, qs, full, relu)
    o.dsa_token_scores = dsa_token_scores


def _mut_dsa_tie_higher_index(o):
    def dsa_ranked_tokens(row, pos):
        return sorted(range(pos + 1), key=lambda s: (-float(row[s]), -s))
    o.dsa_ranked_tokens = dsa_ranked_tokens


def _mut_dsa_k_minus_one(o):
    orig = o.dsa_select_one

    def dsa_select_one(row, pos, top_k):
        return orig(row, pos, top_k)[:max(1, top_k - 1)] if pos + 1 > top_k else orig(row, pos, top_k)
    o.dsa_select_one = dsa_select_one


def _mut_dsa_group_zero(o):
    def dsa_sparse_attention(q, k, v, sel, qs, qp, scale=None):
        return orig(q, k[:, :1].expand_as(k), v[:, :1].expand_as(v), sel, qs, qp, scale)
    orig = o.dsa_sparse_attention
    o.dsa_sparse_attention = dsa_sparse_attention


MUTATIONS = [_mut_causal_off_by_one, _mut_no_causal_mask, _mut_tie_higher_index, _mut_no_bias,
             _mut_gqa_modulo, _mut_no_scale, _mut_nvis_off_by_one, _mut_transposed_scores,
             _mut_dropped_term, _mut_future_rows, _mut_sign, _mut_k_minus_one,
             _mut_unsorted_ids, _mut_lowest_scores, _mut_nan_unordered, _mut_append_swapped, _mut_paged_table_transposed,
             _mut_paged_slots_reversed, _mut_paged_append_next_slot, _mut_dsa_no_relu, _mut_dsa_unweighted,
             _mut_dsa_future_tokens, _mut_dsa_tie_higher_index, _mut_dsa_k_minus_one, _mut_dsa_group_zero]


@pytest.mark.parametrize("mut", MUTATIONS, ids=lambda f: f.__name__[5:])
def test_mutation_is_caught(mut):
    o = fresh_oracle(mut.__name__)
    mut(o)
    failed = []
    for pin in P.ALL_PINS:
        try:
            pin(o)
        except Exception:        # AssertionError, or a crash the mistake causes
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mut.__name__}"


def test_unmutated_copy_passes():
    P.run_all(fresh_oracle("clean"))
