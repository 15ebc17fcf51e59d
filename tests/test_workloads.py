"""The seeded input generators that both the CUDA path and the oracle draw
from: deterministic, laid out as the library expects, and sampled streams
identical to the same streams of the full draw (the host-core baseline and
every bench rank draw sub-ranges of streams)."""
import pytest
import torch

import workloads as W


def _small(queries, quantize=False):
    # 4 streams, 300 existing + 40 new tokens (a ragged last block), 2 groups
    return W.Workload(f"small_{queries}", 4, 300, 340, queries, n_q_heads=32, n_kv_heads=2, quantize_idx=quantize)


@pytest.mark.parametrize("queries", ["last", "new"])
def test_same_seed_same_inputs(queries):
    w = _small(queries)
    a, b = W.make_inputs(w, seed=5), W.make_inputs(w, seed=5)
    for name in ("idx_k_cache", "k_cache", "v_cache", "idx_k_new", "k_new", "v_new", "idx_q", "q",
                 "tok_stream", "tok_pos", "q_stream", "q_pos"):
        assert torch.equal(getattr(a, name), getattr(b, name)), name
    c = W.make_inputs(w, seed=6)
    assert not torch.equal(a.k_cache, c.k_cache)


@pytest.mark.parametrize("queries", ["last", "new"])
def test_layout_and_positions(queries):
    w = _small(queries)
    inp = W.make_inputs(w, seed=1)
    S, G, cap = w.n_streams, w.n_kv_heads, w.capacity
    assert cap % 128 == 0 and cap >= w.l_total
    assert inp.idx_k_cache.shape == (S, G, cap, w.idx_dim) and inp.idx_k_cache.dtype == torch.float32
    assert inp.k_cache.shape == (S, G, cap, w.head_dim) and inp.k_cache.dtype == torch.bfloat16
    # the cache holds the existing tokens only; the new ones arrive through the append inputs
    assert torch.count_nonzero(inp.k_cache[:, :, w.l_existing:]) == 0
    assert torch.count_nonzero(inp.k_cache[:, :, :w.l_existing]) > 0
    n_new = w.l_total - w.l_existing
    assert inp.tok_stream.tolist() == [s for s in range(S) for _ in range(n_new)]
    assert inp.tok_pos.tolist() == list(range(w.l_existing, w.l_total)) * S
    if queries == "last":
        assert inp.q_stream.tolist() == list(range(S)) and inp.q_pos.tolist() == [w.l_total - 1] * S
    else:
        assert torch.equal(inp.q_stream, inp.tok_stream) and torch.equal(inp.q_pos, inp.tok_pos)
    n_q = inp.q_pos.numel()
    assert inp.idx_q.shape == (n_q, G, w.idx_dim) and inp.q.shape == (n_q, w.n_q_heads, w.head_dim)


@pytest.mark.parametrize("queries", ["last", "new"])
def test_sampled_streams_match_the_full_draw(queries):
    w = _small(queries)
    full = W.make_inputs(w, seed=3)
    part = W.make_inputs(w, seed=3, streams=range(2, 4))
    for name in ("idx_k_cache", "k_cache", "v_cache"):
        assert torch.equal(getattr(part, name), getattr(full, name)[2:4]), name
    # new tokens and queries of streams 2 and 3, in the same order
    keep_tok = full.tok_stream >= 2
    for name in ("idx_k_new", "k_new", "v_new"):
        assert torch.equal(getattr(part, name), getattr(full, name)[keep_tok]), name
    keep_q = full.q_stream >= 2
    assert torch.equal(part.q, full.q[keep_q]) and torch.equal(part.idx_q, full.idx_q[keep_q])
    assert torch.equal(part.q_pos, full.q_pos[keep_q])
    # stream ids are local to the sample
    assert part.q_stream.tolist() == (full.q_stream[keep_q] - 2).tolist()


def test_quantised_indexer_keys_make_ties():
    # the tie workloads draw indexer values on a coarse grid, so equal block
    # scores occur and the selection's tie rule is exercised
    w = _small("new", quantize=True)
    inp = W.make_inputs(w, seed=2)
    vals = inp.idx_k_cache[:, :, :w.l_existing].flatten()
    assert vals.unique().numel() < vals.numel() // 100


def test_step_sets_redraw_the_new_token_and_query_only():
    """The benchmark's second decode input set: same layouts and
    distributions as the workload's own new token and query, different
    values, deterministic, and the same per stream whatever streams are
    drawn."""
    w = W.Workload("small_decode", 5, 299, 300, "last", n_q_heads=32, n_kv_heads=2)
    inp = W.make_inputs(w, seed=0)
    a, b = W.make_step_set(w, seed=1001), W.make_step_set(w, seed=1001)
    for name in ("idx_k_new", "k_new", "v_new", "idx_q", "q"):
        got, base = a[name], getattr(inp, name)
        assert got.shape == base.shape and got.dtype == base.dtype, name
        assert torch.equal(got, b[name]), name
        assert not torch.equal(got, base), name
    part = W.make_step_set(w, seed=1001, streams=range(2, 4))
    assert torch.equal(part["q"], a["q"][2:4]) and torch.equal(part["idx_k_new"], a["idx_k_new"][2:4])
    with pytest.raises(ValueError):
        W.make_step_set(_small("new"), seed=1)
