"""Paged caches on the GPU: the *_paged calls against the oracle's logical view
of the same page pools, and against the contiguous calls on the same data.

The pools are shuffled (every block at a random page, spare pages filled
with a poison value that would dominate any score or output it reached),
and some cases let several streams share prefix pages."""
import math

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
import oracle
import workloads as W
from tests import parity as PT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_attention_maxpool_b200 import build as msa_build
    msa_build.build()
    msa.msa_get_device_error()


def test_paged_decode_shared_prefix():
    w = W.Workload("paged_decode_6x3000", 6, 2999, 3000, "last")
    inp = W.make_inputs(w, seed=41)
    rep = PT.full_parity(inp, paged=dict(seed=1, spare_pages=5, shared_prefix_blocks=7))
    print("\n[paged] decode shared prefix:", rep)
    assert rep["near_ties"] == 0


def test_paged_decode_f16_keys():
    w = W.Workload("paged_decode_f16_5x2600", 5, 2599, 2600, "last")
    inp = W.make_inputs(w, seed=42)
    rep = PT.full_parity(inp, idx_f16=True, paged=dict(seed=2, spare_pages=2, shared_prefix_blocks=3))
    print("\n[paged] decode f16:", rep)


def test_paged_prefill_tile_path():
    # 2 x 1100 new tokens on 300 existing: prefill-shaped, the block scores take the tile path
    w = W.Workload("paged_prefill_2x1400", 2, 300, 1400, "new")
    inp = W.make_inputs(w, seed=43)
    rep = PT.full_parity(inp, prefill=True, paged=dict(seed=3, spare_pages=4, shared_prefix_blocks=2))
    print("\n[paged] prefill:", rep)


def test_paged_prefill_ties_f16():
    w = W.Workload("paged_prefill_ties_2x700_on_1500", 2, 1500, 2200, "new", quantize_idx=True)
    inp = W.make_inputs(w, seed=44)
    rep = PT.full_parity(inp, prefill=True, idx_f16=True, paged=dict(seed=4, spare_pages=1))
    print("\n[paged] prefill ties f16:", rep)
    assert rep["max_score_err"] == 0.0


def test_paged_prefill_long_context():
    # 33K-token caches on pages: long block tables, few blocks shared per tile
    w = W.Workload("paged_prefill_2x64_on_33000", 2, 33000, 33064, "new")
    inp = W.make_inputs(w, seed=49)
    rep = PT.full_parity(inp, prefill=True, paged=dict(seed=7, spare_pages=3, shared_prefix_blocks=4))
    print("\n[paged] prefill long context:", rep)


def _contiguous_vs_paged(w, seed, prefill):
    inp = W.make_inputs(w, seed=seed)
    shape = PT.shape_of(w)
    d = PT.to_dev(inp)
    out_c, sel_c, nsel_c, bs_c, err_c = PT.run_step(shape, d, prefill)
    lay = W.page_layout(inp, seed=seed, spare_pages=7)
    dp = PT.to_dev(inp)
    dp["idx_k_cache"], dp["k_cache"], dp["v_cache"] = (lay.idx_pool.cuda(), lay.k_pool.cuda(), lay.v_pool.cuda())
    pages = msa.Pages(lay.block_table.cuda(), lay.n_pages)
    out_p, sel_p, nsel_p, bs_p, err_p = PT.run_step(shape, dp, prefill, pages)
    assert err_c == 0 and err_p == 0
    # same arithmetic on the same rows: bit-identical results
    assert torch.equal(bs_c, bs_p)
    assert torch.equal(sel_c, sel_p) and torch.equal(nsel_c, nsel_p)
    assert torch.equal(out_c, out_p)


def test_paged_equals_contiguous_bitwise_decode():
    _contiguous_vs_paged(W.Workload("bitwise_decode_9x5000", 9, 4999, 5000, "last"), 45, False)


def test_paged_equals_contiguous_bitwise_prefill():
    _contiguous_vs_paged(W.Workload("bitwise_prefill_2x900", 2, 200, 1100, "new"), 46, True)


def test_paged_equals_contiguous_bitwise_long_prefill():
    _contiguous_vs_paged(W.Workload("bitwise_prefill_2x80_on_33000", 2, 33000, 33080, "new"), 50, True)


def test_paged_equals_contiguous_bitwise_full_size_decode():
    """The 32-stream x 32K decode workload, paged with every block shuffled."""
    _contiguous_vs_paged(W.DECODE_32K_X32, 0, False)


def test_unmapped_page_is_skipped_and_flagged():
    """A visible block whose table entry is -1 scores -inf and is left out of
    attention; MSA_DEVERR_PAGE_RANGE is set; every other result is the one the
    mapped layout gives with that block unselected."""
    w = W.Workload("unmapped_4x3000", 4, 3000, 3000, "last")
    inp = W.make_inputs(w, seed=47)
    shape = PT.shape_of(w)
    lay = W.page_layout(inp, seed=5, spare_pages=2)
    dev = "cuda"
    idx_pool, k_pool, v_pool = lay.idx_pool.to(dev), lay.k_pool.to(dev), lay.v_pool.to(dev)
    qs, qp = inp.q_stream.to(dev), inp.q_pos.to(dev)
    idx_q, q = inp.idx_q.to(dev), inp.q.to(dev)
    good = msa.Pages(lay.block_table.to(dev), lay.n_pages)
    bs_ok = msa.msa_block_scores_paged(shape, good, idx_q, idx_pool, qs, qp)
    sel_ok, _ = msa.msa_select_topk(shape, bs_ok, qp)
    assert msa.msa_get_device_error() == 0
    # unmap one block that stream 1's query selects (not its local block)
    s_bad = 1
    b_bad = int([b for b in sel_ok[s_bad, 0].tolist() if 0 <= b < 3000 // 128][0])
    table = lay.block_table.clone()
    table[s_bad, b_bad] = -1
    bad = msa.Pages(table.to(dev), lay.n_pages)
    bs = msa.msa_block_scores_paged(shape, bad, idx_q, idx_pool, qs, qp)
    assert msa.msa_get_device_error() & 0x10
    want = bs_ok.clone()
    want[s_bad, :, b_bad] = float("-inf")
    assert torch.equal(bs, want)
    # attention with the mapped selection but the unmapped table: the block drops out
    out = msa.msa_sparse_attn_decode_paged(shape, bad, q, k_pool, v_pool, sel_ok, qs, qp)
    assert msa.msa_get_device_error() & 0x10
    sel_drop = sel_ok.clone()
    row = sel_drop[s_bad]
    row[row == b_bad] = -1
    out_ref = msa.msa_sparse_attn_decode_paged(shape, good, q, k_pool, v_pool, sel_drop, qs, qp)
    assert msa.msa_get_device_error() == 0
    assert torch.equal(out, out_ref)
    # the oracle agrees on the dropped-block output of the affected stream
    logical_k = oracle.logical_cache(lay.k_pool, lay.block_table, w.block)
    logical_v = oracle.logical_cache(lay.v_pool, lay.block_table, w.block)
    o = oracle.sparse_attention(inp.q, logical_k, logical_v, sel_drop.cpu(), inp.q_stream, inp.q_pos, w.block,
                                1.0 / math.sqrt(w.head_dim))
    PT.check_attention(out.cpu(), o)


@pytest.mark.parametrize("cap_blocks", [24, 260], ids=["short_cache", "long_cache"])
def test_unmapped_page_is_skipped_in_prefill(cap_blocks):
    """Prefill attention with a selected block on an unmapped page: the block
    drops out of that query's attention (bit-identical to dropping it from the
    selection) and MSA_DEVERR_PAGE_RANGE is set."""
    n_new = 40
    L = cap_blocks * 128
    w = W.Workload(f"unmapped_prefill_{cap_blocks}", 2, L - n_new, L, "new")
    inp = W.make_inputs(w, seed=51)
    shape = PT.shape_of(w)
    lay = W.page_layout(inp, seed=8, spare_pages=2)
    dev = "cuda"
    k_pool, v_pool = lay.k_pool.to(dev), lay.v_pool.to(dev)
    qs, qp, q = inp.q_stream.to(dev), inp.q_pos.to(dev), inp.q.to(dev)
    good = msa.Pages(lay.block_table.to(dev), lay.n_pages)
    g = torch.Generator().manual_seed(cap_blocks)
    from tests.test_gpu_parity import _random_selection
    sel = _random_selection(g, inp.q_pos, w.n_kv_heads).to(dev)
    # unmap a block that query 5 (stream 1) selects, other than its local block
    s_bad = int(inp.q_stream[5])
    b_bad = int([b for b in sel[5, 0].tolist() if 0 <= b < int(inp.q_pos[5]) // 128][0])
    table = lay.block_table.clone()
    table[s_bad, b_bad] = -1
    bad = msa.Pages(table.to(dev), lay.n_pages)
    out = msa.msa_sparse_attn_prefill_paged(shape, bad, q, k_pool, v_pool, sel, qs, qp)
    assert msa.msa_get_device_error() & 0x10
    sel_drop = sel.clone()
    for i in range(sel.shape[0]):
        if int(inp.q_stream[i]) == s_bad:
            row = sel_drop[i]
            row[row == b_bad] = -1
    out_ref = msa.msa_sparse_attn_prefill_paged(shape, good, q, k_pool, v_pool, sel_drop, qs, qp)
    assert msa.msa_get_device_error() == 0
    assert torch.equal(out, out_ref)


def test_paged_append_flags_unmapped_token():
    w = W.Workload("append_unmapped_2x600", 2, 500, 600, "last", n_q_heads=16, n_kv_heads=1)
    inp = W.make_inputs(w, seed=48)
    shape = PT.shape_of(w)
    lay = W.page_layout(inp, seed=6, spare_pages=1, unmapped_from=4)   # blocks 4.. (slots 512..) unmapped
    dev = "cuda"
    pool = lay.idx_pool.to(dev)
    pages = msa.Pages(lay.block_table.to(dev), lay.n_pages)
    msa.msa_indexer_append_paged(shape, pages, pool, inp.idx_k_new.to(dev), inp.tok_stream.to(dev),
                                 inp.tok_pos.to(dev))
    assert msa.msa_get_device_error() & 0x10
    keep = inp.tok_pos < 512
    want = oracle.paged_append(lay.idx_pool, inp.idx_k_new[keep], inp.tok_stream[keep], inp.tok_pos[keep],
                               lay.block_table, w.block)
    assert torch.equal(pool.cpu(), want)
