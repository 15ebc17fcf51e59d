"""The token-level (lightning-indexer) variant on the GPU against the oracle:
top-k selection bit-exact from identical scores, token scores within their
float32 bound, attention given a selection, whole steps (ragged, ties, short
contexts, paged caches) and the 32-stream x 32K decode workload."""
import math

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
import oracle
import workloads as W
from tests import parity as PT
from tests import parity_dsa as PD

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_attention_maxpool_b200 import build as msa_build
    msa_build.build()
    msa.msa_get_device_error()


def _scores_with_ties(n_q, cap, seed):
    g = torch.Generator().manual_seed(seed)
    sc = torch.randn((n_q, cap), generator=g)
    sc[:, ::7] = torch.round(sc[:, ::7] * 4) / 4          # many exact ties
    sc[:, 3::11] = 0.0
    sc[:, 5::13] = -0.0                                    # -0 equals +0
    sc[0, 10] = float("nan")                               # ranks as -inf
    sc[:, 17::19] = float("-inf")
    return sc


@pytest.mark.parametrize("cap,top_k", [(4096, 2048), (4096, 7), (4096, 1), (9984, 100), (32768, 2048),
                                       (32768, 100), (65536, 2048), (131072, 2048)])
def test_select_bitexact_from_identical_scores(cap, top_k):
    n_q = 12
    sc = _scores_with_ties(n_q, cap, seed=cap + top_k)
    g = torch.Generator().manual_seed(top_k)
    q_pos = torch.randint(0, cap, (n_q,), generator=g, dtype=torch.int32)
    q_pos[0] = cap - 1
    q_pos[1] = min(top_k - 1, cap - 1)        # exactly top_k visible: all kept
    q_pos[2] = 0
    ds = msa.DsaShape(n_streams=1, capacity=cap, top_k=top_k)
    sel, n_sel = msa.msa_dsa_select_topk(ds, sc.cuda(), q_pos.cuda())
    assert msa.msa_get_device_error() == 0
    sel_o, nsel_o = oracle.dsa_select_tokens(sc.double(), q_pos, top_k, msa.DSA_SEL_WIDTH)
    assert torch.equal(n_sel.cpu(), nsel_o)
    assert torch.equal(sel.cpu(), sel_o)


def test_select_constant_and_two_valued_rows():
    """Rows where the sample bracket keeps too many keys (all equal) or where
    the k-th key sits in a huge tie run: the exact fallback must agree."""
    cap = 32768
    sc = torch.zeros((3, cap))
    sc[1, ::2] = 1.0
    sc[2] = torch.randn(cap, generator=torch.Generator().manual_seed(3))
    sc[2, 5000:30000] = 0.25
    q_pos = torch.full((3,), cap - 1, dtype=torch.int32)
    ds = msa.DsaShape(n_streams=1, capacity=cap, top_k=2048)
    sel, n_sel = msa.msa_dsa_select_topk(ds, sc.cuda(), q_pos.cuda())
    assert msa.msa_get_device_error() == 0
    sel_o, nsel_o = oracle.dsa_select_tokens(sc.double(), q_pos, 2048, msa.DSA_SEL_WIDTH)
    assert torch.equal(sel.cpu(), sel_o) and torch.equal(n_sel.cpu(), nsel_o)


def test_select_invalid_query_flags():
    ds = msa.DsaShape(n_streams=1, capacity=1024, top_k=16)
    sc = torch.randn((2, 1024)).cuda()
    sel, n_sel = msa.msa_dsa_select_topk(ds, sc, torch.tensor([5, 1024], dtype=torch.int32).cuda())
    assert msa.msa_get_device_error() & 0x1
    assert n_sel.tolist() == [6, 0] and bool((sel[1] == -1).all())


@pytest.mark.parametrize("relu", [True, False])
def test_token_scores_within_bound(relu):
    w = W.Workload("dsa_scores_3x3000", 3, 3000, 3000, "last")
    dinp = W.make_dsa_inputs(w, seed=61)
    inp = dinp.base
    # ragged positions: one query per stream plus extra ones
    qs = torch.tensor([0, 1, 2, 2, 0], dtype=torch.int32)
    qp = torch.tensor([2999, 1500, 127, 128, 0], dtype=torch.int32)
    g = torch.Generator().manual_seed(5)
    q_idx = (torch.randn((5, 64, 128), generator=g) / math.sqrt(128)).half()
    wts = torch.randn((5, 64), generator=g) / 8
    ds = PD.dsa_shape_of(w, relu=relu)
    keys = dinp.k_idx_cache.half()
    sc = msa.msa_dsa_token_scores(ds, q_idx.cuda(), wts.cuda(), keys.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() == 0
    sc_o = oracle.dsa_token_scores(q_idx, wts, keys, qs, qp, relu)
    err = PD.check_scores(sc.cpu(), sc_o, PD.score_bounds(q_idx, wts, keys, qs, qp))
    print(f"\n[dsa] token scores relu={relu}: max err {err:.3e}")
    del inp


def test_attention_given_selection():
    w = W.Workload("dsa_attn_5x4000", 5, 4000, 4000, "last")
    inp = W.make_inputs(w, seed=62)
    shape = PT.shape_of(w)
    g = torch.Generator().manual_seed(62)
    n_q = 7
    qs = torch.tensor([0, 1, 2, 3, 4, 0, 1], dtype=torch.int32)
    qp = torch.tensor([3999, 2047, 100, 3000, 129, 2048, 0], dtype=torch.int32)
    q = torch.randn((n_q, 64, 128), generator=g).to(torch.bfloat16)
    sel = torch.full((n_q, msa.DSA_SEL_WIDTH), -1, dtype=torch.int32)
    for t in range(n_q):
        p = int(qp[t])
        k = min(p + 1, [2048, 2048, 60, 1000, 130, 2048, 1][t])
        ids = torch.randperm(p + 1, generator=g)[:k].sort().values
        sel[t, :k] = ids.to(torch.int32)
    d = PT.to_dev(inp)
    out = msa.msa_dsa_sparse_attn_decode(shape, q.cuda(), d["k_cache"], d["v_cache"], sel.cuda(), qs.cuda(),
                                         qp.cuda())
    assert msa.msa_get_device_error() == 0
    want = oracle.dsa_sparse_attention(q, inp.k_cache, inp.v_cache, sel, qs, qp)
    mx, mean, _ = PT.check_attention(out.cpu(), want)
    print(f"\n[dsa] attention given selection: max {mx:.3e} mean {mean:.3e}")


def test_attention_flags_token_past_query():
    w = W.Workload("dsa_attn_bad_1x600", 1, 600, 600, "last", n_q_heads=16, n_kv_heads=1)
    inp = W.make_inputs(w, seed=63)
    shape = PT.shape_of(w)
    q = torch.randn((1, 16, 128)).to(torch.bfloat16)
    sel = torch.full((1, msa.DSA_SEL_WIDTH), -1, dtype=torch.int32)
    sel[0, :300] = torch.arange(0, 600, 2, dtype=torch.int32)[:300]     # 0, 2, .., 598: 201 visible
    qp = torch.tensor([400], dtype=torch.int32)
    d = PT.to_dev(inp)
    out = msa.msa_dsa_sparse_attn_decode(shape, q.cuda(), d["k_cache"], d["v_cache"], sel.cuda(),
                                         torch.zeros(1, dtype=torch.int32).cuda(), qp.cuda())
    assert msa.msa_get_device_error() & 0x4
    ok = sel.clone()
    ok[ok > 400] = -1
    want = oracle.dsa_sparse_attention(q, inp.k_cache, inp.v_cache, ok, torch.zeros(1, dtype=torch.int32), qp)
    PT.check_attention(out.cpu(), want)


def test_step_decode_ragged():
    w = W.Workload("dsa_decode_6x5000", 6, 4999, 5000, "last")
    rep = PD.full_parity(W.make_dsa_inputs(w, seed=64))
    print("\n[dsa] decode 6x5000:", rep)


def test_step_small_top_k_no_relu():
    w = W.Workload("dsa_decode_3x3000_k300", 3, 2999, 3000, "last")
    rep = PD.full_parity(W.make_dsa_inputs(w, seed=65), top_k=300, relu=False)
    print("\n[dsa] decode k=300 no relu:", rep)


def test_step_ties_exact():
    w = W.Workload("dsa_ties_4x4000", 4, 3999, 4000, "last")
    rep = PD.full_parity(W.make_dsa_inputs(w, seed=66, quantize=True), top_k=512)
    print("\n[dsa] ties:", rep)
    assert rep["max_score_err"] == 0.0 and rep["boundary_swaps"] == 0


def test_step_short_context_keeps_everything():
    w = W.Workload("dsa_short_3x1500", 3, 1499, 1500, "last")
    rep = PD.full_parity(W.make_dsa_inputs(w, seed=67))
    print("\n[dsa] short context:", rep)
    assert rep["boundary_swaps"] == 0


def test_step_paged_bitwise_equal_to_contiguous():
    w = W.Workload("dsa_paged_5x3500", 5, 3499, 3500, "last")
    dinp = W.make_dsa_inputs(w, seed=68)
    inp = dinp.base
    shape, ds = PT.shape_of(w), PD.dsa_shape_of(w)
    d = PD.to_dev(dinp)
    caches = {k: d[k] for k in ("k_idx_cache", "k_cache", "v_cache")}
    out_c, sel_c, n_c, sc_c = msa.dsa_decode_step(shape, ds, caches, d)
    # the same caches as shuffled pools: K/V pages (4 groups) and key pages (one group)
    lay = W.page_layout(inp, seed=3, spare_pages=3)
    nb = w.capacity // 128
    perm = torch.randperm(5 * nb + 2, generator=torch.Generator().manual_seed(9))
    ktab = perm[:5 * nb].view(5, nb).to(torch.int32)
    kpool = torch.full((5 * nb + 2, 128, 128), 64.0, dtype=torch.float16)
    keys16 = dinp.k_idx_cache.half()
    for s in range(5):
        for b in range(nb):
            kpool[int(ktab[s, b])] = keys16[s, b * 128:(b + 1) * 128]
    dp = PD.to_dev(dinp)
    caches_p = {"k_idx_cache": kpool.cuda(), "k_cache": lay.k_pool.cuda(), "v_cache": lay.v_pool.cuda()}
    out_p, sel_p, n_p, sc_p = msa.dsa_decode_step(shape, ds, caches_p, dp,
                                                  pages=msa.Pages(lay.block_table.cuda(), lay.n_pages),
                                                  idx_pages=msa.Pages(ktab.cuda(), 5 * nb + 2))
    assert msa.msa_get_device_error() == 0
    assert torch.equal(sc_c, sc_p) and torch.equal(sel_c, sel_p) and torch.equal(n_c, n_p)
    assert torch.equal(out_c, out_p)


def test_step_full_size_decode_32x32k():
    """The 32-stream x 32K decode workload with 2048 kept tokens; the oracle
    checks 3 of the 32 streams."""
    dinp = W.make_dsa_inputs(W.DECODE_32K_X32, seed=0)
    rep = PD.full_parity(dinp, queries=[0, 17, 31])
    print("\n[dsa] decode_32x32k:", rep)
