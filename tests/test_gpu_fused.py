"""The whole decode step as one persistent kernel (msa_decode_step_fused)
against the separate calls (themselves checked against the oracle in the
other GPU tests): caches after the appends, block scores, selection and
output must be bit-identical, since every phase does the same arithmetic.
One case is also checked against the oracle directly."""
import math

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
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


def _both(w, seed, mutate=None):
    inp = W.make_inputs(w, seed=seed)
    if mutate is not None:
        mutate(inp)
    shape = PT.shape_of(w)
    d1 = PT.to_dev(inp)
    d2 = PT.to_dev(inp)
    c1 = {k: d1[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    c2 = {k: d2[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    r1 = msa.decode_step(shape, c1, d1)
    e1 = msa.msa_get_device_error()
    r2 = msa.decode_step_fused(shape, c2, d2)
    e2 = msa.msa_get_device_error()
    assert e1 == e2
    for k in ("idx_k_cache", "k_cache", "v_cache"):
        assert torch.equal(c1[k], c2[k]), k
    for a, b, name in zip(r1, r2, ("out", "sel", "n_sel", "block_scores")):
        assert torch.equal(a, b), name
    return inp, r2, e2


@pytest.mark.parametrize("w", [
    W.DECODE_4K,
    W.Workload("fused_32x3000", 32, 2999, 3000, "last"),
    W.Workload("fused_5x20000", 5, 19999, 20000, "last"),
    W.Workload("fused_g1_7x2500", 7, 2499, 2500, "last", n_q_heads=16, n_kv_heads=1),
    W.Workload("fused_g8_3x2000", 3, 1999, 2000, "last", n_q_heads=128, n_kv_heads=8),
    W.Workload("fused_short_6x300", 6, 299, 300, "last"),
], ids=lambda w: w.name)
def test_fused_equals_separate_calls(w):
    _both(w, seed=71)


def test_fused_with_invalid_query_and_ragged_positions():
    w = W.Workload("fused_ragged_4x5000", 4, 4999, 5000, "last")

    def mutate(inp):
        inp.q_pos[1] = 2047          # an earlier position of its stream
        inp.q_pos[2] = 1 << 20       # past the cache: flagged, -inf scores, zero output
    _, r, err = _both(w, seed=72, mutate=mutate)
    assert err & 0x1


def test_fused_matches_oracle():
    w = W.Workload("fused_oracle_3x2600", 3, 2599, 2600, "last")
    inp = W.make_inputs(w, seed=73)
    shape = PT.shape_of(w)
    d = PT.to_dev(inp)
    caches = {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    out, sel, n_sel, bs = msa.decode_step_fused(shape, caches, d)
    assert msa.msa_get_device_error() == 0
    import oracle
    idx_o, k_o, v_o = PT.oracle_caches(inp)
    assert torch.equal(caches["idx_k_cache"].cpu(), idx_o)
    bs_o = oracle.block_scores(inp.idx_q, idx_o, inp.q_stream, inp.q_pos, w.block)
    PT.check_scores(bs.cpu(), bs_o, PT.score_bounds(inp.idx_q, idx_o, inp.q_stream, inp.q_pos, w.block))
    merged, _ = PT.check_selection(sel.cpu(), n_sel.cpu(), bs_o, inp.q_pos, w.block, w.top_k)
    out_o = oracle.sparse_attention(inp.q, k_o, v_o, merged, inp.q_stream, inp.q_pos, w.block,
                                    1.0 / math.sqrt(w.head_dim))
    PT.check_attention(out.cpu(), out_o)


def test_fused_full_size_decode_32x32k():
    _both(W.DECODE_32K_X32, seed=0)


def test_fused_rejects_prefill_shaped_batches():
    w = W.Workload("fused_prefill_1x600", 1, 0, 600, "new")
    inp = W.make_inputs(w, seed=74)
    shape = PT.shape_of(w)
    d = PT.to_dev(inp)
    caches = {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    with pytest.raises(msa.MsaError):
        msa.decode_step_fused(shape, caches, d)
