"""A layer that reuses another layer's selection (the GLM-DSA pull request's
IndexShare review comment: shared layers take the top-k of the previous full
layer instead of running their own indexer).  Layer A runs the whole MSA
step; layer B, with its own K/V caches and queries at the same positions,
only appends its K/V rows and attends over layer A's selection: no block
scores, no top-k.  Checked against the oracle: layer A's selection, and
layer B's attention over that selection on layer B's caches."""
import dataclasses
import math

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
import oracle
import workloads as W
from block_sparse_attention_maxpool_b200 import build as msa_build
from tests import parity as PT

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    msa_build.build()
    msa.msa_get_device_error()


@pytest.mark.parametrize("w", [
    W.Workload("shared_decode_9x5000", 9, 4999, 5000, "last"),
    W.Workload("shared_prefill_1x1800", 1, 0, 1800, "new"),
    W.Workload("shared_chunk_2x300_on_2500", 2, 2500, 2800, "new"),
], ids=lambda w: w.name)
def test_shared_layer_attends_over_the_previous_layers_selection(w):
    prefill = w.queries == "new"
    a = W.make_inputs(w, seed=50)                    # layer A: runs the indexer
    b = W.make_inputs(w, seed=51)                    # layer B: own K/V and queries, same positions
    shape = PT.shape_of(w)
    da = PT.to_dev(a)
    ca = {k: da[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    _, sel_a, n_sel_a, bs_a = msa.decode_step(shape, ca, da, prefill=prefill)
    db = PT.to_dev(b)
    msa.msa_kv_append(shape, db["k_cache"], db["v_cache"], db["k_new"], db["v_new"], db["tok_stream"], db["tok_pos"])
    attn = msa.msa_sparse_attn_prefill if prefill else msa.msa_sparse_attn_decode
    out_b = attn(shape, db["q"], db["k_cache"], db["v_cache"], sel_a, db["q_stream"], db["q_pos"])
    assert msa.msa_get_device_error() == 0
    # layer A's selection against the oracle (no near-tie met on these seeds)
    idx_a, _, _ = PT.oracle_caches(a)
    bs_o = oracle.block_scores(a.idx_q, idx_a, a.q_stream, a.q_pos, w.block)
    sel_o, nsel_o = oracle.select_blocks(bs_o, a.q_pos, w.block, w.top_k)
    assert torch.equal(sel_a.cpu(), sel_o) and torch.equal(n_sel_a.cpu(), nsel_o)
    # layer B: its caches after its own append, layer A's selection
    _, k_b, v_b = PT.oracle_caches(b)
    assert torch.equal(db["k_cache"].cpu(), k_b) and torch.equal(db["v_cache"].cpu(), v_b)
    n_q = b.q_pos.numel()
    rows = list(range(n_q)) if n_q <= 64 else sorted(set(range(0, n_q, 13)) | {n_q - 1})
    r = torch.tensor(rows, dtype=torch.long)
    want = oracle.sparse_attention(b.q[r], k_b, v_b, sel_o[r], b.q_stream[r], b.q_pos[r], w.block,
                                   1.0 / math.sqrt(w.head_dim))
    print(f"\n[parity] {w.name} shared layer:", PT.check_attention(out_b.cpu()[r], want))
