"""msa_select_attn_decode (the top-16 taken inside the decode attention
kernel) against msa_select_topk followed by msa_sparse_attn_decode on the
same inputs: selection, counts, output and device error word must be
bit-identical.  Both separate calls are themselves checked against the
oracle in the other GPU tests; one case here is also checked against the
oracle directly.  Batches of up to about 900 (query, group) pairs take the
in-kernel selection on a 148-SM B200, larger ones the selection kernel
first; both are covered."""
import math
import types

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


def _scores(g, n_q, G, nblk, q_pos, ties):
    bs = torch.randn((n_q, G, nblk), generator=g)
    if ties:
        bs = (bs * 2).round() / 2                      # many equal scores
    bs[torch.rand((n_q, G, nblk), generator=g) < 0.05] = float("nan")
    bs[torch.rand((n_q, G, nblk), generator=g) < 0.05] = float("-inf")
    for i in range(n_q):
        p = int(q_pos[i])
        if 0 <= p < nblk * 128:
            bs[i, :, p // 128] += 2.0 ** 100           # the local block's bias
    return bs


def _case(S, nblk, n_q, seed, ties=False, bad=(), pages=False):
    g = torch.Generator().manual_seed(seed)
    cap = nblk * 128
    G = 4
    lengths = [cap] + [int(x) for x in torch.randint(1, cap + 1, (S - 1,), generator=g)]
    qpos = []
    for i in range(n_q):
        s = i % S
        qpos.append((s, int(torch.randint(0, lengths[s], (1,), generator=g))))
    qpos[0] = (0, cap - 1)
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=seed)
    for i in bad:                                      # queries outside the cache
        qp[i] = cap + 5 if i % 2 else -1
    bs = _scores(g, n_q, G, nblk, qp, ties)
    sh = msa.Shape(n_streams=S, capacity=cap)
    dev = {"bs": bs.cuda(), "q": q.cuda(), "k": k.cuda(), "v": v.cuda(), "qs": qs.cuda(), "qp": qp.cuda()}
    pg = None
    if pages:
        caches = types.SimpleNamespace(idx_k_cache=idx, k_cache=k, v_cache=v, w=types.SimpleNamespace(block=128))
        lay = W.page_layout(caches, seed=seed)
        dev["k"], dev["v"] = lay.k_pool.cuda(), lay.v_pool.cuda()
        pg = msa.Pages(lay.block_table.cuda(), lay.n_pages)
    return sh, dev, pg, (k, v, q, qs, qp, bs)


def _compare(sh, d, pg):
    sel1, n1 = msa.msa_select_topk(sh, d["bs"], d["qp"])
    fn = msa.msa_sparse_attn_decode if pg is None else \
        (lambda *a, **kw: msa.msa_sparse_attn_decode_paged(sh, pg, *a[1:], **kw))
    out1 = fn(sh, d["q"], d["k"], d["v"], sel1, d["qs"], d["qp"])
    e1 = msa.msa_get_device_error()
    if pg is None:
        out2, sel2, n2 = msa.msa_select_attn_decode(sh, d["bs"], d["q"], d["k"], d["v"], d["qs"], d["qp"])
    else:
        out2, sel2, n2 = msa.msa_select_attn_decode_paged(sh, pg, d["bs"], d["q"], d["k"], d["v"], d["qs"], d["qp"])
    e2 = msa.msa_get_device_error()
    assert e1 == e2, (hex(e1), hex(e2))
    assert torch.equal(sel1, sel2), "selection"
    assert torch.equal(n1, n2), "counts"
    assert torch.equal(out1, out2), "attention output"
    return out2, sel2, n2, e2


@pytest.mark.parametrize("n_q", [1, 2, 3, 37, 128, 225, 300, 400])
@pytest.mark.parametrize("nblk", [1, 9, 20, 200])
def test_select_attn_equals_the_two_calls(n_q, nblk):
    S = min(n_q, 3)
    sh, d, pg, _ = _case(S, nblk, n_q, seed=n_q * 31 + nblk, ties=(n_q % 2 == 0))
    _compare(sh, d, pg)


@pytest.mark.parametrize("n_q", [1, 37])
def test_select_attn_more_blocks_than_the_shared_memory_keys(n_q):
    """1100 blocks: the top-16 re-reads the scores from global memory."""
    sh, d, pg, _ = _case(1, 1100, n_q, seed=n_q + 1100, ties=True)
    _compare(sh, d, pg)


def test_select_attn_invalid_queries_flag_and_write_empty_selections():
    sh, d, pg, _ = _case(3, 24, 20, seed=5, bad=(3, 4, 11))
    out, sel, n_sel, err = _compare(sh, d, pg)
    assert err & 0x1
    for i in (3, 4, 11):
        assert sel[i].eq(-1).all() and n_sel[i].eq(0).all()
        assert out[i].eq(0).all()


def test_select_attn_paged_caches():
    sh, d, pg, _ = _case(3, 30, 24, seed=9, ties=True, pages=True)
    _compare(sh, d, pg)


def test_select_attn_against_the_oracle():
    sh, d, pg, (k, v, q, qs, qp, bs) = _case(3, 40, 12, seed=17, ties=True)
    out, sel, n_sel, err = _compare(sh, d, pg)
    assert err == 0
    sel_o, nsel_o = oracle.select_blocks(bs.double(), qp, 128, 16)
    assert torch.equal(sel.cpu(), sel_o) and torch.equal(n_sel.cpu(), nsel_o)
    want = oracle.sparse_attention(q, k, v, sel_o, qs, qp, 128, 1 / math.sqrt(128))
    PT.check_attention(out.cpu(), want)


def test_select_attn_workspace_and_argument_errors():
    sh, d, pg, _ = _case(2, 10, 4, seed=3)
    with pytest.raises(msa.MsaError):
        msa.msa_select_attn_decode(sh, d["bs"], d["q"], d["k"], d["v"], d["qs"], d["qp"],
                                   workspace=torch.empty((16,), dtype=torch.uint8, device="cuda"))
