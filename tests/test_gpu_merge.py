"""Pairs cut between CTAs of the decode attention are merged inside the
kernel, with bookkeeping (publication flags and epochs) that lives in the
workspace from call to call and has no initial value.  These tests reuse one
workspace across calls whose unit splits differ, after filling it with random
bytes and after a prefill call wrote its plans there, and check that every
result is bit-identical to the same call on a fresh zeroed workspace, with no
device error; one sequence is also checked against the oracle."""
import math

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
import oracle
import workloads as W
from tests import parity as PT

pytestmark = pytest.mark.gpu

S, NBLK, G = 3, 24, 4
N_QS = (1, 2, 3, 7, 20, 37, 70, 150)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from block_sparse_attention_maxpool_b200 import build as msa_build
    msa_build.build()
    msa.msa_get_device_error()


def _random_selection(g, q_pos, top_k=16):
    n_q = q_pos.numel()
    sel = torch.full((n_q, G, top_k), -1, dtype=torch.int32)
    for i in range(n_q):
        nvis = int(q_pos[i]) // 128 + 1
        for gg in range(G):
            k = int(torch.randint(1, min(top_k, nvis) + 1, (1,), generator=g))
            others = torch.randperm(nvis - 1, generator=g)[:k - 1].tolist() if nvis > 1 else []
            ids = sorted(set(others) | {nvis - 1})
            sel[i, gg, :len(ids)] = torch.tensor(ids, dtype=torch.int32)
    return sel


@pytest.fixture(scope="module")
def case():
    g = torch.Generator().manual_seed(77)
    cap = NBLK * 128
    lengths = [cap, 2000, 700]
    n_max = max(N_QS)
    qpos = [(i % S, int(torch.randint(0, lengths[i % S], (1,), generator=g))) for i in range(n_max)]
    qpos[0] = (0, cap - 1)
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=77)
    sel = _random_selection(g, qp)
    sh = msa.Shape(n_streams=S, capacity=cap)
    d = {"q": q.cuda(), "k": k.cuda(), "v": v.cuda(), "qs": qs.cuda(), "qp": qp.cuda(), "sel": sel.cuda()}
    return sh, d, (k, v, q, qs, qp, sel)


def _call(sh, d, n, ws):
    return msa.msa_sparse_attn_decode(sh, d["q"][:n], d["k"], d["v"], d["sel"][:n], d["qs"][:n], d["qp"][:n],
                                      workspace=ws)


def _reference(sh, d):
    ref = {}
    for n in N_QS:
        ws = torch.zeros((msa.msa_workspace_bytes(sh, n, msa.MODE_DECODE),), dtype=torch.uint8, device="cuda")
        ref[n] = _call(sh, d, n, ws)
        assert msa.msa_get_device_error() == 0
    return ref


def test_reused_workspace_with_changing_splits_is_bit_identical(case):
    sh, d, _ = case
    ref = _reference(sh, d)
    size = max(msa.msa_workspace_bytes(sh, n, msa.MODE_DECODE) for n in N_QS)
    g = torch.Generator(device="cuda").manual_seed(5)
    ws = torch.randint(0, 256, (size,), dtype=torch.uint8, device="cuda", generator=g)   # arbitrary contents
    order = list(N_QS) + list(reversed(N_QS)) + [7, 150, 1, 70, 70, 2, 37, 20, 150, 3]
    for n in order:
        out = _call(sh, d, n, ws)
        assert msa.msa_get_device_error() == 0, n
        assert torch.equal(out, ref[n]), n


def test_workspace_left_by_a_prefill_call(case):
    sh, d, _ = case
    ref = _reference(sh, d)
    n_pf = 150
    size = max(max(msa.msa_workspace_bytes(sh, n, msa.MODE_DECODE) for n in N_QS),
               msa.msa_workspace_bytes(sh, n_pf, msa.MODE_PREFILL))
    ws = torch.zeros((size,), dtype=torch.uint8, device="cuda")
    for n in (70, 20, 150):
        msa.msa_sparse_attn_prefill(sh, d["q"][:n_pf], d["k"], d["v"], d["sel"][:n_pf], d["qs"][:n_pf],
                                    d["qp"][:n_pf], workspace=ws)      # plans over the bookkeeping
        out = _call(sh, d, n, ws)
        assert msa.msa_get_device_error() == 0, n
        assert torch.equal(out, ref[n]), n


def test_in_kernel_merges_against_the_oracle(case):
    """Many pairs cut across several CTAs each (150 queries x 4 groups of 16
    units over the SMs), on a workspace reused from calls with other splits."""
    sh, d, (k, v, q, qs, qp, sel) = case
    size = max(msa.msa_workspace_bytes(sh, n, msa.MODE_DECODE) for n in N_QS)
    ws = torch.full((size,), 0x4d, dtype=torch.uint8, device="cuda")
    for n in (3, 37, 150):
        out = _call(sh, d, n, ws)
        assert msa.msa_get_device_error() == 0
        want = oracle.sparse_attention(q[:n], k, v, sel[:n], qs[:n], qp[:n], 128, 1 / math.sqrt(128))
        PT.check_attention(out.cpu(), want)
