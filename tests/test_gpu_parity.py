"""GPU parity of every step of the MSA hot path against the CPU oracle, through
the C ABI: cache append, block scores, top-k selection, block-sparse
attention, and the whole step on small ragged cases and on the five
benchmark workloads (full size, sampled where the oracle would be slow)."""
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
def gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    msa_build.build()
    msa.msa_get_device_error()          # clear leftovers
    yield
    torch.cuda.synchronize()


def report(name, rep):
    print(f"\n[parity] {name}: {rep}")


# ---------------------------------------------------------------------------
# step by step
# ---------------------------------------------------------------------------
def test_append_bit_exact_and_range_errors():
    g = torch.Generator().manual_seed(11)
    sh = msa.Shape(n_streams=3, capacity=384, n_kv_heads=2, n_q_heads=32)
    idx = torch.randn((3, 2, 384, 128), generator=g)
    k = torch.randn((3, 2, 384, 128), generator=g).to(torch.bfloat16)
    v = torch.randn((3, 2, 384, 128), generator=g).to(torch.bfloat16)
    n = 50
    ts = torch.randint(0, 3, (n,), generator=g, dtype=torch.int32)
    tp = torch.randperm(384, generator=g)[:n].to(torch.int32)
    new_i = torch.randn((n, 2, 128), generator=g)
    new_k = torch.randn((n, 2, 128), generator=g).to(torch.bfloat16)
    new_v = torch.randn((n, 2, 128), generator=g).to(torch.bfloat16)
    di, dk, dv = idx.cuda(), k.cuda(), v.cuda()
    msa.msa_indexer_append(sh, di, new_i.cuda(), ts.cuda(), tp.cuda())
    msa.msa_kv_append(sh, dk, dv, new_k.cuda(), new_v.cuda(), ts.cuda(), tp.cuda())
    assert msa.msa_get_device_error() == 0
    assert torch.equal(di.cpu(), oracle.indexer_append(idx, new_i, ts, tp))
    assert torch.equal(dk.cpu(), oracle.indexer_append(k, new_k, ts, tp))
    assert torch.equal(dv.cpu(), oracle.indexer_append(v, new_v, ts, tp))
    # out-of-range tokens are skipped and reported
    bad_s = torch.tensor([3, 0], dtype=torch.int32).cuda()
    bad_p = torch.tensor([0, 384], dtype=torch.int32).cuda()
    before = di.clone()
    msa.msa_indexer_append(sh, di, new_i[:2].cuda(), bad_s, bad_p)
    assert msa.msa_get_device_error() & 0x2
    assert torch.equal(di, before)


def test_step_append_matches_the_separate_appends_and_flags_bad_tokens():
    """msa_step_append (indexer keys + K/V in one launch) writes what
    msa_indexer_append and msa_kv_append write, bit for bit, skips a token
    outside the cache and sets the same error bit."""
    g = torch.Generator().manual_seed(12)
    sh = msa.Shape(n_streams=3, capacity=384, n_kv_heads=2, n_q_heads=32)
    idx = torch.randn((3, 2, 384, 128), generator=g)
    k = torch.randn((3, 2, 384, 128), generator=g).to(torch.bfloat16)
    v = torch.randn((3, 2, 384, 128), generator=g).to(torch.bfloat16)
    n = 60
    ts = torch.randint(0, 3, (n,), generator=g, dtype=torch.int32)
    tp = torch.randperm(384, generator=g)[:n].to(torch.int32)
    ts[7], tp[9] = 3, 384                       # no such stream; past the capacity
    new_i = torch.randn((n, 2, 128), generator=g)
    new_k = torch.randn((n, 2, 128), generator=g).to(torch.bfloat16)
    new_v = torch.randn((n, 2, 128), generator=g).to(torch.bfloat16)
    di, dk, dv = idx.cuda(), k.cuda(), v.cuda()
    msa.msa_step_append(sh, di, dk, dv, new_i.cuda(), new_k.cuda(), new_v.cuda(), ts.cuda(), tp.cuda())
    assert msa.msa_get_device_error() == 0x2
    ok = torch.ones(n, dtype=torch.bool)
    ok[7] = ok[9] = False
    assert torch.equal(di.cpu(), oracle.indexer_append(idx, new_i[ok], ts[ok], tp[ok]))
    assert torch.equal(dk.cpu(), oracle.indexer_append(k, new_k[ok], ts[ok], tp[ok]))
    assert torch.equal(dv.cpu(), oracle.indexer_append(v, new_v[ok], ts[ok], tp[ok]))


def _rand_scores(g, n_q, G, nblk, q_pos, ties):
    bs = torch.randn((n_q, G, nblk), generator=g)
    if ties:
        bs = torch.round(bs * 2) / 2          # many exact ties, both signs of zero
    for i in range(n_q):
        p = int(q_pos[i])
        bs[i, :, p // 128 + 1:] = float("-inf")
        bs[i, :, p // 128] += 2.0 ** 100
    return bs


@pytest.mark.parametrize("nblk", [1, 9, 200, 256, 600, 1024, 1500])
@pytest.mark.parametrize("ties", [False, True])
def test_select_bit_exact_from_identical_scores(nblk, ties):
    g = torch.Generator().manual_seed(nblk * 2 + ties)
    cap = nblk * 128
    G, n_q = 4, 40
    q_pos = torch.randint(0, cap, (n_q,), generator=g, dtype=torch.int32)
    q_pos[0], q_pos[1] = cap - 1, 0
    q_pos[2] = min(cap - 1, 15 * 128 + 5)     # exactly 16 visible blocks
    q_pos[3] = min(cap - 1, 16 * 128)         # 17 visible blocks
    bs = _rand_scores(g, n_q, G, nblk, q_pos, ties)
    sh = msa.Shape(n_streams=1, capacity=cap)
    sel, n_sel = msa.msa_select_topk(sh, bs.cuda(), q_pos.cuda())
    assert msa.msa_get_device_error() == 0
    sel_o, nsel_o = oracle.select_blocks(bs.double(), q_pos, 128, 16)
    assert torch.equal(sel.cpu(), sel_o)
    assert torch.equal(n_sel.cpu(), nsel_o)


def test_select_nan_ranks_last_and_bad_positions():
    """NaN scores rank as -inf (tied with -inf, lower index first), as the
    oracle ranks them; a query past the capacity selects nothing."""
    sh = msa.Shape(n_streams=1, capacity=128 * 40)
    g = torch.Generator().manual_seed(40)
    bs = torch.zeros((3, 4, 40))
    bs[:, :, 0] = float("nan")
    bs[:, :, 39] += 2.0 ** 100
    bs[2] = torch.randn((4, 40), generator=g)
    bs[2, :, 5:30:3] = float("nan")                # many NaN blocks ...
    bs[2, :, 7:33:4] = float("-inf")               # ... mixed with -inf ones
    bs[2, 1, :] = float("nan")                     # a group with nothing but NaN and the local block
    bs[2, :, 20] = 2.0 ** 100
    q_pos = torch.tensor([128 * 40 - 1, 128 * 40, 128 * 20 + 3], dtype=torch.int32)   # second is out of range
    sel, n_sel = msa.msa_select_topk(sh, bs.cuda(), q_pos.cuda())
    assert msa.msa_get_device_error() & 0x1
    sel, n_sel = sel.cpu(), n_sel.cpu()
    assert 0 not in sel[0, 0].tolist()             # the NaN block loses to every finite one
    assert sel[0, 0].tolist() == list(range(1, 16)) + [39]
    assert sel[1].eq(-1).all() and n_sel[1].eq(0).all()
    good = torch.tensor([0, 2])
    sel_o, nsel_o = oracle.select_blocks(bs[good].double(), q_pos[good], 128, 16)
    assert torch.equal(sel[good], sel_o) and torch.equal(n_sel[good], nsel_o)


def _random_selection(g, q_pos, G, top_k=16):
    n_q = q_pos.numel()
    sel = torch.full((n_q, G, top_k), -1, dtype=torch.int32)
    for i in range(n_q):
        p = int(q_pos[i])
        nvis = p // 128 + 1
        for gg in range(G):
            k = int(torch.randint(1, min(top_k, nvis) + 1, (1,), generator=g))
            others = torch.randperm(nvis - 1, generator=g)[:k - 1].tolist() if nvis > 1 else []
            ids = sorted(set(others) | {nvis - 1})
            sel[i, gg, :len(ids)] = torch.tensor(ids, dtype=torch.int32)
    return sel


@pytest.mark.parametrize("n_q,mode", [(1, "decode"), (3, "decode"), (20, "decode"), (40, "decode"),
                                      (70, "decode"), (150, "decode"), (300, "decode"), (37, "prefill")])
def test_attention_given_selection(n_q, mode):
    g = torch.Generator().manual_seed(n_q)
    S, cap, G = 3, 128 * 24, 4
    lengths = [cap, 1000, 129]
    qpos = []
    for i in range(n_q):
        s = i % S
        qpos.append((s, int(torch.randint(0, lengths[s], (1,), generator=g))))
    qpos[0] = (0, cap - 1)
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=n_q)
    sel = _random_selection(g, qp, G)
    sh = msa.Shape(n_streams=S, capacity=cap)
    fn = msa.msa_sparse_attn_decode if mode == "decode" else msa.msa_sparse_attn_prefill
    out = fn(sh, q.cuda(), k.cuda(), v.cuda(), sel.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() == 0
    want = oracle.sparse_attention(q, k, v, sel, qs, qp, 128, 1 / math.sqrt(128))
    report(f"attention n_q={n_q} {mode}", PT.check_attention(out.cpu(), want))


def test_prefill_attention_long_context():
    """Caches of 38400 tokens per stream (300 blocks): few blocks shared
    between the queries of a tile, the same oracle check."""
    g = torch.Generator().manual_seed(91)
    S, cap, G = 2, 128 * 300, 4
    lengths = [cap, 20000]
    qpos = [(i % S, int(torch.randint(0, lengths[i % S], (1,), generator=g))) for i in range(37)]
    qpos[0] = (0, cap - 1)
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=91)
    sel = _random_selection(g, qp, G)
    sh = msa.Shape(n_streams=S, capacity=cap)
    out = msa.msa_sparse_attn_prefill(sh, q.cuda(), k.cuda(), v.cuda(), sel.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() == 0
    want = oracle.sparse_attention(q, k, v, sel, qs, qp, 128, 1 / math.sqrt(128))
    report("prefill attention, 38400-token caches", PT.check_attention(out.cpu(), want))


@pytest.mark.parametrize("cap", [1024, 128 * 260], ids=["short_cache", "long_cache"])
def test_prefill_attention_edge_queries(cap):
    """Prefill attention on a ragged batch (21 queries: two 8-query tiles and
    a tail of 5) whose tiles mix streams, with shuffled selection lists (-1
    in the middle), an invalid selected block, an empty selection, a
    position past the cache and a bad stream id: the invalid block is skipped
    (SEL_RANGE), the bad queries give zeros (QUERY_RANGE), everything else
    matches the oracle."""
    g = torch.Generator().manual_seed(cap)
    S, G = 2, 4
    lengths = [cap, cap // 2]
    qpos = [(int(torch.randint(0, S, (1,), generator=g)), 0) for _ in range(21)]
    qpos = [(st, int(torch.randint(0, lengths[st], (1,), generator=g))) for st, _ in qpos]
    qpos[0] = (0, 700)
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=cap)
    sel = _random_selection(g, qp, G)
    # a selection is a set of blocks: lists in any order, -1 anywhere
    for i in range(4, 21, 3):
        for gg in range(G):
            sel[i, gg] = sel[i, gg][torch.randperm(16, generator=g)]
    sel[0, 2, 15] = 6                 # block 6 starts past position 700: invalid, skipped
    sel[1] = -1                       # empty selection: zeros
    qp_dev = qp.clone()
    qs_dev = qs.clone()
    qp_dev[2] = cap                   # past the capacity: zeros, QUERY_RANGE
    qs_dev[3] = -1                    # no such stream: zeros, QUERY_RANGE
    sh = msa.Shape(n_streams=S, capacity=cap)
    out = msa.msa_sparse_attn_prefill(sh, q.cuda(), k.cuda(), v.cuda(), sel.cuda(), qs_dev.cuda(), qp_dev.cuda())
    err = msa.msa_get_device_error()
    assert err & 0x1 and err & 0x4 and not err & ~0x5, err
    sel_clean = sel.clone()
    sel_clean[0, 2, 15] = -1
    want = oracle.sparse_attention(q, k, v, sel_clean, qs, qp, 128, 1 / math.sqrt(128))
    want[1:4] = 0.0
    report(f"prefill attention edge queries, cap {cap}", PT.check_attention(out.cpu(), want))


def test_prefill_attention_every_tile_spans_eight_streams():
    """Prefill queries interleaved over 8 streams, so each 8-query tile of the
    union kernel holds 8 segments (one per stream, each with its own blocks)."""
    g = torch.Generator().manual_seed(77)
    S, cap, G = 8, 128 * 12, 4
    lengths = [cap - 97 * s for s in range(S)]
    qpos = [(i % S, int(torch.randint(0, lengths[i % S], (1,), generator=g))) for i in range(83)]
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=77)
    sel = _random_selection(g, qp, G)
    sh = msa.Shape(n_streams=S, capacity=cap)
    out = msa.msa_sparse_attn_prefill(sh, q.cuda(), k.cuda(), v.cuda(), sel.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() == 0
    want = oracle.sparse_attention(q, k, v, sel, qs, qp, 128, 1 / math.sqrt(128))
    report("prefill attention, 8 streams per tile", PT.check_attention(out.cpu(), want))


def test_attention_empty_and_invalid_selection():
    S, cap = 1, 512
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, [512], [(0, 300), (0, 100)], seed=5)
    sel = torch.full((2, 4, 16), -1, dtype=torch.int32)
    sel[0, :, 0] = 2
    sel[0, 1, 1] = 3                 # block 3 starts past position 300: invalid, skipped
    sh = msa.Shape(n_streams=S, capacity=cap)
    out = msa.msa_sparse_attn_decode(sh, q.cuda(), k.cuda(), v.cuda(), sel.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() & 0x4
    sel_clean = sel.clone()
    sel_clean[0, 1, 1] = -1
    want = oracle.sparse_attention(q, k, v, sel_clean, qs, qp, 128)
    want[1] = 0.0                    # query 1 has an empty selection: zeros
    PT.check_attention(out.cpu(), want)


def test_block_scores_ragged_multi_stream():
    S, cap = 3, 128 * 10
    lengths = [cap, 700, 129]
    qpos = [(0, 0), (0, 127), (0, 128), (0, 129), (0, cap - 1), (1, 699), (1, 383), (2, 128), (2, 5),
            (1, 256), (0, 640), (0, 1000)]
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=3)
    sh = msa.Shape(n_streams=S, capacity=cap)
    bs = msa.msa_block_scores(sh, iq.cuda(), idx.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() == 0
    bs_o = oracle.block_scores(iq, idx, qs, qp, 128)
    PT.check_scores(bs.cpu(), bs_o, PT.score_bounds(iq, idx, qs, qp, 128))


def test_block_scores_tile_path_mixed_streams_and_padding():
    """A prefill-shaped batch (tensor-core tiles): 3 streams, queries in
    stream-contiguous runs that do not align with the 128-query tiles (so
    mixed tiles send some queries to the streaming kernel), unsorted
    positions, a padded last tile, 40 key blocks (two 32-block chunks) and
    two invalid queries."""
    S, cap = 3, 128 * 40
    lengths = [cap, 4000, 3000]
    g = torch.Generator().manual_seed(12)
    qpos = []
    for s, n in ((0, 300), (1, 200), (2, 150)):
        pos = torch.randint(0, lengths[s], (n,), generator=g).tolist()
        qpos += [(s, p) for p in pos]
    qpos[5] = (0, cap - 1)
    qpos[301] = (1, 0)
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, lengths, qpos, seed=12)
    qs_bad, qp_bad = qs.clone(), qp.clone()
    qs_bad[10] = 7                   # no such stream
    qp_bad[400] = cap                # past the capacity
    sh = msa.Shape(n_streams=S, capacity=cap)
    assert msa.msa_workspace_bytes(sh, len(qpos), msa.MODE_PREFILL) > 0     # tile path
    bs = msa.msa_block_scores(sh, iq.cuda(), idx.cuda(), qs_bad.cuda(), qp_bad.cuda())
    assert msa.msa_get_device_error() & 0x1
    bs = bs.cpu()
    for bad in (10, 400):
        assert torch.isinf(bs[bad]).all() and (bs[bad] < 0).all()
    good = [i for i in range(len(qpos)) if i not in (10, 400)]
    bs_o = oracle.block_scores(iq[good], idx, qs[good], qp[good], 128)
    err = PT.check_scores(bs[good], bs_o, PT.score_bounds(iq[good], idx, qs[good], qp[good], 128))
    report("tile path scores", {"queries": len(good), "max_err": err})


def test_block_scores_out_of_range_query():
    sh = msa.Shape(n_streams=1, capacity=256)
    idx, k, v, qs, qp, iq, q = W.make_custom(1, 256, [256], [(0, 10), (0, 10)], seed=4)
    qs[1] = 1                        # stream 1 does not exist
    bs = msa.msa_block_scores(sh, iq.cuda(), idx.cuda(), qs.cuda(), qp.cuda())
    assert msa.msa_get_device_error() & 0x1
    bs = bs.cpu()
    assert torch.isinf(bs[1]).all() and (bs[1] < 0).all()
    assert torch.isfinite(bs[0, :, 0]).all()


# ---------------------------------------------------------------------------
# whole step
# ---------------------------------------------------------------------------
def test_step_small_prefill_ragged_tail():
    w = W.Workload("prefill_1x2500", 1, 0, 2500, "new")
    inp = W.make_inputs(w, seed=1)
    q = list(range(0, 2500, 7)) + [2047, 2048, 2049, 2499]
    report(w.name, PT.full_parity(inp, queries=q, prefill=True))


def test_step_small_chunked_prefill_with_ties():
    w = W.Workload("chunk_2x600_on_2000_ties", 2, 2000, 2600, "new", quantize_idx=True)
    inp = W.make_inputs(w, seed=2)
    rep = PT.full_parity(inp, prefill=True)
    report(w.name, rep)
    assert rep["near_ties"] == 0          # quantised scores are exact in float32: no excuses


def test_step_decode_mixed_streams():
    w = W.Workload("decode_6x3000", 6, 2999, 3000, "last")
    report(w.name, PT.full_parity(W.make_inputs(w, seed=3)))


@pytest.mark.parametrize("G", [1, 2, 8])
def test_step_other_group_counts(G):
    """1, 2 or 8 KV/indexer groups (16 query heads each): decode across
    streams, and a prefill batch that takes the tensor-core tile path."""
    dec = W.Workload(f"decode_3x1500_g{G}", 3, 1499, 1500, "last", n_kv_heads=G, n_q_heads=16 * G)
    report(dec.name, PT.full_parity(W.make_inputs(dec, seed=20 + G)))
    pre = W.Workload(f"prefill_1x700_g{G}", 1, 0, 700, "new", n_kv_heads=G, n_q_heads=16 * G)
    report(pre.name, PT.full_parity(W.make_inputs(pre, seed=30 + G), prefill=True))


def test_step_single_block_capacity():
    """Capacity of one 128-slot block: every query sees one (partial) block."""
    w = W.Workload("prefill_2x100_cap128", 2, 0, 100, "new")
    report(w.name, PT.full_parity(W.make_inputs(w, seed=9), prefill=True))
    d = W.Workload("decode_5x128", 5, 127, 128, "last")
    report(d.name, PT.full_parity(W.make_inputs(d, seed=10)))


def test_decode_attention_invalid_query_in_shared_pair():
    """An invalid query among valid ones in the stream-K decode kernel: its
    pairs write zeros and set the error bit, the others stay exact."""
    S, cap = 2, 128 * 20
    qpos = [(0, cap - 1), (1, 1700), (0, 900)]
    idx, k, v, qs, qp, iq, q = W.make_custom(S, cap, [cap, 1800], qpos, seed=14)
    g = torch.Generator().manual_seed(14)
    sel = _random_selection(g, qp, 4)
    qs_bad = qs.clone()
    qs_bad[1] = 5                      # stream 5 does not exist
    sh = msa.Shape(n_streams=S, capacity=cap)
    out = msa.msa_sparse_attn_decode(sh, q.cuda(), k.cuda(), v.cuda(), sel.cuda(), qs_bad.cuda(), qp.cuda())
    assert msa.msa_get_device_error() & 0x1
    out = out.cpu()
    assert out[1].eq(0).all()
    want = oracle.sparse_attention(q, k, v, sel, qs, qp, 128, queries=[0, 2])
    PT.check_attention(out[[0, 2]], want[[0, 2]])


@pytest.mark.parametrize("case", ["decode", "prefill", "ties"])
def test_step_f16_indexer_cache(case):
    """F16 indexer-key cache variant: append rounds keys to fp16 (bit-exact
    with torch's rounding), block scores on fp16 keys within the float32
    bound, selection and attention as for the F32 cache."""
    if case == "decode":
        w, kw = W.Workload("decode_5x2600_f16", 5, 2599, 2600, "last"), {}
    elif case == "prefill":
        w, kw = W.Workload("prefill_1x1500_f16", 1, 0, 1500, "new"), {"prefill": True}
    else:
        w, kw = W.Workload("chunk_2x400_on_1600_ties_f16", 2, 1600, 2000, "new", quantize_idx=True), {"prefill": True}
    rep = PT.full_parity(W.make_inputs(w, seed=41), idx_f16=True, **kw)
    report(w.name, rep)
    if case == "ties":
        assert rep["near_ties"] == 0 and rep["max_score_err"] == 0.0


def test_step_is_deterministic():
    w = W.Workload("decode_4x2200", 4, 2199, 2200, "last")
    inp = W.make_inputs(w, seed=4)
    sh = PT.shape_of(w)
    outs = []
    for _ in range(2):
        d = PT.to_dev(inp)
        out, sel, n_sel, bs, err = PT.run_step(sh, d)
        outs.append((out.cpu(), sel.cpu(), bs.cpu()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


# ---------------------------------------------------------------------------
# the five benchmark workloads at full size
# ---------------------------------------------------------------------------
def test_workload_decode_1x4k_full():
    report(W.DECODE_4K.name, PT.full_parity(W.make_inputs(W.DECODE_4K)))


def test_workload_decode_32x32k_full():
    inp = W.make_inputs(W.DECODE_32K_X32)
    report(W.DECODE_32K_X32.name, PT.full_parity(inp))
    report(W.DECODE_32K_X32.name + " f16 indexer cache", PT.full_parity(inp, queries=[3, 30], idx_f16=True))


def test_workload_decode_8x128k_full():
    inp = W.make_inputs(W.DECODE_128K_X8)
    report(W.DECODE_128K_X8.name, PT.full_parity(inp))


def _spread_tiles(n_q, every=32, tile=8, extra=()):
    """Queries of every ``every``-th attention tile (``tile`` consecutive
    queries), plus ``extra``: a spread of whole tiles across the batch."""
    q = set(extra)
    for t0 in range(0, n_q, every * tile):
        q.update(range(t0, min(t0 + tile, n_q)))
    return sorted(q)


def test_workload_prefill_16k_every_query():
    """Block scores and selection of all 16384 queries against the oracle;
    attention on every 32nd 8-query tile (512 queries) and the edges of the
    dense/sparse boundary."""
    inp = W.make_inputs(W.PREFILL_16K)
    attn = _spread_tiles(16384, extra=[1, 127, 128, 129, 2046, 2047, 2048, 2049, 4095, 4096, 8191, 16383])
    rep = PT.full_parity(inp, prefill=True, attn_queries=attn)
    report(W.PREFILL_16K.name, rep)
    assert rep["queries"] == 16384 and rep["attn_queries"] >= 256


def test_workload_chunked_prefill_ties_every_query():
    """All 8192 queries of the tie workload: scores, and selection bit-exact
    with no near-tie excused (every score is exact in float32); attention on
    every 32nd 8-query tile of the four streams (256 queries) plus the
    chunk edges."""
    inp = W.make_inputs(W.CHUNKED_PREFILL_TIES)
    attn = _spread_tiles(8192, extra=[1, 2047, 2048, 4095, 6143, 8191])
    rep = PT.full_parity(inp, prefill=True, attn_queries=attn)
    report(W.CHUNKED_PREFILL_TIES.name, rep)
    assert rep["queries"] == 8192 and rep["attn_queries"] >= 256
    assert rep["near_ties"] == 0 and rep["max_score_err"] == 0.0
