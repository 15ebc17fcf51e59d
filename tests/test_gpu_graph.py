"""DecodeGraph: a step captured once and replayed on new inputs copied into
its buffers gives exactly what the direct calls give on those inputs."""
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


NAMES = ("tok_stream", "tok_pos", "idx_k_new", "k_new", "v_new", "q_stream", "q_pos", "idx_q", "q")


@pytest.mark.parametrize("prefill", [False, True])
def test_replay_with_new_inputs_matches_direct_calls(prefill):
    if prefill:
        w = W.Workload("graph_prefill_2x700", 2, 300, 1000, "new")
    else:
        w = W.Workload("graph_decode_9x3000", 9, 2999, 3000, "last")
    first = W.make_inputs(w, seed=81)
    second = W.make_inputs(w, seed=82)
    shape = PT.shape_of(w)
    # graph path: capture on the first step's buffers, then feed the second step's inputs
    dg_dev = PT.to_dev(first)
    caches_g = {k: dg_dev[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    graph = msa.DecodeGraph(shape, caches_g, dg_dev, prefill=prefill)
    # the second step's inputs arrive in one copy of a packed pinned buffer
    host = {n: getattr(second, n).contiguous() for n in NAMES}
    out_g = graph.replay_from(graph.pack(host, graph.host_buffer())).clone()
    torch.cuda.synchronize()
    # direct path: the first step, then the second, on their own caches
    d = PT.to_dev(first)
    caches_d = {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    msa.decode_step(shape, caches_d, d, prefill=prefill)
    d2 = PT.to_dev(second)
    out_d, sel_d, n_d, bs_d = msa.decode_step(shape, caches_d, d2, prefill=prefill)
    assert msa.msa_get_device_error() == 0
    for k in ("idx_k_cache", "k_cache", "v_cache"):
        assert torch.equal(caches_g[k], caches_d[k]), k
    assert torch.equal(out_g, out_d)
    assert torch.equal(graph.sel, sel_d) and torch.equal(graph.block_scores, bs_d)


@pytest.mark.parametrize("prefill", [False, True])
def test_step_pipeline_matches_direct_calls(prefill):
    """Four steps through StepPipeline (overlapped host transfers, two
    alternating captures) give the outputs and caches of four direct steps."""
    if prefill:
        ws = [W.Workload("pipe_prefill_2x200", 2, 200 * i, 200 * (i + 1), "new") for i in range(1, 5)]
    else:
        ws = [W.Workload("pipe_decode_5x2000", 5, 1995 + i, 1996 + i, "last") for i in range(4)]
    steps = [W.make_inputs(w, seed=90 + i) for i, w in enumerate(ws)]
    shape = PT.shape_of(ws[-1])                  # every step's positions fit the last one's capacity
    base = steps[0]
    cache_src = W.make_inputs(ws[-1], seed=89)

    # the same starting caches twice (pipeline / direct)
    def fresh():
        return {k: getattr(cache_src, k).clone().cuda() for k in ("idx_k_cache", "k_cache", "v_cache")}
    cache_p, cache_d = fresh(), fresh()
    first = {n: getattr(base, n).cuda() for n in NAMES}
    pipe = msa.StepPipeline(shape, cache_p, first, prefill=prefill)
    host_bufs = [pipe.host_buffer() for _ in steps]
    outs = []
    for st, hb in zip(steps, host_bufs):
        h, ev = pipe.step(pipe.pack({n: getattr(st, n).contiguous() for n in NAMES}, hb))
        ev.synchronize()
        outs.append(h.clone())
    torch.cuda.synchronize()
    # direct: the two set-up runs of the first inputs, then the four steps
    first_d = {n: getattr(base, n).cuda() for n in NAMES}
    msa.decode_step(shape, cache_d, first_d, prefill=prefill)
    msa.decode_step(shape, cache_d, first_d, prefill=prefill)
    for st, got in zip(steps, outs):
        out, _, _, _ = msa.decode_step(shape, cache_d, {n: getattr(st, n).cuda() for n in NAMES}, prefill=prefill)
        assert torch.equal(got, out.cpu())
    assert msa.msa_get_device_error() == 0
    for k in ("idx_k_cache", "k_cache", "v_cache"):
        assert torch.equal(cache_p[k], cache_d[k]), k
