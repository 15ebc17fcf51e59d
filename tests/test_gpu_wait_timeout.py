"""Failure detection without a GPU fault: the library's bounded device waits
(the grid barrier of the one-kernel decode step, an mbarrier wait) are driven
to a short limit by msa_wait_selftest.  Each wait must give up, record
MSA_DEVERR_TIMEOUT and let its kernel return; the context must stay usable,
so the calls made right after are exact against the oracle and the one-kernel
step is bit-identical to the separate calls."""
import time

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
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


@pytest.mark.parametrize("cycles", [1, 20_000, 2_000_000])
def test_waits_run_out_and_the_context_stays_usable(cycles):
    ws = torch.full((msa.WAIT_SELFTEST_WORKSPACE_BYTES,), 7, dtype=torch.uint8, device="cuda")
    t0 = time.perf_counter()
    msa.msa_wait_selftest(cycles, ws)
    err = msa.msa_get_device_error()           # waits for the stream
    elapsed = time.perf_counter() - t0
    assert err == 0x8, f"device error word {err:#x}: expected TIMEOUT only"
    assert int(ws.view(torch.int32)[2]) == 0, "a wait that could not end did not give up"
    assert elapsed < 5.0
    # the same context, right after: a whole step against the oracle, and the
    # one-kernel step (whose grid barriers now complete) against the separate calls
    w = W.Workload("after_timeout_5x2300", 5, 2299, 2300, "last")
    inp = W.make_inputs(w, seed=cycles % 1000)
    rep = PT.full_parity(inp)
    assert rep["near_ties"] == 0
    shape = PT.shape_of(w)
    d1, d2 = PT.to_dev(inp), PT.to_dev(inp)
    c1 = {k: d1[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    c2 = {k: d2[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
    r1 = msa.decode_step(shape, c1, d1)
    r2 = msa.decode_step_fused(shape, c2, d2)
    assert msa.msa_get_device_error() == 0
    for a, b in zip(r1, r2):
        assert torch.equal(a, b)
