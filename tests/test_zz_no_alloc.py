"""msa_sparse_attn_decode_noalloc: decode attention for callers that cannot
allocate device memory when they run attention (a runtime whose device
memory all belongs to a pool sized at start-up, or a program using the C ABI
from a language with no CUDA allocator).  Instead of a caller workspace it
uses the library's fixed file-scope device buffer.

The GPU test calls the new entry point through the C ABI twice in a row, with
different batch sizes (so the second call runs over the first call's leftover
buffer contents), and checks that each output is bit-identical to the
workspace entry point msa_sparse_attn_decode (same kernels, same split).
This file is collected last so a failure here never hides another test."""
import ctypes

import pytest
import torch

import block_sparse_attention_maxpool_b200 as msa
import workloads as W
from block_sparse_attention_maxpool_b200 import build as msa_build
from tests import parity as PT


def test_noalloc_buffer_covers_every_batch_and_checks_shapes():
    """Host-side checks (no GPU needed): the decode workspace of any batch
    (merge bookkeeping and at most 256 CTAs x 1 partial) fits the fixed
    buffer, and bad arguments are rejected before any device work."""
    msa_build.build()
    lib = msa.library()
    # many streams: decode-shaped batches, so the query measures the attention workspace only
    many = msa.Shape(n_streams=20000, capacity=128).c()
    for n_q in (1, 3, 127, 128, 4096, 1 << 20):
        assert 0 < lib.msa_workspace_bytes(ctypes.byref(many), n_q, msa.MODE_DECODE) <= msa.NOALLOC_SCRATCH_BYTES
    sh = msa.Shape(n_streams=1, capacity=4096)
    s = sh.c()
    fake = 0x10000
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(s), fake, fake, fake, fake, fake, fake, -1,
                                              ctypes.c_float(0.088), fake, None) == -4
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(s), 0, fake, fake, fake, fake, fake, 3,
                                              ctypes.c_float(0.088), fake, None) == -1
    bad = msa.Shape(n_streams=1, capacity=1000).c()
    assert lib.msa_sparse_attn_decode_noalloc(ctypes.byref(bad), fake, fake, fake, fake, fake, fake, 1,
                                              ctypes.c_float(0.088), fake, None) == -3


def test_binding_scratch_size_matches_header():
    """The binding's copy of the buffer size is the header's constant."""
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "msa.h")).read()
    m = re.search(r"#define\s+MSA_NOALLOC_SCRATCH_BYTES\s+\(([^)]*)\)", hdr)
    assert m is not None
    assert eval(m.group(1).replace("u", "").replace("ll", ""), {}) == msa.NOALLOC_SCRATCH_BYTES


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    msa_build.build()
    for call, (n_streams, ctx, seed) in enumerate(((32, 3000, 31), (5, 2600, 32))):
        w = W.Workload(f"noalloc_{n_streams}x{ctx}", n_streams, ctx - 1, ctx, "last")
        inp = W.make_inputs(w, seed=seed)
        shape = PT.shape_of(w)
        d = PT.to_dev(inp)
        caches = {k: d[k] for k in ("idx_k_cache", "k_cache", "v_cache")}
        out_ws, sel, n_sel, bs = msa.decode_step(shape, caches, d)      # workspace entry point
        assert msa.msa_workspace_bytes(shape, w.n_queries, msa.MODE_DECODE) > 0   # split path used
        out_na = torch.full_like(out_ws, float("nan"))
        msa.msa_sparse_attn_decode_noalloc(shape, d["q"], d["k_cache"], d["v_cache"], sel, d["q_stream"],
                                           d["q_pos"], out=out_na)
        assert msa.msa_get_device_error() == 0
        # the same kernels with the same split: bit-identical, so a stale
        # partial left in the shared buffer by the first call cannot hide
        assert torch.equal(out_na, out_ws), f"call {call}: differs from the workspace entry point"
