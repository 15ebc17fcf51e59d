"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every function include/msa.h declares, and rejects bad arguments with the
documented status codes before any CUDA call is made."""
import ctypes
import os
import re

import pytest

import block_sparse_attention_maxpool_b200 as msa
from block_sparse_attention_maxpool_b200 import build as msa_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "msa.h")


@pytest.fixture(scope="module")
def lib():
    msa_build.build()
    return msa.library()


def header_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MSA_API\s+[\w\s\*]+?\b(msa_\w+)\s*\(", text)))


def header_constants():
    text = open(HEADER).read()
    return {m[0]: int(m[1]) for m in re.findall(r"#define\s+(MSA_(?:OK|ERR_\w+))\s+\(?(-?\d+)\)?", text)}


def test_header_declares_the_boundary():
    fns = header_functions()
    for name in ("msa_indexer_append", "msa_block_scores", "msa_select_topk",
                 "msa_sparse_attn_decode", "msa_sparse_attn_prefill"):
        assert name in fns


def test_every_declared_symbol_is_exported(lib):
    for name in header_functions():
        assert hasattr(lib, name), name


def test_binding_status_table_matches_header():
    consts = header_constants()
    for name, value in consts.items():
        assert msa.STATUS[value] == name


def test_version_and_status_strings(lib):
    assert lib.msa_version() >= 100
    assert lib.msa_status_string(0) == b"MSA_OK"
    assert lib.msa_status_string(-5).startswith(b"MSA_ERR_WORKSPACE")


GOOD = msa.Shape(n_streams=2, capacity=1024)
FAKE = 0x10000          # a 16-byte aligned address that is never dereferenced


def call_scores(lib, shape, n_q=4, **over):
    a = dict(idx_q=FAKE, idx_k=FAKE, qs=FAKE, qp=FAKE, bs=FAKE, ws=0, ws_bytes=0)
    a.update(over)
    s = shape.c()
    return lib.msa_block_scores(ctypes.byref(s), a["idx_q"], a["idx_k"], a["qs"], a["qp"], n_q,
                                a["bs"], a["ws"], a["ws_bytes"], None)


@pytest.mark.parametrize("bad", [
    dict(capacity=1000), dict(capacity=0), dict(n_streams=0), dict(head_dim=64), dict(idx_dim=64),
    dict(block=64), dict(top_k=8), dict(n_q_heads=32), dict(n_kv_heads=0), dict(n_kv_heads=17, n_q_heads=272),
    dict(n_streams=4096, capacity=1 << 20),
])
def test_shape_rejected(lib, bad):
    sh = msa.Shape(**{**GOOD.__dict__, **bad})
    assert call_scores(lib, sh) == -3


def test_null_and_alignment(lib):
    assert lib.msa_block_scores(None, FAKE, FAKE, FAKE, FAKE, 1, FAKE, 0, 0, None) == -1
    assert call_scores(lib, GOOD, idx_k=0) == -1
    assert call_scores(lib, GOOD, bs=0) == -1
    assert call_scores(lib, GOOD, idx_q=FAKE + 4) == -2
    assert call_scores(lib, GOOD, n_q=-1) == -4
    assert call_scores(lib, GOOD, n_q=0, idx_q=0, idx_k=0) == 0      # empty batch is a no-op


def test_tile_path_requires_workspace(lib):
    sh = msa.Shape(n_streams=1, capacity=4096)
    s = sh.c()
    need = lib.msa_workspace_bytes(ctypes.byref(s), 512, msa.MODE_PREFILL)
    assert need > 0
    assert call_scores(lib, sh, n_q=512) == -5                               # none given
    assert call_scores(lib, sh, n_q=512, ws=FAKE, ws_bytes=need - 1) == -5   # too small
    assert call_scores(lib, sh, n_q=512, ws=FAKE + 16, ws_bytes=need) == -2  # not 256-B aligned


def test_select_and_append_validation(lib):
    s = GOOD.c()
    assert lib.msa_select_topk(ctypes.byref(s), FAKE, FAKE, 3, 0, 0, None) == -1
    assert lib.msa_select_topk(ctypes.byref(s), FAKE + 8, FAKE, 3, FAKE, 0, None) == -2
    assert lib.msa_select_topk(ctypes.byref(s), FAKE, FAKE, 0, 0, 0, None) == 0
    assert lib.msa_indexer_append(ctypes.byref(s), FAKE, FAKE, FAKE, 0, 2, None) == -1
    assert lib.msa_indexer_append(ctypes.byref(s), FAKE + 4, FAKE, FAKE, FAKE, 2, None) == -2
    assert lib.msa_indexer_append(ctypes.byref(s), FAKE, FAKE, FAKE, FAKE, -2, None) == -4
    assert lib.msa_kv_append(ctypes.byref(s), FAKE, 0, FAKE, FAKE, FAKE, FAKE, 2, None) == -1
    assert lib.msa_kv_append(ctypes.byref(s), 0, 0, 0, 0, 0, 0, 0, None) == 0


def test_attention_validation_and_workspace(lib):
    s = GOOD.c()
    # decode: the merge bookkeeping of 256 CTA slots (16 bytes each), then one
    # partial (16 heads x (128 + 2) floats) per CTA, one CTA per (pair,
    # block) unit at most, 256 CTAs at most
    need = lib.msa_workspace_bytes(ctypes.byref(s), 2, msa.MODE_DECODE)
    assert need == 256 * 16 + min(2 * 4 * 16, 256) * 16 * 130 * 4
    assert lib.msa_workspace_bytes(ctypes.byref(s), 1000, msa.MODE_DECODE) >= 256 * 16 + 256 * 16 * 130 * 4
    # prefill attention: the plan of every 8-query tile (844 bytes) per group
    plans = lambda n_q, G=4: G * ((n_q + 7) // 8) * 844          # noqa: E731
    assert lib.msa_workspace_bytes(ctypes.byref(s), 2, msa.MODE_PREFILL) == plans(2)
    long_cap = msa.Shape(n_streams=2, capacity=65536).c()
    assert lib.msa_workspace_bytes(ctypes.byref(long_cap), 2, msa.MODE_PREFILL) == plans(2)
    # 4096 queries over 2 streams: prefill-shaped, the block scores take the tile path
    big = lib.msa_workspace_bytes(ctypes.byref(s), 4096, msa.MODE_DECODE)
    assert big > 0 and big == lib.msa_workspace_bytes(ctypes.byref(s), 4096, msa.MODE_PREFILL)
    # 600 decode queries over 600 streams keep the streaming score kernel (no
    # score workspace): only the attention partials remain
    many = msa.Shape(n_streams=600, capacity=1024).c()
    assert lib.msa_workspace_bytes(ctypes.byref(many), 600, msa.MODE_DECODE) == 256 * 16 + 256 * 16 * 130 * 4
    assert lib.msa_workspace_bytes(ctypes.byref(many), 600, msa.MODE_PREFILL) == plans(600)
    bad = msa.Shape(n_streams=2, capacity=1000).c()
    assert lib.msa_workspace_bytes(ctypes.byref(bad), 2, 0) == ctypes.c_size_t(-1).value
    args = [FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, ctypes.c_float(0.088), FAKE]
    assert lib.msa_sparse_attn_decode(ctypes.byref(s), *args, 0, 0, None) == -5
    assert lib.msa_sparse_attn_decode(ctypes.byref(s), *args, FAKE, need - 1, None) == -5
    assert lib.msa_sparse_attn_decode(ctypes.byref(s), *args, FAKE + 4, need, None) == -2
    nan_args = list(args)
    nan_args[7] = ctypes.c_float(float("nan"))
    assert lib.msa_sparse_attn_decode(ctypes.byref(s), *nan_args, FAKE, need, None) == -4
    null_args = list(args)
    null_args[1] = 0
    assert lib.msa_sparse_attn_prefill(ctypes.byref(s), *null_args, 0, 0, None) == -1
    assert lib.msa_sparse_attn_prefill(ctypes.byref(s), *args[:6], 0, args[7], FAKE, 0, 0, None) == 0


def test_select_attn_validation(lib):
    """msa_select_attn_decode checks its block scores and selection buffer on
    top of the decode attention's arguments, before any device work."""
    s = GOOD.c()
    need = lib.msa_workspace_bytes(ctypes.byref(s), 2, msa.MODE_DECODE)
    scale = ctypes.c_float(0.088)

    def call(bs=FAKE, q=FAKE, sel=FAKE, n_q=2, scale=scale, ws=FAKE, ws_bytes=need):
        return lib.msa_select_attn_decode(ctypes.byref(s), bs, q, FAKE, FAKE, FAKE, FAKE, n_q, scale, sel, 0,
                                          FAKE, ws, ws_bytes, None)
    assert call(bs=0) == -1
    assert call(sel=0) == -1
    assert call(q=0) == -1
    assert call(bs=FAKE + 4) == -2
    assert call(sel=FAKE + 8) == -2
    assert call(ws_bytes=need - 1) == -5
    assert call(ws=0) == -5
    assert call(scale=ctypes.c_float(float("nan"))) == -4
    assert call(n_q=-1) == -4
    assert call(bs=0, sel=0, n_q=0) == 0
    assert lib.msa_select_attn_decode_paged(ctypes.byref(s), None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 2, scale,
                                            FAKE, 0, FAKE, FAKE, need, None) == -1


def test_binding_rejects_cpu_tensors():
    import torch
    sh = msa.Shape(n_streams=1, capacity=128)
    with pytest.raises(ValueError):
        msa.msa_select_topk(sh, torch.zeros((1, 4, 1)), torch.zeros(1, dtype=torch.int32),
                            sel=torch.zeros((1, 4, 16), dtype=torch.int32),
                            n_sel=torch.zeros((1, 4), dtype=torch.int32), stream=0)


def test_paged_calls_validate_the_page_table(lib):
    s = GOOD.c()
    fake = FAKE

    def pages(table, n):
        return ctypes.byref(msa.CPages(table, n))

    # a NULL msa_pages is rejected by every paged call
    assert lib.msa_indexer_append_paged(ctypes.byref(s), None, fake, fake, fake, fake, 2, None) == -1
    assert lib.msa_kv_append_paged(ctypes.byref(s), None, fake, fake, fake, fake, fake, fake, 2, None) == -1
    assert lib.msa_block_scores_paged(ctypes.byref(s), None, fake, fake, fake, fake, 2, fake, 0, 0, None) == -1
    assert lib.msa_sparse_attn_decode_paged(ctypes.byref(s), None, fake, fake, fake, fake, fake, fake, 2,
                                            ctypes.c_float(0.088), fake, fake, 1 << 24, None) == -1
    # the table itself: NULL, misaligned, no pages, a pool too large for 31-bit rows
    args = (fake, fake, fake, fake, 2, None)
    assert lib.msa_indexer_append_paged(ctypes.byref(s), pages(None, 4), *args) == -1
    assert lib.msa_indexer_append_paged(ctypes.byref(s), pages(fake + 2, 4), *args) == -2
    assert lib.msa_indexer_append_paged(ctypes.byref(s), pages(fake, 0), *args) == -4
    assert lib.msa_indexer_append_f16_paged(ctypes.byref(s), pages(fake, (1 << 31) // (4 * 128)), *args) == -3
    assert lib.msa_indexer_append_paged(ctypes.byref(s), pages(fake, 4), fake, fake, fake, fake, 0, None) == 0
    assert lib.msa_block_scores_f16_paged(ctypes.byref(s), pages(fake, 0), fake, fake, fake, fake, 2, fake,
                                          0, 0, None) == -4
    assert lib.msa_sparse_attn_prefill_paged(ctypes.byref(s), pages(None, 4), fake, fake, fake, fake, fake, fake,
                                             2, ctypes.c_float(0.088), fake, 0, 0, None) == -1


def test_dsa_calls_validate_shapes(lib):
    fake = FAKE
    good = msa.DsaShape(n_streams=2, capacity=1024).c()
    for bad in (msa.DsaShape(n_streams=2, capacity=1000), msa.DsaShape(n_streams=2, capacity=1024, top_k=0),
                msa.DsaShape(n_streams=2, capacity=1024, top_k=2049), msa.DsaShape(n_streams=2, capacity=1024,
                                                                                   n_index_heads=32)):
        b = bad.c()
        assert lib.msa_dsa_select_topk(ctypes.byref(b), fake, fake, 1, fake, 0, None) == -3
        assert lib.msa_dsa_token_scores(ctypes.byref(b), None, fake, fake, fake, fake, fake, 1, fake, None) == -3
    assert lib.msa_dsa_select_topk(ctypes.byref(good), fake, fake, 0, fake, 0, None) == 0
    assert lib.msa_dsa_select_topk(ctypes.byref(good), 0, fake, 2, fake, 0, None) == -1
    assert lib.msa_dsa_select_topk(ctypes.byref(good), fake + 4, fake, 2, fake, 0, None) == -2
    assert lib.msa_dsa_token_scores(ctypes.byref(good), None, fake, 0, fake, fake, fake, 2, fake, None) == -1
    assert lib.msa_dsa_token_scores(ctypes.byref(good), None, fake, fake, fake, fake, fake, -1, fake, None) == -4
    assert lib.msa_dsa_token_scores(ctypes.byref(good), ctypes.byref(msa.CPages(fake, 0)), fake, fake, fake,
                                    fake, fake, 2, fake, None) == -4
    assert lib.msa_dsa_indexer_append(ctypes.byref(good), None, fake, fake, fake, 0, 2, None) == -1
    s = GOOD.c()
    assert lib.msa_dsa_sparse_attn_decode(ctypes.byref(s), None, fake, fake, fake, 0, fake, fake, 2,
                                          ctypes.c_float(0.088), fake, 0, 0, None) == -1
    assert lib.msa_dsa_sparse_attn_decode(ctypes.byref(s), None, fake, fake, fake, fake, fake, fake, 2,
                                          ctypes.c_float(0.088), fake, 0, 0, None) == -5


def test_fused_step_validation(lib):
    s = GOOD.c()
    fake = FAKE
    ws = lib.msa_decode_step_fused_workspace_bytes(ctypes.byref(s), 2)
    assert 0 < ws < (1 << 24)
    assert lib.msa_decode_step_fused_workspace_bytes(ctypes.byref(s), 0) == ctypes.c_size_t(-1).value
    assert lib.msa_decode_step_fused_workspace_bytes(ctypes.byref(s), 4096) == ctypes.c_size_t(-1).value  # prefill-shaped
    f = lib.msa_decode_step_fused

    def call(n_tok=1, n_q=2, null_at=None, ws_ptr=fake, ws_bytes=1 << 24):
        args = [fake] * 8 + [n_tok] + [fake] * 4 + [n_q, ctypes.c_float(0.088)] + [fake] * 4 + [ws_ptr, ws_bytes, None]
        if null_at is not None:
            args[null_at] = 0
        return f(ctypes.byref(s), *args)
    assert call(n_q=-1) == -4
    assert call(null_at=0) == -1                      # idx_k_cache
    assert call(null_at=9) == -1                      # idx_q
    assert call(n_q=4096) == -3                       # prefill-shaped batch
    assert call(ws_ptr=0, ws_bytes=0) == -5
    assert call(ws_ptr=fake + 16) == -2               # workspace not 256-byte aligned


def test_wait_selftest_validation(lib):
    """Argument checks of msa_wait_selftest, made before any device work."""
    fake = 0x10000
    assert lib.msa_wait_selftest(0, fake, 16, None) == -4                 # limit out of range
    assert lib.msa_wait_selftest(10 ** 9 + 1, fake, 16, None) == -4
    assert lib.msa_wait_selftest(1000, None, 16, None) == -1
    assert lib.msa_wait_selftest(1000, fake, 8, None) == -5               # too small
    assert lib.msa_wait_selftest(1000, fake + 4, 16, None) == -2          # not 16-byte aligned


def test_step_append_validation(lib):
    """msa_step_append (indexer keys + K/V in one launch): null, alignment,
    count and shape errors before any device work."""
    s = msa.Shape(n_streams=1, capacity=256).c()
    fake = 0x10000
    args = [fake] * 6 + [fake, fake]
    assert lib.msa_step_append(ctypes.byref(s), *args, 0, None) == 0            # nothing to append
    assert lib.msa_step_append(ctypes.byref(s), *args, -1, None) == -4
    for i in range(8):
        bad = list(args)
        bad[i] = None
        assert lib.msa_step_append(ctypes.byref(s), *bad, 3, None) == -1, i
    for i in range(6):
        bad = list(args)
        bad[i] = fake + 8
        assert lib.msa_step_append(ctypes.byref(s), *bad, 3, None) == -2, i
    bad_shape = msa.Shape(n_streams=1, capacity=200).c()
    assert lib.msa_step_append(ctypes.byref(bad_shape), *args, 3, None) == -3
    assert lib.msa_step_append_paged(ctypes.byref(s), None, *args, 3, None) == -1
