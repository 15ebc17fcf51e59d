"""MiniMax Sparse Attention (MSA) hot path on B200: Python binding.

Thin ctypes layer over ``libmsa.so`` (the C ABI declared in include/msa.h):
it checks tensor dtypes, devices and shapes, passes raw device pointers and
the current CUDA stream, and turns a non-zero status into ``MsaError``.  All
computation runs in the library's CUDA kernels; there is no fallback.  If the
library has not been built, every call raises.

Build:  python -m block_sparse_attention_maxpool_b200.build
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass

import torch

__all__ = ["MsaError", "Shape", "msa_indexer_append", "msa_kv_append", "msa_step_append", "msa_block_scores",
           "msa_indexer_append_f16",
           "msa_select_topk", "msa_sparse_attn_decode", "msa_sparse_attn_prefill", "msa_select_attn_decode",
           "msa_select_attn_decode_paged",
           "msa_workspace_bytes", "msa_get_device_error", "msa_sparse_attn_decode_noalloc", "msa_version", "library", "LIB_PATH",
           "MODE_DECODE", "MODE_PREFILL", "LOCAL_BIAS", "decode_step",
           "Pages", "msa_indexer_append_paged", "msa_indexer_append_f16_paged", "msa_kv_append_paged",
           "msa_block_scores_paged", "msa_block_scores_f16_paged", "msa_sparse_attn_decode_paged",
           "msa_sparse_attn_prefill_paged", "DsaShape", "DSA_SEL_WIDTH", "msa_dsa_indexer_append",
           "msa_dsa_token_scores", "msa_dsa_select_topk", "msa_dsa_sparse_attn_decode", "dsa_decode_step",
           "msa_decode_step_fused", "msa_decode_step_fused_workspace_bytes", "decode_step_fused", "DecodeGraph",
           "StepPipeline", "msa_wait_selftest", "WAIT_SELFTEST_WORKSPACE_BYTES"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmsa.so")
MODE_DECODE = 0
MODE_PREFILL = 1
LOCAL_BIAS = 2.0 ** 100

STATUS = {0: "MSA_OK", -1: "MSA_ERR_NULL", -2: "MSA_ERR_ALIGN", -3: "MSA_ERR_SHAPE",
          -4: "MSA_ERR_RANGE", -5: "MSA_ERR_WORKSPACE", -6: "MSA_ERR_CUDA"}
DEVERR = {0x1: "QUERY_RANGE", 0x2: "TOKEN_RANGE", 0x4: "SEL_RANGE", 0x8: "TIMEOUT", 0x10: "PAGE_RANGE"}


class MsaError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS.get(status, status)}")
        self.status = status


class CShape(ctypes.Structure):
    _fields_ = [("n_streams", ctypes.c_int32), ("capacity", ctypes.c_int32),
                ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
                ("block", ctypes.c_int32), ("top_k", ctypes.c_int32)]


@dataclass(frozen=True)
class Shape:
    """Geometry of one MSA layer's caches (msa_shape)."""
    n_streams: int
    capacity: int
    n_q_heads: int = 64
    n_kv_heads: int = 4
    head_dim: int = 128
    idx_dim: int = 128
    block: int = 128
    top_k: int = 16

    @property
    def n_blocks(self) -> int:
        return self.capacity // self.block

    def c(self) -> CShape:
        return CShape(self.n_streams, self.capacity, self.n_q_heads, self.n_kv_heads,
                      self.head_dim, self.idx_dim, self.block, self.top_k)


class CPages(ctypes.Structure):
    _fields_ = [("block_table", ctypes.c_void_p), ("n_pages", ctypes.c_int32)]


@dataclass(frozen=True)
class Pages:
    """Block table of paged caches (msa_pages): ``block_table`` is an int32
    device tensor [n_streams][capacity / 128] naming the pool page that holds
    each logical block; pools are [n_pages][G][128][row]."""
    block_table: torch.Tensor
    n_pages: int

    def c(self, shape: "Shape") -> CPages:
        t = _ptr(self.block_table, torch.int32, (shape.n_streams, shape.n_blocks), "block_table")
        return CPages(t, int(self.n_pages))


class CDsaShape(ctypes.Structure):
    _fields_ = [("n_streams", ctypes.c_int32), ("capacity", ctypes.c_int32), ("n_index_heads", ctypes.c_int32),
                ("index_dim", ctypes.c_int32), ("top_k", ctypes.c_int32), ("relu", ctypes.c_int32)]


DSA_SEL_WIDTH = 2048


@dataclass(frozen=True)
class DsaShape:
    """Geometry of the token-level (lightning-indexer) variant (msa_dsa_shape)."""
    n_streams: int
    capacity: int
    n_index_heads: int = 64
    index_dim: int = 128
    top_k: int = 2048
    relu: bool = True

    def c(self) -> CDsaShape:
        return CDsaShape(self.n_streams, self.capacity, self.n_index_heads, self.index_dim, self.top_k,
                         int(bool(self.relu)))


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32
_SIGS = {
    "msa_indexer_append": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _I, _P]),
    "msa_kv_append": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _I, _P]),
    "msa_step_append": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "msa_block_scores": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _I, _P, _P, ctypes.c_size_t,
                                        _P]),
    "msa_block_scores_f16": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _I, _P, _P,
                                            ctypes.c_size_t, _P]),
    "msa_indexer_append_f16": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _I, _P]),
    "msa_select_topk": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _I, _P, _P, _P]),
    "msa_sparse_attn_decode": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _I,
                                              ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "msa_sparse_attn_prefill": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _I,
                                               ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "msa_select_attn_decode": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _I,
                                              ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "msa_sparse_attn_decode_noalloc": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P,
                                                      _I, ctypes.c_float, _P, _P]),
    "msa_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(CShape), _I, _I]),
    "msa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "msa_get_device_error": (ctypes.c_int, [ctypes.POINTER(ctypes.c_uint32), _P]),
    "msa_version": (ctypes.c_int, []),
}
_PG = ctypes.POINTER(CPages)
_DS = ctypes.POINTER(CDsaShape)
_SIGS.update({
    "msa_indexer_append_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _I, _P]),
    "msa_indexer_append_f16_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _I, _P]),
    "msa_kv_append_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _P, _P, _I, _P]),
    "msa_step_append_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "msa_block_scores_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _I, _P, _P,
                                              ctypes.c_size_t, _P]),
    "msa_block_scores_f16_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _I, _P, _P,
                                                  ctypes.c_size_t, _P]),
    "msa_sparse_attn_decode_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _P, _P, _I,
                                                    ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "msa_sparse_attn_prefill_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _P, _P, _I,
                                                     ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "msa_select_attn_decode_paged": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _P, _P, _I,
                                                    ctypes.c_float, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "msa_dsa_indexer_append": (ctypes.c_int, [_DS, _PG, _P, _P, _P, _P, _I, _P]),
    "msa_dsa_token_scores": (ctypes.c_int, [_DS, _PG, _P, _P, _P, _P, _P, _I, _P, _P]),
    "msa_dsa_select_topk": (ctypes.c_int, [_DS, _P, _P, _I, _P, _P, _P]),
    "msa_dsa_sparse_attn_decode": (ctypes.c_int, [ctypes.POINTER(CShape), _PG, _P, _P, _P, _P, _P, _P, _I,
                                                  ctypes.c_float, _P, _P, ctypes.c_size_t, _P]),
    "msa_decode_step_fused": (ctypes.c_int, [ctypes.POINTER(CShape), _P, _P, _P, _P, _P, _P, _P, _P, _I, _P, _P,
                                             _P, _P, _I, ctypes.c_float, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "msa_decode_step_fused_workspace_bytes": (ctypes.c_size_t, [ctypes.POINTER(CShape), _I]),
    "msa_wait_selftest": (ctypes.c_int, [ctypes.c_longlong, _P, ctypes.c_size_t, _P]),
})


def library() -> ctypes.CDLL:
    """The loaded libmsa.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "'python -m block_sparse_attention_maxpool_b200.build'")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


# ---------------------------------------------------------------------------
def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: torch.Tensor | None, dtype, shape, name: str) -> int:
    if t is None:
        return 0
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise MsaError(fn, status)


def _n(t: torch.Tensor, name: str) -> int:
    if t.dim() != 1:
        raise ValueError(f"{name} must be 1-D")
    return t.shape[0]


def _cache_shape(shape: Shape, pages: Pages | None, row: int) -> tuple:
    """[S][G][capacity][row] for a contiguous cache, [n_pages][G][128][row] for a pool."""
    if pages is None:
        return (shape.n_streams, shape.n_kv_heads, shape.capacity, row)
    return (pages.n_pages, shape.n_kv_heads, shape.block, row)


def _call(fn: str, shape: Shape, pages: Pages | None, *args) -> None:
    """Call fn (or fn + '_paged' with the page table after the shape)."""
    s = shape.c()
    if pages is None:
        _check(fn, getattr(library(), fn)(ctypes.byref(s), *args))
    else:
        pg = pages.c(shape)
        _check(fn + "_paged", getattr(library(), fn + "_paged")(ctypes.byref(s), ctypes.byref(pg), *args))


def msa_indexer_append(shape: Shape, idx_k_cache, idx_k_new, tok_stream, tok_pos, stream=None, pages=None):
    n = _n(tok_stream, "tok_stream")
    _call("msa_indexer_append", shape, pages,
          _ptr(idx_k_cache, torch.float32, _cache_shape(shape, pages, shape.idx_dim), "idx_k_cache"),
          _ptr(idx_k_new, torch.float32, (n, shape.n_kv_heads, shape.idx_dim), "idx_k_new"),
          _ptr(tok_stream, torch.int32, (n,), "tok_stream"), _ptr(tok_pos, torch.int32, (n,), "tok_pos"),
          n, _stream(stream))


def msa_kv_append(shape: Shape, k_cache, v_cache, k_new, v_new, tok_stream, tok_pos, stream=None, pages=None):
    n = _n(tok_stream, "tok_stream")
    cs = _cache_shape(shape, pages, shape.head_dim)
    ns = (n, shape.n_kv_heads, shape.head_dim)
    _call("msa_kv_append", shape, pages,
          _ptr(k_cache, torch.bfloat16, cs, "k_cache"), _ptr(v_cache, torch.bfloat16, cs, "v_cache"),
          _ptr(k_new, torch.bfloat16, ns, "k_new"), _ptr(v_new, torch.bfloat16, ns, "v_new"),
          _ptr(tok_stream, torch.int32, (n,), "tok_stream"), _ptr(tok_pos, torch.int32, (n,), "tok_pos"),
          n, _stream(stream))


def msa_step_append(shape: Shape, idx_k_cache, k_cache, v_cache, idx_k_new, k_new, v_new, tok_stream, tok_pos,
                    stream=None, pages=None):
    """The step's appends in one launch: F32 indexer keys and K/V rows
    (msa_indexer_append + msa_kv_append)."""
    n = _n(tok_stream, "tok_stream")
    cs = _cache_shape(shape, pages, shape.head_dim)
    ns = (n, shape.n_kv_heads, shape.head_dim)
    _call("msa_step_append", shape, pages,
          _ptr(idx_k_cache, torch.float32, _cache_shape(shape, pages, shape.idx_dim), "idx_k_cache"),
          _ptr(k_cache, torch.bfloat16, cs, "k_cache"), _ptr(v_cache, torch.bfloat16, cs, "v_cache"),
          _ptr(idx_k_new, torch.float32, (n, shape.n_kv_heads, shape.idx_dim), "idx_k_new"),
          _ptr(k_new, torch.bfloat16, ns, "k_new"), _ptr(v_new, torch.bfloat16, ns, "v_new"),
          _ptr(tok_stream, torch.int32, (n,), "tok_stream"), _ptr(tok_pos, torch.int32, (n,), "tok_pos"),
          n, _stream(stream))


def _workspace(shape: Shape, n: int, mode: int, workspace, device):
    """(pointer, bytes) of the caller's workspace, allocating one if needed."""
    need = msa_workspace_bytes(shape, n, mode)
    if workspace is None and need > 0:
        workspace = torch.empty((need,), dtype=torch.uint8, device=device)
    if workspace is None:
        return 0, 0, None
    return _ptr(workspace, torch.uint8, None, "workspace"), workspace.numel(), workspace


def msa_indexer_append_f16(shape: Shape, idx_k_cache, idx_k_new, tok_stream, tok_pos, stream=None,
                           pages=None):
    """F16 indexer-key cache variant of msa_indexer_append (float16 cache;
    the new F32 keys are rounded to fp16 as they are written)."""
    n = _n(tok_stream, "tok_stream")
    _call("msa_indexer_append_f16", shape, pages,
          _ptr(idx_k_cache, torch.float16, _cache_shape(shape, pages, shape.idx_dim), "idx_k_cache"),
          _ptr(idx_k_new, torch.float32, (n, shape.n_kv_heads, shape.idx_dim), "idx_k_new"),
          _ptr(tok_stream, torch.int32, (n,), "tok_stream"), _ptr(tok_pos, torch.int32, (n,), "tok_pos"),
          n, _stream(stream))


def msa_block_scores(shape: Shape, idx_q, idx_k_cache, q_stream, q_pos, block_scores=None, stream=None,
                     workspace=None, pages=None):
    """Block scores over the F32 indexer-key cache, or over the F16 cache
    variant when idx_k_cache is a float16 tensor."""
    n = _n(q_pos, "q_pos")
    if idx_k_cache.dtype == torch.float16:
        fn, kdt = "msa_block_scores_f16", torch.float16
    else:
        fn, kdt = "msa_block_scores", torch.float32
    if block_scores is None:
        block_scores = torch.empty((n, shape.n_kv_heads, shape.n_blocks), dtype=torch.float32,
                                   device=idx_q.device)
    ws_ptr, ws_bytes, _keep = _workspace(shape, n, MODE_DECODE, workspace, idx_q.device)
    _call(fn, shape, pages, _ptr(idx_q, torch.float32, (n, shape.n_kv_heads, shape.idx_dim), "idx_q"),
          _ptr(idx_k_cache, kdt, _cache_shape(shape, pages, shape.idx_dim), "idx_k_cache"),
          _ptr(q_stream, torch.int32, (n,), "q_stream"), _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
          _ptr(block_scores, torch.float32, (n, shape.n_kv_heads, shape.n_blocks), "block_scores"),
          ws_ptr, ws_bytes, _stream(stream))
    return block_scores


def msa_select_topk(shape: Shape, block_scores, q_pos, sel=None, n_sel=None, stream=None):
    n = _n(q_pos, "q_pos")
    dev = block_scores.device
    if sel is None:
        sel = torch.empty((n, shape.n_kv_heads, shape.top_k), dtype=torch.int32, device=dev)
    if n_sel is None:
        n_sel = torch.empty((n, shape.n_kv_heads), dtype=torch.int32, device=dev)
    s = shape.c()
    _check("msa_select_topk", library().msa_select_topk(
        ctypes.byref(s),
        _ptr(block_scores, torch.float32, (n, shape.n_kv_heads, shape.n_blocks), "block_scores"),
        _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
        _ptr(sel, torch.int32, (n, shape.n_kv_heads, shape.top_k), "sel"),
        _ptr(n_sel, torch.int32, (n, shape.n_kv_heads), "n_sel"), _stream(stream)))
    return sel, n_sel


def msa_workspace_bytes(shape: Shape, n_q: int, mode: int) -> int:
    s = shape.c()
    v = library().msa_workspace_bytes(ctypes.byref(s), n_q, mode)
    if v == ctypes.c_size_t(-1).value:
        raise MsaError("msa_workspace_bytes", -3)
    return v


def _attn(fn_name: str, mode: int, shape: Shape, q, k_cache, v_cache, sel, q_stream, q_pos,
          softmax_scale=None, out=None, workspace=None, stream=None, pages=None):
    n = _n(q_pos, "q_pos")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(shape.head_dim)
    if out is None:
        out = torch.empty((n, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=q.device)
    ws_ptr, ws_bytes, _keep = _workspace(shape, n, mode, workspace, q.device)
    cs = _cache_shape(shape, pages, shape.head_dim)
    _call(fn_name, shape, pages, _ptr(q, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "q"),
          _ptr(k_cache, torch.bfloat16, cs, "k_cache"), _ptr(v_cache, torch.bfloat16, cs, "v_cache"),
          _ptr(sel, torch.int32, (n, shape.n_kv_heads, shape.top_k), "sel"),
          _ptr(q_stream, torch.int32, (n,), "q_stream"), _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
          float(softmax_scale), _ptr(out, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "out"),
          ws_ptr, ws_bytes, _stream(stream))
    return out


def msa_sparse_attn_decode(shape: Shape, q, k_cache, v_cache, sel, q_stream, q_pos, softmax_scale=None,
                           out=None, workspace=None, stream=None, pages=None):
    return _attn("msa_sparse_attn_decode", MODE_DECODE, shape, q, k_cache, v_cache, sel, q_stream,
                 q_pos, softmax_scale, out, workspace, stream, pages)


def msa_sparse_attn_prefill(shape: Shape, q, k_cache, v_cache, sel, q_stream, q_pos, softmax_scale=None,
                            out=None, workspace=None, stream=None, pages=None):
    return _attn("msa_sparse_attn_prefill", MODE_PREFILL, shape, q, k_cache, v_cache, sel, q_stream,
                 q_pos, softmax_scale, out, workspace, stream, pages)


def msa_select_attn_decode(shape: Shape, block_scores, q, k_cache, v_cache, q_stream, q_pos, softmax_scale=None,
                           sel=None, n_sel=None, out=None, workspace=None, stream=None, pages=None):
    """Top-16 selection and decode attention in one call (msa_select_attn_decode,
    or its _paged form with ``pages``).  Returns (out, sel, n_sel)."""
    n = _n(q_pos, "q_pos")
    dev = q.device
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(shape.head_dim)
    if sel is None:
        sel = torch.empty((n, shape.n_kv_heads, shape.top_k), dtype=torch.int32, device=dev)
    if n_sel is None:
        n_sel = torch.empty((n, shape.n_kv_heads), dtype=torch.int32, device=dev)
    if out is None:
        out = torch.empty((n, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=dev)
    ws_ptr, ws_bytes, _keep = _workspace(shape, n, MODE_DECODE, workspace, dev)
    cs = _cache_shape(shape, pages, shape.head_dim)
    _call("msa_select_attn_decode", shape, pages,
          _ptr(block_scores, torch.float32, (n, shape.n_kv_heads, shape.n_blocks), "block_scores"),
          _ptr(q, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "q"),
          _ptr(k_cache, torch.bfloat16, cs, "k_cache"), _ptr(v_cache, torch.bfloat16, cs, "v_cache"),
          _ptr(q_stream, torch.int32, (n,), "q_stream"), _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
          float(softmax_scale), _ptr(sel, torch.int32, (n, shape.n_kv_heads, shape.top_k), "sel"),
          _ptr(n_sel, torch.int32, (n, shape.n_kv_heads), "n_sel"),
          _ptr(out, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "out"), ws_ptr, ws_bytes,
          _stream(stream))
    return out, sel, n_sel


def msa_select_attn_decode_paged(shape: Shape, pages: Pages, block_scores, q, k_pool, v_pool, q_stream, q_pos,
                                 softmax_scale=None, sel=None, n_sel=None, out=None, workspace=None, stream=None):
    return msa_select_attn_decode(shape, block_scores, q, k_pool, v_pool, q_stream, q_pos, softmax_scale, sel,
                                  n_sel, out, workspace, stream, pages)


# ---- paged caches: the C ABI's *_paged calls --------------------------------
def msa_indexer_append_paged(shape: Shape, pages: Pages, idx_k_pool, idx_k_new, tok_stream, tok_pos,
                             stream=None):
    msa_indexer_append(shape, idx_k_pool, idx_k_new, tok_stream, tok_pos, stream, pages)


def msa_indexer_append_f16_paged(shape: Shape, pages: Pages, idx_k_pool, idx_k_new, tok_stream, tok_pos,
                                 stream=None):
    msa_indexer_append_f16(shape, idx_k_pool, idx_k_new, tok_stream, tok_pos, stream, pages)


def msa_kv_append_paged(shape: Shape, pages: Pages, k_pool, v_pool, k_new, v_new, tok_stream, tok_pos,
                        stream=None):
    msa_kv_append(shape, k_pool, v_pool, k_new, v_new, tok_stream, tok_pos, stream, pages)


def msa_block_scores_paged(shape: Shape, pages: Pages, idx_q, idx_k_pool, q_stream, q_pos, block_scores=None,
                           stream=None, workspace=None):
    """Paged block scores; a float16 pool selects msa_block_scores_f16_paged."""
    return msa_block_scores(shape, idx_q, idx_k_pool, q_stream, q_pos, block_scores, stream, workspace, pages)


def msa_block_scores_f16_paged(shape: Shape, pages: Pages, idx_q, idx_k_pool, q_stream, q_pos,
                               block_scores=None, stream=None, workspace=None):
    if idx_k_pool.dtype != torch.float16:
        raise ValueError("idx_k_pool must be float16")
    return msa_block_scores(shape, idx_q, idx_k_pool, q_stream, q_pos, block_scores, stream, workspace, pages)


def msa_sparse_attn_decode_paged(shape: Shape, pages: Pages, q, k_pool, v_pool, sel, q_stream, q_pos,
                                 softmax_scale=None, out=None, workspace=None, stream=None):
    return msa_sparse_attn_decode(shape, q, k_pool, v_pool, sel, q_stream, q_pos, softmax_scale, out,
                                  workspace, stream, pages)


def msa_sparse_attn_prefill_paged(shape: Shape, pages: Pages, q, k_pool, v_pool, sel, q_stream, q_pos,
                                  softmax_scale=None, out=None, workspace=None, stream=None):
    return msa_sparse_attn_prefill(shape, q, k_pool, v_pool, sel, q_stream, q_pos, softmax_scale, out,
                                   workspace, stream, pages)


NOALLOC_SCRATCH_BYTES = 8 * 1024 * 1024


def msa_sparse_attn_decode_noalloc(shape: Shape, q, k_cache, v_cache, sel, q_stream, q_pos,
                                   softmax_scale=None, out=None, stream=None):
    """Decode attention for callers that cannot allocate device memory: the
    merge bookkeeping and partials go to the library's fixed 8 MiB device
    buffer instead of a workspace.  ``out`` is still the caller's (allocated here only when
    None, for convenience).  Calls sharing the buffer at the same time on the
    GPU race; see include/msa.h."""
    n = _n(q_pos, "q_pos")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(shape.head_dim)
    if out is None:
        out = torch.empty((n, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=q.device)
    cs = (shape.n_streams, shape.n_kv_heads, shape.capacity, shape.head_dim)
    s = shape.c()
    _check("msa_sparse_attn_decode_noalloc", library().msa_sparse_attn_decode_noalloc(
        ctypes.byref(s), _ptr(q, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "q"),
        _ptr(k_cache, torch.bfloat16, cs, "k_cache"), _ptr(v_cache, torch.bfloat16, cs, "v_cache"),
        _ptr(sel, torch.int32, (n, shape.n_kv_heads, shape.top_k), "sel"),
        _ptr(q_stream, torch.int32, (n,), "q_stream"), _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
        float(softmax_scale), _ptr(out, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "out"),
        _stream(stream)))
    return out


def msa_get_device_error(stream=None) -> int:
    """Wait for the stream, then read and clear the device error word."""
    v = ctypes.c_uint32(0)
    _check("msa_get_device_error", library().msa_get_device_error(ctypes.byref(v), _stream(stream)))
    return v.value


WAIT_SELFTEST_WORKSPACE_BYTES = 16


def msa_wait_selftest(wait_cycles: int, workspace: torch.Tensor, stream=None) -> None:
    """Run the library's bounded waits against conditions that never come
    true (see include/msa.h); each gives up after ``wait_cycles`` SM clock
    cycles and records the TIMEOUT bit of the device error word.
    ``workspace``: a uint8 CUDA tensor of at least 16 bytes; its third
    32-bit word is 0 afterwards when every wait ran out."""
    _check("msa_wait_selftest", library().msa_wait_selftest(
        int(wait_cycles), _ptr(workspace, torch.uint8, None, "workspace"), workspace.numel(), _stream(stream)))


def msa_version() -> int:
    return library().msa_version()


def decode_step(shape: Shape, caches: dict, new: dict, bufs: dict | None = None, stream=None,
                prefill: bool = False, pages: Pages | None = None):
    """One MSA step through the C ABI: append the new tokens' indexer keys
    and K/V rows, score blocks, select the top-k and attend.

    caches: idx_k_cache (float32, or float16 for the F16 cache variant),
    k_cache, v_cache (device); new: tok_stream, tok_pos,
    idx_k_new, k_new, v_new, q_stream, q_pos, idx_q, q (device).  ``bufs`` may
    hold preallocated block_scores / sel / n_sel / out / workspace.  With
    ``pages`` the caches are page pools addressed through its block table.
    Returns (out, sel, n_sel, block_scores).
    """
    b = bufs or {}
    if caches["idx_k_cache"].dtype == torch.float16:
        msa_indexer_append_f16(shape, caches["idx_k_cache"], new["idx_k_new"], new["tok_stream"], new["tok_pos"],
                               stream, pages)
        msa_kv_append(shape, caches["k_cache"], caches["v_cache"], new["k_new"], new["v_new"],
                      new["tok_stream"], new["tok_pos"], stream, pages)
    else:
        msa_step_append(shape, caches["idx_k_cache"], caches["k_cache"], caches["v_cache"], new["idx_k_new"],
                        new["k_new"], new["v_new"], new["tok_stream"], new["tok_pos"], stream, pages)
    n = new["q_pos"].shape[0]
    mode = MODE_PREFILL if prefill else MODE_DECODE
    if b.get("workspace") is None and msa_workspace_bytes(shape, n, mode) > 0:
        b = dict(b, workspace=torch.empty((msa_workspace_bytes(shape, n, mode),), dtype=torch.uint8,
                                          device=new["q"].device))
    bs = msa_block_scores(shape, new["idx_q"], caches["idx_k_cache"], new["q_stream"], new["q_pos"],
                          b.get("block_scores"), stream, b.get("workspace"), pages)
    if not prefill:                         # the top-16 inside the attention kernel
        out, sel, n_sel = msa_select_attn_decode(shape, bs, new["q"], caches["k_cache"], caches["v_cache"],
                                                 new["q_stream"], new["q_pos"], None, b.get("sel"), b.get("n_sel"),
                                                 b.get("out"), b.get("workspace"), stream, pages)
        return out, sel, n_sel, bs
    sel, n_sel = msa_select_topk(shape, bs, new["q_pos"], b.get("sel"), b.get("n_sel"), stream)
    out = msa_sparse_attn_prefill(shape, new["q"], caches["k_cache"], caches["v_cache"], sel, new["q_stream"],
                                  new["q_pos"], None, b.get("out"), b.get("workspace"), stream, pages)
    return out, sel, n_sel, bs


# ---- token-level variant (lightning indexer) --------------------------------
def _dsa_pages(shape, pages):
    """ctypes argument for an optional page table (None: contiguous)."""
    if pages is None:
        return None
    return ctypes.byref(pages.c(shape))


def _dsa_key_shape(shape: DsaShape, pages: Pages | None) -> tuple:
    if pages is None:
        return (shape.n_streams, shape.capacity, shape.index_dim)
    return (pages.n_pages, 128, shape.index_dim)


def _as_msa_shape(shape: DsaShape) -> Shape:
    return Shape(n_streams=shape.n_streams, capacity=shape.capacity, n_q_heads=16, n_kv_heads=1)


def msa_dsa_indexer_append(shape: DsaShape, k_idx_cache, k_idx_new, tok_stream, tok_pos, stream=None,
                           pages: Pages | None = None):
    """Write new tokens' F32 indexer keys (rounded to fp16) into the F16 key cache."""
    n = _n(tok_stream, "tok_stream")
    s = shape.c()
    _check("msa_dsa_indexer_append", library().msa_dsa_indexer_append(
        ctypes.byref(s), _dsa_pages(_as_msa_shape(shape), pages),
        _ptr(k_idx_cache, torch.float16, _dsa_key_shape(shape, pages), "k_idx_cache"),
        _ptr(k_idx_new, torch.float32, (n, shape.index_dim), "k_idx_new"),
        _ptr(tok_stream, torch.int32, (n,), "tok_stream"), _ptr(tok_pos, torch.int32, (n,), "tok_pos"),
        n, _stream(stream)))


def msa_dsa_token_scores(shape: DsaShape, q_idx, weights, k_idx_cache, q_stream, q_pos, scores=None,
                         stream=None, pages: Pages | None = None):
    """Lightning-indexer scores [n_q][capacity] (float32, -inf past each query)."""
    n = _n(q_pos, "q_pos")
    if scores is None:
        scores = torch.empty((n, shape.capacity), dtype=torch.float32, device=q_idx.device)
    s = shape.c()
    _check("msa_dsa_token_scores", library().msa_dsa_token_scores(
        ctypes.byref(s), _dsa_pages(_as_msa_shape(shape), pages),
        _ptr(q_idx, torch.float16, (n, shape.n_index_heads, shape.index_dim), "q_idx"),
        _ptr(weights, torch.float32, (n, shape.n_index_heads), "weights"),
        _ptr(k_idx_cache, torch.float16, _dsa_key_shape(shape, pages), "k_idx_cache"),
        _ptr(q_stream, torch.int32, (n,), "q_stream"), _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
        _ptr(scores, torch.float32, (n, shape.capacity), "scores"), _stream(stream)))
    return scores


def msa_dsa_select_topk(shape: DsaShape, scores, q_pos, sel=None, n_sel=None, stream=None):
    """Top-k tokens per query: sel [n_q][2048] ascending ids (-1 padded), n_sel [n_q]."""
    n = _n(q_pos, "q_pos")
    dev = scores.device
    if sel is None:
        sel = torch.empty((n, DSA_SEL_WIDTH), dtype=torch.int32, device=dev)
    if n_sel is None:
        n_sel = torch.empty((n,), dtype=torch.int32, device=dev)
    s = shape.c()
    _check("msa_dsa_select_topk", library().msa_dsa_select_topk(
        ctypes.byref(s), _ptr(scores, torch.float32, (n, shape.capacity), "scores"),
        _ptr(q_pos, torch.int32, (n,), "q_pos"), n, _ptr(sel, torch.int32, (n, DSA_SEL_WIDTH), "sel"),
        _ptr(n_sel, torch.int32, (n,), "n_sel"), _stream(stream)))
    return sel, n_sel


def msa_dsa_sparse_attn_decode(shape: Shape, q, k_cache, v_cache, sel, q_stream, q_pos, softmax_scale=None,
                               out=None, workspace=None, stream=None, pages: Pages | None = None):
    """Attention of every head over its query's kept tokens (MSA K/V caches)."""
    n = _n(q_pos, "q_pos")
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(shape.head_dim)
    if out is None:
        out = torch.empty((n, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=q.device)
    ws_ptr, ws_bytes, _keep = _workspace(shape, n, MODE_DECODE, workspace, q.device)
    cs = _cache_shape(shape, pages, shape.head_dim)
    s = shape.c()
    _check("msa_dsa_sparse_attn_decode", library().msa_dsa_sparse_attn_decode(
        ctypes.byref(s), _dsa_pages(shape, pages),
        _ptr(q, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "q"),
        _ptr(k_cache, torch.bfloat16, cs, "k_cache"), _ptr(v_cache, torch.bfloat16, cs, "v_cache"),
        _ptr(sel, torch.int32, (n, DSA_SEL_WIDTH), "sel"),
        _ptr(q_stream, torch.int32, (n,), "q_stream"), _ptr(q_pos, torch.int32, (n,), "q_pos"), n,
        float(softmax_scale), _ptr(out, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "out"),
        ws_ptr, ws_bytes, _stream(stream)))
    return out


def dsa_decode_step(shape: Shape, dshape: DsaShape, caches: dict, new: dict, bufs: dict | None = None,
                    stream=None, pages: Pages | None = None, idx_pages: Pages | None = None):
    """One token-level step through the C ABI: append the new tokens' F16
    indexer keys and K/V rows, score every visible token, keep the top-k and
    attend.  caches: k_idx_cache (float16 [S][cap][128]), k_cache, v_cache;
    new: tok_stream, tok_pos, k_idx_new, k_new, v_new, q_stream, q_pos,
    q_idx (float16 [n_q][64][128]), weights ([n_q][64]), q.
    Returns (out, sel, n_sel, scores)."""
    b = bufs or {}
    msa_dsa_indexer_append(dshape, caches["k_idx_cache"], new["k_idx_new"], new["tok_stream"], new["tok_pos"],
                           stream, idx_pages)
    msa_kv_append(shape, caches["k_cache"], caches["v_cache"], new["k_new"], new["v_new"],
                  new["tok_stream"], new["tok_pos"], stream, pages)
    sc = msa_dsa_token_scores(dshape, new["q_idx"], new["weights"], caches["k_idx_cache"], new["q_stream"],
                              new["q_pos"], b.get("scores"), stream, idx_pages)
    sel, n_sel = msa_dsa_select_topk(dshape, sc, new["q_pos"], b.get("sel"), b.get("n_sel"), stream)
    out = msa_dsa_sparse_attn_decode(shape, new["q"], caches["k_cache"], caches["v_cache"], sel, new["q_stream"],
                                     new["q_pos"], None, b.get("out"), b.get("workspace"), stream, pages)
    return out, sel, n_sel, sc


# ---- the whole decode step in one kernel ---------------------------------------
def msa_decode_step_fused_workspace_bytes(shape: Shape, n_q: int) -> int:
    s = shape.c()
    v = library().msa_decode_step_fused_workspace_bytes(ctypes.byref(s), n_q)
    if v == ctypes.c_size_t(-1).value:
        raise MsaError("msa_decode_step_fused_workspace_bytes", -3)
    return v


def msa_decode_step_fused(shape: Shape, caches: dict, new: dict, bufs: dict | None = None, stream=None,
                          softmax_scale=None):
    """One decode step (appends, block scores, top-16, attention) as a single
    persistent kernel; same inputs and results as ``decode_step`` (F32
    indexer cache, decode-shaped batches).  Returns (out, sel, n_sel,
    block_scores)."""
    b = bufs or {}
    n = _n(new["q_pos"], "q_pos")
    nt = _n(new["tok_stream"], "tok_stream")
    dev = new["q"].device
    G = shape.n_kv_heads
    if softmax_scale is None:
        softmax_scale = 1.0 / math.sqrt(shape.head_dim)
    bs = b.get("block_scores")
    if bs is None:
        bs = torch.empty((n, G, shape.n_blocks), dtype=torch.float32, device=dev)
    sel = b.get("sel")
    if sel is None:
        sel = torch.empty((n, G, shape.top_k), dtype=torch.int32, device=dev)
    n_sel = b.get("n_sel")
    if n_sel is None:
        n_sel = torch.empty((n, G), dtype=torch.int32, device=dev)
    out = b.get("out")
    if out is None:
        out = torch.empty((n, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=dev)
    ws = b.get("workspace_fused")
    need = msa_decode_step_fused_workspace_bytes(shape, n) if n > 0 else 0
    if ws is None and need > 0:
        ws = torch.empty((need,), dtype=torch.uint8, device=dev)
    cs = (shape.n_streams, G, shape.capacity)
    s = shape.c()
    _check("msa_decode_step_fused", library().msa_decode_step_fused(
        ctypes.byref(s), _ptr(caches["idx_k_cache"], torch.float32, cs + (shape.idx_dim,), "idx_k_cache"),
        _ptr(caches["k_cache"], torch.bfloat16, cs + (shape.head_dim,), "k_cache"),
        _ptr(caches["v_cache"], torch.bfloat16, cs + (shape.head_dim,), "v_cache"),
        _ptr(new["idx_k_new"], torch.float32, (nt, G, shape.idx_dim), "idx_k_new"),
        _ptr(new["k_new"], torch.bfloat16, (nt, G, shape.head_dim), "k_new"),
        _ptr(new["v_new"], torch.bfloat16, (nt, G, shape.head_dim), "v_new"),
        _ptr(new["tok_stream"], torch.int32, (nt,), "tok_stream"), _ptr(new["tok_pos"], torch.int32, (nt,), "tok_pos"),
        nt, _ptr(new["idx_q"], torch.float32, (n, G, shape.idx_dim), "idx_q"),
        _ptr(new["q"], torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "q"),
        _ptr(new["q_stream"], torch.int32, (n,), "q_stream"), _ptr(new["q_pos"], torch.int32, (n,), "q_pos"), n,
        float(softmax_scale), _ptr(bs, torch.float32, (n, G, shape.n_blocks), "block_scores"),
        _ptr(sel, torch.int32, (n, G, shape.top_k), "sel"), _ptr(n_sel, torch.int32, (n, G), "n_sel"),
        _ptr(out, torch.bfloat16, (n, shape.n_q_heads, shape.head_dim), "out"),
        _ptr(ws, torch.uint8, None, "workspace") if ws is not None else 0, ws.numel() if ws is not None else 0,
        _stream(stream)))
    return out, sel, n_sel, bs


decode_step_fused = msa_decode_step_fused


# ---- replaying a captured step ----------------------------------------------
STEP_INPUTS = ("tok_stream", "tok_pos", "idx_k_new", "k_new", "v_new", "q_stream", "q_pos", "idx_q", "q")


class DecodeGraph:
    """One MSA step (``decode_step``: appends, block scores, top-k, attention)
    captured once as a CUDA graph on fixed device buffers and replayed.

    The step's inputs (tok_stream, tok_pos, idx_k_new, k_new, v_new,
    q_stream, q_pos, idx_q, q) live in one device staging buffer; ``inputs``
    holds views of it, and every replay reads whatever they hold.  A caller
    either writes the views directly, or packs a step's host tensors into
    one pinned buffer (``host_buffer`` + ``pack``) and calls
    ``replay_from(buffer)``, which moves all of them in a single
    host-to-device copy before the replay.  ``out`` holds the result.  The
    graph's kernels are the library's own; shapes are fixed at capture;
    ``caches`` are updated in place by every replay."""

    def __init__(self, shape: Shape, caches: dict, inputs: dict, bufs: dict | None = None, prefill: bool = False,
                 pages: Pages | None = None):
        self.shape, self.caches, self.prefill, self.pages = shape, caches, prefill, pages
        dev = inputs["q"].device
        self._layout = []
        off = 0
        for name in STEP_INPUTS:
            t = inputs[name]
            off = (off + 255) // 256 * 256
            self._layout.append((name, off, t.numel() * t.element_size(), t.dtype, tuple(t.shape)))
            off += t.numel() * t.element_size()
        self.staging = torch.empty((max(off, 16),), dtype=torch.uint8, device=dev)
        self.inputs = {name: self.staging[o:o + nb].view(dt).view(shp) for name, o, nb, dt, shp in self._layout}
        for name in STEP_INPUTS:
            self.inputs[name].copy_(inputs[name])
        n = inputs["q_pos"].shape[0]
        G = shape.n_kv_heads
        b = dict(bufs or {})
        b.setdefault("block_scores", torch.empty((n, G, shape.n_blocks), dtype=torch.float32, device=dev))
        b.setdefault("sel", torch.empty((n, G, shape.top_k), dtype=torch.int32, device=dev))
        b.setdefault("n_sel", torch.empty((n, G), dtype=torch.int32, device=dev))
        b.setdefault("out", torch.empty((n, shape.n_q_heads, shape.head_dim), dtype=torch.bfloat16, device=dev))
        mode = MODE_PREFILL if prefill else MODE_DECODE
        b.setdefault("workspace", torch.empty((max(16, msa_workspace_bytes(shape, n, mode)),), dtype=torch.uint8,
                                              device=dev))
        self.bufs = b
        self.out, self.sel, self.n_sel, self.block_scores = b["out"], b["sel"], b["n_sel"], b["block_scores"]
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):                # first run outside the capture (one-time set-up)
            decode_step(shape, caches, self.inputs, b, side, prefill, pages)
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            decode_step(shape, caches, self.inputs, b, None, prefill, pages)

    def host_buffer(self) -> torch.Tensor:
        """A pinned host buffer with the staging buffer's layout."""
        return torch.empty(self.staging.shape, dtype=torch.uint8).pin_memory()

    def pack(self, host_inputs: dict, buffer: torch.Tensor) -> torch.Tensor:
        """Copy a step's host tensors (same names, dtypes and shapes as the
        captured inputs) into ``buffer`` (a ``host_buffer()``)."""
        for name, o, nb, dt, shp in self._layout:
            t = host_inputs[name]
            if t.dtype != dt or tuple(t.shape) != shp:
                raise ValueError(f"{name} must be {dt} {shp}")
            buffer[o:o + nb].view(dt).view(shp).copy_(t)
        return buffer

    def replay(self):
        """Run the captured step on the current stream."""
        self.graph.replay()
        return self.out

    def replay_from(self, buffer: torch.Tensor):
        """One host-to-device copy of a packed step, then the replay."""
        self.staging.copy_(buffer, non_blocking=True)
        return self.replay()


class StepPipeline:
    """Back-to-back steps with their host transfers overlapped.

    Two ``DecodeGraph`` captures on the same caches alternate (each with its
    own staging buffer and result buffers).  ``step(buffer)`` queues, for the
    next step, the host-to-device copy of its packed inputs on one copy
    stream, the replay on the current stream, and the device-to-host copy of
    its output on a second copy stream; events order them, so step i+1's
    inputs and step i-1's output move while step i runs, and the steps
    still run one after another on the caches.  It returns the pinned host
    tensor that will hold the output and an event recorded when it has
    landed; that tensor is reused two steps later, so read it (after
    ``event.synchronize()``) before then.  Building the pipeline runs the
    first inputs twice (one step per capture, as ``DecodeGraph`` does)."""

    def __init__(self, shape: Shape, caches: dict, inputs: dict, prefill: bool = False,
                 pages: Pages | None = None):
        dev = inputs["q"].device
        self.graphs = [DecodeGraph(shape, caches, inputs, None, prefill, pages) for _ in range(2)]
        self.h2d = torch.cuda.Stream(device=dev)
        self.d2h = torch.cuda.Stream(device=dev)
        self.host_out = [torch.empty(g.out.shape, dtype=g.out.dtype).pin_memory() for g in self.graphs]
        self.ev_in = [torch.cuda.Event() for _ in range(2)]      # inputs of the slot's step are on the device
        self.ev_done = [torch.cuda.Event() for _ in range(2)]    # the slot's replay has finished
        self.ev_out = [torch.cuda.Event() for _ in range(2)]     # the slot's output is on the host
        self.used = [False, False]
        self.n = 0

    def host_buffer(self) -> torch.Tensor:
        """A pinned host buffer with the staging layout (both captures share it)."""
        return self.graphs[0].host_buffer()

    def pack(self, host_inputs: dict, buffer: torch.Tensor) -> torch.Tensor:
        return self.graphs[0].pack(host_inputs, buffer)

    def step(self, buffer: torch.Tensor):
        """Queue one step whose packed inputs are in ``buffer`` (pinned; not
        to be rewritten before the returned event).  Returns (host output,
        event)."""
        i = self.n % 2
        g = self.graphs[i]
        cur = torch.cuda.current_stream(g.out.device)
        if self.used[i]:
            self.h2d.wait_event(self.ev_done[i])      # the slot's staging buffer is free again
            cur.wait_event(self.ev_out[i])            # and its output has been read
        with torch.cuda.stream(self.h2d):
            g.staging.copy_(buffer, non_blocking=True)
            self.ev_in[i].record(self.h2d)
        cur.wait_event(self.ev_in[i])
        g.graph.replay()
        self.ev_done[i].record(cur)
        self.d2h.wait_event(self.ev_done[i])
        with torch.cuda.stream(self.d2h):
            self.host_out[i].copy_(g.out, non_blocking=True)
            self.ev_out[i].record(self.d2h)
        self.used[i] = True
        self.n += 1
        return self.host_out[i], self.ev_out[i]

    def wait_all(self):
        """Make the current stream wait until every queued output has landed."""
        cur = torch.cuda.current_stream(self.graphs[0].out.device)
        for i in range(2):
            if self.used[i]:
                cur.wait_event(self.ev_out[i])
