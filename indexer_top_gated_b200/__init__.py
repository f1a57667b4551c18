"""Python binding of libdsa.so, the B200 gated Indexer + Top-K sparse-attention layer.

Argument marshalling only: every step of the layer runs in the library's CUDA kernels.
Functions carry the C names (``dsa_index_scores``, ``dsa_topk``,
``dsa_sparse_attn_gated``, ``dsa_prefill``, ``dsa_decode``, ...) and take torch CUDA
tensors, which supply device memory and the current stream.  There is no fallback:
if the library cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import math
import os
from dataclasses import dataclass
from typing import Optional, Sequence

from . import _build

DSA_OK, DSA_ERR_INVALID_ARG, DSA_ERR_UNSUPPORTED, DSA_ERR_WORKSPACE, DSA_ERR_CUDA, \
    DSA_ERR_TIMEOUT = range(6)
DSA_BF16, DSA_FP8_E4M3 = 0, 1

LIB_PATH = _build.LIB


class DsaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {status_string(status)} ({status})")
        self.status = status


class Params(ctypes.Structure):
    _fields_ = [
        ("n_idx_heads", ctypes.c_int32), ("idx_dim", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32), ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32), ("top_k", ctypes.c_int32),
        ("idx_dtype", ctypes.c_int32), ("idx_scale_q", ctypes.c_float),
        ("idx_scale_k", ctypes.c_float), ("attn_scale", ctypes.c_float),
        ("w_row_stride", ctypes.c_int32),
    ]


class Ragged(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("q_offsets", ctypes.c_void_p),
        ("kv_offsets", ctypes.c_void_p), ("max_q_len", ctypes.c_int32),
        ("max_kv_len", ctypes.c_int32), ("total_q", ctypes.c_int64),
        ("total_kv", ctypes.c_int64), ("block_table", ctypes.c_void_p),
        ("max_pages", ctypes.c_int32), ("page_size", ctypes.c_int32),
        ("q_offsets_host", ctypes.c_void_p), ("kv_offsets_host", ctypes.c_void_p),
    ]


class LayerBuffers(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "q_offsets", "kv_offsets", "q_idx", "k_idx", "w", "q", "k_cache", "v_cache", "gate", "out")]


LAYER_BUFFER_KEYS = ("q_offsets", "kv_offsets", "q_idx", "k_idx", "w", "q", "k", "v", "gate", "out")


def layer_buffers(t: dict) -> LayerBuffers:
    """dsa_layer_buffers from a dict of tensors keyed q_offsets, kv_offsets, q_idx, k_idx, w,
    q, k, v, gate (optional), out."""
    return LayerBuffers(*[_ptr(t.get(k)) for k in LAYER_BUFFER_KEYS])


EXPORTS = [
    "dsa_status_string", "dsa_version", "dsa_index_scores", "dsa_topk",
    "dsa_sparse_attn_gated", "dsa_workspace_size", "dsa_prefill", "dsa_decode",
    "dsa_device_status", "dsa_launch_count", "dsa_stage_timing", "dsa_stage_times",
    "dsa_decode_noalloc", "dsa_index_topk", "dsa_index_topk_workspace_size",
    "dsa_sparse_attn_gated_mix", "dsa_index_topk_blocks", "dsa_index_topk_blocks_workspace_size",
    "dsa_prefill_from_host", "dsa_fused_rows",
]


def _load():
    _build.build()
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    PP, RP = ctypes.POINTER(Params), ctypes.POINTER(Ragged)
    L.dsa_status_string.argtypes = [ctypes.c_int]
    L.dsa_status_string.restype = ctypes.c_char_p
    L.dsa_version.argtypes = []
    L.dsa_version.restype = i32
    L.dsa_index_scores.argtypes = [PP, RP, vp, vp, vp, i64, i64, vp, i64, vp]
    L.dsa_topk.argtypes = [PP, RP, vp, i64, i64, i64, vp, i64, vp, vp]
    L.dsa_sparse_attn_gated.argtypes = [PP, RP, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp, vp]
    LB = ctypes.POINTER(LayerBuffers)
    L.dsa_prefill_from_host.argtypes = [PP, RP, LB, LB, i32, i32, vp, sz, vp]
    L.dsa_index_topk_blocks_workspace_size.argtypes = [PP, RP, i32, i64, ctypes.POINTER(sz),
                                                       ctypes.POINTER(sz)]
    L.dsa_index_topk_blocks.argtypes = [PP, RP, vp, vp, vp, i32, i64, i64, vp, i64, vp, vp, sz, vp]
    L.dsa_sparse_attn_gated_mix.argtypes = [PP, RP, vp, vp, vp, vp, i64, i64, i64, vp, vp, vp, vp,
                                            vp, vp]
    L.dsa_workspace_size.argtypes = [PP, RP, ctypes.c_int, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.dsa_index_topk_workspace_size.argtypes = [PP, RP, i64, ctypes.POINTER(sz), ctypes.POINTER(sz)]
    L.dsa_index_topk.argtypes = [PP, RP, vp, vp, vp, i64, i64, vp, i64, vp, vp, sz, vp]
    L.dsa_prefill.argtypes = [PP, RP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
    L.dsa_decode.argtypes = L.dsa_prefill.argtypes
    L.dsa_decode_noalloc.argtypes = [PP, RP, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
    L.dsa_device_status.argtypes = [vp, ctypes.POINTER(i32), ctypes.c_int]
    L.dsa_launch_count.argtypes = []
    L.dsa_launch_count.restype = i64
    L.dsa_fused_rows.argtypes = [ctypes.c_int]
    L.dsa_fused_rows.restype = i64
    L.dsa_stage_timing.argtypes = [ctypes.c_int]
    L.dsa_stage_times.argtypes = [ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64), ctypes.c_int]
    for name in ("dsa_index_scores", "dsa_topk", "dsa_sparse_attn_gated", "dsa_workspace_size",
                 "dsa_prefill", "dsa_decode", "dsa_decode_noalloc", "dsa_device_status",
                 "dsa_stage_timing",
                 "dsa_stage_times"):
        getattr(L, name).restype = ctypes.c_int
    return L


lib = _load()


def status_string(s: int) -> str:
    return lib.dsa_status_string(int(s)).decode()


def _check(rc: int, where: str):
    if rc != DSA_OK:
        raise DsaError(rc, where)


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


@dataclass
class LayerShape:
    n_idx_heads: int = 4
    idx_dim: int = 64
    n_q_heads: int = 32
    n_kv_heads: int = 4
    head_dim: int = 128
    top_k: int = 2048
    idx_dtype: int = DSA_BF16
    idx_scale_q: float = 1.0
    idx_scale_k: float = 1.0
    attn_scale: float = 0.0
    w_row_stride: int = 0

    def params(self) -> Params:
        return Params(self.n_idx_heads, self.idx_dim, self.n_q_heads, self.n_kv_heads,
                      self.head_dim, self.top_k, self.idx_dtype, self.idx_scale_q,
                      self.idx_scale_k, self.attn_scale, self.w_row_stride)


def ragged(q_offsets, kv_offsets, q_lens: Sequence[int], kv_lens: Sequence[int],
           block_table=None, page_size: int = 0, cache_rows: Optional[int] = None) -> Ragged:
    """Build a dsa_ragged from device int32 offset tensors and host lengths; with a device
    int32 block table [batch, max_pages] the cache arrays are paged (cache_rows rows).
    Host copies of the offsets are made from the lengths and attached (they let the layer
    plan per sequence).  The descriptor holds only the tensors' addresses: keep them alive
    while it is used."""
    import numpy as np
    qoh = np.concatenate([[0], np.cumsum(np.asarray(q_lens, dtype=np.int64))]).astype(np.int32)
    koh = np.concatenate([[0], np.cumsum(np.asarray(kv_lens, dtype=np.int64))]).astype(np.int32)
    rg = Ragged(len(q_lens), q_offsets.data_ptr(), kv_offsets.data_ptr(),
                int(max(q_lens)) if len(q_lens) else 0,
                int(max(kv_lens)) if len(kv_lens) else 0, int(sum(q_lens)), int(sum(kv_lens)),
                None, 0, 0, qoh.ctypes.data, koh.ctypes.data)
    rg.host_offsets = (qoh, koh)  # keeps the host copies alive with the descriptor
    if block_table is not None:
        rg.block_table = block_table.data_ptr()
        rg.max_pages = int(block_table.shape[1])
        rg.page_size = int(page_size)
        rg.total_kv = int(cache_rows)
    return rg


def dsa_index_scores(shape: LayerShape, rg: Ragged, q_idx, k_idx, w, q_begin: int, q_count: int,
                     scores, ld_scores: int, stream=None):
    p = shape.params()
    _check(lib.dsa_index_scores(ctypes.byref(p), ctypes.byref(rg), _ptr(q_idx), _ptr(k_idx),
                                _ptr(w), q_begin, q_count, _ptr(scores), ld_scores,
                                _stream(stream)), "dsa_index_scores")


def dsa_topk(shape: LayerShape, rg: Ragged, scores, ld_scores: int, q_begin: int, q_count: int,
             idx, ld_idx: int, cnt=None, stream=None):
    p = shape.params()
    _check(lib.dsa_topk(ctypes.byref(p), ctypes.byref(rg), _ptr(scores), ld_scores, q_begin,
                        q_count, _ptr(idx), ld_idx, _ptr(cnt), _stream(stream)), "dsa_topk")


def dsa_sparse_attn_gated(shape: LayerShape, rg: Ragged, q, k_cache, v_cache, idx, ld_idx: int,
                          q_begin: int, q_count: int, gate, out, lse=None, err_count=None,
                          stream=None):
    p = shape.params()
    _check(lib.dsa_sparse_attn_gated(ctypes.byref(p), ctypes.byref(rg), _ptr(q), _ptr(k_cache),
                                     _ptr(v_cache), _ptr(idx), ld_idx, q_begin, q_count,
                                     _ptr(gate), _ptr(out), _ptr(lse), _ptr(err_count),
                                     _stream(stream)), "dsa_sparse_attn_gated")


def dsa_prefill_from_host(shape: LayerShape, rg: Ragged, host: dict, dev: dict, n_chunks: int = 0,
                          workspace=None, ws_bytes=None, stream=None, order: int = 0):
    """dsa_prefill with inputs and output in (page-locked) host tensors, copies overlapped
    with the computation; dev holds the device buffers of the same shapes."""
    p = shape.params()
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    hb, db = layer_buffers(host), layer_buffers(dev)
    _check(lib.dsa_prefill_from_host(ctypes.byref(p), ctypes.byref(rg), ctypes.byref(hb),
                                     ctypes.byref(db), n_chunks, order, _ptr(workspace), ws_bytes,
                                     _stream(stream)), "dsa_prefill_from_host")


def dsa_index_topk_blocks_workspace_size(shape: LayerShape, rg: Ragged, block: int,
                                         q_count: int):
    p = shape.params()
    mn, rec = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.dsa_index_topk_blocks_workspace_size(ctypes.byref(p), ctypes.byref(rg), block,
                                                    q_count, ctypes.byref(mn), ctypes.byref(rec)),
           "dsa_index_topk_blocks_workspace_size")
    return mn.value, rec.value


def dsa_index_topk_blocks(shape: LayerShape, rg: Ragged, q_idx, k_idx, w, block: int, q_begin: int,
                          q_count: int, idx, ld_idx: int, cnt=None, workspace=None, ws_bytes=None,
                          stream=None):
    """top_k of `shape` counts blocks; idx receives positions (ld_idx >= top_k * block)."""
    p = shape.params()
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.dsa_index_topk_blocks(ctypes.byref(p), ctypes.byref(rg), _ptr(q_idx), _ptr(k_idx),
                                     _ptr(w), block, q_begin, q_count, _ptr(idx), ld_idx,
                                     _ptr(cnt), _ptr(workspace), ws_bytes, _stream(stream)),
           "dsa_index_topk_blocks")


def dsa_sparse_attn_gated_mix(shape: LayerShape, rg: Ragged, q, k_cache, v_cache, idx, ld_idx: int,
                              q_begin: int, q_count: int, gate, other, out, lse=None,
                              err_count=None, stream=None):
    p = shape.params()
    _check(lib.dsa_sparse_attn_gated_mix(ctypes.byref(p), ctypes.byref(rg), _ptr(q),
                                         _ptr(k_cache), _ptr(v_cache), _ptr(idx), ld_idx, q_begin,
                                         q_count, _ptr(gate), _ptr(other), _ptr(out), _ptr(lse),
                                         _ptr(err_count), _stream(stream)),
           "dsa_sparse_attn_gated_mix")


def dsa_workspace_size(shape: LayerShape, rg: Ragged, is_decode: bool = False):
    p = shape.params()
    mn, rec = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.dsa_workspace_size(ctypes.byref(p), ctypes.byref(rg), int(is_decode),
                                  ctypes.byref(mn), ctypes.byref(rec)), "dsa_workspace_size")
    return mn.value, rec.value


def dsa_index_topk_workspace_size(shape: LayerShape, rg: Ragged, q_count: int):
    p = shape.params()
    mn, rec = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _check(lib.dsa_index_topk_workspace_size(ctypes.byref(p), ctypes.byref(rg), q_count,
                                             ctypes.byref(mn), ctypes.byref(rec)),
           "dsa_index_topk_workspace_size")
    return mn.value, rec.value


def dsa_index_topk(shape: LayerShape, rg: Ragged, q_idx, k_idx, w, q_begin: int, q_count: int,
                   idx, ld_idx: int, cnt=None, workspace=None, ws_bytes=None, stream=None):
    p = shape.params()
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.dsa_index_topk(ctypes.byref(p), ctypes.byref(rg), _ptr(q_idx), _ptr(k_idx),
                              _ptr(w), q_begin, q_count, _ptr(idx), ld_idx, _ptr(cnt),
                              _ptr(workspace), ws_bytes, _stream(stream)), "dsa_index_topk")


def _layer(fn, name, shape, rg, q_idx, k_idx, w, q, k_cache, v_cache, gate, out, idx_out,
           err_count, workspace, ws_bytes, stream):
    p = shape.params()
    if ws_bytes is None:
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(fn(ctypes.byref(p), ctypes.byref(rg), _ptr(q_idx), _ptr(k_idx), _ptr(w), _ptr(q),
              _ptr(k_cache), _ptr(v_cache), _ptr(gate), _ptr(out), _ptr(idx_out), _ptr(err_count),
              _ptr(workspace), ws_bytes, _stream(stream)), name)


def dsa_prefill(shape: LayerShape, rg: Ragged, q_idx, k_idx, w, q, k_cache, v_cache, gate, out,
                idx_out=None, err_count=None, workspace=None, ws_bytes=None, stream=None):
    _layer(lib.dsa_prefill, "dsa_prefill", shape, rg, q_idx, k_idx, w, q, k_cache, v_cache, gate,
           out, idx_out, err_count, workspace, ws_bytes, stream)


def dsa_decode(shape: LayerShape, rg: Ragged, q_idx, k_idx, w, q, k_cache, v_cache, gate, out,
               idx_out=None, err_count=None, workspace=None, ws_bytes=None, stream=None):
    _layer(lib.dsa_decode, "dsa_decode", shape, rg, q_idx, k_idx, w, q, k_cache, v_cache, gate,
           out, idx_out, err_count, workspace, ws_bytes, stream)


def dsa_decode_noalloc(shape: LayerShape, rg: Ragged, q_idx, k_idx, w, q, k_cache, v_cache, gate,
                       out, idx_out=None, err_count=None, stream=None):
    """dsa_decode whose scratch is the library's fixed per-device array (no allocation)."""
    p = shape.params()
    _check(lib.dsa_decode_noalloc(ctypes.byref(p), ctypes.byref(rg), _ptr(q_idx), _ptr(k_idx),
                                  _ptr(w), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(gate),
                                  _ptr(out), _ptr(idx_out), _ptr(err_count), _stream(stream)),
           "dsa_decode_noalloc")


def dsa_device_status(clear: bool = True, stream=None) -> int:
    v = ctypes.c_int32(0)
    _check(lib.dsa_device_status(_stream(stream), ctypes.byref(v), int(clear)), "dsa_device_status")
    return v.value


def dsa_launch_count() -> int:
    return int(lib.dsa_launch_count())


def dsa_fused_rows(reset: bool = False) -> int:
    return int(lib.dsa_fused_rows(int(reset)))


def dsa_stage_timing(enable: bool):
    _check(lib.dsa_stage_timing(int(enable)), "dsa_stage_timing")


def dsa_stage_times(reset: bool = True):
    ms = (ctypes.c_double * 3)()
    n = (ctypes.c_int64 * 3)()
    _check(lib.dsa_stage_times(ms, n, int(reset)), "dsa_stage_times")
    return list(ms), list(n)


def workload_shape(w) -> LayerShape:
    """LayerShape of a dsa_synth.Workload."""
    return LayerShape(w.n_idx_heads, w.idx_dim, w.n_q_heads, w.n_kv_heads, w.head_dim, w.top_k,
                      DSA_FP8_E4M3 if w.idx_dtype == "fp8" else DSA_BF16)
