"""ctypes binding of the plain CPU oracle (oracle.cpp).

TEST INFRASTRUCTURE ONLY: imported by the tests, by ``__graft_entry__.smoke()``
and by the benchmark's CPU-baseline / reference leg.  The product package never
imports it.  Arrays are numpy: bf16 tensors as uint16 bit patterns, fp8 e4m3 as
uint8, weights fp32, offsets int64.  Results are fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Dict, Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    subprocess.check_call(["g++", "-O2", "-std=c++17", "-shared", "-fPIC", "-pthread",
                           "-ffp-contract=off", "-o", _LIB_PATH, _SRC])
    return _LIB_PATH


class Problem(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("q_off", ctypes.c_void_p),
        ("kv_off", ctypes.c_void_p),
        ("n_idx_heads", ctypes.c_int32),
        ("idx_dim", ctypes.c_int32),
        ("n_q_heads", ctypes.c_int32),
        ("n_kv_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("top_k", ctypes.c_int32),
        ("idx_is_fp8", ctypes.c_int32),
        ("idx_scale_q", ctypes.c_double),
        ("idx_scale_k", ctypes.c_double),
        ("attn_scale", ctypes.c_double),
        ("w_row_stride", ctypes.c_int32),
    ]


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        L.oracle_index_scores_row.argtypes = [ctypes.POINTER(Problem), vp, vp, vp, i64, vp]
        L.oracle_index_scores_row.restype = i64
        L.oracle_topk_row.argtypes = [vp, i64, i32, vp]
        L.oracle_topk_row.restype = i32
        L.oracle_sparse_attn_row.argtypes = [ctypes.POINTER(Problem), vp, vp, vp, vp, vp, i64, vp, vp]
        L.oracle_sparse_attn_row.restype = None
        L.oracle_layer_rows.argtypes = [ctypes.POINTER(Problem), vp, vp, vp, vp, vp, vp, vp, vp, i64,
                                        i32, vp, vp, vp]
        L.oracle_layer_rows.restype = None
        L.oracle_block_topk_row.argtypes = [vp, i64, i32, i32, vp]
        L.oracle_block_topk_row.restype = i32
        L.oracle_gate_mix.argtypes = [vp, vp, vp, i64, vp]
        L.oracle_gate_mix.restype = None
        L.oracle_hardware_threads.argtypes = []
        L.oracle_hardware_threads.restype = i32
        _lib = L
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


class Oracle:
    """One problem description plus the host arrays it reads."""

    def __init__(self, arrays: Dict[str, np.ndarray], *, top_k: int, n_idx_heads: int,
                 idx_dim: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                 idx_fp8: bool = False, idx_scale_q: float = 1.0, idx_scale_k: float = 1.0,
                 attn_scale: float = 0.0, w_row_stride: int = 0):
        self.a = {k: (np.ascontiguousarray(v) if isinstance(v, np.ndarray) else v)
                  for k, v in arrays.items()}
        self.q_off = np.ascontiguousarray(self.a["q_offsets"], dtype=np.int64)
        self.kv_off = np.ascontiguousarray(self.a["kv_offsets"], dtype=np.int64)
        self.P = Problem(len(self.q_off) - 1, self.q_off.ctypes.data, self.kv_off.ctypes.data,
                         n_idx_heads, idx_dim, n_q_heads, n_kv_heads, head_dim, top_k,
                         1 if idx_fp8 else 0, idx_scale_q, idx_scale_k, attn_scale, w_row_stride)
        self.top_k, self.Hq, self.d = top_k, n_q_heads, head_dim

    @classmethod
    def for_workload(cls, w, arrays):
        return cls(arrays, top_k=w.top_k, n_idx_heads=w.n_idx_heads, idx_dim=w.idx_dim,
                   n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   idx_fp8=(w.idx_dtype == "fp8"))

    def position(self, r: int) -> int:
        b = int(np.searchsorted(self.q_off, r, side="right") - 1)
        L = self.kv_off[b + 1] - self.kv_off[b]
        Q = self.q_off[b + 1] - self.q_off[b]
        return int(L - Q + (r - self.q_off[b]))

    def index_scores_row(self, r: int) -> np.ndarray:
        s = np.empty(self.position(r) + 1, dtype=np.float64)
        n = lib().oracle_index_scores_row(ctypes.byref(self.P), _ptr(self.a["q_idx"]),
                                          _ptr(self.a["k_idx"]), _ptr(self.a["w"]), r,
                                          s.ctypes.data)
        assert n == len(s)
        return s

    def sparse_attn_row(self, r: int, idx: np.ndarray):
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        assert idx.shape == (self.top_k,)
        out = np.empty((self.Hq, self.d), dtype=np.float64)
        lse = np.empty((self.Hq,), dtype=np.float64)
        lib().oracle_sparse_attn_row(ctypes.byref(self.P), _ptr(self.a["q"]), _ptr(self.a["k"]),
                                     _ptr(self.a["v"]), _ptr(self.a.get("gate")), idx.ctypes.data,
                                     r, out.ctypes.data, lse.ctypes.data)
        return out, lse

    def sparse_attn_mix_row(self, r: int, idx: np.ndarray, o2: np.ndarray):
        """Gated mixing with the second branch: sigmoid(g) * o + (1 - sigmoid(g)) * o2 for
        packed query row r (o the ungated attention over idx; o2 [Hq, d] bf16 bits)."""
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        o = np.empty((self.Hq, self.d), dtype=np.float64)
        lib().oracle_sparse_attn_row(ctypes.byref(self.P), _ptr(self.a["q"]), _ptr(self.a["k"]),
                                     _ptr(self.a["v"]), None, idx.ctypes.data, r, o.ctypes.data,
                                     None)
        g = np.ascontiguousarray(self.a["gate"][r], dtype=np.uint16)
        o2 = np.ascontiguousarray(o2, dtype=np.uint16)
        return gate_mix(o, g, o2)

    def layer_rows(self, rows: Sequence[int], nthreads: int = 0):
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        nr = len(rows)
        if nthreads <= 0:
            nthreads = hardware_threads()
        idx = np.empty((nr, self.top_k), dtype=np.int32)
        out = np.empty((nr, self.Hq, self.d), dtype=np.float64)
        lse = np.empty((nr, self.Hq), dtype=np.float64)
        lib().oracle_layer_rows(ctypes.byref(self.P), _ptr(self.a["q_idx"]), _ptr(self.a["k_idx"]),
                                _ptr(self.a["w"]), _ptr(self.a["q"]), _ptr(self.a["k"]),
                                _ptr(self.a["v"]), _ptr(self.a.get("gate")), rows.ctypes.data, nr,
                                nthreads, idx.ctypes.data, out.ctypes.data, lse.ctypes.data)
        return idx, out, lse


def block_topk_row(s: np.ndarray, B: int, Kb: int) -> np.ndarray:
    """Oracle block-granular Top-K of one score row: positions of the Kb blocks (of B
    positions) with the largest maxima, ascending, -1 up to Kb * B."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    idx = np.empty(Kb * B, dtype=np.int32)
    lib().oracle_block_topk_row(s.ctypes.data, len(s), B, Kb, idx.ctypes.data)
    return idx


def gate_mix(o: np.ndarray, gate_bits: np.ndarray, o2_bits: np.ndarray) -> np.ndarray:
    """Oracle step 4 with the second branch, elementwise over equally shaped arrays: o fp64,
    gate logits and o2 as bf16 bit patterns (uint16)."""
    o = np.ascontiguousarray(o, dtype=np.float64)
    g = np.ascontiguousarray(gate_bits, dtype=np.uint16)
    o2 = np.ascontiguousarray(o2_bits, dtype=np.uint16)
    assert o.shape == g.shape == o2.shape
    out = np.empty_like(o)
    lib().oracle_gate_mix(o.ctypes.data, g.ctypes.data, o2.ctypes.data, o.size, out.ctypes.data)
    return out


def topk_row(s: np.ndarray, K: int) -> np.ndarray:
    """Oracle Top-K of one score row (fp64 values; fp32 inputs convert exactly)."""
    s = np.ascontiguousarray(s, dtype=np.float64)
    idx = np.empty(K, dtype=np.int32)
    lib().oracle_topk_row(s.ctypes.data, len(s), K, idx.ctypes.data)
    return idx


def hardware_threads() -> int:
    return int(lib().oracle_hardware_threads())
