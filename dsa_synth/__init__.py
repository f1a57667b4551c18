"""Seeded synthetic inputs for the gated Indexer + Top-K sparse-attention layer.

This package is the one piece that both the CPU oracle and the CUDA path
consume: it turns (seed, tensor id, flat element index) into input values via
the counter-based generator in ``synth.h`` (host and device give identical
bits).  It holds no arithmetic of the layer itself.

``Workload`` describes one input recipe (shapes, ragged lengths, value
families, planted structure).  ``make_device_inputs`` fills device tensors;
``make_host_sequence`` regenerates one sequence's inputs on the host so the
oracle can check sampled rows of workloads far larger than host memory.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libdsasynth.so")
_SRC = [os.path.join(_HERE, "synth.cu"), os.path.join(_HERE, "synth.h")]

# tensor ids and value families; must match synth.h
T_Q_IDX, T_K_IDX, T_W, T_Q, T_K, T_V, T_GATE, T_SCORES, T_LAYOUT = range(1, 10)
GRID, NORMAL, WEIGHT, ZERO, ONE = range(5)

INV_SQRT_128 = float(np.float32(1.0 / math.sqrt(128.0)))


def build(force: bool = False) -> str:
    """Compile libdsasynth.so in place (host + sm_100a device fills)."""
    newest = max(os.path.getmtime(p) for p in _SRC)
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= newest:
        return _LIB_PATH
    cmd = [
        "nvcc", "-O3", "-shared", "-Xcompiler", "-fPIC", "-std=c++17",
        "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
        "-o", _LIB_PATH, os.path.join(_HERE, "synth.cu"),
    ]
    subprocess.check_call(cmd)
    return _LIB_PATH


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        i64, u64, u32, f32, vp, ci = (ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                      ctypes.c_float, ctypes.c_void_p, ctypes.c_int)
        L.synth_fill_bf16_device.argtypes = [vp, i64, ci, u64, u32, u64, f32, vp]
        L.synth_fill_bf16_device.restype = ci
        L.synth_fill_e4m3_grid_device.argtypes = [vp, i64, u64, u32, u64, vp]
        L.synth_fill_e4m3_grid_device.restype = ci
        L.synth_fill_f32_device.argtypes = [vp, i64, ci, u64, u32, u64, f32, vp]
        L.synth_fill_f32_device.restype = ci
        L.synth_fill_bf16_host.argtypes = [vp, i64, ci, u64, u32, u64, f32]
        L.synth_fill_bf16_host.restype = None
        L.synth_fill_e4m3_grid_host.argtypes = [vp, i64, u64, u32, u64]
        L.synth_fill_e4m3_grid_host.restype = None
        L.synth_fill_f32_host.argtypes = [vp, i64, ci, u64, u32, u64, f32]
        L.synth_fill_f32_host.restype = None
        L.synth_u64_host.argtypes = [vp, i64, u64, u32, u64]
        L.synth_u64_host.restype = None
        _lib = L
    return _lib


# ----------------------------------------------------------------------------- host fills

def host_bf16(count: int, family: int, seed: int, tensor: int, start: int = 0,
              scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of elements [start, start+count)."""
    out = np.empty(count, dtype=np.uint16)
    lib().synth_fill_bf16_host(out.ctypes.data, count, family, seed, tensor, start, scale)
    return out


def host_e4m3_grid(count: int, seed: int, tensor: int, start: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.uint8)
    lib().synth_fill_e4m3_grid_host(out.ctypes.data, count, seed, tensor, start)
    return out


def host_f32(count: int, family: int, seed: int, tensor: int, start: int = 0,
             scale: float = 1.0) -> np.ndarray:
    out = np.empty(count, dtype=np.float32)
    lib().synth_fill_f32_host(out.ctypes.data, count, family, seed, tensor, start, scale)
    return out


def host_u64(count: int, seed: int, tensor: int, start: int = 0) -> np.ndarray:
    out = np.empty(count, dtype=np.uint64)
    lib().synth_u64_host(out.ctypes.data, count, seed, tensor, start)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite values)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


# ----------------------------------------------------------------------------- workloads

@dataclass
class Workload:
    """One synthetic input recipe for the layer (a ragged batch of sequences).

    Sequence b has ``kv_lens[b]`` cache positions; its ``q_lens[b]`` queries are
    the last ``q_lens[b]`` of them, so query i sits at position
    ``kv_lens[b] - q_lens[b] + i`` and may attend to positions 0..that one.
    """
    name: str
    q_lens: List[int]
    kv_lens: List[int]
    top_k: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int = 128
    n_idx_heads: int = 4
    idx_dim: int = 64
    idx_dtype: str = "bf16"          # "bf16" or "fp8"
    qkv_scale: float = INV_SQRT_128  # q, k, v ~ N(0,1) * qkv_scale
    gate: bool = True
    seed: int = 0
    # planted needles: list of key positions (sequence 0) and the designated query rows
    needle_pos: List[int] = field(default_factory=list)
    needle_rows: List[int] = field(default_factory=list)
    needle_dims: int = 42
    w_family: int = WEIGHT
    idx_family: int = GRID

    @property
    def batch(self) -> int:
        return len(self.q_lens)

    @property
    def q_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.q_lens)]).astype(np.int64)

    @property
    def kv_offsets(self) -> np.ndarray:
        return np.concatenate([[0], np.cumsum(self.kv_lens)]).astype(np.int64)

    @property
    def total_q(self) -> int:
        return int(sum(self.q_lens))

    @property
    def total_kv(self) -> int:
        return int(sum(self.kv_lens))

    def row_position(self, r: int) -> int:
        qo = self.q_offsets
        b = int(np.searchsorted(qo, r, side="right") - 1)
        return self.kv_lens[b] - self.q_lens[b] + (r - int(qo[b]))

    def row_seq(self, r: int) -> int:
        return int(np.searchsorted(self.q_offsets, r, side="right") - 1)

    def device_bytes(self) -> int:
        e_idx = 1 if self.idx_dtype == "fp8" else 2
        tq, tk = self.total_q, self.total_kv
        b = tq * self.n_idx_heads * self.idx_dim * e_idx + tk * self.n_idx_heads * self.idx_dim * e_idx
        b += 3 * tq * self.n_q_heads * self.head_dim * 2  # q, gate, out
        b += 2 * tk * self.n_kv_heads * self.head_dim * 2  # k, v
        return b

    # ---- planted structure (needles): u vector and needle key rows
    def needle_u(self) -> np.ndarray:
        """[H_i, D_i] values +-1/2; signs drawn from the layout stream."""
        h = host_u64(self.n_idx_heads * self.idx_dim, self.seed, T_LAYOUT, 1000)
        return np.where((h & np.uint64(1)) == 1, 0.5, -0.5).astype(np.float32).reshape(
            self.n_idx_heads, self.idx_dim)

    def needle_key_row(self) -> np.ndarray:
        u = self.needle_u()
        row = np.zeros_like(u)
        row[:, : self.needle_dims] = np.sign(u[:, : self.needle_dims]) * 0.5
        return row


def _needle_positions(seed: int, T: int, block: int, count: int) -> List[int]:
    out: List[int] = []
    k = 0
    while len(out) < count:
        p = int(host_u64(1, seed, T_LAYOUT, 2000 + k)[0] % np.uint64(T - block))
        k += 1
        if p not in out:
            out.append(p)
    return sorted(out)


def workload(name: str, scale_down: int = 1) -> Workload:
    """The five named input recipes (sizes of the layer's published configuration).

    ``scale_down`` > 1 shrinks sequence lengths (and K) for quick parity cases
    while keeping head counts, dims, value families and structure.
    """
    s = max(1, int(scale_down))
    if name == "prefill_t4096_k256":
        T = max(1, 4096 // s)
        return Workload(name, [T], [T], top_k=max(1, 256 // s), n_q_heads=8, n_kv_heads=8)
    if name == "prefill_t32768_k2048":
        T = max(1, 32768 // s)
        return Workload(name, [T], [T], top_k=max(1, 2048 // s), n_q_heads=32, n_kv_heads=4)
    if name == "decode_b64_l131072":
        B = 64 if s == 1 else max(2, 64 // s)
        L = max(1, 131072 // s)
        return Workload(name, [1] * B, [L] * B, top_k=max(1, 2048 // s), n_q_heads=32,
                        n_kv_heads=4)
    if name == "prefill_t131072_needles":
        T = max(256, 131072 // s)
        block = 128
        w = Workload(name, [T], [T], top_k=max(16, 2048 // s), n_q_heads=32, n_kv_heads=4)
        w.needle_pos = _needle_positions(w.seed, T, block, 16)
        w.needle_rows = list(range(T - block, T))
        return w
    if name == "mixed_serving":
        n_pre, chunk = 8, max(1, 8192 // s)
        hist_max = 262144 // s
        hh = host_u64(n_pre, 0, T_LAYOUT, 3000)
        hist = [int(x % np.uint64(hist_max + 1)) for x in hh]
        n_dec = 256 if s == 1 else max(4, 256 // s)
        lo, hi = max(1, 4096 // s), max(2, 262144 // s)
        ud = host_u64(n_dec, 0, T_LAYOUT, 4000)
        dec = []
        for x in ud:
            u = float(int(x) >> 11) * (2.0 ** -53)
            dec.append(int(math.floor(lo * (hi / lo) ** u)))
        q_lens = [chunk] * n_pre + [1] * n_dec
        kv_lens = [h + chunk for h in hist] + dec
        return Workload(name, q_lens, kv_lens, top_k=max(1, 2048 // s), n_q_heads=64,
                        n_kv_heads=8)
    raise KeyError(name)


WORKLOADS = ["prefill_t4096_k256", "prefill_t32768_k2048", "decode_b64_l131072",
             "prefill_t131072_needles", "mixed_serving"]


# ----------------------------------------------------------------------------- host inputs

def make_host_sequence(w: Workload, b: int, rows: Optional[np.ndarray] = None) -> Dict[str, np.ndarray]:
    """Regenerate sequence b's inputs on the host, exactly as the device fill made them.

    Returns bf16 tensors as uint16 bit arrays (fp8 indexer tensors as uint8),
    shaped [rows, heads, dim]; query-side tensors cover all of the sequence's
    query rows.  Also returns the per-sequence offsets for a batch-of-one view.
    """
    Hi, Di, Hq, Hkv, d = w.n_idx_heads, w.idx_dim, w.n_q_heads, w.n_kv_heads, w.head_dim
    qo, ko = int(w.q_offsets[b]), int(w.kv_offsets[b])
    Q, L = w.q_lens[b], w.kv_lens[b]
    out: Dict[str, np.ndarray] = {}
    if w.idx_dtype == "fp8":
        out["q_idx"] = host_e4m3_grid(Q * Hi * Di, w.seed, T_Q_IDX, qo * Hi * Di).reshape(Q, Hi, Di)
        out["k_idx"] = host_e4m3_grid(L * Hi * Di, w.seed, T_K_IDX, ko * Hi * Di).reshape(L, Hi, Di)
    else:
        out["q_idx"] = host_bf16(Q * Hi * Di, w.idx_family, w.seed, T_Q_IDX, qo * Hi * Di,
                                 w.qkv_scale).reshape(Q, Hi, Di)
        out["k_idx"] = host_bf16(L * Hi * Di, w.idx_family, w.seed, T_K_IDX, ko * Hi * Di,
                                 w.qkv_scale).reshape(L, Hi, Di)
    out["q"] = host_bf16(Q * Hq * d, NORMAL, w.seed, T_Q, qo * Hq * d, w.qkv_scale).reshape(Q, Hq, d)
    out["k"] = host_bf16(L * Hkv * d, NORMAL, w.seed, T_K, ko * Hkv * d, w.qkv_scale).reshape(L, Hkv, d)
    out["v"] = host_bf16(L * Hkv * d, NORMAL, w.seed, T_V, ko * Hkv * d, w.qkv_scale).reshape(L, Hkv, d)
    if w.gate:
        out["gate"] = host_bf16(Q * Hq * d, NORMAL, w.seed, T_GATE, qo * Hq * d, 1.0).reshape(Q, Hq, d)
    out["w"] = host_f32(Hi, w.w_family, w.seed, T_W, 0)
    if w.needle_pos and b == 0:
        _plant_host(w, out, qo)
    out["q_offsets"] = np.array([0, Q], dtype=np.int64)
    out["kv_offsets"] = np.array([0, L], dtype=np.int64)
    return out


def _encode_idx(w: Workload, vals: np.ndarray) -> np.ndarray:
    if w.idx_dtype == "fp8":
        table = {0.5: 0x30, 0.375: 0x2C, 0.25: 0x28, 0.125: 0x20, 0.0: 0x00}
        mag = np.vectorize(lambda x: table[abs(float(x))])(vals).astype(np.uint8)
        return np.where(vals < 0, mag | 0x80, mag).astype(np.uint8)
    return f32_to_bf16_bits(vals)


def needle_arrays(w: Workload):
    """(u rows for the designated queries, needle key row) encoded in the indexer dtype."""
    return _encode_idx(w, w.needle_u()), _encode_idx(w, w.needle_key_row())


def _plant_host(w: Workload, seq: Dict[str, np.ndarray], qo: int) -> None:
    u_enc, key_enc = needle_arrays(w)
    for p in w.needle_pos:
        seq["k_idx"][p] = key_enc
    for r in w.needle_rows:
        seq["q_idx"][r - qo] = u_enc


def make_host_inputs(w: Workload) -> Dict[str, np.ndarray]:
    """All inputs of a (small) workload on the host, packed ragged."""
    Hi, Di, Hq, Hkv, d = w.n_idx_heads, w.idx_dim, w.n_q_heads, w.n_kv_heads, w.head_dim
    tq, tk = w.total_q, w.total_kv
    out: Dict[str, np.ndarray] = {}
    if w.idx_dtype == "fp8":
        out["q_idx"] = host_e4m3_grid(tq * Hi * Di, w.seed, T_Q_IDX).reshape(tq, Hi, Di)
        out["k_idx"] = host_e4m3_grid(tk * Hi * Di, w.seed, T_K_IDX).reshape(tk, Hi, Di)
    else:
        out["q_idx"] = host_bf16(tq * Hi * Di, w.idx_family, w.seed, T_Q_IDX, 0,
                                 w.qkv_scale).reshape(tq, Hi, Di)
        out["k_idx"] = host_bf16(tk * Hi * Di, w.idx_family, w.seed, T_K_IDX, 0,
                                 w.qkv_scale).reshape(tk, Hi, Di)
    out["q"] = host_bf16(tq * Hq * d, NORMAL, w.seed, T_Q, 0, w.qkv_scale).reshape(tq, Hq, d)
    out["k"] = host_bf16(tk * Hkv * d, NORMAL, w.seed, T_K, 0, w.qkv_scale).reshape(tk, Hkv, d)
    out["v"] = host_bf16(tk * Hkv * d, NORMAL, w.seed, T_V, 0, w.qkv_scale).reshape(tk, Hkv, d)
    if w.gate:
        out["gate"] = host_bf16(tq * Hq * d, NORMAL, w.seed, T_GATE, 0, 1.0).reshape(tq, Hq, d)
    out["w"] = host_f32(Hi, w.w_family, w.seed, T_W, 0)
    if w.needle_pos:
        _plant_host(w, out, 0)
    out["q_offsets"] = w.q_offsets
    out["kv_offsets"] = w.kv_offsets
    return out


# ----------------------------------------------------------------------------- device inputs

def make_device_inputs(w: Workload, device="cuda", stream=None):
    """Fill device tensors for the whole workload with the device generator.

    Returns a dict of torch tensors (bf16 as torch.bfloat16, fp8 as uint8,
    offsets as int32), generated in place on the device; nothing is copied from
    the host except the small planted rows and the offsets.
    """
    import torch

    L = lib()
    Hi, Di, Hq, Hkv, d = w.n_idx_heads, w.idx_dim, w.n_q_heads, w.n_kv_heads, w.head_dim
    tq, tk = w.total_q, w.total_kv
    st = torch.cuda.current_stream(device) if stream is None else stream
    sp = ctypes.c_void_p(st.cuda_stream)
    out = {}

    def bf16(shape, family, tensor, scale):
        t = torch.empty(shape, dtype=torch.bfloat16, device=device)
        rc = L.synth_fill_bf16_device(t.data_ptr(), t.numel(), family, w.seed, tensor, 0, scale, sp)
        assert rc == 0, f"synth fill failed: {rc}"
        return t

    if w.idx_dtype == "fp8":
        for key, tid, rows in (("q_idx", T_Q_IDX, tq), ("k_idx", T_K_IDX, tk)):
            t = torch.empty((rows, Hi, Di), dtype=torch.uint8, device=device)
            rc = L.synth_fill_e4m3_grid_device(t.data_ptr(), t.numel(), w.seed, tid, 0, sp)
            assert rc == 0
            out[key] = t
    else:
        out["q_idx"] = bf16((tq, Hi, Di), w.idx_family, T_Q_IDX, w.qkv_scale)
        out["k_idx"] = bf16((tk, Hi, Di), w.idx_family, T_K_IDX, w.qkv_scale)
    out["q"] = bf16((tq, Hq, d), NORMAL, T_Q, w.qkv_scale)
    out["k"] = bf16((tk, Hkv, d), NORMAL, T_K, w.qkv_scale)
    out["v"] = bf16((tk, Hkv, d), NORMAL, T_V, w.qkv_scale)
    out["gate"] = bf16((tq, Hq, d), NORMAL, T_GATE, 1.0) if w.gate else None
    wt = torch.empty((Hi,), dtype=torch.float32, device=device)
    rc = L.synth_fill_f32_device(wt.data_ptr(), Hi, w.w_family, w.seed, T_W, 0, 1.0, sp)
    assert rc == 0
    out["w"] = wt
    if w.needle_pos:
        u_enc, key_enc = needle_arrays(w)
        dt = torch.uint8 if w.idx_dtype == "fp8" else torch.int16
        u_t = torch.from_numpy(u_enc.view(np.uint8) if w.idx_dtype == "fp8" else u_enc.view(np.int16))
        k_t = torch.from_numpy(key_enc.view(np.uint8) if w.idx_dtype == "fp8" else key_enc.view(np.int16))
        qi = out["q_idx"].view(dt)
        ki = out["k_idx"].view(dt)
        for p in w.needle_pos:
            ki[p].copy_(k_t.to(device))
        rows = torch.tensor(w.needle_rows, dtype=torch.long, device=device)
        qi[rows] = u_t.to(device).unsqueeze(0).expand(len(w.needle_rows), Hi, Di)
    out["q_offsets"] = torch.from_numpy(w.q_offsets.astype(np.int32)).to(device)
    out["kv_offsets"] = torch.from_numpy(w.kv_offsets.astype(np.int32)).to(device)
    return out
